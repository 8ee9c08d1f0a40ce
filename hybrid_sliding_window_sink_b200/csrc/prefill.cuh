// prefill.cuh - sm_100a prefill of one SWA or GA layer with the attention sink.
//
// Math ("MiMo-V2-Flash: Hybrid Sliding Window Attention Architecture", §4.4 and §5
// steps 2-5; partial RoPE from "...MiMo-V2.6-Flash-MOPD混合SWA设计原理" §5):
//   q_i, k_j rotated on dims [0, rot) at positions i, j (rotate-half pairing);
//   a_ij = q_i.k_j * scale for j in J_i (SWA: [max(0, i-W+1), i]; GA: [0, i]);
//   m_i = max(sink_h, max_j a_ij); l_i = exp(sink_h - m_i) + sum_j exp(a_ij - m_i);
//   o_i = sum_j exp(a_ij - m_i) v_j / l_i; lse_i = m_i + ln l_i.
// The running max and denominator of the online softmax start at (sink_h, 1), so
// the sink enters the denominator exactly once and carries no value vector.
//
// Tiling. One tile row block = 128 MMA rows = P positions x G query heads of one
// KV group (G = Hq/Hkv, P = 128/G; row r = position p0 + r/G, head g*G + r%G), so
// every K/V tile is loaded once for all G heads that share it. Key tiles of BN rows
// cover only [lo, p0+P-1] with lo = max(0, p0-W+1) (SWA) or 0 (GA): tiles outside
// the window or the causal prefix are never loaded. For W = 128 and G >= 8 a single
// 144-key tile covers the whole window of a row block.
//
// CTA roles (192 threads, one CTA per SM, persistent over row blocks):
//   warp 0     TMA producer: Q (3 x 64-dim chunks), K (3 chunks), V (2 chunks),
//              128-byte swizzled tiles, completion on mbarriers (expect-tx).
//   warp 1     allocates 512 TMEM columns; one thread issues tcgen05.mma:
//              S = Q K^T into a double-buffered TMEM S tile, O += P V into TMEM O.
//   warps 2-5  compute group: RoPE of Q and K tiles in shared memory (fp64 angle
//              reduction, fp32 sin/cos, rotated dims kept as f16), sink-seeded
//              online softmax from TMEM S,
//              P (bf16) to shared memory, O rescale in TMEM, epilogue O / l -> bf16.
// Every wait is bounded in time; on a timeout all roles leave their loops, the
// producer and MMA thread wait (bounded) for their in-flight work, TMEM is freed
// and the device error word is set.
#pragma once

#include "ptx.cuh"

namespace mimo {

constexpr int kPfThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct PrefillParams {
  const float* sink;       // [Hq] or null
  __nv_bfloat16* out;      // [B, n, Hq, 128]
  float* lse;              // [B, Hq, n] or null
  int B, n, Hq, Hkv, window, rot_dims;
  double rope_theta;
  float scale_log2;        // softmax scale * log2(e)
  int n_qtiles, num_work;
  // chunked prefill (generic kernel only): query row i sits at position q_off + i; keys
  // cover positions 0 .. nk-1; key rows at positions < krot_from are stored rotated.
  // Whole-sequence prefill: q_off = 0, nk = n, krot_from = 0.
  int q_off, nk, krot_from;
  unsigned* err;
  unsigned long long* trace;   // debug timestamps (builds with -DMIMO_TRACE only), else null
};

template <int G, int BN, int NKS>
struct PfCfg {
  static constexpr int P = 128 / G;
  static constexpr int Q_CHUNK = 128 * 128;      // 128 rows x 64 dims bf16
  static constexpr int K_CHUNK = BN * 128;       // BN rows x 64 dims bf16
  static constexpr int Q_BYTES = 3 * Q_CHUNK;
  static constexpr int K_BYTES = 3 * K_CHUNK;
  static constexpr int V_BYTES = 2 * K_CHUNK;
  static constexpr int P_CHUNK = 128 * 128;      // 128 rows x 64 keys bf16
  static constexpr int P_CHUNKS = (BN + 63) / 64;
  static constexpr int P_BYTES = P_CHUNKS * P_CHUNK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NKS * K_BYTES;
  static constexpr int OFF_P = OFF_V + V_BYTES;
  static constexpr int OFF_MISC = OFF_P + P_BYTES;
  static constexpr int MISC_BYTES = 256 + 96 * 8;   // barriers + flags, inverse frequencies
  static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;   // + alignment slack
  static constexpr int S1_COL = (BN + 31) / 32 * 32;
  static constexpr int O_COL = (S1_COL + BN + 31) / 32 * 32;
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
  static constexpr uint32_t IDESC_S_F16 = idesc_f16kind(128, BN, 0, 0, 1);   // rotated dims
  static constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, 0, 1);
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(K_CHUNK % 1024 == 0, "swizzle atoms");
  static_assert(O_COL + 128 <= 512, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

// Barrier slots inside the misc area.
enum : int {
  kBarQFull = 0, kBarQReady, kBarQEmpty, kBarVFull, kBarVEmpty, kBarPReady, kBarPVDone,
  kBarFinal, kBarSFull0, kBarSFull1, kBarSFree0, kBarSFree1,
  kBarKFull0, kBarKFull1, kBarKReady0, kBarKReady1, kBarKEmpty0, kBarKEmpty1,
  kNumBars
};

// Rotates dims [0, rot) of one tile row in place (rotate-half pairing (d, d + rot/2)).
// The row lives in 64-dim chunks of `chunk_bytes`, 128 bytes per row, with the
// 16-byte units XOR-swizzled by (row & 7) as the 128-byte TMA swizzle writes them.
// Inputs are bf16; the rotated values are written back as f16 (11 significant bits
// instead of 8), and the QK^T k-steps over [0, rot) run as f16 x f16 MMAs. Rounding
// the rotated q and k to bf16 would perturb the scores by ~1e-3 (the size of the
// LSE tolerance); f16 cuts that eightfold. Values are clamped to the f16 range.
__device__ __forceinline__ void rope_row(uint32_t base, int chunk_bytes, int row, int pos, int rot,
                                         const double* invf) {
  const int nun = rot >> 4;   // 8-dim units per half
  const double dpos = static_cast<double>(pos);
  for (int u = 0; u < nun; ++u) {
    const int u2 = u + nun;
    const uint32_t a1 = base + (u >> 3) * chunk_bytes + row * 128 + (((u & 7) ^ (row & 7)) << 4);
    const uint32_t a2 = base + (u2 >> 3) * chunk_bytes + row * 128 + (((u2 & 7) ^ (row & 7)) << 4);
    uint32_t x[4], y[4];
    ld_shared_v4(a1, x[0], x[1], x[2], x[3]);
    ld_shared_v4(a2, y[0], y[1], y[2], y[3]);
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      float r1[2], r2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = u * 8 + e2 * 2 + h;
        // angle = pos * theta^(-2k/rot), reduced modulo 2*pi in double precision
        const double ang = dpos * invf[k];
        const double nrev = rint(ang * 0.15915494309189535);
        const float red = static_cast<float>(fma(-nrev, 6.283185307179586, ang));
        float s, c;
        __sincosf(red, &s, &c);
        const float v1 = h ? bf16_hi(x[e2]) : bf16_lo(x[e2]);
        const float v2 = h ? bf16_hi(y[e2]) : bf16_lo(y[e2]);
        r1[h] = v1 * c - v2 * s;
        r2[h] = v2 * c + v1 * s;
      }
      x[e2] = pack_f16_sat(r1[0], r1[1]);
      y[e2] = pack_f16_sat(r2[0], r2[1]);
    }
    st_shared_v4(a1, x[0], x[1], x[2], x[3]);
    st_shared_v4(a2, y[0], y[1], y[2], y[3]);
  }
}

// A key row stored already rotated (a cached prefix): its first `rot` dims only change
// format, bf16 -> f16, to match the f16 MMA k-steps over the rotated dims.
__device__ __forceinline__ void f16_row(uint32_t base, int chunk_bytes, int row, int rot) {
  for (int u = 0; u < (rot >> 3); ++u) {
    const uint32_t a = base + (u >> 3) * chunk_bytes + row * 128 + (((u & 7) ^ (row & 7)) << 4);
    uint32_t x[4];
    ld_shared_v4(a, x[0], x[1], x[2], x[3]);
    st_shared_v4(a, bf16x2_to_f16x2(x[0]), bf16x2_to_f16x2(x[1]), bf16x2_to_f16x2(x[2]),
                 bf16x2_to_f16x2(x[3]));
  }
}

template <int G, int BN, int NKS>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PfCfg<G, BN, NKS>;
  static_assert(NKS == 1 || NKS == 2, "K stages");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK0 = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  const uint32_t sP = sbase + C::OFF_P;
  const uint32_t sBar = sbase + C::OFF_MISC;
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8 * kNumBars);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + 8 * kNumBars + 4);
  double* s_invf = reinterpret_cast<double*>(smem + C::OFF_MISC + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned* err = p.err;

  if (threadIdx.x == 0) {
    const uint32_t counts[kNumBars] = {1, 128, 1, 1, 1, 128, 1, 1, 1, 1, 128, 128,
                                       1, 1, 128, 128, 1, 1};
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), counts[i]);
    *s_abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), 512);
    tmem_relinquish();
  }
  if (warp >= 2) {
    const int half = p.rot_dims >> 1;
    for (int k = threadIdx.x - 64; k < half; k += 128)
      s_invf[k] = pow(p.rope_theta, -2.0 * k / static_cast<double>(p.rot_dims));
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  const bool swa = p.window > 0 && p.window < p.nk;
  const int BG = p.B * p.Hkv;
  auto work_of = [&](int w, int& b, int& g, int& qt) {
    if (swa) {   // neighbouring CTAs take neighbouring row blocks: K/V windows overlap in L2
      qt = w % p.n_qtiles;
      const int bg = w / p.n_qtiles;
      b = bg / p.Hkv;
      g = bg - b * p.Hkv;
    } else {     // causal: longest row blocks first
      const int bg = w % BG;
      qt = p.n_qtiles - 1 - w / BG;
      b = bg / p.Hkv;
      g = bg - b * p.Hkv;
    }
  };
  auto kv_range = [&](int qt, int& lo, int& ntiles) {
    const int p0 = p.q_off + qt * C::P;                  // absolute position of the block
    const int hi = min(p0 + C::P - 1, p.q_off + p.n - 1);
    lo = swa ? max(0, p0 - p.window + 1) : 0;
    ntiles = (hi - lo + BN) / BN;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it_q = 0, it_kv = 0, nk[2] = {0, 0}, nv = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.num_work && ok; w += gridDim.x, ++it_q) {
        int b, g, qt, lo, T;
        work_of(w, b, g, qt);
        kv_range(qt, lo, T);
        if (it_q > 0 && !mbar_wait(bar(kBarQEmpty), (it_q - 1) & 1, s_abort, err)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(kBarQFull), C::Q_BYTES);
        for (int c = 0; c < 3; ++c)
          tma_load_4d(sQ + c * C::Q_CHUNK, &tmQ, bar(kBarQFull), 64 * c, g * G, qt * C::P, b);
        for (int j = 0; j < T; ++j) {
          const int it = it_kv + j, ks = it % NKS;
          if (it >= NKS && !mbar_wait(bar(kBarKEmpty0 + ks), ((it / NKS) - 1) & 1, s_abort, err)) { ok = false; break; }
          const uint32_t sK = sK0 + ks * C::K_BYTES;
          mbar_arrive_expect_tx(bar(kBarKFull0 + ks), C::K_BYTES);
          for (int c = 0; c < 3; ++c)
            tma_load_4d(sK + c * C::K_CHUNK, &tmK, bar(kBarKFull0 + ks), 64 * c, g, lo + j * BN, b);
          ++nk[ks];
          if (it >= 1 && !mbar_wait(bar(kBarVEmpty), (it - 1) & 1, s_abort, err)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(kBarVFull), C::V_BYTES);
          for (int c = 0; c < 2; ++c)
            tma_load_4d(sV + c * C::K_CHUNK, &tmV, bar(kBarVFull), 64 * c, g, lo + j * BN, b);
          ++nv;
        }
        it_kv += T;
      }
      if (!ok) {   // let every issued copy land before the CTA can exit
        if (it_q > 0) mbar_wait_drain(bar(kBarQFull), (it_q - 1) & 1, err);
        for (int s = 0; s < NKS; ++s)
          if (nk[s] > 0) mbar_wait_drain(bar(kBarKFull0 + s), (nk[s] - 1) & 1, err);
        if (nv > 0) mbar_wait_drain(bar(kBarVFull), (nv - 1) & 1, err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it_q = 0, it_kv = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.num_work && ok; w += gridDim.x, ++it_q) {
        int b, g, qt, lo, T;
        work_of(w, b, g, qt);
        kv_range(qt, lo, T);
        if (!mbar_wait(bar(kBarQReady), it_q & 1, s_abort, err)) { ok = false; break; }
        tc_fence_after();
        const int it_last = it_kv + T - 1;
        auto issue_s = [&](int it) -> bool {
          const int ks = it % NKS, sb = it & 1;
          if (!mbar_wait(bar(kBarKReady0 + ks), (it / NKS) & 1, s_abort, err)) return false;
          if (it >= 2 && !mbar_wait(bar(kBarSFree0 + sb), ((it >> 1) - 1) & 1, s_abort, err)) return false;
          tc_fence_after();
          const uint32_t sK = sK0 + ks * C::K_BYTES;
          const uint32_t d = tmem + (sb ? C::S1_COL : 0);
#pragma unroll
          for (int kk = 0; kk < 12; ++kk) {
            const uint32_t off = (kk & 3) * 32u;   // 16-dim step inside the 128-byte row
            const uint64_t a = smem_desc(sQ + (kk >> 2) * C::Q_CHUNK + off, 16, 1024);
            const uint64_t bd = smem_desc(sK + (kk >> 2) * C::K_CHUNK + off, 16, 1024);
            const uint32_t idesc = kk * 16 < p.rot_dims ? C::IDESC_S_F16 : C::IDESC_S;
            umma_ss(d, a, bd, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(kBarKEmpty0 + ks));
          umma_commit(bar(kBarSFull0 + sb));
          if (it == it_last) umma_commit(bar(kBarQEmpty));
          return true;
        };
        if (!issue_s(it_kv)) { ok = false; break; }
        for (int j = 0; j < T; ++j) {
          const int it = it_kv + j;
          if (j + 1 < T && !issue_s(it + 1)) { ok = false; break; }
          if (!mbar_wait(bar(kBarPReady), it & 1, s_abort, err)) { ok = false; break; }
          if (!mbar_wait(bar(kBarVFull), it & 1, s_abort, err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < BN / 16; ++s) {
            const uint64_t a = smem_desc(sP + (s >> 2) * C::P_CHUNK + (s & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc(sV + s * 2048, C::K_CHUNK, 1024);
            umma_ss(tmem + C::O_COL, a, bd, C::IDESC_PV, (j > 0 || s > 0) ? 1u : 0u);
          }
          umma_commit(bar(kBarVEmpty));
          umma_commit(bar(kBarPVDone));
        }
        it_kv += T;
      }
      // all issued MMAs must finish before TMEM is released
      umma_commit(bar(kBarFinal));
      mbar_wait_drain(bar(kBarFinal), 0, err);
    }
  } else {
    // ------------------------------------------------------------ compute group
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                       // tile row == TMEM lane
    const int ctid = threadIdx.x - 64;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    int it_q = 0, it_kv = 0;
    bool ok = true;
    auto wait_all = [&](uint32_t b_, uint32_t par) -> bool {
      const bool w_ok = mbar_wait(b_, par, s_abort, err);
      return __all_sync(0xffffffffu, w_ok);
    };
    auto rope_k = [&](int it, int key0) -> bool {
      const int ks = it % NKS;
      if (!wait_all(bar(kBarKFull0 + ks), (it / NKS) & 1)) return false;
      if (p.rot_dims > 0) {
        const uint32_t sK = sK0 + ks * C::K_BYTES;
        for (int t = ctid; t < BN; t += 128) {
          const int pos = key0 + t;
          if (pos >= p.krot_from && pos < p.nk) rope_row(sK, C::K_CHUNK, t, pos, p.rot_dims, s_invf);
          else if (pos >= 0 && pos < p.krot_from) f16_row(sK, C::K_CHUNK, t, p.rot_dims);
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(bar(kBarKReady0 + ks));
      return true;
    };

    for (int w = blockIdx.x; w < p.num_work && ok; w += gridDim.x, ++it_q) {
      int b, g, qt, lo, T;
      work_of(w, b, g, qt);
      kv_range(qt, lo, T);
      const int qi = qt * C::P + r / G;                  // query row within the call
      const int pos = p.q_off + qi;                      // its position
      const int h = g * G + (r % G);
      const bool row_ok = qi < p.n;
      const int klo = swa ? pos - p.window + 1 : 0;   // valid keys: [klo, pos]

      if (!wait_all(bar(kBarQFull), it_q & 1)) { ok = false; break; }
      if (p.rot_dims > 0) {
        if (row_ok) rope_row(sQ, C::Q_CHUNK, r, pos, p.rot_dims, s_invf);
        fence_proxy_async_smem();
      }
      mbar_arrive(bar(kBarQReady));

      const float sink2 = p.sink ? p.sink[h] * kLog2e : -INFINITY;
      float m = sink2, l = p.sink ? 1.f : 0.f;
      if (!rope_k(it_kv, lo)) { ok = false; break; }

      for (int j = 0; j < T; ++j) {
        const int it = it_kv + j;
        if (NKS >= 2 && j + 1 < T && !rope_k(it + 1, lo + (j + 1) * BN)) { ok = false; break; }
        if (!wait_all(bar(kBarSFull0 + (it & 1)), (it >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sc = trow + ((it & 1) ? C::S1_COL : 0);
        const int kt0 = lo + j * BN;

        // pass 1: row max over the valid keys of this tile
        float mx = -INFINITY;
#pragma unroll 1
        for (int cb = 0; cb < BN / 16; ++cb) {
          uint32_t v[16];
          tmem_ld16(sc + cb * 16, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int key = kt0 + cb * 16 + e;
            if (key >= klo && key <= pos) mx = fmaxf(mx, __uint_as_float(v[e]));
          }
        }
        const float mnew = fmaxf(m, mx * p.scale_log2);
        const float ref = mnew == -INFINITY ? 0.f : mnew;
        const float alpha = ex2(m - ref);

        // P and O are still in use by the previous PV MMA until it completes
        if (j > 0) {
          if (!wait_all(bar(kBarPVDone), (it - 1) & 1)) { ok = false; break; }
          tc_fence_after();
        }
        // pass 2: p = exp2(a*scale*log2e - ref) -> bf16 P tile in shared memory
        float sum = 0.f;
#pragma unroll 1
        for (int cb = 0; cb < BN / 16; ++cb) {
          uint32_t v[16];
          tmem_ld16(sc + cb * 16, v);
          tmem_wait_ld();
          float pe[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int key = kt0 + cb * 16 + e;
            const bool valid = key >= klo && key <= pos;
            pe[e] = valid ? ex2(__uint_as_float(v[e]) * p.scale_log2 - ref) : 0.f;
            sum += pe[e];
          }
          const uint32_t prow = sP + (cb >> 2) * C::P_CHUNK + r * 128;
          const int u0 = 2 * (cb & 3);
          st_shared_v4(prow + (((u0) ^ (r & 7)) << 4), pack_bf16(pe[0], pe[1]),
                       pack_bf16(pe[2], pe[3]), pack_bf16(pe[4], pe[5]), pack_bf16(pe[6], pe[7]));
          st_shared_v4(prow + (((u0 + 1) ^ (r & 7)) << 4), pack_bf16(pe[8], pe[9]),
                       pack_bf16(pe[10], pe[11]), pack_bf16(pe[12], pe[13]),
                       pack_bf16(pe[14], pe[15]));
        }
        tc_fence_before();
        mbar_arrive(bar(kBarSFree0 + (it & 1)));

        // rescale the running O when the max moved (warp-uniform TMEM access)
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int cb = 0; cb < 8; ++cb) {
            uint32_t v[16];
            tmem_ld16(trow + C::O_COL + cb * 16, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st16(trow + C::O_COL + cb * 16, v);
          }
          tmem_wait_st();
        }
        l = l * alpha + sum;
        m = mnew;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(kBarPReady));
      }
      if (!ok) break;

      // epilogue: o = O / l -> bf16, lse = (m + log2 l) ln 2
      if (!wait_all(bar(kBarPVDone), (it_kv + T - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.out + ((static_cast<long long>(b) * p.n + qi) * p.Hq + h) * 128;
#pragma unroll 1
      for (int cb = 0; cb < 8; ++cb) {
        uint32_t v[16];
        tmem_ld16(trow + C::O_COL + cb * 16, v);
        tmem_wait_ld();
        if (row_ok) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            pk[e] = pack_bf16(__uint_as_float(v[2 * e]) * inv_l, __uint_as_float(v[2 * e + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + cb * 16);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (row_ok && p.lse)
        p.lse[(static_cast<long long>(b) * p.Hq + h) * p.n + qi] =
            l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
      tc_fence_before();
      it_kv += T;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Appends a chunk of n tokens (positions off .. off+n-1) to a KV cache: K rotated at its
// position (rotate-half pairing over the first rot dims, angles reduced in double precision)
// and rounded to bf16, V copied. One thread per 16-byte unit of an output row; slot =
// p mod cap (ring, only the chunk's last cap tokens) or p (linear).
struct CacheAppendParams {
  const __nv_bfloat16* k;     // [B, n, Hkv, 192]
  const __nv_bfloat16* v;     // [B, n, Hkv, 128]
  __nv_bfloat16* kc;          // [B, stride, Hkv, 192]
  __nv_bfloat16* vc;          // [B, stride, Hkv, 128]
  long long stride;
  int B, n, Hkv, off, rot, ring, cap;
  double theta;
};

__global__ void __launch_bounds__(256) cache_append_kernel(const CacheAppendParams p) {
  constexpr int kUnits = 24 + 16;                       // K units, then V units, per row
  const long long total = static_cast<long long>(p.B) * p.n * p.Hkv * kUnits;
  const int first = p.ring && p.n > p.cap ? p.n - p.cap : 0;   // older chunk tokens are overwritten
  const int half = p.rot >> 1;
  for (long long it = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; it < total;
       it += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int u = static_cast<int>(it % kUnits);
    const long long row = it / kUnits;                  // (b, i, g)
    const int g = static_cast<int>(row % p.Hkv);
    const long long bi = row / p.Hkv;
    const int i = static_cast<int>(bi % p.n), b = static_cast<int>(bi / p.n);
    if (i < first) continue;
    const int pos = p.off + i;
    const long long slot = p.ring ? pos % p.cap : pos;
    const long long dst_row = (static_cast<long long>(b) * p.stride + slot) * p.Hkv + g;
    if (u >= 24) {                                      // V: copy 16 bytes
      const int vu = u - 24;
      *reinterpret_cast<uint4*>(p.vc + dst_row * 128 + vu * 8) =
          *reinterpret_cast<const uint4*>(p.v + row * 128 + vu * 8);
      continue;
    }
    const __nv_bfloat16* src = p.k + row * 192;
    uint4 x = *reinterpret_cast<const uint4*>(src + u * 8);
    if (u * 8 < p.rot) {
      // dims d = 8u .. 8u+7: partner dims d -+ half
      const bool first_half = u * 8 < half;
      const int pu = first_half ? u + (half >> 3) : u - (half >> 3);
      const uint4 y = *reinterpret_cast<const uint4*>(src + pu * 8);
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
      uint32_t out[4];
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        float r[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int d = u * 8 + e2 * 2 + hh;
          const int k = first_half ? d : d - half;
          const double ang = static_cast<double>(pos) * pow(p.theta, -2.0 * k / static_cast<double>(p.rot));
          const double nrev = rint(ang * 0.15915494309189535);
          float sn, cs;
          sincosf(static_cast<float>(fma(-nrev, 6.283185307179586, ang)), &sn, &cs);
          const float a = hh ? bf16_hi(xs[e2]) : bf16_lo(xs[e2]);
          const float bp = hh ? bf16_hi(ys[e2]) : bf16_lo(ys[e2]);
          r[hh] = first_half ? a * cs - bp * sn : a * cs + bp * sn;
        }
        out[e2] = pack_bf16(r[0], r[1]);
      }
      x = make_uint4(out[0], out[1], out[2], out[3]);
    }
    *reinterpret_cast<uint4*>(p.kc + dst_row * 192 + u * 8) = x;
  }
}

}  // namespace mimo
