// prefill_ga.cuh - sm_100a prefill of a GA layer (full causal prefix) with 8 or 16 query
// heads per KV head (MiMo GA layers: 64 Q / 4 KV heads).
//
// Math as in prefill.cuh ("MiMo-V2-Flash: Hybrid Sliding Window Attention Architecture",
// §4.4, §5 steps 2-5; RoPE from "...MiMo-V2.6-Flash-MOPD混合SWA设计原理" §5): online softmax
// over 128-key tiles of [0, i], running max and denominator seeded with the sink.
//
// Work item = two row blocks (A, B) of P = 128/G consecutive positions x G heads, so every
// K/V tile a CTA loads serves 256 query rows. Items are taken longest first (causal).
// Roles (448 threads, one CTA per SM):
//   warp 0       TMA producer: Q of both blocks (one buffer), K tiles (2 stages), V (1).
//   warp 1       TMEM allocator (512 columns) and event-driven tcgen05.mma issuer:
//                S_w = Q_w K^T (SS), O_w += P_w V (TS, P from TMEM) for w in {A, B}.
//   warps 2-5    RoPE group: Q of a new item (cos/sin table per position), and every K
//                tile once per CTA. K rows use no MUFU: thread t keeps (cos, sin)(t w_k) of
//                its tile row in registers and multiplies by the tile's base
//                (cos, sin)(kt0 w_k), computed by 32 threads per tile.
//   warps 6-9    softmax group A, warps 10-13 softmax group B: each owns 256 TMEM columns,
//                S in [0, 128) (P, bf16, overwrites it in [0, 64)) and O in [128, 256).
// The MMA issues S_w of tile j+1 only after PV_w of tile j has completed (P aliases S),
// so a softmax group always finds its O stable and never waits for PV inside a row block.
// Lazy rescaling: a row keeps its reference max until a tile raises it by more than 8 (log2
// units); P = 2^(a - ref) then stays below 2^8, and O / l are rescaled only when the
// reference moves.
#pragma once

#include <type_traits>

#include "ptx.cuh"
#include "prefill.cuh"

namespace mimo {

// Optional per-tile timestamps (debug builds with -DMIMO_TRACE; compiled out otherwise):
// events 0/1 S issued (group A/B), 2/3 PV issued, 4/5 S seen by the softmax group, 6/7 P
// written, 9 K tile rotated, 10/11 S issue started, 12/13 PV issue started, 14/15 row max
// done, 18/19 first half of P written.
#ifdef MIMO_TRACE
#define GA_TRACE(tile, ev)                                                             \
  do {                                                                                 \
    if (p.trace && blockIdx.x < 8 && (tile) < 256)                                     \
      p.trace[(static_cast<size_t>(blockIdx.x) * 256 + (tile)) * 32 + (ev)] = clock64(); \
  } while (0)
#else
#define GA_TRACE(tile, ev) \
  do {                     \
  } while (0)
#endif

// 32 consecutive TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
  tmem_ld16(taddr + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
}
// Placed right after tmem_wait_ld(): makes every later use of r depend on this point, so
// the compiler cannot move arithmetic on TMEM-loaded registers above the wait.
__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}
__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
  reg_fence16(*reinterpret_cast<uint32_t(*)[16]>(r));
  reg_fence16(*reinterpret_cast<uint32_t(*)[16]>(r + 16));
}

constexpr int kGaThreads = 448;
constexpr int kGaBN = 128;

template <int G>
struct GaLayout {
  static constexpr int P = 128 / G;                 // positions per row block
  static constexpr int Q_CHUNK = 128 * 128;
  static constexpr int Q_BLOCK = 3 * Q_CHUNK;      // 48 KB per row block
  static constexpr int K_CHUNK = kGaBN * 128;
  static constexpr int K_TILE = 3 * K_CHUNK;       // 48 KB
  static constexpr int V_TILE = 2 * K_CHUNK;       // 32 KB
  static constexpr int OFF_Q = 0;                  // blocks A, B
  static constexpr int OFF_K = OFF_Q + 2 * Q_BLOCK;
  static constexpr int OFF_V = OFF_K + 2 * K_TILE;
  static constexpr int OFF_MISC = OFF_V + V_TILE;
  static constexpr int MISC_BYTES = 512 + 32 * 8 + 4 * 32 * 8;   // barriers, inv freqs, 4 base tables
  static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;
  static constexpr uint32_t IDESC_S = idesc_bf16(128, kGaBN, 0, 0);
  static constexpr uint32_t IDESC_S_F16 = idesc_f16kind(128, kGaBN, 0, 0, 1);
  static constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, 0, 1);
  static_assert(SMEM <= 232448, "shared memory budget");
};

enum : int {
  kGaQFull = 0, kGaQReady = 1, kGaQEmpty = 2,
  kGaKFull = 3,    // [2]
  kGaKReady = 5,   // [2] (128 arrivals)
  kGaKEmpty = 7,   // [2]
  kGaVFull = 9, kGaVEmpty = 10,
  kGaSFull = 11,   // [2] per softmax group
  kGaPReady = 13,  // [2] (128 arrivals)
  kGaPVDone = 15,  // [2]
  kGaBase = 17,    // [4] K-tile base table written (32 arrivals)
  kGaFinal = 21,
  kGaNumBars = 22
};

template <int G>
__global__ void __launch_bounds__(kGaThreads, 1)
    prefill_ga_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using L = GaLayout<G>;
  constexpr int P = L::P;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::OFF_Q;
  const uint32_t sK = sbase + L::OFF_K;
  const uint32_t sV = sbase + L::OFF_V;
  const uint32_t sBar = sbase + L::OFF_MISC;
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8 * kGaNumBars);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC + 8 * kGaNumBars + 4);
  double* s_invf = reinterpret_cast<double*>(smem + L::OFF_MISC + 512);
  float2* s_base = reinterpret_cast<float2*>(smem + L::OFF_MISC + 512 + 256);   // [4][32]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned* err = p.err;
  const int half = p.rot_dims >> 1;   // <= 32

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGaNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == kGaQReady || (i >= kGaKReady && i < kGaKReady + 2) || (i >= kGaPReady && i < kGaPReady + 2))
        cnt = 128;
      if (i >= kGaBase && i < kGaBase + 4) cnt = 32;
      mbar_init(bar(i), cnt);
    }
    *s_abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), 512);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 6 && threadIdx.x - 64 < half)
    s_invf[threadIdx.x - 64] = pow(p.rope_theta, -2.0 * (threadIdx.x - 64) / static_cast<double>(p.rot_dims));
  // Q rows past the sequence end are never loaded: start them (and all of Q) at zero
  for (int i = threadIdx.x; i < 2 * L::Q_BLOCK / 16; i += kGaThreads)
    reinterpret_cast<uint4*>(smem + L::OFF_Q)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  const int BG = p.B * p.Hkv;
  const int npairs = p.n_qtiles;   // work items per (b, g): pairs of row blocks
  // round r of this CTA takes item r * grid + c, with c running backwards on odd rounds
  // (zig-zag), so that every CTA sees long and short items alike
  auto work_of = [&](int r) -> int {
    return r * static_cast<int>(gridDim.x) +
           ((r & 1) ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x));
  };
  // item w: longest first; (b, g) fastest so that concurrent CTAs share K/V tiles in L2
  auto item_of = [&](int w, int& b, int& g, int& p0, int& ntiles) {
    const int bg = w % BG;
    const int pi = npairs - 1 - w / BG;
    b = bg / p.Hkv;
    g = bg - b * p.Hkv;
    p0 = pi * 2 * P;                               // first query row of block A in the call
    const int hi = p.q_off + min(p0 + 2 * P - 1, p.n - 1);   // last position of the item
    ntiles = hi / kGaBN + 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int nq = 0, nk = 0, nv = 0;   // loads issued
      bool ok = true;
      for (int rd = 0, w = work_of(0); w < p.num_work && ok; w = work_of(++rd)) {
        int b, g, p0, T;
        item_of(w, b, g, p0, T);
        if (nq > 0 && !mbar_wait(bar(kGaQEmpty), (nq - 1) & 1, s_abort, err)) { ok = false; break; }
        const int nblk = p0 + P < p.n ? 2 : 1;   // block B may lie wholly past the end
        mbar_arrive_expect_tx(bar(kGaQFull), nblk * L::Q_BLOCK);
        for (int blk = 0; blk < nblk; ++blk)
          for (int c = 0; c < 3; ++c)
            tma_load_4d(sQ + blk * L::Q_BLOCK + c * L::Q_CHUNK, &tmQ, bar(kGaQFull), 64 * c, g * G,
                        p0 + blk * P, b);
        ++nq;
        // K runs one tile ahead of V: K(j + 1) needs only S of tile j - 1 to be done,
        // while the single V buffer frees up only when PV of tile j - 1 is done
        for (int j = 0; j <= T && ok; ++j) {
          if (j < T) {
            const int ks = nk & 1;
            if (nk >= 2 && !mbar_wait(bar(kGaKEmpty + ks), ((nk >> 1) - 1) & 1, s_abort, err)) { ok = false; break; }
            mbar_arrive_expect_tx(bar(kGaKFull + ks), L::K_TILE);
            for (int c = 0; c < 3; ++c)
              tma_load_4d(sK + ks * L::K_TILE + c * L::K_CHUNK, &tmK, bar(kGaKFull + ks), 64 * c, g,
                          j * kGaBN, b);
            ++nk;
          }
          if (j >= 1) {
            if (nv >= 1 && !mbar_wait(bar(kGaVEmpty), (nv - 1) & 1, s_abort, err)) { ok = false; break; }
            mbar_arrive_expect_tx(bar(kGaVFull), L::V_TILE);
            for (int c = 0; c < 2; ++c)
              tma_load_4d(sV + c * L::K_CHUNK, &tmV, bar(kGaVFull), 64 * c, g, (j - 1) * kGaBN, b);
            ++nv;
          }
        }
      }
      if (!ok) {   // let every issued copy land before the CTA can exit
        if (nq > 0) mbar_wait_drain(bar(kGaQFull), (nq - 1) & 1, err);
        for (int t = nk - 2 < 0 ? 0 : nk - 2; t < nk; ++t)
          mbar_wait_drain(bar(kGaKFull + (t & 1)), (t >> 1) & 1, err);
        if (nv > 0) mbar_wait_drain(bar(kGaVFull), (nv - 1) & 1, err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // queues: S ops (tile, group) in order A, B per tile; PV ops likewise
      int s_r = 0, s_w = work_of(0), s_it = 0, s_j = 0, s_T = 0, s_gt = 0, s_grp = 0;
      int v_r = 0, v_w = work_of(0), v_j = 0, v_T = 0, v_gt = 0, v_grp = 0;
      int b_, g_, p0_;
      bool s_done = s_w >= p.num_work, v_done = v_w >= p.num_work;
      if (!s_done) item_of(s_w, b_, g_, p0_, s_T);
      if (!v_done) item_of(v_w, b_, g_, p0_, v_T);
      bool ok = true;
      uint32_t idle = 0;
      unsigned long long t_prog = globaltimer_ns();
      while (!v_done && ok) {
        bool prog = false;
        if (!s_done) {
          bool ready = true;
          if (s_j == 0 && s_grp == 0) ready = mbar_test(bar(kGaQReady), s_it & 1);
          if (ready) ready = mbar_test(bar(kGaKReady + (s_gt & 1)), (s_gt >> 1) & 1);
          if (ready && s_gt >= 1) ready = mbar_test(bar(kGaPVDone + s_grp), (s_gt - 1) & 1);
          if (ready) {
            tc_fence_after();
            GA_TRACE(s_gt, 10 + s_grp);
            const uint32_t d = tmem + s_grp * 256;
            const uint32_t kb = sK + (s_gt & 1) * L::K_TILE;
#pragma unroll
            for (int kk = 0; kk < 12; ++kk) {
              const uint64_t a = smem_desc(sQ + s_grp * L::Q_BLOCK + (kk >> 2) * L::Q_CHUNK + (kk & 3) * 32, 16, 1024);
              const uint64_t bd = smem_desc(kb + (kk >> 2) * L::K_CHUNK + (kk & 3) * 32, 16, 1024);
              umma_ss(d, a, bd, kk * 16 < p.rot_dims ? L::IDESC_S_F16 : L::IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar(kGaSFull + s_grp));
            GA_TRACE(s_gt, s_grp);
            if (s_grp == 1) {
              umma_commit(bar(kGaKEmpty + (s_gt & 1)));
              if (s_j == s_T - 1) umma_commit(bar(kGaQEmpty));
              s_grp = 0;
              ++s_gt;
              if (++s_j == s_T) {
                s_j = 0;
                ++s_it;
                s_w = work_of(++s_r);
                s_done = s_w >= p.num_work;
                if (!s_done) item_of(s_w, b_, g_, p0_, s_T);
              }
            } else {
              s_grp = 1;
            }
            prog = true;
          }
        }
        if (v_gt < s_gt || (v_gt == s_gt && v_grp < s_grp)) {   // PV only after its S
          bool ready = mbar_test(bar(kGaPReady + v_grp), v_gt & 1);
          if (ready && v_grp == 0) ready = mbar_test(bar(kGaVFull), v_gt & 1);
          if (ready) {
            tc_fence_after();
            GA_TRACE(v_gt, 12 + v_grp);
            const uint32_t base = tmem + v_grp * 256;
#pragma unroll
            for (int s2 = 0; s2 < kGaBN / 16; ++s2) {
              const uint64_t bd = smem_desc(sV + s2 * 2048, L::K_CHUNK, 1024);
              umma_ts(base + 128, base + 8 * s2, bd, L::IDESC_PV, (v_j > 0 || s2 > 0) ? 1u : 0u);
            }
            umma_commit(bar(kGaPVDone + v_grp));
            GA_TRACE(v_gt, 2 + v_grp);
            if (v_grp == 1) {
              umma_commit(bar(kGaVEmpty));
              v_grp = 0;
              ++v_gt;
              if (++v_j == v_T) {
                v_j = 0;
                v_w = work_of(++v_r);
                v_done = v_w >= p.num_work;
                if (!v_done) item_of(v_w, b_, g_, p0_, v_T);
              }
            } else {
              v_grp = 1;
            }
            prog = true;
          }
        }
        if (prog) {
          idle = 0;
        } else if ((++idle & 1023u) == 0) {
          if (idle == 1024u) t_prog = globaltimer_ns();
          if (*s_abort) {
            ok = false;
          } else if (globaltimer_ns() - t_prog > kWaitLimitNs) {
            *s_abort = 1;
            atomicOr(err, kErrWaitTimeout);
            ok = false;
          }
        }
      }
      umma_commit(bar(kGaFinal));
      mbar_wait_drain(bar(kGaFinal), 0, err);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ RoPE group
    const int ctid = threadIdx.x - 64;
    auto wait_all = [&](uint32_t b_, uint32_t par) -> bool {
      const bool w_ok = mbar_wait(b_, par, s_abort, err);
      return __all_sync(0xffffffffu, w_ok);
    };
    // (cos, sin)(t w_k) of this thread's K tile row t = ctid, kept in registers
    float oc[32], os[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      oc[k] = 1.f;
      os[k] = 0.f;
      if (k < half) {
        const double ang = static_cast<double>(ctid) * s_invf[k];
        const double nrev = rint(ang * 0.15915494309189535);
        sincosf(static_cast<float>(fma(-nrev, 6.283185307179586, ang)), &os[k], &oc[k]);
      }
    }
    int it = 0, gt = 0;
    bool ok = true;
    for (int rd = 0, w = work_of(0); w < p.num_work && ok; w = work_of(++rd), ++it) {
      int b, g, p0, T;
      item_of(w, b, g, p0, T);
      // Q of both blocks: rows ctid (block A) and ctid (block B), fp64-reduced angles
      if (!wait_all(bar(kGaQFull), it & 1)) { ok = false; break; }
      if (half > 0) {
        for (int blk = 0; blk < 2; ++blk) {
          const int qi = p0 + blk * P + ctid / G;
          if (qi < p.n)
            rope_row(sQ + blk * L::Q_BLOCK, L::Q_CHUNK, ctid, p.q_off + qi, p.rot_dims, s_invf);
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(bar(kGaQReady));
      for (int j = 0; j < T; ++j, ++gt) {
        const int ks = gt & 1;
        const int kt0 = j * kGaBN;
        if (half > 0) {
          // base (cos, sin)(kt0 w_k) of this tile, by the first warp. Four buffers: a warp
          // that writes the table of tile t has seen K tile t-1 land, which needs every
          // thread to have finished tile t-3, so readers are at tile t-2 or later.
          const int tb = gt & 3;
          float2* base = s_base + tb * 32;
          if (ctid < 32) {
            if (ctid < half) {
              const double ang = static_cast<double>(kt0) * s_invf[ctid];
              const double nrev = rint(ang * 0.15915494309189535);
              float sn, cs;
              sincosf(static_cast<float>(fma(-nrev, 6.283185307179586, ang)), &sn, &cs);
              base[ctid] = make_float2(cs, sn);
            }
            mbar_arrive(bar(kGaBase + tb));
          }
          if (!wait_all(bar(kGaBase + tb), (gt >> 2) & 1)) { ok = false; break; }
          if (!wait_all(bar(kGaKFull + ks), (gt >> 1) & 1)) { ok = false; break; }
          if (kt0 + ctid < p.nk && kt0 + ctid < p.krot_from) {
            // a prefix row stored rotated (from a KV cache): only bf16 -> f16 for the f16
            // MMA k-steps over the rotated dims
            uint8_t* row = smem + L::OFF_K + ks * L::K_TILE + ctid * 128;
            for (int u = 0; u < (half >> 2); ++u) {
              uint4* px = reinterpret_cast<uint4*>(row + ((u ^ (ctid & 7)) << 4));
              const uint4 xv = *px;
              *px = make_uint4(bf16x2_to_f16x2(xv.x), bf16x2_to_f16x2(xv.y), bf16x2_to_f16x2(xv.z),
                               bf16x2_to_f16x2(xv.w));
            }
          } else if (kt0 + ctid < p.nk) {
            // rotate row ctid of the tile: angle (kt0 + t) w_k from base_k and own_k
            uint8_t* row = smem + L::OFF_K + ks * L::K_TILE + ctid * 128;
            const int nun = half >> 3;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (u < nun) {
                uint4* px = reinterpret_cast<uint4*>(row + ((u ^ (ctid & 7)) << 4));
                uint4* py = reinterpret_cast<uint4*>(row + (((u + nun) ^ (ctid & 7)) << 4));
                const uint4 xv = *px, yv = *py;
                uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, ys[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                  float r1[2], r2[2];
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const int k = u * 8 + e2 * 2 + h;
                    const float2 bs = base[k];
                    const float c = bs.x * oc[k] - bs.y * os[k];
                    const float sn = bs.y * oc[k] + bs.x * os[k];
                    const float x1 = h ? bf16_hi(xs[e2]) : bf16_lo(xs[e2]);
                    const float x2 = h ? bf16_hi(ys[e2]) : bf16_lo(ys[e2]);
                    r1[h] = x1 * c - x2 * sn;
                    r2[h] = x2 * c + x1 * sn;
                  }
                  xs[e2] = pack_f16_sat(r1[0], r1[1]);
                  ys[e2] = pack_f16_sat(r2[0], r2[1]);
                }
                *px = make_uint4(xs[0], xs[1], xs[2], xs[3]);
                *py = make_uint4(ys[0], ys[1], ys[2], ys[3]);
              }
            }
          }
          fence_proxy_async_smem();
        } else {
          if (!wait_all(bar(kGaKFull + ks), (gt >> 1) & 1)) { ok = false; break; }
        }
        mbar_arrive(bar(kGaKReady + ks));
        if (ctid == 0) GA_TRACE(gt, 9);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax groups A, B
    const int grp = (warp - 6) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t trow = tmem + grp * 256 + (static_cast<uint32_t>(q4 * 32) << 16);
    auto wait_all = [&](uint32_t b_, uint32_t par) -> bool {
      const bool w_ok = mbar_wait(b_, par, s_abort, err);
      return __all_sync(0xffffffffu, w_ok);
    };
    int gt = 0;
    bool ok = true;
    for (int rd = 0, w = work_of(0); w < p.num_work && ok; w = work_of(++rd)) {
      int b, g, p0, T;
      item_of(w, b, g, p0, T);
      const int pmin = p.q_off + p0 + grp * P;    // first position of this row block
      const int pos = pmin + r / G;
      const int qi = pos - p.q_off;               // query row within the call
      const int hq = g * G + (r % G);
      const bool row_ok = qi < p.n;
      const float sink2 = p.sink ? p.sink[hq] * kLog2e : -INFINITY;
      float m = sink2;                             // reference max (log2 units)
      float l = p.sink ? 1.f : 0.f;
      for (int j = 0; j < T; ++j, ++gt) {
        if (!wait_all(bar(kGaSFull + grp), gt & 1)) { ok = false; break; }
        tc_fence_after();
        if (q4 == 0 && lane == 0) GA_TRACE(gt, 4 + grp);
        const int kt0 = j * kGaBN;
        const bool full = kt0 + kGaBN - 1 <= pmin;   // every key of the tile is <= every row's pos
        // pass 1: tile max of the valid keys, 64 columns per TMEM round trip
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < kGaBN; c += 64) {
          uint32_t v[64];
          tmem_ld32(trow + c, *reinterpret_cast<uint32_t(*)[32]>(v));
          tmem_ld32(trow + c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
          tmem_wait_ld();
          reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(v));
          reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(v + 32));
          if (full) {
#pragma unroll
            for (int e = 0; e < 64; e += 4) {
              mx0 = fmax3(mx0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
              mx1 = fmax3(mx1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
            }
          } else {
            const int lim = pos - kt0 - c;   // columns e <= lim are keys <= pos
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              if (e <= lim) mx0 = fmaxf(mx0, __uint_as_float(v[e]));
              if (e + 1 <= lim) mx1 = fmaxf(mx1, __uint_as_float(v[e + 1]));
            }
          }
        }
        if (q4 == 0 && lane == 0) GA_TRACE(gt, 14 + grp);
        const float tmax = fmaxf(mx0, mx1) * p.scale_log2;
        // Reference update: the first tile of a row moves it to the tile max (the dominant P
        // is then exactly 1); later tiles move it only when their max is 2^8 above it, so
        // P = 2^(a - ref) stays below 2^8 and O, l are rescaled only when the reference moves.
        const bool move = (j == 0) ? (tmax > m) : (tmax > m + 8.f);
        float alpha = 1.f;
        if (move) {
          alpha = ex2(m - tmax);                  // 0 when m = -inf
          m = tmax;
          l *= alpha;
        }
        if (j > 0 && __any_sync(0xffffffffu, move)) {   // rescale O rows (warp-collective)
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            uint32_t v[32];
            tmem_ld32(trow + 128 + c, v);
            tmem_wait_ld();
            reg_fence32(v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st16(trow + 128 + c, *reinterpret_cast<const uint32_t(*)[16]>(v));
            tmem_st16(trow + 128 + c + 16, *reinterpret_cast<const uint32_t(*)[16]>(v + 16));
          }
        }
        const float ref = m == -INFINITY ? 0.f : m;
        // pass 2: P = 2^(a - ref) (0 above the diagonal), bf16 into S columns [0, 64)
        const unsigned long long sc2 = f2_pack(p.scale_log2, p.scale_log2);
        const unsigned long long nref2 = f2_pack(-ref, -ref);
        unsigned long long sab = f2_pack(0.f, 0.f);   // row sums of even and odd columns
        auto pass2 = [&](auto masked) {
#pragma unroll 1
          for (int c = 0; c < kGaBN; c += 64) {
            uint32_t v[64];
            tmem_ld32(trow + c, *reinterpret_cast<uint32_t(*)[32]>(v));
            tmem_ld32(trow + c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
            tmem_wait_ld();
            reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(v));
            reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(v + 32));
            const int lim = pos - kt0 - c;   // columns e <= lim are keys <= pos
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t pk[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int col = 16 * q + 2 * e;
                const float2 y = f2_unpack(f2_fma(f2_bits(v[col], v[col + 1]), sc2, nref2));
                float a0 = ex2(y.x);
                float a1 = ex2(y.y);
                if (decltype(masked)::value) {
                  a0 = col <= lim ? a0 : 0.f;
                  a1 = col + 1 <= lim ? a1 : 0.f;
                }
                sab = f2_add(sab, f2_pack(a0, a1));
                pk[e] = pack_bf16(a0, a1);
              }
              tmem_st8(trow + (c >> 1) + 8 * q, pk);
            }
            if (c == 0 && q4 == 0 && lane == 0) GA_TRACE(gt, 18 + grp);
          }
        };
        if (full)
          pass2(std::false_type{});
        else
          pass2(std::true_type{});
        tmem_wait_st();
        tc_fence_before();
        if (q4 == 0 && lane == 0) GA_TRACE(gt, 6 + grp);
        mbar_arrive(bar(kGaPReady + grp));
        const float2 s2 = f2_unpack(sab);
        l += s2.x + s2.y;
      }
      if (!ok) break;
      // epilogue after the item's last PV: o = O / l, lse = (m + log2 l) ln 2
      if (!wait_all(bar(kGaPVDone + grp), (gt - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.out + ((static_cast<long long>(b) * p.n + qi) * p.Hq + hq) * 128;
#pragma unroll 1
      for (int c = 0; c < 8; c += 2) {
        uint32_t v0[16], v1[16];
        tmem_ld16(trow + 128 + c * 16, v0);
        tmem_ld16(trow + 128 + (c + 1) * 16, v1);
        tmem_wait_ld();
        if (row_ok) {
          uint32_t pk[16];
          const unsigned long long il2 = f2_pack(inv_l, inv_l);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 o0 = f2_unpack(f2_mul(f2_bits(v0[2 * e], v0[2 * e + 1]), il2));
            const float2 o1 = f2_unpack(f2_mul(f2_bits(v1[2 * e], v1[2 * e + 1]), il2));
            pk[e] = pack_bf16(o0.x, o0.y);
            pk[8 + e] = pack_bf16(o1.x, o1.y);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 16);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
          dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
        }
      }
      if (row_ok && p.lse)
        p.lse[(static_cast<long long>(b) * p.Hq + hq) * p.n + qi] =
            l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mimo
