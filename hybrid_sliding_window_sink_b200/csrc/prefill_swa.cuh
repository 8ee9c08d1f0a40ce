// prefill_swa.cuh - sm_100a prefill of an SWA layer with window W <= 129 and 8 query
// heads per KV head (the MiMo SWA layout, 64 Q / 8 KV heads, W = 128).
//
// Same math as prefill.cuh ("MiMo-V2-Flash: Hybrid Sliding Window Attention
// Architecture", §2.1 window, §4.4 sink softmax; RoPE from "...MiMo-V2.6-Flash-MOPD
// 混合SWA设计原理" §5). A row block is 16 positions x 8 heads = 128 MMA rows; its keys
// lie in the 144-key span [p0 - 128, p0 + 16) (9 units of 16 keys), so one S tile
// covers all of them and the softmax of a row block needs no rescaling across tiles.
//
// Chunked prefill: query row i of the call sits at position q_off + i (q_off a multiple of
// 16, so blocks stay on 16-key units); keys come from a prefix + the chunk (nk rows), and
// prefix rows below krot_from are stored rotated (their rotated dims only turn into f16).
//
// Layout of the work. Each persistent CTA takes a contiguous run of row blocks of the
// flattened (sequence, KV head, block) order, so consecutive blocks share 128 of their
// 144 keys. K and V live in a shared-memory ring of 11 units of 16 rows (176 rows):
// a block brings in only its 16 new key rows (one TMA box per 64-dim chunk), which are
// rotated once and then serve the next 9 blocks. The S MMA multiplies Q against the whole
// ring in slot order (N = 176, one MMA per k-step, never split at the wrap-around); the
// softmax maps each 16-column slot block to the keys it holds and masks the two slots
// outside the window (they may be refilling for later blocks; the ring starts zeroed, so
// their values are finite, and their P is exactly 0). Softmax and PV do not depend on the
// order of the keys.
//
// Roles (448 threads):
//   warp 0       TMA producer: Q row blocks (2 stages), K/V units into the ring.
//   warp 1       TMEM allocator (512 columns) and single-thread tcgen05.mma issuer, event
//                driven (issues whichever of S / PV has its inputs ready).
//   warps 2-5    RoPE group: per block, a cos/sin table of its 16 positions (double
//                precision angle reduction), RoPE of the 128 Q rows and of the block's 16
//                new K rows, V of the new unit to f16. Runs ahead of the softmax groups.
//   warps 6-9    softmax group 0 (even blocks), warps 10-13 softmax group 1 (odd blocks):
//                sink softmax from TMEM S into P, then the epilogue O / l -> bf16.
// Each softmax group owns 256 TMEM columns: S in [0, 176), overwritten in place by P
// (f16, two keys per column) in [0, 88), and O in [128, 256) (S is dead by then). The
// PV MMA takes A = P from TMEM and B = V from the ring.
// Precision: rotated Q/K dims are stored as f16 and their QK^T k-steps run as f16 MMAs
// (see prefill.cuh); P and V are f16 too (each V unit is converted in place once when it
// enters the ring; P in [0, 1] keeps 11 significant bits instead of 8). P is scaled by the
// row's largest score, so it never underflows when the sink dominates; the sink joins the
// denominator at the epilogue. Inputs must lie inside the f16 range (|x| < 65504).
#pragma once

#include "ptx.cuh"
#include "prefill.cuh"

namespace mimo {

// Optional per-phase timestamps (debug builds with -DMIMO_TRACE; compiled out otherwise).
#ifdef MIMO_TRACE
#define SWA_TRACE(tile, ev)                                                            \
  do {                                                                                 \
    if (p.trace && blockIdx.x < 8 && (tile) < 256)                                     \
      p.trace[(static_cast<size_t>(blockIdx.x) * 256 + (tile)) * 32 + (ev)] = clock64(); \
  } while (0)
#else
#define SWA_TRACE(tile, ev) \
  do {                      \
  } while (0)
#endif

constexpr int kSwaThreads = 448;
constexpr int kSwaG = 8;            // query heads per KV head
constexpr int kSwaP = 16;           // positions per row block
constexpr int kSwaUnits = 11;       // 16-row units in the ring
constexpr int kSwaR = 16 * kSwaUnits;
constexpr int kSwaWin = 9;          // units holding the 144-key span of a row block
constexpr int kSwaN = kSwaR;        // S columns: the whole ring, in slot order

struct SwaLayout {
  static constexpr int Q_CHUNK = 128 * 128;
  static constexpr int Q_STAGE = 3 * Q_CHUNK;
  static constexpr int R_CHUNK = kSwaR * 128;          // 176 rows x 64 dims
  static constexpr int UNIT_BYTES = 16 * 128;          // one unit inside one 64-dim chunk
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_STAGE;
  static constexpr int OFF_V = OFF_K + 3 * R_CHUNK;
  static constexpr int OFF_TAB = OFF_V + 2 * R_CHUNK;
  static constexpr int TAB_BYTES = kSwaP * 32 * 8;     // 16 positions x 32 frequencies x (cos, sin)
  static constexpr int OFF_MISC = OFF_TAB + 2 * TAB_BYTES;
  static constexpr int MISC_BYTES = 512 + 32 * 8;
  static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;
  static constexpr uint32_t IDESC_PV = idesc_f16kind(128, 128, 0, 1, 1);   // P and V in f16
  static constexpr uint32_t IDESC_S = idesc_bf16(128, kSwaN, 0, 0);
  static constexpr uint32_t IDESC_S_F16 = idesc_f16kind(128, kSwaN, 0, 0, 1);   // rotated dims
  static_assert(R_CHUNK % 1024 == 0, "ring chunks stay on swizzle atoms");
  static_assert(SMEM <= 232448, "shared memory budget");
};

enum : int {
  kSwQFull = 0,      // [2] Q stage landed
  kSwQEmpty = 2,     // [2] S MMA done with the Q stage
  kSwQReady = 4,     // [2] RoPE group rotated the Q stage (128 arrivals)
  kSwSFull = 6,      // [2] S tile of a softmax group ready in TMEM
  kSwPReady = 8,     // [2] P written to TMEM (128 arrivals)
  kSwPVDone = 10,    // [2] O of a softmax group ready
  kSwTmFree = 12,    // [2] softmax group read its O: its TMEM region is free (128 arrivals)
  kSwTab = 14,       // [2] RoPE group's cos/sin table written (128 arrivals)
  kSwFinal = 16,
  kSwKVFull = 17,    // [11] unit landed
  kSwKReady = 28,    // [11] unit rotated (128 arrivals)
  kSwSlotFree = 39,  // [11] last MMA reading the unit finished
  kSwNumBars = 50
};

// (x, y) <- (x cos - y sin, y cos + x sin) for two rotation pairs: xw and yw each hold two
// bf16 (dims k, k+1 of the first and of the second half), cs = (cos k, cos k+1, sin k,
// sin k+1). Packed f32x2 arithmetic, results rounded to f16 with clamping.
__device__ __forceinline__ void rot_pair(uint32_t& xw, uint32_t& yw, const float4 cs) {
  unsigned long long x, y, c, s, ys, xc, yc, xr, yr;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(xw << 16), "r"(xw & 0xFFFF0000u));
  asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "r"(yw << 16), "r"(yw & 0xFFFF0000u));
  asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(cs.x), "f"(cs.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(s) : "f"(cs.z), "f"(cs.w));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(ys) : "l"(y), "l"(s));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(xc) : "l"(x), "l"(c));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(xr) : "l"(xc), "l"(ys));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(yc) : "l"(y), "l"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(yr) : "l"(x), "l"(s), "l"(yc));
  float a0, a1, b0, b1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(xr));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(yr));
  xw = pack_f16_sat(a0, a1);
  yw = pack_f16_sat(b0, b1);
}

// Rotates dims [0, 16 * nun) (nun <= 4, i.e. rot_dims <= 64, all in the first 64-dim
// chunk) of one tile row with its table row (float4 per two dims, see rot_pair). Two unit
// pairs at a time: loads first, then the math, then the stores, as plain shared-memory
// accesses.
__device__ __forceinline__ void rope_half(uint8_t* row_base, int row, int nun, const float4* t4,
                                          int ubeg) {
  uint4 x[2], y[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int u = ubeg + q;
    if (u < nun) {
      x[q] = *reinterpret_cast<const uint4*>(row_base + ((u ^ (row & 7)) << 4));
      y[q] = *reinterpret_cast<const uint4*>(row_base + (((u + nun) ^ (row & 7)) << 4));
    }
  }
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int u = ubeg + q;
    if (u < nun) {
      uint32_t xs[4] = {x[q].x, x[q].y, x[q].z, x[q].w};
      uint32_t ys[4] = {y[q].x, y[q].y, y[q].z, y[q].w};
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) rot_pair(xs[e2], ys[e2], t4[u * 4 + e2]);   // k = 8u + 2e2
      *reinterpret_cast<uint4*>(row_base + ((u ^ (row & 7)) << 4)) =
          make_uint4(xs[0], xs[1], xs[2], xs[3]);
      *reinterpret_cast<uint4*>(row_base + (((u + nun) ^ (row & 7)) << 4)) =
          make_uint4(ys[0], ys[1], ys[2], ys[3]);
    }
  }
}

// Rotates one 8-dim unit u (< nun) of the first half of a tile row and its partner u + nun.
__device__ __forceinline__ void rope_unit(uint8_t* row_base, int row, int nun, const float4* t4, int u) {
  uint4* px = reinterpret_cast<uint4*>(row_base + ((u ^ (row & 7)) << 4));
  uint4* py = reinterpret_cast<uint4*>(row_base + (((u + nun) ^ (row & 7)) << 4));
  const uint4 x = *px, y = *py;
  uint32_t xs[4] = {x.x, x.y, x.z, x.w};
  uint32_t ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int e2 = 0; e2 < 4; ++e2) rot_pair(xs[e2], ys[e2], t4[u * 4 + e2]);
  *px = make_uint4(xs[0], xs[1], xs[2], xs[3]);
  *py = make_uint4(ys[0], ys[1], ys[2], ys[3]);
}

__device__ __forceinline__ void rope_row_tab(uint8_t* row_base, int row, int nun, const float4* t4) {
  rope_half(row_base, row, nun, t4, 0);
  rope_half(row_base, row, nun, t4, 2);
}

__global__ void __launch_bounds__(kSwaThreads, 1)
    prefill_swa_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using L = SwaLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::OFF_Q;
  const uint32_t sK = sbase + L::OFF_K;
  const uint32_t sV = sbase + L::OFF_V;
  const uint32_t sBar = sbase + L::OFF_MISC;
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8 * kSwNumBars);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC + 8 * kSwNumBars + 4);
  double* s_invf = reinterpret_cast<double*>(smem + L::OFF_MISC + 512);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned* err = p.err;
  const int half = p.rot_dims >> 1;   // <= 32

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSwNumBars; ++i) {
      const bool many = (i >= kSwQReady && i < kSwQReady + 2) || (i >= kSwPReady && i < kSwPReady + 2) ||
                        (i >= kSwTmFree && i < kSwTab + 2) ||
                        (i >= kSwKReady && i < kSwKReady + kSwaUnits);
      mbar_init(bar(i), many ? 128u : 1u);
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
  // the ring starts zeroed: slots outside a window are read (masked) before they are filled
  for (int o = threadIdx.x * 16; o < 3 * L::R_CHUNK + 2 * L::R_CHUNK; o += kSwaThreads * 16)
    *reinterpret_cast<uint4*>(smem + L::OFF_K + o) = make_uint4(0u, 0u, 0u, 0u);
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

  // this CTA's contiguous run [f0, f1) of the flattened (b, g, block) order
  const long long F = static_cast<long long>(p.num_work);
  const long long f0 = F * blockIdx.x / gridDim.x;
  const long long f1 = F * (blockIdx.x + 1) / gridDim.x;
  const int nqt = p.n_qtiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int seq = 0, nq = 0;
      bool ok = true;
      auto load_unit = [&](int b, int g, int u) -> bool {
        const int slot = seq % kSwaUnits;
        if (seq >= kSwaUnits &&
            !mbar_wait(bar(kSwSlotFree + slot), ((seq / kSwaUnits) - 1) & 1, s_abort, err))
          return false;
        mbar_arrive_expect_tx(bar(kSwKVFull + slot), 16 * (kDQK + kDV) * 2);
        for (int c = 0; c < 3; ++c)
          tma_load_4d(sK + c * L::R_CHUNK + slot * L::UNIT_BYTES, &tmK, bar(kSwKVFull + slot),
                      64 * c, g, 16 * u, b);
        for (int c = 0; c < 2; ++c)
          tma_load_4d(sV + c * L::R_CHUNK + slot * L::UNIT_BYTES, &tmV, bar(kSwKVFull + slot),
                      64 * c, g, 16 * u, b);
        ++seq;
        return true;
      };
      for (long long f = f0; f < f1 && ok; ++f) {
        const int bg = static_cast<int>(f / nqt), t = static_cast<int>(f % nqt);
        const int b = bg / p.Hkv, g = bg - b * p.Hkv;
        const int ua = t + (p.q_off >> 4);   // K/V unit holding the block's own positions
        if (f == f0 || t == 0)
          for (int u = ua - 8; u < ua && ok; ++u) ok = load_unit(b, g, u);
        if (!ok) break;
        const int st = nq & 1;
        if (nq >= 2 && !mbar_wait(bar(kSwQEmpty + st), ((nq >> 1) - 1) & 1, s_abort, err)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(kSwQFull + st), L::Q_STAGE);
        for (int c = 0; c < 3; ++c)
          tma_load_4d(sQ + st * L::Q_STAGE + c * L::Q_CHUNK, &tmQ, bar(kSwQFull + st), 64 * c,
                      g * kSwaG, t * kSwaP, b);
        SWA_TRACE(nq, 9);
        ++nq;
        ok = load_unit(b, g, ua);
      }
      if (!ok) {   // let every issued copy land before the CTA can exit
        for (int s = seq - kSwaUnits < 0 ? 0 : seq - kSwaUnits; s < seq; ++s)
          mbar_wait_drain(bar(kSwKVFull + s % kSwaUnits), (s / kSwaUnits) & 1, err);
        for (int i = nq - 2 < 0 ? 0 : nq - 2; i < nq; ++i)
          mbar_wait_drain(bar(kSwQFull + (i & 1)), (i >> 1) & 1, err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const int ntiles = static_cast<int>(f1 - f0);
      int ns = 0, npv = 0, seq = 0;
      int useq_of[4] = {0, 0, 0, 0};
      bool last_of[4] = {false, false, false, false};
      int s_useq = 0, kwait = 0;
      bool s_last = false, s_q = false, s_free = false, ok = true;
      auto prep_s = [&]() {
        const long long f = f0 + ns;
        const int t = static_cast<int>(f % nqt);
        const bool first = (ns == 0 || t == 0);
        s_last = (f == f1 - 1 || t == nqt - 1);
        if (first) seq += 8;
        s_useq = seq++;
        kwait = first ? s_useq - 8 : s_useq;
        s_q = false;
        s_free = ns < 2;
      };
      if (ntiles > 0) prep_s();
      unsigned long long t_prog = globaltimer_ns();
      uint32_t idle = 0;
      while (npv < ntiles && ok) {
        bool prog = false;
        if (ns < ntiles) {
          const int wg = ns & 1;
          if (!s_q) s_q = mbar_test(bar(kSwQReady + wg), (ns >> 1) & 1);
          if (!s_free) s_free = mbar_test(bar(kSwTmFree + wg), ((ns >> 1) - 1) & 1);
          while (s_q && kwait <= s_useq &&
                 mbar_test(bar(kSwKReady + kwait % kSwaUnits), (kwait / kSwaUnits) & 1))
            ++kwait;
          if (s_q && s_free && kwait > s_useq) {
            SWA_TRACE(ns, 17);
            tc_fence_after();
            const uint32_t d = tmem + wg * 256;
#pragma unroll
            for (int kk = 0; kk < 12; ++kk) {
              const uint64_t a =
                  smem_desc(sQ + wg * L::Q_STAGE + (kk >> 2) * L::Q_CHUNK + (kk & 3) * 32, 16, 1024);
              const uint64_t bd = smem_desc(sK + (kk >> 2) * L::R_CHUNK + (kk & 3) * 32, 16, 1024);
              umma_ss(d, a, bd, kk * 16 < p.rot_dims ? L::IDESC_S_F16 : L::IDESC_S, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar(kSwQEmpty + wg));
            umma_commit(bar(kSwSFull + wg));
            SWA_TRACE(ns, 7);
            useq_of[ns & 3] = s_useq;
            last_of[ns & 3] = s_last;
            ++ns;
            if (ns < ntiles) prep_s();
            prog = true;
          }
        }
        if (npv < ns) {
          const int wg = npv & 1;
          if (mbar_test(bar(kSwPReady + wg), (npv >> 1) & 1)) {
            SWA_TRACE(npv, 18);
            tc_fence_after();
            const int uq = useq_of[npv & 3];
            const uint32_t base = tmem + wg * 256;
#pragma unroll
            for (int s2 = 0; s2 < kSwaUnits; ++s2) {
              const uint64_t bd = smem_desc(sV + s2 * L::UNIT_BYTES, L::R_CHUNK, 1024);
              umma_ts(base + 128, base + 8 * s2, bd, L::IDESC_PV, s2 > 0 ? 1u : 0u);
            }
            umma_commit(bar(kSwPVDone + wg));
            umma_commit(bar(kSwSlotFree + (uq - 8) % kSwaUnits));
            if (last_of[npv & 3])
              for (int s2 = 1; s2 < kSwaWin; ++s2)
                umma_commit(bar(kSwSlotFree + (uq - 8 + s2) % kSwaUnits));
            SWA_TRACE(npv, 8);
            ++npv;
            prog = true;
          }
        }
        if (prog) {
          idle = 0;
        } else if ((++idle & 1023u) == 0) {   // look at the clock only now and then
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
      umma_commit(bar(kSwFinal));
      mbar_wait_drain(bar(kSwFinal), 0, err);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ RoPE group
    const int ctid = threadIdx.x - 64;             // 0..127, also the Q row it rotates
    const int nun = p.rot_dims >> 4;
    auto wait_all = [&](uint32_t b_, uint32_t par) -> bool {
      const bool w_ok = mbar_wait(b_, par, s_abort, err);
      return __all_sync(0xffffffffu, w_ok);
    };
    int seq = 0, i = 0;
    for (long long f = f0; f < f1; ++f, ++i) {
      const int t = static_cast<int>(f % nqt);
      const bool first = (f == f0 || t == 0);
      if (first) seq += 8;
      const int useq = seq++;
      const int p0 = p.q_off + t * kSwaP;            // absolute position of the block
      float* tab = reinterpret_cast<float*>(smem + L::OFF_TAB + (i & 1) * L::TAB_BYTES);
      if (ctid == 0) SWA_TRACE(i, 0);
      // (cos, sin) of the block's 16 positions (double buffered: tile i - 1 may still read)
      if (half > 0) {
        for (int e = ctid; e < kSwaP * half; e += 128) {
          const int pp = e / half, k = e - pp * half;
          const double ang = static_cast<double>(p0 + pp) * s_invf[k];
          const double nrev = rint(ang * 0.15915494309189535);
          float sn, cs;
          __sincosf(static_cast<float>(fma(-nrev, 6.283185307179586, ang)), &sn, &cs);
          float* tk = tab + pp * 64 + (k >> 1) * 4 + (k & 1);   // (cos k, cos k+1, sin k, sin k+1)
          tk[0] = cs;
          tk[2] = sn;
        }
        mbar_arrive(bar(kSwTab + (i & 1)));   // (bounded waits only: no hardware named barrier)
        if (!wait_all(bar(kSwTab + (i & 1)), (i >> 1) & 1)) break;
      }
      if (!wait_all(bar(kSwQFull + (i & 1)), (i >> 1) & 1)) break;
      if (ctid == 0) SWA_TRACE(i, 1);
      if (half > 0 && t * kSwaP + (ctid >> 3) < p.n)
        rope_row_tab(smem + L::OFF_Q + (i & 1) * L::Q_STAGE + ctid * 128, ctid, nun,
                     reinterpret_cast<const float4*>(tab + (ctid >> 3) * 64));
      // K units of this block: the new one, or the whole window at the start of a run
      bool ok = true;
      const int s_first = first ? useq - 8 : useq;
      for (int s = s_first; s <= useq && ok; ++s) ok = wait_all(bar(kSwKVFull + s % kSwaUnits), (s / kSwaUnits) & 1);
      if (!ok) break;
      for (int s = s_first; s <= useq; ++s) {   // V units entering the ring: bf16 -> f16 in place
        uint8_t* vb = smem + L::OFF_V + (s % kSwaUnits) * L::UNIT_BYTES;
        uint4 xv[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
          xv[h2] = *reinterpret_cast<const uint4*>(vb + h2 * L::R_CHUNK + ctid * 16);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2)
          *reinterpret_cast<uint4*>(vb + h2 * L::R_CHUNK + ctid * 16) =
              make_uint4(bf16x2_to_f16x2(xv[h2].x), bf16x2_to_f16x2(xv[h2].y),
                         bf16x2_to_f16x2(xv[h2].z), bf16x2_to_f16x2(xv[h2].w));
      }
      if (half > 0) {
        if (first) {
          for (int rr = ctid; rr < 16 * kSwaWin; rr += 128) {
            const int kpos = p0 - 128 + rr;
            const int ring_row = ((s_first + rr / 16) % kSwaUnits) * 16 + (rr & 15);
            if (kpos >= p.krot_from && kpos < p.nk) rope_row(sK, L::R_CHUNK, ring_row, kpos, p.rot_dims, s_invf);
            else if (kpos >= 0 && kpos < p.krot_from) f16_row(sK, L::R_CHUNK, ring_row, p.rot_dims);
          }
        } else if (ctid < 64) {   // the 16 new K rows, one (row, unit pair) per thread
          const int rr = ctid >> 2, u = ctid & 3;
          const int ring_row = (useq % kSwaUnits) * 16 + rr;
          if (u < nun && p0 + rr < p.nk)   // a block's own keys lie in the chunk: never stored rotated
            rope_unit(smem + L::OFF_K + ring_row * 128, ring_row, nun,
                      reinterpret_cast<const float4*>(tab + rr * 64), u);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(kSwQReady + (i & 1)));
      for (int s = s_first; s <= useq; ++s) mbar_arrive(bar(kSwKReady + s % kSwaUnits));
      if (lane == 0) SWA_TRACE(i, 21 + (ctid >> 5));
    }
  } else {
    // ------------------------------------------------------------ softmax groups
    const int w = (warp - 6) >> 2;                 // group 0 or 1
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                  // row == TMEM lane
    const int ctid = (warp - 6 - 4 * w) * 32 + lane;
    const int pl = r >> 3, hl = r & 7;
    const uint32_t trow = tmem + w * 256 + (static_cast<uint32_t>(q4 * 32) << 16);
    auto wait_all = [&](uint32_t b_, uint32_t par) -> bool {
      const bool w_ok = mbar_wait(b_, par, s_abort, err);
      return __all_sync(0xffffffffu, w_ok);
    };
    int seq = 0, i = 0;
    for (long long f = f0; f < f1; ++f, ++i) {
      const int bg = static_cast<int>(f / nqt), t = static_cast<int>(f % nqt);
      const bool first = (f == f0 || t == 0);
      if (first) seq += 8;
      const int useq = seq++;
      if ((i & 1) != w) continue;
      const int b = bg / p.Hkv, g = bg - b * p.Hkv;
      const int qi = t * kSwaP + pl;                 // query row within the call
      const int p0 = p.q_off + t * kSwaP;            // absolute positions
      const int pos = p.q_off + qi;
      const int hq = g * kSwaG + hl;
      const bool row_ok = qi < p.n;

      // Softmax over the row block's keys, two passes over TMEM. Slot block c (columns
      // 16c..16c+15) holds the unit d = (useq - c) mod 11 blocks back: keys kb + e with
      // kb = p0 - 16 d. A block is empty, full or partial for every row of the tile alike
      // (the class depends on p0, W and d only); only partial blocks mask per element.
      const float sink2 = p.sink ? p.sink[hq] * kLog2e : -INFINITY;
      const int klo = max(0, pos - p.window + 1);          // valid keys of this row: [klo, pos]
      const int klo_min = max(0, p0 - p.window + 1);       // over the tile's rows
      const int klo_max = max(0, p0 + kSwaP - 1 - p.window + 1);
      const int um = useq % kSwaUnits;
      // 0 = empty, 1 = partial, 2 = full; elo/ehi: valid e of this row (partial blocks)
      auto block_class = [&](int c, int& elo, int& ehi) -> int {
        int d = um - c;
        d += d < 0 ? kSwaUnits : 0;
        const int kb = p0 - 16 * d;
        elo = max(klo - kb, 0);
        ehi = min(pos - kb, 15);
        if (d >= kSwaWin || kb + 15 < klo_min || kb > p0 + kSwaP - 1) return 0;
        return (kb >= klo_max && kb + 15 <= p0) ? 2 : 1;
      };
      if (!wait_all(bar(kSwSFull + w), (i >> 1) & 1)) break;
      tc_fence_after();
      if (ctid == 0) SWA_TRACE(i, 3);
      // pass 1: row max over the valid keys (four slot blocks per TMEM round trip)
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < kSwaUnits; c += 2) {
        uint32_t v[2][16];
        int elo[2], ehi[2], k[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          k[q] = c + q < kSwaUnits ? block_class(c + q, elo[q], ehi[q]) : 0;
          if (k[q]) tmem_ld16(trow + (c + q) * 16, v[q]);
        }
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float mq = -INFINITY;
          if (k[q] == 2) {
            float mb = -INFINITY;
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              mq = fmax3_v(mq, __uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1]));
              mb = fmax3_v(mb, __uint_as_float(v[q][e + 2]), __uint_as_float(v[q][e + 3]));
            }
            mq = fmaxf(mq, mb);
          } else if (k[q] == 1) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (e >= elo[q] && e <= ehi[q]) mq = fmaxf(mq, __uint_as_float(v[q][e]));
          }
          if (q & 1) mx1 = fmaxf(mx1, mq); else mx0 = fmaxf(mx0, mq);
        }
      }
      const float mx = fmaxf(mx0, mx1);
      const float amax = mx * p.scale_log2;                 // -inf when the row has no key
      const float ref = amax == -INFINITY ? 0.f : amax;
      // pass 2: P = exp2(a - amax) (0 outside the window), packed f16 into the S columns
      float sum0 = 0.f, sum1 = 0.f;
      // P of one slot block into pk; returns its sum
      const unsigned long long sc2 = f2_pack(p.scale_log2, p.scale_log2), nref2 = f2_pack(-ref, -ref);
      auto p_block = [&](const uint32_t (&v)[16], int k, int elo, int ehi, uint32_t (&pk)[8]) -> float {
        if (k == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = 0u;
          return 0.f;
        }
        unsigned long long acc = f2_pack(0.f, 0.f);   // even and odd columns
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 y = f2_unpack(f2_fma(f2_bits(v[2 * e], v[2 * e + 1]), sc2, nref2));
          float a0 = ex2(y.x);
          float a1 = ex2(y.y);
          if (k == 1) {
            a0 = (2 * e >= elo && 2 * e <= ehi) ? a0 : 0.f;
            a1 = (2 * e + 1 >= elo && 2 * e + 1 <= ehi) ? a1 : 0.f;
          }
          acc = f2_add(acc, f2_pack(a0, a1));
          pk[e] = pack_f16(a0, a1);
        }
        const float2 sab = f2_unpack(acc);
        return sab.x + sab.y;
      };
#pragma unroll 1
      for (int c = 0; c < kSwaUnits; c += 2) {
        uint32_t v[2][16];
        int elo[2], ehi[2], k[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          k[q] = c + q < kSwaUnits ? block_class(c + q, elo[q], ehi[q]) : 0;
          if (k[q]) tmem_ld16(trow + (c + q) * 16, v[q]);
        }
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          if (c + q < kSwaUnits) {
            uint32_t pk[8];
            const float sq = p_block(v[q], k[q], elo[q], ehi[q], pk);
            if (q & 1) sum1 += sq; else sum0 += sq;
            tmem_st8(trow + (c + q) * 8, pk);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kSwPReady + w));
      if (lane == 0) SWA_TRACE(i, 25 + (ctid >> 5));
      const float sum = sum0 + sum1;
      // denominator with the sink: M = max(amax, sink); l = sum 2^(amax-M) + 2^(sink-M)
      const float M = fmaxf(ref, sink2);
      const float sc = ex2(ref - M);
      const float lt = sum * sc + (p.sink ? ex2(sink2 - M) : 0.f);

      // epilogue: o = O sc / lt -> bf16, lse = (M + log2 lt) ln 2
      if (!wait_all(bar(kSwPVDone + w), (i >> 1) & 1)) break;
      tc_fence_after();
      if (ctid == 0) SWA_TRACE(i, 5);
      const float inv_l = lt > 0.f ? sc / lt : 0.f;
      __nv_bfloat16* orow = p.out + ((static_cast<long long>(b) * p.n + qi) * p.Hq + hq) * 128;
      // O columns [128, 192) overlap the S columns of this group's next tile: read them
      // first, release the TMEM region, then finish with columns [192, 256)
#pragma unroll 1
      for (int hh = 0; hh < 4; ++hh) {
        uint32_t v[2][16];
#pragma unroll
        for (int q = 0; q < 2; ++q) tmem_ld16(trow + 128 + (2 * hh + q) * 16, v[q]);
        tmem_wait_ld();
        if (hh == 1) {
          tc_fence_before();
          mbar_arrive(bar(kSwTmFree + w));
        }
        if (row_ok) {
          const unsigned long long il2 = f2_pack(inv_l, inv_l);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 o = f2_unpack(f2_mul(f2_bits(v[q][2 * e], v[q][2 * e + 1]), il2));
              pk[e] = pack_bf16(o.x, o.y);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + (2 * hh + q) * 16);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      if (row_ok && p.lse)
        p.lse[(static_cast<long long>(b) * p.Hq + hq) * p.n + qi] =
            lt > 0.f ? (M + log2f(lt)) * kLn2 : -INFINITY;
      if (ctid == 0) SWA_TRACE(i, 6);
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
