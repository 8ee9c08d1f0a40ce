// decode_mq_tma.cuh - multi-query decode (MTP draft verification) over a linear (GA) cache with
// both products on the 5th-generation tensor cores.
//
// Math, key sets and the chunk / combine split are those of decode_mq.cuh: draft token t of
// sequence b sits at position p_t = L - T + t and attends the keys [0, p_t] of the GA pool with
// the attention sink of "MiMo-V2-Flash: Hybrid Sliding Window Attention Architecture" §4.4; the
// MTP section of the syt-nju "mimo-mtp-swa-not-mla" page has the main model verify the draft
// tokens in one pass.
//
// Design. One CTA per (sequence, KV head, chunk of keys); the T*G (draft token, head) rows,
// zero-padded to 64, are the M = 64 rows of every MMA. Six warps:
//  * warp 4, the producer: K and V of each 64-key subtile by TMA (three 64-dim K slabs and two
//    64-dim V slabs, 128-byte swizzle: the K-major B operand of S and the MN-major B operand of
//    PV), four subtiles in flight.
//  * warp 5, the MMA issuer (and TMEM allocator): S_j = Q K_j^T (N = 64, K = 192) into one of
//    two TMEM buffers, O += P_j V_j (N = 128, K = 64) with P from shared memory and O in TMEM.
//    Once P_j is written it issues PV_j and S_{j+2} together (one fence, one commit), so the
//    tensor core computes those while the warps take the softmax of subtile j + 1.
//  * warps 0-3, the softmax: with M = 64 row r of an accumulator sits in TMEM lane
//    32 (r / 16) + r % 16, so warp w owns rows 16 w .. 16 w + 15 and reads them with
//    tcgen05.ld.16x256b (rows gq and gq + 8 of each thread, columns 2 tq, 2 tq + 1 of every 8).
//    It masks each row to [0, p_t], keeps a lazy reference max (moved only when a subtile's max
//    exceeds it by 2^8, then it rescales its own rows of O in TMEM after the previous PV has
//    completed), writes P = 2^(a - ref) as bf16 into the 128-byte-swizzled K-major A operand in
//    shared memory, and sums the unrounded P in fp32.
// Keys past the chunk or the cache end: their scores are masked; their V rows (whatever the
// cache holds there) are zeroed in shared memory before PV reads them, so 0 * V stays 0.
// Every wait is bounded; on a time-out all roles leave their loops, the producer waits for its
// copies, the issuer for its MMAs, TMEM is freed and the CTA returns without writing.
#pragma once

#include "ptx.cuh"
#include "decode.cuh"
#include "decode_mq.cuh"

namespace mimo {

// Optional per-subtile timestamps (debug builds with -DMIMO_TRACE; compiled out otherwise), for
// the first chunk of KV head 0 of sequences 0-7: events 0 S issued, 1 PV issued, 2 S seen by the
// softmax, 3 P written, 4 K/V subtile loads issued.
#ifdef MIMO_TRACE
#define MT_TRACE(sub, ev)                                                                       \
  do {                                                                                          \
    if (p.trace && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z < 8 && (sub) < 256)         \
      p.trace[(static_cast<size_t>(blockIdx.z) * 256 + (sub)) * 32 + (ev)] = clock64();         \
  } while (0)
#else
#define MT_TRACE(sub, ev) \
  do {                    \
  } while (0)
#endif

constexpr int kMtThreads = 192;
constexpr int kMtKeys = 64;                                   // keys per subtile
constexpr int kMtStages = 4;                                  // K/V subtiles in flight
constexpr int kMtSlab = kMtKeys * 128;                        // 64 rows x 64 bf16 (8 KB)
constexpr int kMtQBytes = 3 * kMtSlab;                        // Q: 64 rows x 192
constexpr int kMtKBytes = 3 * kMtSlab;                        // K subtile: 64 keys x 192
constexpr int kMtVBytes = 2 * kMtSlab;                        // V subtile: 64 keys x 128
constexpr int kMtOffK = kMtQBytes;
constexpr int kMtOffV = kMtOffK + kMtStages * kMtKBytes;
constexpr int kMtOffP = kMtOffV + kMtStages * kMtVBytes;      // two P buffers, 64 rows x 64 keys
constexpr int kMtOffMisc = kMtOffP + 2 * kMtSlab;
constexpr int kMtSmemBytes = kMtOffMisc + 256 + 1024;         // + room to align the base to 1024
constexpr int kMtTmemCols = 256;                              // S buffers [0, 128), O [128, 256)
constexpr uint32_t kMtIdescS = idesc_bf16(64, kMtKeys, 0, 0);
constexpr uint32_t kMtIdescPV = idesc_bf16(64, kDV, 0, 1);

enum : int {
  kMtKVFull = 0,                      // [4] K and V of a subtile landed
  kMtKVEmpty = kMtKVFull + kMtStages, // [4] PV of that subtile done: the stage is free
  kMtDone = kMtKVEmpty + kMtStages,   // [4] batch j (PV_j, S_{j+2}) done, in barrier j % 4
  kMtInit = kMtDone + kMtStages,      // S_0 and S_1 done
  kMtPReady = kMtInit + 1,            // [2] P written (128 arrivals): S buffer read, P buffer full
  kMtFinal = kMtPReady + 2,
  kMtNumBars = kMtFinal + 1
};

// 16 TMEM lanes x 256 bits, eight times along the columns: r[4 n .. 4 n + 3] hold lanes
// base + gq and base + gq + 8, columns 8 n + 2 tq and 8 n + 2 tq + 1.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_16x256b_x8(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

template <int G>
__global__ void __launch_bounds__(kMtThreads, 1)
    decode_mq_tma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const DecodeMqParams p) {
  static_assert(G >= 1 && G <= 16, "group size");
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = p.T * G;

  int klo;
  const int L = mq_range(p, b, klo);
  const int nkeys = L - klo > 0 ? L - klo : 0;
  const int k_begin = c * p.chunk;
  if (k_begin >= nkeys && !p.direct) return;   // empty chunk: the combine skips it
  int n_here = nkeys - k_begin;
  n_here = n_here < 0 ? 0 : (n_here < p.chunk ? n_here : p.chunk);
  const int tok0 = klo + k_begin;                // token (= cache slot) of key 0 of this chunk
  const int nsub = (n_here + kMtKeys - 1) / kMtKeys;

  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase, sK = sbase + kMtOffK, sV = sbase + kMtOffV, sP = sbase + kMtOffP;
  auto bar = [&](int i) -> uint32_t { return sbase + kMtOffMisc + 8u * static_cast<uint32_t>(i); };
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kMtOffMisc + 8 * kMtNumBars);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kMtOffMisc + 8 * kMtNumBars + 4);
  unsigned* err = p.err;

  if (tid == 0) {
    for (int i = 0; i < kMtNumBars; ++i) mbar_init(bar(i), (i == kMtPReady || i == kMtPReady + 1) ? 128u : 1u);
    *s_abort = 0;
    mbar_fence_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(s_tmem), kMtTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  // Q rows r = t G + h (zero beyond R) into three swizzled 64-dim slabs
  for (int idx = tid; idx < 64 * 24; idx += kMtThreads) {
    const int r = idx / 24, u = idx - r * 24;
    const bool ok = r < R;
    const int t = ok ? r / G : 0, hh = ok ? r - t * G : 0;
    const __nv_bfloat16* src = p.q + ((static_cast<long long>(b) * p.T + t) * p.Hq + g * G + hh) * kDQK + u * 8;
    cp_async16(sQ + (u >> 3) * kMtSlab + r * 128 + (((u & 7) ^ (r & 7)) << 4), src, ok ? 16u : 0u);
  }
  cp_async_commit();
  cp_async_wait<0>();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int j = 0;
      bool ok = true;
      for (; j < nsub; ++j) {
        const int s = j % kMtStages;
        if (j >= kMtStages && !mbar_wait(bar(kMtKVEmpty + s), ((j / kMtStages) - 1) & 1, s_abort, err)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(kMtKVFull + s), kMtKBytes + kMtVBytes);
        const int key0 = tok0 + j * kMtKeys;
        for (int cc = 0; cc < 3; ++cc)
          tma_load_4d(sK + s * kMtKBytes + cc * kMtSlab, &tmK, bar(kMtKVFull + s), 64 * cc, g, key0, b);
        for (int cc = 0; cc < 2; ++cc)
          tma_load_4d(sV + s * kMtVBytes + cc * kMtSlab, &tmV, bar(kMtKVFull + s), 64 * cc, g, key0, b);
        MT_TRACE(j, 4);
      }
      if (!ok)   // let every issued copy land before the CTA can exit
        for (int t = j - kMtStages < 0 ? 0 : j - kMtStages; t < j; ++t)
          mbar_wait_drain(bar(kMtKVFull + t % kMtStages), (t / kMtStages) & 1, err);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    // Batches: S_0 and S_1 first; then, once P_j is written, batch j = PV_j and S_{j+2} (which
    // overwrites the S buffer P_j was taken from) under one fence. A tcgen05 fence or commit
    // between two MMAs makes the issuing thread wait for the MMAs in flight, so a batch holds
    // one commit besides its last: after PV_j, which frees the K/V stage for the producer.
    if (lane == 0) {
      bool ok = true;
      auto wait = [&](int i, int par) {
        if (ok && !mbar_wait(bar(i), static_cast<uint32_t>(par & 1), s_abort, err)) ok = false;
      };
      auto issue_s = [&](int j) {
        const uint32_t kb = sK + (j % kMtStages) * kMtKBytes;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const uint64_t a = smem_desc(sQ + (kk >> 2) * kMtSlab + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc(kb + (kk >> 2) * kMtSlab + (kk & 3) * 32, 16, 1024);
          umma_ss(tmem + (j & 1) * kMtKeys, a, bd, kMtIdescS, kk > 0 ? 1u : 0u);
        }
        MT_TRACE(j, 0);
      };
      auto issue_pv = [&](int j) {
        const uint32_t pb = sP + (j & 1) * kMtSlab, vb = sV + (j % kMtStages) * kMtVBytes;
#pragma unroll
        for (int s2 = 0; s2 < kMtKeys / 16; ++s2) {
          const uint64_t a = smem_desc(pb + s2 * 32, 16, 1024);
          const uint64_t bd = smem_desc(vb + s2 * 2048, kMtSlab, 1024);
          umma_ss(tmem + 128, a, bd, kMtIdescPV, (j > 0 || s2 > 0) ? 1u : 0u);
        }
        MT_TRACE(j, 1);
      };
      if (nsub > 0) {
        wait(kMtKVFull, 0);
        if (nsub > 1) wait(kMtKVFull + 1, 0);
        if (ok) {
          tc_fence_after();
          issue_s(0);
          if (nsub > 1) issue_s(1);
          umma_commit(bar(kMtInit));
        }
      }
      for (int j = 0; j < nsub && ok; ++j) {
        wait(kMtPReady + (j & 1), j >> 1);
        if (j + 2 < nsub) wait(kMtKVFull + (j + 2) % kMtStages, (j + 2) / kMtStages);
        if (!ok) break;
        tc_fence_after();
        issue_pv(j);
        umma_commit(bar(kMtKVEmpty + j % kMtStages));   // the producer may refill the stage now
        if (j + 2 < nsub) issue_s(j + 2);
        umma_commit(bar(kMtDone + j % kMtStages));
      }
      umma_commit(bar(kMtFinal));
      mbar_wait_drain(bar(kMtFinal), 0, err);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int gq = lane >> 2, tq = lane & 3;
    const int r0 = warp * 16 + gq, r1 = r0 + 8;
    const bool ok0 = r0 < R, ok1 = r1 < R;
    const int t0 = ok0 ? r0 / G : 0, t1 = ok1 ? r1 / G : 0;
    const int h0 = g * G + (ok0 ? r0 - t0 * G : 0), h1 = g * G + (ok1 ? r1 - t1 * G : 0);
    const int hi0 = ok0 ? L - p.T + t0 : -1, hi1 = ok1 ? L - p.T + t1 : -1;   // last key token of each row
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * warp) << 16);
    auto wait_all = [&](uint32_t b_, uint32_t par) -> bool {
      const bool w_ok = mbar_wait(b_, par, s_abort, err);
      return __all_sync(0xffffffffu, w_ok);
    };
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;
    for (int j = 0; j < nsub; ++j) {
      // S_j: in the first batch for j < 2, else in batch j - 2 (which also freed P buffer j & 1)
      if (!wait_all(bar(j < 2 ? kMtInit : kMtDone + (j - 2) % kMtStages), j < 2 ? 0u : ((j - 2) / kMtStages) & 1)) {
        ok = false;
        break;
      }
      if (warp == 0 && lane == 0) MT_TRACE(j, 2);
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld_16x256b_x8(trow + (j & 1) * kMtKeys, sr);
      tmem_wait_ld();
      // mask: key k of the chunk is token tok0 + k; row limits hi0 / hi1 and the chunk end. A
      // subtile inside every row's interval (the usual case) needs no per-score test.
      const int first_tok = tok0 + j * kMtKeys;
      const int nvalid = n_here - j * kMtKeys;       // keys of this subtile inside the chunk
      const bool whole = nvalid >= kMtKeys && __all_sync(0xffffffffu, (!ok0 || first_tok + kMtKeys - 1 <= hi0) &&
                                                                         (!ok1 || first_tok + kMtKeys - 1 <= hi1));
      float s[8][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = __uint_as_float(sr[4 * n + e]) * p.scale_log2;
          if (whole) {
            s[n][e] = x;
          } else {
            const int k = n * 8 + tq * 2 + (e & 1);
            const bool in = k < nvalid && first_tok + k <= (e < 2 ? hi0 : hi1);
            s[n][e] = in ? x : -INFINITY;
          }
        }
        mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
        mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      // lazy reference: the first subtile sets it; later ones move it only when their max is
      // 2^8 above it (P then stays below 2^8), and the rows that move rescale O and l
      const bool mv0 = j == 0 ? mx0 > m0 : mx0 > m0 + 8.f;
      const bool mv1 = j == 0 ? mx1 > m1 : mx1 > m1 + 8.f;
      float a0 = 1.f, a1 = 1.f;
      if (mv0) { a0 = ex2(m0 - mx0); m0 = mx0; l0 *= a0; }
      if (mv1) { a1 = ex2(m1 - mx1); m1 = mx1; l1 *= a1; }
      if (j > 0 && __any_sync(0xffffffffu, mv0 || mv1)) {
        // O must hold the PV of subtile j - 1 first
        if (!wait_all(bar(kMtDone + (j - 1) % kMtStages), ((j - 1) / kMtStages) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t ov[32];
          tmem_ld_16x256b_x8(trow + 128 + hh * 64, ov);
          tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            ov[4 * n + 0] = __float_as_uint(__uint_as_float(ov[4 * n + 0]) * a0);
            ov[4 * n + 1] = __float_as_uint(__uint_as_float(ov[4 * n + 1]) * a0);
            ov[4 * n + 2] = __float_as_uint(__uint_as_float(ov[4 * n + 2]) * a1);
            ov[4 * n + 3] = __float_as_uint(__uint_as_float(ov[4 * n + 3]) * a1);
          }
          tmem_st_16x256b_x8(trow + 128 + hh * 64, ov);
        }
        tmem_wait_st();
      }
      const float ref0 = m0 == -INFINITY ? 0.f : m0, ref1 = m1 == -INFINITY ? 0.f : m1;
      // (the P buffer was last read by PV of subtile j - 2, in the batch waited for above)
      const uint32_t pb = sP + (j & 1) * kMtSlab;
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const float p0 = ex2(s[n][0] - ref0), p1 = ex2(s[n][1] - ref0);
        const float p2 = ex2(s[n][2] - ref1), p3 = ex2(s[n][3] - ref1);
        sum0 += p0 + p1;
        sum1 += p2 + p3;
        // rows r0 / r1 of the 128-byte-swizzled K-major A operand: keys 8 n + 2 tq, + 1
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(pb + r0 * 128 + ((n ^ (r0 & 7)) << 4) + 4 * tq),
                     "r"(pack_bf16(p0, p1)) : "memory");
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(pb + r1 * 128 + ((n ^ (r1 & 7)) << 4) + 4 * tq),
                     "r"(pack_bf16(p2, p3)) : "memory");
      }
      l0 += sum0;
      l1 += sum1;
      if (nvalid < kMtKeys) {
        // V rows past the chunk hold whatever the cache holds there: zero them (both slabs),
        // after acquiring the stage's copy directly (it cannot have been reused yet: that
        // needs the PV this subtile has not released)
        if (!wait_all(bar(kMtKVFull + j % kMtStages), (j / kMtStages) & 1)) { ok = false; break; }
        const uint32_t vb = sV + (j % kMtStages) * kMtVBytes;
        const int rows = kMtKeys - (nvalid > 0 ? nvalid : 0);
        for (int idx = warp * 32 + lane; idx < rows * 16; idx += 128) {
          const int rr = kMtKeys - rows + (idx >> 4), cc = idx & 15;
          st_shared_v4(vb + (cc >> 3) * kMtSlab + rr * 128 + ((cc & 7) << 4), 0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (warp == 0 && lane == 0) MT_TRACE(j, 3);
      mbar_arrive(bar(kMtPReady + (j & 1)));
    }
    if (ok) {
      // O after the last PV; rows past R are not written
      float o[16][4];
      if (nsub > 0) {
        if (!wait_all(bar(kMtDone + (nsub - 1) % kMtStages), ((nsub - 1) / kMtStages) & 1)) ok = false;
        tc_fence_after();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t ov[32];
          if (ok) {
            tmem_ld_16x256b_x8(trow + 128 + hh * 64, ov);
            tmem_wait_ld();
          }
#pragma unroll
          for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[hh * 8 + n][e] = ok ? __uint_as_float(ov[4 * n + e]) : 0.f;
        }
      } else {
#pragma unroll
        for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
      }
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
#pragma unroll
      for (int half = 0; half < 2 && ok; ++half) {
        const bool okr = half == 0 ? ok0 : ok1;
        if (!okr) continue;
        const int t = half == 0 ? t0 : t1, h = half == 0 ? h0 : h1;
        const float m = half == 0 ? m0 : m1, l = half == 0 ? l0 : l1;
        const long long row = (static_cast<long long>(b) * p.T + t) * p.Hq + h;
        if (p.direct) {
          const float sk = p.sink ? p.sink[h] * 1.4426950408889634f : -INFINITY;
          const float M = fmaxf(m, sk);
          const float ref = M == -INFINITY ? 0.f : M;
          const float sc = ex2(m - ref);
          const float Lt = l * sc + (p.sink ? ex2(sk - ref) : 0.f);
          const float inv = Lt > 0.f ? sc / Lt : 0.f;
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const float a = half == 0 ? o[n][0] : o[n][2], bb = half == 0 ? o[n][1] : o[n][3];
            *reinterpret_cast<uint32_t*>(p.out + row * kDV + n * 8 + tq * 2) = pack_bf16(a * inv, bb * inv);
          }
          if (tq == 0 && p.lse) p.lse[row] = Lt > 0.f ? (ref + log2f(Lt)) * 0.6931471805599453f : -INFINITY;
        } else {
          const long long slot = row * p.nchunks + c;
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const float a = half == 0 ? o[n][0] : o[n][2], bb = half == 0 ? o[n][1] : o[n][3];
            *reinterpret_cast<float2*>(p.part_o + slot * kDV + n * 8 + tq * 2) = make_float2(a, bb);
          }
          if (tq == 0) {
            p.part_ml[slot * 2 + 0] = m;
            p.part_ml[slot * 2 + 1] = l;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kMtTmemCols);
  }
}

}  // namespace mimo
