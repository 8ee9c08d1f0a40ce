// decode.cuh - one-token decode over a KV cache (SWA ring pool, GA linear pool) and
// token-level sparse decode (recent window + selected indices), as split-KV kernels.
//
// Math ("MiMo-V2-Flash: Hybrid Sliding Window Attention Architecture", §4.4): for the
// query of sequence b (position L_b - 1) and query head h,
//   a_j = q.k_j * scale,  m = max(sink_h, max_j a_j),
//   o = sum_j exp(a_j - m) v_j / (exp(sink_h - m) + sum_j exp(a_j - m)).
// The key list of one (b, kv-head g) is cut into chunks; each CTA streams one chunk
// and produces the chunk's (m_c, l_c, o_c) WITHOUT the sink. The combine kernel
// merges chunks and adds exp(sink - M) exactly once. A unit whose key list fits in
// one chunk is finalised in place (sink included) with no workspace.
//
// Key lists (token indices within the sequence):
//   ring   (SWA pool of O(W) slots, "...MiMo-V2.5..." dual-pool cache): slots
//          [0, min(L, cap)); slot order does not matter since K is stored rotated.
//   linear (GA pool): slots [0, L).
//   sparse ("小米MiMo-V3的核心架构HySparse2" §四.3): {L - recent, ..., L - 1} followed by
//          sel[b, g, 0..n_sel) - one merged softmax over both parts.
//
// Work per CTA (4 warps): subtiles of 64 keys double-buffered in shared memory by
// 16-byte cp.async gathers (rows XOR-swizzled for conflict-free ldmatrix). Each warp
// owns 16 keys of a subtile: S = Q K^T and O += P V as m16n8k16 bf16 MMAs with the
// group's (up to 16) query heads as the M dimension; online softmax per warp; the
// four warp states are merged at the end.
//
// FP8 caches have kernels of their own (decode_fp8.cuh).
#pragma once

#include "ptx.cuh"

namespace mimo {

constexpr int kDQK = 192;
constexpr int kDV = 128;
constexpr int kDecThreads = 128;
constexpr int kDecSub = 64;                        // keys per subtile (16 per warp)
constexpr int kDecStages = 2;
constexpr int kKRow = kDQK * 2;                    // 384 bytes
constexpr int kVRow = kDV * 2;                     // 256 bytes
constexpr int kDecStageBytes = kDecSub * (kKRow + kVRow);   // 40960
constexpr int kDecMaxTokList = 512;                // sparse chunk limit (tokens staged in smem)
constexpr int kDecSmemBytes = kDecStages * kDecStageBytes + kDecMaxTokList * 4;
constexpr int kKRow8 = kDQK, kVRow8 = kDV;                    // FP8 bytes per cached row

enum : int { kModeRing = 0, kModeLinear = 1, kModeSparse = 2 };

struct DecodeParams {
  const __nv_bfloat16* q;     // [B, Hq, 192]
  const __nv_bfloat16* k;     // [B, seq_stride, Hkv, 192]
  const __nv_bfloat16* v;     // [B, seq_stride, Hkv, 128]
  const int* lengths;         // [B]
  const int* sel;             // [B, Hkv, n_sel] (sparse)
  const float* sink;          // [Hq] or null
  __nv_bfloat16* out;         // [B, Hq, 128]
  float* lse;                 // [B, Hq] or null
  float* part_ml;             // [B*Hq, nchunks, 2]  (m in log2 units, l)
  float* part_o;              // [B*Hq, nchunks, 128]
  long long seq_stride;       // tokens between sequences
  const uint8_t* k8;          // FP8 caches: [B, seq_stride, Hkv, 192] / [.., 128] E4M3 bytes
  const uint8_t* v8;
  const float* k_scale;       // [B, seq_stride, Hkv] fp32 (FP8 only)
  const float* v_scale;
  int B, Hq, Hkv, group, cap, mode, chunk, nchunks, recent, n_sel, direct;
  int nstages;                // stages in flight per CTA (decode_warp_kernel)
  float scale_log2;           // softmax scale * log2(e)
  unsigned* err;
};

// Number of keys of unit (b, .) and the size of the recent part (sparse). Lengths outside
// [0, capacity] (linear and sparse) are clamped; debug builds also record them.
__device__ __forceinline__ int dec_unit_keys(const DecodeParams& p, int b, int& nw, int& L) {
  L = p.lengths[b];
#ifdef MIMO_DEBUG
  if (L < 0 || (p.mode != kModeRing && L > p.cap)) atomicOr(p.err, kErrBadLength);
#endif
  L = L < 0 ? 0 : L;
  if (p.mode == kModeRing) {
    nw = 0;
    return L < p.cap ? L : p.cap;
  }
  L = L < p.cap ? L : p.cap;
  if (p.mode == kModeLinear) {
    nw = 0;
    return L;
  }
  nw = p.recent < L ? p.recent : L;
  return nw + p.n_sel;
}

// Token (row within the sequence) of key t of unit (b, g); -1 for a selected entry that
// names no token (the -1 padding of a short selection row), which is a masked key.
__device__ __forceinline__ int dec_token(const DecodeParams& p, int b, int g, int t, int nw,
                                         int L) {
  if (p.mode != kModeSparse) return t;
  if (t < nw) return L - nw + t;
  const int x = __ldg(p.sel + (static_cast<long long>(b) * p.Hkv + g) * p.n_sel + (t - nw));
#ifdef MIMO_DEBUG
  // a real entry must lie outside the recent window and above its predecessor
  if (x < -1 || x >= L - nw || (x >= 0 && t > nw && __ldg(p.sel + (static_cast<long long>(b) * p.Hkv + g) * p.n_sel +
                                                          (t - nw - 1)) >= x))
    atomicOr(p.err, kErrBadIndex);
#endif
  if (x < 0) return -1;
  return x < p.cap - 1 ? x : p.cap - 1;
}

// 4-byte cp.async (zero-filled when src_bytes = 0).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two E4M3 bytes (lo = first) -> packed f16x2, exactly.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}

template <int G>
__global__ void __launch_bounds__(kDecThreads, 2) decode_split_kernel(const DecodeParams p) {
  static_assert(G >= 1 && G <= 16, "group size");
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem[];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;   // mma fragment row / column pair

  int nw, L;
  const int nkeys = dec_unit_keys(p, b, nw, L);
  const int k_begin = c * p.chunk;
  if (k_begin >= nkeys && !p.direct) return;   // empty chunk: the combine skips it
  int n_here = nkeys - k_begin;
  n_here = n_here < 0 ? 0 : (n_here < p.chunk ? n_here : p.chunk);

  int* s_tok = reinterpret_cast<int*>(smem + kDecStages * kDecStageBytes);
  if (p.mode == kModeSparse) {
    for (int i = tid; i < n_here; i += kDecThreads) s_tok[i] = dec_token(p, b, g, k_begin + i, nw, L);
    __syncthreads();
  }
  const uint32_t s_base = smem_u32(smem);
  const long long seq0 = static_cast<long long>(b) * p.seq_stride;
  const __nv_bfloat16* kbase = p.k + g * kDQK;
  const __nv_bfloat16* vbase = p.v + g * kDV;
  const long long krow_stride = static_cast<long long>(p.Hkv) * kDQK;
  const long long vrow_stride = static_cast<long long>(p.Hkv) * kDV;

  auto token_of = [&](int key) -> int {
    return p.mode == kModeSparse ? s_tok[key] : k_begin + key;
  };

  // Thread t serves rows 16 i + t / 8 of the subtile and, in each, the 16-byte units 8 p + t % 8:
  // every warp instruction reads 128 contiguous bytes from each of 4 rows, and a row (token,
  // global and shared addresses) is resolved once for all of its units.
  auto load_sub = [&](int st, int stage) {
    const uint32_t sK = s_base + stage * kDecStageBytes;
    const uint32_t sV = sK + kDecSub * kKRow;
    const int base = st * kDecSub;
    const int lr = tid >> 3, lu = tid & 7;
#pragma unroll
    for (int i = 0; i < kDecSub / (kDecThreads / 8); ++i) {
      const int row = (kDecThreads / 8) * i + lr;
      const int key = base + row;
      int tok = key < n_here ? token_of(key) : -1;
      const uint32_t sz = tok >= 0 ? 16u : 0u;
      tok = tok >= 0 ? tok : 0;
      const __nv_bfloat16* kg = kbase + (seq0 + tok) * krow_stride + lu * 8;
      const __nv_bfloat16* vg = vbase + (seq0 + tok) * vrow_stride + lu * 8;
      // unit 8 p + lu lands at unit 8 p + (lu ^ (row & 7)) (the XOR keeps the low 3 bits)
      const uint32_t sw = static_cast<uint32_t>((lu ^ (row & 7)) << 4);
      const uint32_t sk = sK + row * kKRow + sw, sv = sV + row * kVRow + sw;
#pragma unroll
      for (int pp = 0; pp < kKRow / 128; ++pp) cp_async16(sk + pp * 128, kg + pp * 64, sz);
#pragma unroll
      for (int pp = 0; pp < kVRow / 128; ++pp) cp_async16(sv + pp * 128, vg + pp * 64, sz);
    }
  };

  const int nsub = (n_here + kDecSub - 1) / kDecSub;
  if (nsub > 0) load_sub(0, 0);
  cp_async_commit();
  if (nsub > 1) load_sub(1, 1);
  cp_async_commit();

  // Query fragments (A operand, rows = the group's heads, zero-padded to 16).
  uint32_t qa[12][4];
  {
    const __nv_bfloat16* qg = p.q + (static_cast<long long>(b) * p.Hq + g * G) * kDQK;
    const bool r0ok = gq < G, r1ok = gq + 8 < G;
#pragma unroll
    for (int kk = 0; kk < 12; ++kk) {
      const int d0 = kk * 16 + tq * 2;
      qa[kk][0] = r0ok ? *reinterpret_cast<const uint32_t*>(qg + gq * kDQK + d0) : 0u;
      qa[kk][1] = r1ok ? *reinterpret_cast<const uint32_t*>(qg + (gq + 8) * kDQK + d0) : 0u;
      qa[kk][2] = r0ok ? *reinterpret_cast<const uint32_t*>(qg + gq * kDQK + d0 + 8) : 0u;
      qa[kk][3] = r1ok ? *reinterpret_cast<const uint32_t*>(qg + (gq + 8) * kDQK + d0 + 8) : 0u;
    }
  }

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int st = 0; st < nsub; ++st) {
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sK = s_base + (st & 1) * kDecStageBytes;
    const uint32_t sV = sK + kDecSub * kKRow;
    const int mi = lane >> 3, r8 = lane & 7;

    // S = Q K^T for this warp's 16 keys (two n-tiles of 8 keys).
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int krow = warp * 16 + ((mi >> 1) << 3) + r8;
      const uint32_t rowaddr = sK + krow * kKRow;
#pragma unroll
      for (int kk = 0; kk < 12; ++kk) {
        const int unit = 2 * kk + (mi & 1);
        uint32_t b00, b01, b10, b11;
        ldmatrix_x4(rowaddr + ((unit ^ (krow & 7)) << 4), b00, b01, b10, b11);
        mma_16816(sacc[0], qa[kk], b00, b01);
        mma_16816(sacc[1], qa[kk], b10, b11);
      }
    }

    // Online softmax (log2 domain); masked keys (past the end, or a selected entry that
    // names no token) contribute nothing.
    const int keybase = st * kDecSub + warp * 16 + tq * 2;
    float s[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = keybase + nt * 8 + (e & 1);
        const bool ok = key < n_here && (p.mode != kModeSparse || s_tok[key] >= 0);
        s[nt][e] = ok ? sacc[nt][e] * p.scale_log2 : -INFINITY;
      }
    }
    float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float ref0 = mn0 == -INFINITY ? 0.f : mn0;
    const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = ex2(m0 - ref0), al1 = ex2(m1 - ref1);
    float pv[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pv[nt][0] = ex2(s[nt][0] - ref0);
      pv[nt][1] = ex2(s[nt][1] - ref0);
      pv[nt][2] = ex2(s[nt][2] - ref1);
      pv[nt][3] = ex2(s[nt][3] - ref1);
    }
    l0 = l0 * al0 + (pv[0][0] + pv[0][1] + pv[1][0] + pv[1][1]);
    l1 = l1 * al1 + (pv[0][2] + pv[0][3] + pv[1][2] + pv[1][3]);
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j][0] *= al0; o[j][1] *= al0;
      o[j][2] *= al1; o[j][3] *= al1;
    }
    uint32_t pa[4];
    pa[0] = pack_bf16(pv[0][0], pv[0][1]);
    pa[1] = pack_bf16(pv[0][2], pv[0][3]);
    pa[2] = pack_bf16(pv[1][0], pv[1][1]);
    pa[3] = pack_bf16(pv[1][2], pv[1][3]);

    // O += P V (V fragments through transposed ldmatrix).
    {
      const int vrow = warp * 16 + ((mi & 1) << 3) + r8;
      const uint32_t rowaddr = sV + vrow * kVRow;
#pragma unroll
      for (int jp = 0; jp < 8; ++jp) {
        const int unit = 2 * jp + (mi >> 1);
        uint32_t v0, v1, v2, v3;
        ldmatrix_x4_trans(rowaddr + ((unit ^ (vrow & 7)) << 4), v0, v1, v2, v3);
        mma_16816(o[2 * jp], pa, v0, v1);
        mma_16816(o[2 * jp + 1], pa, v2, v3);
      }
    }
    __syncthreads();
    if (st + 2 < nsub) load_sub(st + 2, st & 1);
    cp_async_commit();
  }
  cp_async_wait<0>();

  // Merge the four warp states through shared memory (stage buffers are free now).
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();
  float* s_o = reinterpret_cast<float*>(smem);                 // [4][16][128]
  float* s_m = s_o + 4 * 16 * kDV;                              // [4][16]
  float* s_l = s_m + 4 * 16;                                    // [4][16]
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float* r0p = s_o + (warp * 16 + gq) * kDV + j * 8 + tq * 2;
    float* r1p = s_o + (warp * 16 + gq + 8) * kDV + j * 8 + tq * 2;
    r0p[0] = o[j][0]; r0p[1] = o[j][1];
    r1p[0] = o[j][2]; r1p[1] = o[j][3];
  }
  if (tq == 0) {
    s_m[warp * 16 + gq] = m0; s_m[warp * 16 + gq + 8] = m1;
    s_l[warp * 16 + gq] = l0; s_l[warp * 16 + gq + 8] = l1;
  }
  __syncthreads();

  const int d = tid;   // one output column per thread
  for (int r = 0; r < G; ++r) {
    const int h = g * G + r;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w * 16 + r]);
    const long long bh = static_cast<long long>(b) * p.Hq + h;
    if (p.direct) {
      const float sk = p.sink ? p.sink[h] * 1.4426950408889634f : -INFINITY;
      const float M2 = fmaxf(M, sk);
      const float ref = M2 == -INFINITY ? 0.f : M2;
      float Lt = p.sink ? ex2(sk - ref) : 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float sc = ex2(s_m[w * 16 + r] - ref);
        Lt += s_l[w * 16 + r] * sc;
        acc += s_o[(w * 16 + r) * kDV + d] * sc;
      }
      const float ov = Lt > 0.f ? acc / Lt : 0.f;
      p.out[bh * kDV + d] = __float2bfloat16_rn(ov);
      if (d == 0 && p.lse) p.lse[bh] = Lt > 0.f ? (ref + log2f(Lt)) * 0.6931471805599453f : -INFINITY;
    } else {
      const float ref = M == -INFINITY ? 0.f : M;
      float Lp = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float sc = ex2(s_m[w * 16 + r] - ref);
        Lp += s_l[w * 16 + r] * sc;
        acc += s_o[(w * 16 + r) * kDV + d] * sc;
      }
      const long long slot = bh * p.nchunks + c;
      p.part_o[slot * kDV + d] = acc;
      if (d == 0) {
        p.part_ml[slot * 2 + 0] = M;
        p.part_ml[slot * 2 + 1] = Lp;
      }
    }
  }
}

// Merges the chunk states of one output row and adds the sink once (one CTA of kDV threads,
// thread d owning column d): M = max(sink, max_c m_c); L = exp2(sink - M) + sum_c l_c exp2(m_c - M);
// o = sum_c o_c exp2(m_c - M) / L; lse = (M + log2 L) ln 2. The chunk states are read in
// parallel (thread t loads chunk t, t + kDV, ...) and the per-column sum runs over weights
// staged in shared memory, so no thread walks the chunks with a chain of dependent loads.
// ml: [nvalid][2] (m in log2 units, l), po: [nvalid][kDV]; sk is sink * log2(e) or -inf.
__device__ __forceinline__ void combine_row(const float* ml, const float* po, int nvalid, float sk,
                                            bool has_sink, __nv_bfloat16* out_row, float* lse) {
  __shared__ float s_w[kDV];
  __shared__ float s_red[kDV / 32];
  const int d = threadIdx.x, lane = d & 31, warp = d >> 5;
  float M = sk;
  for (int c = d; c < nvalid; c += kDV) M = fmaxf(M, ml[2 * c]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) s_red[warp] = M;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kDV / 32; ++w) M = fmaxf(M, s_red[w]);
  const float ref = M == -INFINITY ? 0.f : M;
  float lpart = 0.f, acc = 0.f;
  for (int c0 = 0; c0 < nvalid; c0 += kDV) {
    const int c = c0 + d;
    float w = 0.f;
    if (c < nvalid) {
      w = ex2(ml[2 * c] - ref);
      lpart += ml[2 * c + 1] * w;
    }
    __syncthreads();                 // the previous tile's weights (and s_red) are consumed
    s_w[d] = w;
    __syncthreads();
    const int n = nvalid - c0 < kDV ? nvalid - c0 : kDV;
    const float* pc = po + static_cast<long long>(c0) * kDV + d;
#pragma unroll 8
    for (int i = 0; i < n; ++i) acc += pc[i * kDV] * s_w[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lpart += __shfl_xor_sync(0xffffffffu, lpart, o);
  __syncthreads();
  if (lane == 0) s_red[warp] = lpart;
  __syncthreads();
  float Lt = has_sink ? ex2(sk - ref) : 0.f;
#pragma unroll
  for (int w = 0; w < kDV / 32; ++w) Lt += s_red[w];
  const float ov = Lt > 0.f ? acc / Lt : 0.f;
  out_row[d] = __float2bfloat16_rn(ov);
  if (d == 0 && lse) *lse = Lt > 0.f ? (ref + log2f(Lt)) * 0.6931471805599453f : -INFINITY;
}

// Merges the chunk states of one (b, h) of a decode call (combine_row).
__global__ void __launch_bounds__(kDV) decode_combine_kernel(const DecodeParams p) {
  pdl_wait();
  pdl_trigger();
  const int bh = blockIdx.x;
  const int b = bh / p.Hq, h = bh - b * p.Hq;
  int nw, L;
  const int nkeys = dec_unit_keys(p, b, nw, L);
  int nvalid = (nkeys + p.chunk - 1) / p.chunk;
  nvalid = nvalid < p.nchunks ? nvalid : p.nchunks;
  const float sk = p.sink ? p.sink[h] * 1.4426950408889634f : -INFINITY;
  combine_row(p.part_ml + static_cast<long long>(bh) * p.nchunks * 2,
              p.part_o + static_cast<long long>(bh) * p.nchunks * kDV, nvalid, sk, p.sink != nullptr,
              p.out + static_cast<long long>(bh) * kDV, p.lse ? p.lse + bh : nullptr);
}

// Debug check of sparse preconditions; one thread per (b, g) row. A valid row is a strictly
// increasing run of tokens in [0, L - recent) followed by zero or more -1 entries.
__global__ void check_indices_kernel(const int* lengths, const int* sel, int B, int Hkv, int n_sel,
                                     int recent, int cap, unsigned* violations) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= B * Hkv) return;
  const int b = row / Hkv;
  const int L = lengths[b];
  bool bad = L < 0 || L > cap;
  const int hi = L - recent;
  const int* s = sel + static_cast<long long>(row) * n_sel;
  int prev = -1;
  bool padding = false;
  for (int i = 0; i < n_sel && !bad; ++i) {
    const int x = s[i];
    if (x == -1) {
      padding = true;
      continue;
    }
    if (padding || x <= prev || x < 0 || x >= hi) bad = true;
    prev = x;
  }
  if (bad) atomicAdd(violations, 1u);
}

}  // namespace mimo
