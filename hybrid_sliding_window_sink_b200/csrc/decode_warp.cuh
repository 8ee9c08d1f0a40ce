// decode_warp.cuh - split-KV decode (SWA ring pool, GA linear pool) and token-level sparse
// decode over bf16 caches with one warp per CTA.
//
// Math ("MiMo-V2-Flash: Hybrid Sliding Window Attention Architecture", §4.4) as decode.cuh:
// for the query of sequence b and query head h, a_j = q.k_j * scale, m = max(sink, max_j a_j),
// o = sum_j exp(a_j - m) v_j / (exp(sink - m) + sum_j exp(a_j - m)). The key lists (ring,
// linear, sparse = recent window + selected tokens of "小米MiMo-V3的核心架构HySparse2" §四.3)
// and the chunk / combine split are those of decode.cuh.
//
// Design (for units of at most a few hundred keys: the SWA ring, and the sparse key lists).
// A CTA is one warp and owns one chunk of one (sequence, KV head) unit: no barrier and no
// merge across warps, so the short life of such a CTA is not spent in a CTA-wide epilogue,
// and five CTAs share an SM. The chunk is cut into stages of 32 keys; NS stages are in flight,
// each gathered by 16-byte cp.async (one warp instruction moves 512 bytes; K rows XOR-
// swizzled for conflict-free ldmatrix) and tracked by cp.async groups, so the warp needs no
// mbarrier. Per stage the warp computes S = Q K^T (16 x 32: the group's heads padded to 16
// rows) and O += P V (16 x 128) as m16n8k16 bf16 MMAs with an online softmax. Keys past the
// end of the chunk, and selected entries that name no token (-1), are zero-filled and
// masked. (Per-row bulk copies were measured too: the copy engine then handles about one row
// per 20 cycles per SM, which caps a kernel at about 0.6 of HBM.)
#pragma once

#include "ptx.cuh"
#include "decode.cuh"

namespace mimo {

constexpr int kDwKeys = 32;                                   // keys per stage
constexpr int kDwStageBytes = kDwKeys * (kKRow + kVRow);      // 20480
constexpr int kDwMaxStages = 3;

__host__ __device__ constexpr int dw_smem_bytes(int stages) { return stages * (kDwStageBytes + kDwKeys * 4); }

// The warp copies 32 K and V rows (tokens tk[0..31] of one sequence and KV head; a negative
// token is zero-filled) into a stage by 16-byte cp.async, K rows XOR-swizzled for ldmatrix.
// Lane l serves rows 4 i + l / 8 (i = 0..7) and, in each, the 16-byte units 8 p + l % 8: every
// warp instruction reads 128 contiguous bytes from each of 4 rows, and a lane resolves each of
// its rows (token, global and shared addresses) once for all of that row's units. The caller
// commits the group.
__device__ __forceinline__ void dw_gather(uint32_t sK, uint32_t sV, const int* tk, const __nv_bfloat16* kbase,
                                          const __nv_bfloat16* vbase, long long seq0, long long krow_stride,
                                          long long vrow_stride) {
  const int lane = threadIdx.x & 31, lr = lane >> 3, lu = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = 4 * i + lr;
    const int t = tk[row];
    const uint32_t sz = t < 0 ? 0u : 16u;
    const long long tok = seq0 + (t < 0 ? 0 : t);
    const __nv_bfloat16* kg = kbase + tok * krow_stride + lu * 8;
    const __nv_bfloat16* vg = vbase + tok * vrow_stride + lu * 8;
    // unit 8 p + lu lands at unit 8 p + (lu ^ (row & 7)) of the row (the XOR keeps the low 3 bits)
    const uint32_t sw = static_cast<uint32_t>((lu ^ (row & 7)) << 4);
    const uint32_t sk = sK + row * kKRow + sw, sv = sV + row * kVRow + sw;
#pragma unroll
    for (int pp = 0; pp < kKRow / 128; ++pp) cp_async16(sk + pp * 128, kg + pp * 64, sz);
#pragma unroll
    for (int pp = 0; pp < kVRow / 128; ++pp) cp_async16(sv + pp * 128, vg + pp * 64, sz);
  }
}

// Query fragments of the group's G heads (rows gq, gq + 8 of the m16 A operand; padding
// rows are zero), read once per warp from q [G, 192].
template <int G>
__device__ __forceinline__ void dw_load_q(uint32_t (&qa)[12][4], const __nv_bfloat16* qg) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const bool r0ok = gq < G, r1ok = gq + 8 < G;
#pragma unroll
  for (int kk = 0; kk < 12; ++kk) {
    const int d0 = kk * 16 + tq * 2;
    qa[kk][0] = r0ok ? __ldg(reinterpret_cast<const unsigned*>(qg + gq * kDQK + d0)) : 0u;
    qa[kk][1] = r1ok ? __ldg(reinterpret_cast<const unsigned*>(qg + (gq + 8) * kDQK + d0)) : 0u;
    qa[kk][2] = r0ok ? __ldg(reinterpret_cast<const unsigned*>(qg + gq * kDQK + d0 + 8)) : 0u;
    qa[kk][3] = r1ok ? __ldg(reinterpret_cast<const unsigned*>(qg + (gq + 8) * kDQK + d0 + 8)) : 0u;
  }
}

// One stage of 32 keys for one warp: S = Q K^T (K rows XOR-swizzled at sK), the online
// softmax in the log2 domain (a key whose token tk[key] < 0 is masked), and O += P V (V rows at
// sV). m0 / m1 and l0 / l1 are this thread's running max and (partial) sum of rows gq, gq + 8.
__device__ __forceinline__ void dw_stage(uint32_t sK, uint32_t sV, const int* tk, const uint32_t (&qa)[12][4],
                                         float scale_log2, float (&o)[16][4], float& m0, float& m1,
                                         float& l0, float& l1) {
  const int lane = threadIdx.x & 31, tq = lane & 3;
  const int mi = lane >> 3, r8 = lane & 7;
    // S = Q K^T for the stage's 32 keys: four n-tiles of 8 keys.
    float sacc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 12; ++kk) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int krow = 16 * h + ((mi >> 1) << 3) + r8;
        uint32_t b00, b01, b10, b11;
        ldmatrix_x4(sK + krow * kKRow + (((2 * kk + (mi & 1)) ^ (krow & 7)) << 4), b00, b01, b10, b11);
        mma_16816(sacc[2 * h], qa[kk], b00, b01);
        mma_16816(sacc[2 * h + 1], qa[kk], b10, b11);
      }
    }

    // Online softmax (log2 domain); masked keys contribute nothing.
    float s[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = nt * 8 + tq * 2 + (e & 1);
        s[nt][e] = tk[key] >= 0 ? sacc[nt][e] * scale_log2 : -INFINITY;
      }
    float mx0 = fmaxf(fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1])),
                      fmaxf(fmaxf(s[2][0], s[2][1]), fmaxf(s[3][0], s[3][1])));
    float mx1 = fmaxf(fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3])),
                      fmaxf(fmaxf(s[2][2], s[2][3]), fmaxf(s[3][2], s[3][3])));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float ref0 = mn0 == -INFINITY ? 0.f : mn0;
    const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = ex2(m0 - ref0), al1 = ex2(m1 - ref1);
    float pv[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      pv[nt][0] = ex2(s[nt][0] - ref0);
      pv[nt][1] = ex2(s[nt][1] - ref0);
      pv[nt][2] = ex2(s[nt][2] - ref1);
      pv[nt][3] = ex2(s[nt][3] - ref1);
    }
    l0 = l0 * al0 + ((pv[0][0] + pv[0][1]) + (pv[1][0] + pv[1][1])) + ((pv[2][0] + pv[2][1]) + (pv[3][0] + pv[3][1]));
    l1 = l1 * al1 + ((pv[0][2] + pv[0][3]) + (pv[1][2] + pv[1][3])) + ((pv[2][2] + pv[2][3]) + (pv[3][2] + pv[3][3]));
    m0 = mn0;
    m1 = mn1;
    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        o[j][0] *= al0; o[j][1] *= al0;
        o[j][2] *= al1; o[j][3] *= al1;
      }
    }

    // O += P V over two k-steps of 16 keys (V fragments through transposed ldmatrix).
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t pa[4];
      pa[0] = pack_bf16(pv[2 * ks][0], pv[2 * ks][1]);
      pa[1] = pack_bf16(pv[2 * ks][2], pv[2 * ks][3]);
      pa[2] = pack_bf16(pv[2 * ks + 1][0], pv[2 * ks + 1][1]);
      pa[3] = pack_bf16(pv[2 * ks + 1][2], pv[2 * ks + 1][3]);
      const int vrow = 16 * ks + ((mi & 1) << 3) + r8;
      const uint32_t rowaddr = sV + vrow * kVRow;
#pragma unroll
      for (int jp = 0; jp < 8; ++jp) {
        uint32_t v0, v1, v2, v3;
        ldmatrix_x4_trans(rowaddr + (((2 * jp + (mi >> 1)) ^ (vrow & 7)) << 4), v0, v1, v2, v3);
        mma_16816(o[2 * jp], pa, v0, v1);
        mma_16816(o[2 * jp + 1], pa, v2, v3);
      }
    }
}

template <int G, int NS>
__global__ void __launch_bounds__(32) decode_warp_kernel(const DecodeParams p) {
  static_assert(G >= 1 && G <= 16, "group size");
  static_assert(NS >= 1 && NS <= kDwMaxStages, "stages in flight");
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem[];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x, gq = lane >> 2, tq = lane & 3;

  int nw, L;
  const int nkeys = dec_unit_keys(p, b, nw, L);
  const int k_begin = c * p.chunk;
  int n_here = nkeys - k_begin;
  n_here = n_here < 0 ? 0 : (n_here < p.chunk ? n_here : p.chunk);
  if (n_here == 0 && !p.direct) return;          // empty chunk: the combine skips it

  const uint32_t s_base = smem_u32(smem);
  int* s_tok = reinterpret_cast<int*>(smem + NS * kDwStageBytes);   // [NS][32]
  const int nst = (n_here + kDwKeys - 1) / kDwKeys;
  const long long seq0 = static_cast<long long>(b) * p.seq_stride;
  const __nv_bfloat16* kbase = p.k + g * kDQK;
  const __nv_bfloat16* vbase = p.v + g * kDV;
  const long long krow_stride = static_cast<long long>(p.Hkv) * kDQK;
  const long long vrow_stride = static_cast<long long>(p.Hkv) * kDV;

  // Gathers stage st (keys 32 st .. 32 st + 31 of the chunk) into buffer st % NS: each lane
  // resolves the token of its own key (-1 when masked), then the warp copies the 32 rows.
  auto issue = [&](int st, int tok) {
    const int buf = st % NS;
    int* tk = s_tok + buf * kDwKeys;
    tk[lane] = tok;
    __syncwarp();
    const uint32_t sK = s_base + buf * kDwStageBytes;
    dw_gather(sK, sK + kDwKeys * kKRow, tk, kbase, vbase, seq0, krow_stride, vrow_stride);
  };
  auto token = [&](int st) -> int {
    const int key = st * kDwKeys + lane;
    return key < n_here ? dec_token(p, b, g, k_begin + key, nw, L) : -1;
  };
  {
    int tok[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) tok[s] = s < nst ? token(s) : -1;   // index loads all in flight
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      if (s < nst) issue(s, tok[s]);
      cp_async_commit();
    }
  }

  // Query fragments (A operand, rows = the group's heads, zero-padded to 16).
  uint32_t qa[12][4];
  dw_load_q<G>(qa, p.q + (static_cast<long long>(b) * p.Hq + g * G) * kDQK);

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int st = 0; st < nst; ++st) {
    const int buf = st % NS;
    cp_async_wait<NS - 1>();                       // this lane's copies of stage st have landed
    __syncwarp();                                  // ... and every other lane's
    const int* tk = s_tok + buf * kDwKeys;
    const uint32_t sK = s_base + buf * kDwStageBytes;
    const uint32_t sV = sK + kDwKeys * kKRow;

    dw_stage(sK, sV, tk, qa, p.scale_log2, o, m0, m1, l0, l1);
    __syncwarp();                                  // every lane is done reading the buffer
    if (st + NS < nst) issue(st + NS, token(st + NS));
    cp_async_commit();
  }
  cp_async_wait<0>();

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = gq + 8 * half;
    if (r >= G) continue;
    const int h = g * G + r;
    const long long bh = static_cast<long long>(b) * p.Hq + h;
    const float m = half ? m1 : m0, l = half ? l1 : l0;
    if (p.direct) {
      const float sk = p.sink ? p.sink[h] * 1.4426950408889634f : -INFINITY;
      const float M2 = fmaxf(m, sk);
      const float ref = M2 == -INFINITY ? 0.f : M2;
      const float sc = ex2(m - ref);
      const float Lt = l * sc + (p.sink ? ex2(sk - ref) : 0.f);
      const float inv = Lt > 0.f ? sc / Lt : 0.f;
      unsigned* orow = reinterpret_cast<unsigned*>(p.out + bh * kDV);
#pragma unroll
      for (int j = 0; j < 16; ++j) orow[4 * j + tq] = pack_bf16(o[j][2 * half] * inv, o[j][2 * half + 1] * inv);
      if (tq == 0 && p.lse) p.lse[bh] = Lt > 0.f ? (ref + log2f(Lt)) * 0.6931471805599453f : -INFINITY;
    } else {
      const long long slot = bh * p.nchunks + c;
      float2* po = reinterpret_cast<float2*>(p.part_o + slot * kDV);
#pragma unroll
      for (int j = 0; j < 16; ++j) po[4 * j + tq] = make_float2(o[j][2 * half], o[j][2 * half + 1]);
      if (tq == 0) {
        p.part_ml[slot * 2 + 0] = m;
        p.part_ml[slot * 2 + 1] = l;
      }
    }
  }
}

}  // namespace mimo
