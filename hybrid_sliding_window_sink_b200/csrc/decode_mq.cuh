// decode_mq.cuh - multi-query decode: the T newest tokens of each sequence verified together
// against the KV cache (MTP draft verification).
//
// Math as decode.cuh ("MiMo-V2-Flash: Hybrid Sliding Window Attention Architecture", §4.4),
// with one query row per (draft token t, query head h). Draft token t sits at position
// p_t = L - T + t and attends
//   ring   (SWA pool, token p in slot p mod capacity): tokens [max(0, p_t - W + 1), p_t];
//   linear (GA pool): tokens [0, p_t].
// The MTP section of the syt-nju "mimo-mtp-swa-not-mla" page has the main model verify the
// three draft tokens in one forward pass; all of them are in the cache already.
//
// Work: one CTA (4 warps) per (sequence, KV head, chunk of the unit's key range). The key
// range of a unit is [klo, L) with klo the lowest key of draft token 0, so every key the
// chunk holds is read once and serves all T*G rows. Warp w owns rows [16w, 16w + 16) of the
// T*G (draft token, head) rows and streams every key of the chunk through them: S = Q K^T
// and O += P V as m16n8k16 bf16 MMAs, an online softmax per row with the row's own key
// interval as mask, no merge across warps. K/V subtiles of 64 keys are gathered into shared
// memory by 16-byte cp.async (double buffered, rows XOR-swizzled for ldmatrix). A unit that
// fits one chunk is finalised with the sink in place; otherwise the chunk states go to the
// workspace and decode_mq_combine_kernel adds exp(sink - M) once.
#pragma once

#include "ptx.cuh"
#include "decode.cuh"

namespace mimo {

constexpr int kMqMaxRows = 64;   // T * G <= 64: four m16 row tiles

struct DecodeMqParams {
  const __nv_bfloat16* q;     // [B, T, Hq, 192]
  const __nv_bfloat16* k;     // [B, seq_stride, Hkv, 192]
  const __nv_bfloat16* v;     // [B, seq_stride, Hkv, 128]
  const int* lengths;         // [B], tokens in the cache including the T draft tokens
  const float* sink;          // [Hq] or null
  __nv_bfloat16* out;         // [B, T, Hq, 128]
  float* lse;                 // [B, T, Hq] or null
  float* part_ml;             // [B*T*Hq, nchunks, 2]
  float* part_o;              // [B*T*Hq, nchunks, 128]
  long long seq_stride;
  int B, T, Hq, Hkv, cap, mode, window, chunk, nchunks, direct;
  float scale_log2;
  unsigned* err;
  unsigned long long* trace;  // debug timestamps (builds with -DMIMO_TRACE only), else null
};

// Key range [klo, L) of unit (b, .): the union of the draft tokens' key sets.
__device__ __forceinline__ int mq_range(const DecodeMqParams& p, int b, int& klo) {
  int L = p.lengths[b];
  L = L < 0 ? 0 : (L < p.cap || p.mode == kModeRing ? L : p.cap);
  if (p.mode == kModeRing) {
    const int lo0 = L - p.T - p.window + 1;          // window start of draft token 0
    const int lo_ring = L - p.cap;                   // oldest token the ring still holds
    klo = max(0, max(lo0, lo_ring));
  } else {
    klo = 0;
  }
  return L;
}

// NW warps (16 rows each; NW * 16 >= T * G) and subtiles of SUB keys (64, or 32 for the ring
// layers, whose 131-key units fit in a few subtiles: 40 KB of shared memory then lets five
// CTAs share an SM).
template <int G, int NW, int SUB>
__global__ void __launch_bounds__(NW * 32) decode_mq_kernel(const DecodeMqParams p) {
  constexpr int kThreads = NW * 32;
  constexpr int kStageBytes = SUB * (kKRow + kVRow);
  static_assert(SUB == 32 || SUB == 64, "subtile size");
  static_assert(G >= 1 && G <= 16, "group size");
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem[];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int R = p.T * G;

  int klo;
  const int L = mq_range(p, b, klo);
  const int nkeys = L - klo > 0 ? L - klo : 0;
  const int k_begin = c * p.chunk;
  if (k_begin >= nkeys && !p.direct) return;   // empty chunk: the combine skips it
  int n_here = nkeys - k_begin;
  n_here = n_here < 0 ? 0 : (n_here < p.chunk ? n_here : p.chunk);
  const int tok0 = klo + k_begin;                // token of key 0 of this chunk

  const uint32_t s_base = smem_u32(smem);
  const long long seq0 = static_cast<long long>(b) * p.seq_stride;
  const __nv_bfloat16* kbase = p.k + g * kDQK;
  const __nv_bfloat16* vbase = p.v + g * kDV;
  const long long krow_stride = static_cast<long long>(p.Hkv) * kDQK;
  const long long vrow_stride = static_cast<long long>(p.Hkv) * kDV;
  auto slot_of = [&](int tok) -> int { return p.mode == kModeRing ? tok % p.cap : tok; };

  // Thread t serves rows (kThreads / 8) i + t / 8 of the subtile and, in each, the 16-byte units
  // 8 p + t % 8: every warp instruction reads 128 contiguous bytes from each of 4 rows, and a
  // row (slot, global and shared addresses) is resolved once for all of its units.
  static_assert(SUB % (kThreads / 8) == 0, "rows per pass");
  auto load_sub = [&](int st, int stage) {
    const uint32_t sK = s_base + stage * kStageBytes;
    const uint32_t sV = sK + SUB * kKRow;
    const int base = st * SUB;
    const int lr = tid >> 3, lu = tid & 7;
#pragma unroll
    for (int i = 0; i < SUB / (kThreads / 8); ++i) {
      const int row = (kThreads / 8) * i + lr;
      const int key = base + row;
      const bool ok = key < n_here;
      const int slot = ok ? slot_of(tok0 + key) : 0;
      const uint32_t sz = ok ? 16u : 0u;
      const __nv_bfloat16* kg = kbase + (seq0 + slot) * krow_stride + lu * 8;
      const __nv_bfloat16* vg = vbase + (seq0 + slot) * vrow_stride + lu * 8;
      // unit 8 p + lu lands at unit 8 p + (lu ^ (row & 7)) (the XOR keeps the low 3 bits)
      const uint32_t sw = static_cast<uint32_t>((lu ^ (row & 7)) << 4);
      const uint32_t sk = sK + row * kKRow + sw, sv = sV + row * kVRow + sw;
#pragma unroll
      for (int pp = 0; pp < kKRow / 128; ++pp) cp_async16(sk + pp * 128, kg + pp * 64, sz);
#pragma unroll
      for (int pp = 0; pp < kVRow / 128; ++pp) cp_async16(sv + pp * 128, vg + pp * 64, sz);
    }
  };

  const int nsub = (n_here + SUB - 1) / SUB;
  if (nsub > 0) load_sub(0, 0);
  cp_async_commit();
  if (nsub > 1) load_sub(1, 1);
  cp_async_commit();

  // This warp's two rows per thread: r = t * G + h, padding rows (r >= R) have q = 0 and
  // no keys.
  const bool active = warp * 16 < R;
  const int r0 = warp * 16 + gq, r1 = r0 + 8;
  const bool ok0 = r0 < R, ok1 = r1 < R;
  const int t0 = ok0 ? r0 / G : 0, t1 = ok1 ? r1 / G : 0;
  const int h0 = g * G + (ok0 ? r0 - t0 * G : 0), h1 = g * G + (ok1 ? r1 - t1 * G : 0);
  // key interval [lo_t, p_t] (tokens) of each row; empty for padding rows
  const int pt0 = L - p.T + t0, pt1 = L - p.T + t1;
  int lo0 = p.mode == kModeRing ? max(0, pt0 - p.window + 1) : 0;
  int lo1 = p.mode == kModeRing ? max(0, pt1 - p.window + 1) : 0;
  const int hi0 = ok0 ? pt0 : -1, hi1 = ok1 ? pt1 : -1;

  uint32_t qa[12][4];
  {
    const long long qrow0 = (static_cast<long long>(b) * p.T + t0) * p.Hq + h0;
    const long long qrow1 = (static_cast<long long>(b) * p.T + t1) * p.Hq + h1;
    const __nv_bfloat16* q0 = p.q + qrow0 * kDQK;
    const __nv_bfloat16* q1 = p.q + qrow1 * kDQK;
#pragma unroll
    for (int kk = 0; kk < 12; ++kk) {
      const int d0 = kk * 16 + tq * 2;
      qa[kk][0] = ok0 ? *reinterpret_cast<const uint32_t*>(q0 + d0) : 0u;
      qa[kk][1] = ok1 ? *reinterpret_cast<const uint32_t*>(q1 + d0) : 0u;
      qa[kk][2] = ok0 ? *reinterpret_cast<const uint32_t*>(q0 + d0 + 8) : 0u;
      qa[kk][3] = ok1 ? *reinterpret_cast<const uint32_t*>(q1 + d0 + 8) : 0u;
    }
  }

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int mi = lane >> 3, r8 = lane & 7;

  for (int st = 0; st < nsub; ++st) {
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sK = s_base + (st & 1) * kStageBytes;
    const uint32_t sV = sK + SUB * kKRow;
    if (active) {
      // S = Q K^T over the 64 keys of the subtile (eight n-tiles of 8 keys)
      float sacc[SUB / 8][4];
#pragma unroll
      for (int nt = 0; nt < SUB / 8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
      for (int kg = 0; kg < SUB / 16; ++kg) {
        const int krow = kg * 16 + ((mi >> 1) << 3) + r8;
        const uint32_t rowaddr = sK + krow * kKRow;
#pragma unroll
        for (int kk = 0; kk < 12; ++kk) {
          const int unit = 2 * kk + (mi & 1);
          uint32_t b00, b01, b10, b11;
          ldmatrix_x4(rowaddr + ((unit ^ (krow & 7)) << 4), b00, b01, b10, b11);
          mma_16816(sacc[2 * kg], qa[kk], b00, b01);
          mma_16816(sacc[2 * kg + 1], qa[kk], b10, b11);
        }
      }
      // mask by each row's key interval, online softmax (log2 domain)
      const int tokbase = tok0 + st * SUB + tq * 2;
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < SUB / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = st * SUB + nt * 8 + tq * 2 + (e & 1);
          const int tok = tokbase + nt * 8 + (e & 1);
          const bool in = key < n_here && (e < 2 ? (tok >= lo0 && tok <= hi0) : (tok >= lo1 && tok <= hi1));
          sacc[nt][e] = in ? sacc[nt][e] * p.scale_log2 : -INFINITY;
        }
        mx0 = fmaxf(mx0, fmaxf(sacc[nt][0], sacc[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(sacc[nt][2], sacc[nt][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float ref0 = mn0 == -INFINITY ? 0.f : mn0;
      const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = ex2(m0 - ref0), al1 = ex2(m1 - ref1);
      float s0 = 0.f, s1 = 0.f;
      uint32_t pa[SUB / 16][4];
#pragma unroll
      for (int kg = 0; kg < SUB / 16; ++kg) {
        float pv[2][4];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          pv[q][0] = ex2(sacc[2 * kg + q][0] - ref0);
          pv[q][1] = ex2(sacc[2 * kg + q][1] - ref0);
          pv[q][2] = ex2(sacc[2 * kg + q][2] - ref1);
          pv[q][3] = ex2(sacc[2 * kg + q][3] - ref1);
          s0 += pv[q][0] + pv[q][1];
          s1 += pv[q][2] + pv[q][3];
        }
        pa[kg][0] = pack_bf16(pv[0][0], pv[0][1]);
        pa[kg][1] = pack_bf16(pv[0][2], pv[0][3]);
        pa[kg][2] = pack_bf16(pv[1][0], pv[1][1]);
        pa[kg][3] = pack_bf16(pv[1][2], pv[1][3]);
      }
      l0 = l0 * al0 + s0;
      l1 = l1 * al1 + s1;
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        o[j][0] *= al0; o[j][1] *= al0;
        o[j][2] *= al1; o[j][3] *= al1;
      }
      // O += P V, 16 keys per k-step
#pragma unroll
      for (int kg = 0; kg < SUB / 16; ++kg) {
        const int vrow = kg * 16 + ((mi & 1) << 3) + r8;
        const uint32_t rowaddr = sV + vrow * kVRow;
#pragma unroll
        for (int jp = 0; jp < 8; ++jp) {
          const int unit = 2 * jp + (mi >> 1);
          uint32_t v0, v1, v2, v3;
          ldmatrix_x4_trans(rowaddr + ((unit ^ (vrow & 7)) << 4), v0, v1, v2, v3);
          mma_16816(o[2 * jp], pa[kg], v0, v1);
          mma_16816(o[2 * jp + 1], pa[kg], v2, v3);
        }
      }
    }
    __syncthreads();
    if (st + 2 < nsub) load_sub(st + 2, st & 1);
    cp_async_commit();
  }
  cp_async_wait<0>();
  if (!active) return;

  // Row sums over the quad; each thread then holds columns j*8 + 2 tq + {0, 1} of its rows.
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const bool ok = half == 0 ? ok0 : ok1;
    if (!ok) continue;
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
      for (int j = 0; j < 16; ++j) {
        const float a = half == 0 ? o[j][0] : o[j][2], bb = half == 0 ? o[j][1] : o[j][3];
        *reinterpret_cast<uint32_t*>(p.out + row * kDV + j * 8 + tq * 2) = pack_bf16(a * inv, bb * inv);
      }
      if (tq == 0 && p.lse) p.lse[row] = Lt > 0.f ? (ref + log2f(Lt)) * 0.6931471805599453f : -INFINITY;
    } else {
      const long long slot = row * p.nchunks + c;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float a = half == 0 ? o[j][0] : o[j][2], bb = half == 0 ? o[j][1] : o[j][3];
        *reinterpret_cast<float2*>(p.part_o + slot * kDV + j * 8 + tq * 2) = make_float2(a, bb);
      }
      if (tq == 0) {
        p.part_ml[slot * 2 + 0] = m;
        p.part_ml[slot * 2 + 1] = l;
      }
    }
  }
}

// Merges the chunk states of one (b, t, h) row and adds the sink once (combine_row, over the
// chunks that hold keys of the unit).
__global__ void __launch_bounds__(kDV) decode_mq_combine_kernel(const DecodeMqParams p) {
  pdl_wait();
  pdl_trigger();
  const long long row = blockIdx.x;
  const int h = static_cast<int>(row % p.Hq);
  const int b = static_cast<int>(row / (static_cast<long long>(p.T) * p.Hq));
  int klo;
  const int L = mq_range(p, b, klo);
  const int nkeys = L - klo > 0 ? L - klo : 0;
  int nvalid = (nkeys + p.chunk - 1) / p.chunk;
  nvalid = nvalid < p.nchunks ? nvalid : p.nchunks;
  const float sk = p.sink ? p.sink[h] * 1.4426950408889634f : -INFINITY;
  combine_row(p.part_ml + row * p.nchunks * 2, p.part_o + row * p.nchunks * kDV, nvalid, sk, p.sink != nullptr,
              p.out + row * kDV, p.lse ? p.lse + row : nullptr);
}

}  // namespace mimo
