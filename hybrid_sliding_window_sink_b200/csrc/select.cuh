// select.cuh - token selection for the token-level sparse decode.
//
// "小米MiMo-V3的核心架构HySparse2" §二.2 / §四.3: the selected tokens are chosen token by token
// and reused from the preceding full-attention layer, with no separately trained retrieval
// module. The scoring rule is not given; the one built here: for sequence b and KV head g,
// every token t in [0, L_b - recent) scores max over the group's query heads of q_h . k_t
// (the attention logit up to the positive softmax scale, which does not change the order);
// the n_sel best are kept, equal scores in increasing t, and listed in increasing t.
//
// select_score_kernel: one thread per candidate token, the group's queries in shared memory
// as fp32, the key row read with 16-byte loads; writes an order-preserving uint32 of the
// fp32 score. select_topk_kernel: one CTA per (b, g); a 4-pass radix select (8 bits per
// pass, most significant first) finds the n_sel-th largest key T and how many keys equal to
// T are needed; an ordered compaction (block scans over 1024 candidates at a time) keeps
// every key > T and the first needed keys == T, writing their indices in increasing order.
#pragma once

#include "ptx.cuh"
#include "decode.cuh"

namespace mimo {

constexpr int kSelScoreThreads = 256;
constexpr int kSelThreads = 1024;

struct SelectParams {
  const __nv_bfloat16* q;     // [B, Hq, 192]
  const __nv_bfloat16* k;     // [B, seq_stride, Hkv, 192]
  const int* lengths;         // [B]
  uint32_t* keys;             // workspace [B, Hkv, cap]: order-preserving score bits
  int* sel;                   // [B, Hkv, n_sel]
  long long seq_stride;
  int B, Hq, Hkv, cap, recent, n_sel;
};

__device__ __forceinline__ int sel_candidates(const SelectParams& p, int b) {
  int L = p.lengths[b];
  L = L < 0 ? 0 : (L < p.cap ? L : p.cap);
  const int hi = L - p.recent;
  return hi > 0 ? hi : 0;
}

// fp32 -> uint32 with the same order (negative floats reversed, sign bit set for the rest).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int G>
__global__ void __launch_bounds__(kSelScoreThreads) select_score_kernel(const SelectParams p) {
  __shared__ float s_q[G * kDQK];
  const int g = blockIdx.y, b = blockIdx.z;
  const __nv_bfloat16* qg = p.q + (static_cast<long long>(b) * p.Hq + g * G) * kDQK;
  for (int i = threadIdx.x; i < G * kDQK; i += kSelScoreThreads) s_q[i] = __bfloat162float(qg[i]);
  __syncthreads();
  const int hi = sel_candidates(p, b);
  const int t = blockIdx.x * kSelScoreThreads + threadIdx.x;
  if (t >= hi) return;
  const __nv_bfloat16* krow = p.k + ((static_cast<long long>(b) * p.seq_stride + t) * p.Hkv + g) * kDQK;
  float acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 4
  for (int u = 0; u < kDQK / 8; ++u) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(krow) + u);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float k0 = bf16_lo(w[e]), k1 = bf16_hi(w[e]);
      const int d = u * 8 + 2 * e;
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = fmaf(s_q[h * kDQK + d + 1], k1, fmaf(s_q[h * kDQK + d], k0, acc[h]));
    }
  }
  float best = acc[0];
#pragma unroll
  for (int h = 1; h < G; ++h) best = fmaxf(best, acc[h]);
  p.keys[(static_cast<long long>(b) * p.Hkv + g) * p.cap + t] = order_key(best);
}

// Block-wide exclusive scan of one int per thread (1024 threads); returns the block total.
__device__ __forceinline__ int block_exclusive_scan(int x, int& total, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    s_warp[lane] = wi - w;                 // exclusive prefix of warp totals
    if (lane == 31) s_warp[32] = wi;       // block total
  }
  __syncthreads();
  const int res = s_warp[warp] + incl - x;
  total = s_warp[32];
  __syncthreads();                         // s_warp is reused by the next call
  return res;
}

__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(const SelectParams p) {
  __shared__ int s_hist[256];
  __shared__ int s_warp[33];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  const int g = blockIdx.x, b = blockIdx.y;
  const int hi = sel_candidates(p, b);
  const uint32_t* keys = p.keys + (static_cast<long long>(b) * p.Hkv + g) * p.cap;
  int* out = p.sel + (static_cast<long long>(b) * p.Hkv + g) * p.n_sel;
  const int k = p.n_sel < hi ? p.n_sel : hi;   // fewer candidates than n_sel: keep them all

  // radix select: T = the k-th largest key; need = how many keys equal to T are kept
  uint32_t prefix = 0, mask = 0;
  int need = k;
  if (k > 0 && k < hi) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += kSelThreads) s_hist[i] = 0;
      __syncthreads();
      for (int i = threadIdx.x; i < hi; i += kSelThreads) {
        const uint32_t u = keys[i];
        if ((u & mask) == prefix) atomicAdd(&s_hist[(u >> shift) & 0xFFu], 1);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int above = 0, bin = 255;
        for (; bin > 0; --bin) {
          if (above + s_hist[bin] >= need) break;
          above += s_hist[bin];
        }
        s_prefix = prefix | (static_cast<uint32_t>(bin) << shift);
        s_need = need - above;
      }
      __syncthreads();
      prefix = s_prefix;
      need = s_need;
      mask |= 0xFFu << shift;
      __syncthreads();
    }
  }
  const bool take_all = k >= hi;
  // ordered compaction over the candidates in increasing index
  int out_base = 0, tie_base = 0;
  for (int base = 0; base < hi; base += kSelThreads) {
    const int i = base + threadIdx.x;
    const uint32_t u = i < hi ? keys[i] : 0u;
    const bool valid = i < hi;
    const int eq = valid && !take_all && u == prefix ? 1 : 0;
    int eq_total;
    const int eq_rank = block_exclusive_scan(eq, eq_total, s_warp);
    const int take = valid && (take_all || u > prefix || (eq && tie_base + eq_rank < need)) ? 1 : 0;
    int take_total;
    const int pos = block_exclusive_scan(take, take_total, s_warp);
    if (take && out_base + pos < p.n_sel) out[out_base + pos] = i;
    out_base += take_total;
    tie_base += eq_total;
  }
  for (int j = out_base + threadIdx.x; j < p.n_sel; j += kSelThreads) out[j] = -1;   // too few candidates
}

}  // namespace mimo
