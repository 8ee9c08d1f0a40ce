// select.cuh - token selection for the token-level sparse decode.
//
// "小米MiMo-V3的核心架构HySparse2" §二.2 / §四.3: the selected tokens are chosen token by token
// and reused from the preceding full-attention layer, with no separately trained retrieval
// module. The scoring rule is not given; the one built here: for sequence b and KV head g,
// every token t in [0, L_b - recent) scores max over the group's query heads of q_h . k_t
// (the attention logit up to the positive softmax scale, which does not change the order);
// the n_sel best are kept, equal scores in increasing t, and listed in increasing t.
//
// select_score_kernel: 1024 candidates per CTA, S = Q K^T on the tensor cores (mma.sync,
// fp32 accumulation) and the max over the group's heads; writes an order-preserving uint32
// of the fp32 score and a histogram of its top byte per CTA. select_topk_kernel: one CTA per
// (b, g); a 4-digit radix select (8 bits per digit, most significant first; the first digit's
// histogram comes from the score pass) finds the n_sel-th largest key T and how many keys
// equal to T are needed; an ordered compaction (one block scan per 16384 candidates) keeps
// every key > T and the first needed keys == T, writing their indices in increasing order.
#pragma once

#include "ptx.cuh"
#include "decode.cuh"

namespace mimo {

constexpr int kSelChunk = 1024;   // candidate keys per score CTA
constexpr int kSelScoreSmem = 2 * kDecSub * kKRow + 256 * 4;   // two 64-key K subtiles + histogram
constexpr int kSelThreads = 1024;
constexpr int kSelPerThread = 16;                 // candidates per thread per compaction step
constexpr int kSelBlockKeys = kSelPerThread * kSelThreads;
constexpr int kSelUnroll = 8;                     // 16-byte key loads in flight per thread
constexpr int kSelCluster = 8;                    // CTAs per (b, g) in the top-k of long caches
constexpr int kSelClusterMinCap = 131072;         // capacity from which the top-k uses clusters

struct SelectParams {
  const __nv_bfloat16* q;     // [B, Hq, 192]
  const __nv_bfloat16* k;     // [B, seq_stride, Hkv, 192]
  const int* lengths;         // [B]
  uint32_t* keys;             // workspace [B, Hkv, key_stride]: order-preserving score bits
  uint16_t* hist;             // workspace [B, Hkv, n_chunks, 256]: top-byte histogram per score CTA
  int* sel;                   // [B, Hkv, n_sel]
  long long seq_stride;
  int B, Hq, Hkv, cap, recent, n_sel;
  int key_stride;             // cap rounded up to a multiple of 4 (16-byte aligned rows)
  int n_chunks;               // ceil(cap / kSelChunk)
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

// Scores of 1024 candidate keys per CTA as a small GEMM on the tensor cores: K rows are
// gathered by 16-byte cp.async into double-buffered 64-key subtiles (rows XOR-swizzled for
// ldmatrix, as in the decode kernel), each warp takes 16 keys per subtile and computes
// S = Q K^T with m16n8k16 bf16 MMAs (the group's <= 16 heads as M, zero rows masked), then
// the max over the heads per key.
template <int G>
__global__ void __launch_bounds__(kDecThreads, 4) select_score_kernel(const SelectParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int hi = sel_candidates(p, b);
  const int k_begin = blockIdx.x * kSelChunk;
  if (k_begin >= hi) return;
  const int n_here = min(kSelChunk, hi - k_begin);
  const uint32_t s_base = smem_u32(smem);
  int* s_h = reinterpret_cast<int*>(smem + 2 * kDecSub * kKRow);
  for (int i = tid; i < 256; i += kDecThreads) s_h[i] = 0;   // first use is after a barrier
  const __nv_bfloat16* kbase = p.k + (static_cast<long long>(b) * p.seq_stride) * p.Hkv * kDQK + g * kDQK;
  const long long krow_stride = static_cast<long long>(p.Hkv) * kDQK;
  // Thread t serves rows 16 i + t / 8 of the subtile and, in each, the 16-byte units 8 p + t % 8:
  // every warp instruction reads 128 contiguous bytes from each of 4 rows, and a row is resolved
  // once for all of its units.
  auto load_sub = [&](int st, int stage) {
    const uint32_t sK = s_base + stage * (kDecSub * kKRow);
    const int lr = tid >> 3, lu = tid & 7;
#pragma unroll
    for (int i = 0; i < kDecSub / (kDecThreads / 8); ++i) {
      const int row = (kDecThreads / 8) * i + lr;
      const int key = st * kDecSub + row;
      const bool ok = key < n_here;
      const int t = ok ? k_begin + key : 0;
      const uint32_t sz = ok ? 16u : 0u;
      const __nv_bfloat16* kg = kbase + t * krow_stride + lu * 8;
      // unit 8 p + lu lands at unit 8 p + (lu ^ (row & 7)) (the XOR keeps the low 3 bits)
      const uint32_t sk = sK + row * kKRow + static_cast<uint32_t>((lu ^ (row & 7)) << 4);
#pragma unroll
      for (int pp = 0; pp < kKRow / 128; ++pp) cp_async16(sk + pp * 128, kg + pp * 64, sz);
    }
  };
  const int nsub = (n_here + kDecSub - 1) / kDecSub;
  load_sub(0, 0);
  cp_async_commit();
  if (nsub > 1) load_sub(1, 1);
  cp_async_commit();
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
  uint32_t* keys = p.keys + (static_cast<long long>(b) * p.Hkv + g) * p.key_stride + k_begin;
  const int mi = lane >> 3, r8 = lane & 7;
  for (int st = 0; st < nsub; ++st) {
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sK = s_base + (st & 1) * (kDecSub * kKRow);
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
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
    // sacc[nt][e]: head row gq (e < 2) or gq + 8 (e >= 2), key nt*8 + 2 tq + (e & 1)
    float mx[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float a = gq < G ? sacc[nt][c] : -INFINITY;
        const float bb = gq + 8 < G ? sacc[nt][c + 2] : -INFINITY;
        float m = fmaxf(a, bb);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));    // over gq
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        mx[nt][c] = m;
      }
    if (gq == 0) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int key = st * kDecSub + warp * 16 + nt * 8 + 2 * tq + c;
          if (key < n_here) {
            const uint32_t u = order_key(mx[nt][c]);
            keys[key] = u;
            atomicAdd(&s_h[u >> 24], 1);
          }
        }
    }
    __syncthreads();
    if (st + 2 < nsub) load_sub(st + 2, st & 1);
    cp_async_commit();
  }
  cp_async_wait<0>();
  // first radix digit of this chunk's keys, read back by select_topk_kernel (counts <= 1024)
  uint16_t* h = p.hist + ((static_cast<long long>(b) * p.Hkv + g) * p.n_chunks + blockIdx.x) * 256;
  for (int i = tid; i < 256; i += kDecThreads) h[i] = static_cast<uint16_t>(s_h[i]);
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

// Picks the radix bin holding the need-th largest key among the 256 bins of s_hist (warp 0):
// lane l owns bins 255-8l .. 248-8l, a shuffle scan counts the keys in higher lanes' bins.
__device__ __forceinline__ void select_pick_bin(const int* s_hist, int shift, uint32_t prefix, int need,
                                                uint32_t* s_prefix, int* s_need) {
  const int lane = threadIdx.x & 31;
  int c[8];
  int tot = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = s_hist[255 - 8 * lane - j];
    tot += c[j];
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int excl = incl - tot;
  const unsigned own = __ballot_sync(0xffffffffu, excl < need && need <= incl);
  const int owner = own ? __ffs(own) - 1 : 31;   // the counts always place need in one lane
  if (lane == owner) {
    int above = excl, j = 0;
    for (; j < 7; ++j) {
      if (above + c[j] >= need) break;
      above += c[j];
    }
    *s_prefix = prefix | (static_cast<uint32_t>(255 - 8 * lane - j) << shift);
    *s_need = need - above;
  }
}

// Cluster helpers: the shared-memory address of `saddr` in CTA `rank` of this cluster, a
// 32-bit load from it, and a cluster-wide barrier (release / acquire).
__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

// Top-k per (b, g) on a cluster of CS CTAs (launched with that cluster size; CS = 1 is one CTA
// per (b, g)): CTA `rank` owns the contiguous candidate
// slice [lo, hi_c). Digit 1 of the radix select is summed from the score pass's histograms by
// every CTA (the same decision everywhere); digits 2-4 are counted per slice and the cluster's
// histograms are summed through distributed shared memory. The compaction counts each slice's
// keys > T and == T, takes the exclusive prefix over the lower ranks, and writes the slice's
// indices from there: indices stay increasing and the kept ties are the lowest-indexed ones.
template <int CS>
__global__ void __launch_bounds__(kSelThreads) select_topk_kernel(const SelectParams p) {
  __shared__ int s_hist[256];      // this slice's histogram (read by the whole cluster)
  __shared__ int s_hsum[256];      // the cluster's
  __shared__ int s_warp[33];
  __shared__ int s_cnt[2];         // this slice's keys > T and == T (read by the whole cluster)
  __shared__ int s_base[3];        // out position, ties before this slice, cluster total out
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  uint32_t crank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(crank));
  const int rank = static_cast<int>(crank);
  const int g = blockIdx.x / CS, b = blockIdx.y;
  const int tid = threadIdx.x;
  const int hi = sel_candidates(p, b);
  const long long bg = static_cast<long long>(b) * p.Hkv + g;
  const uint32_t* keys = p.keys + bg * p.key_stride;
  const uint4* keys4 = reinterpret_cast<const uint4*>(keys);
  int* out = p.sel + bg * p.n_sel;
  const int k = p.n_sel < hi ? p.n_sel : hi;   // fewer candidates than n_sel: keep them all
  const int per = (((hi + CS - 1) / CS) + 3) & ~3;   // slice length, 16-byte rows
  const int lo = min(hi, rank * per), hi_c = min(hi, lo + per);

  // radix select: T = the k-th largest key; need = how many keys equal to T are kept
  uint32_t prefix = 0, mask = 0;
  int need = k;
  if (k > 0 && k < hi) {
    {  // digit 1 (bits 31..24): sum the score kernel's per-chunk histograms; lane l of warp w
       // adds bins 8l..8l+7 (one 16-byte load) of chunks w, w + 32, ...
      const int nch = (hi + kSelChunk - 1) / kSelChunk;
      const uint4* h4 = reinterpret_cast<const uint4*>(p.hist + bg * p.n_chunks * 256);
      const int lane = tid & 31, warp = tid >> 5;
      if (tid < 256) s_hsum[tid] = 0;
      int acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 4
      for (int c = warp; c < nch; c += kSelThreads / 32) {
        const uint4 v = h4[c * 32 + lane];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += static_cast<int>(w[e] & 0xFFFFu);
          acc[2 * e + 1] += static_cast<int>(w[e] >> 16);
        }
      }
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (acc[e]) atomicAdd(&s_hsum[8 * lane + e], acc[e]);
      __syncthreads();
      if (tid < 32) select_pick_bin(s_hsum, 24, prefix, need, &s_prefix, &s_need);
      __syncthreads();
      prefix = s_prefix;
      need = s_need;
      mask = 0xFF000000u;
    }
    for (int shift = 16; shift >= 0; shift -= 8) {
      if (tid < 256) s_hist[tid] = 0;
      __syncthreads();
      for (int i4 = (lo >> 2) + tid; i4 < (hi_c + 3) >> 2; i4 += kSelUnroll * kSelThreads) {
        uint4 v[kSelUnroll];
#pragma unroll
        for (int r = 0; r < kSelUnroll; ++r) {
          const int j = i4 + r * kSelThreads;
          v[r] = j < (hi_c + 3) >> 2 ? keys4[j] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int r = 0; r < kSelUnroll; ++r) {
          const int i0 = 4 * (i4 + r * kSelThreads);
          const uint32_t u[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (i0 + e < hi_c && (u[e] & mask) == prefix) atomicAdd(&s_hist[(u[e] >> shift) & 0xFFu], 1);
        }
      }
      __syncthreads();
      cluster_sync_all();   // every slice's histogram is complete and visible
      if (tid < 256) {
        int sum = 0;
        for (int r = 0; r < CS; ++r) sum += ld_cluster_s32(cluster_map(smem_u32(&s_hist[tid]), r));
        s_hsum[tid] = sum;
      }
      __syncthreads();
      if (tid < 32) select_pick_bin(s_hsum, shift, prefix, need, &s_prefix, &s_need);
      __syncthreads();
      prefix = s_prefix;
      need = s_need;
      mask |= 0xFFu << shift;
      cluster_sync_all();   // no CTA clears its histogram while another still reads it
    }
  }
  const bool take_all = k >= hi;
  // per-slice counts of the keys kept outright (> T) and of the ties (== T)
  auto classify = [&](int i0, const uint4 (&v)[kSelPerThread / 4], uint32_t& gt, uint32_t& eq) {
    gt = 0;
    eq = 0;
#pragma unroll
    for (int r = 0; r < kSelPerThread / 4; ++r) {
      const uint32_t u[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int idx = i0 + 4 * r + e;
        const bool valid = idx < hi_c;
        if (valid && (take_all || u[e] > prefix)) gt |= 1u << (4 * r + e);
        if (valid && !take_all && u[e] == prefix) eq |= 1u << (4 * r + e);
      }
    }
  };
  {
    int ngt = 0, neq = 0;
    for (int base = lo; base < hi_c; base += kSelBlockKeys) {
      const int i0 = base + kSelPerThread * tid;
      uint4 v[kSelPerThread / 4];
#pragma unroll
      for (int r = 0; r < kSelPerThread / 4; ++r)
        v[r] = i0 + 4 * r < hi_c ? keys4[(i0 >> 2) + r] : make_uint4(0u, 0u, 0u, 0u);
      uint32_t gt, eq;
      classify(i0, v, gt, eq);
      ngt += __popc(gt);
      neq += __popc(eq);
    }
    int tg, te;   // two scans: a slice may hold more keys than a 16-bit field
    block_exclusive_scan(ngt, tg, s_warp);
    block_exclusive_scan(neq, te, s_warp);
    if (tid == 0) {
      s_cnt[0] = tg;
      s_cnt[1] = te;
    }
  }
  cluster_sync_all();       // every slice's counts are visible
  if (tid == 0) {
    int gt_before = 0, eq_before = 0, gt_all = 0, eq_all = 0;
    for (int r = 0; r < CS; ++r) {
      const int cg = ld_cluster_s32(cluster_map(smem_u32(&s_cnt[0]), r));
      const int ce = ld_cluster_s32(cluster_map(smem_u32(&s_cnt[1]), r));
      if (r < rank) {
        gt_before += cg;
        eq_before += ce;
      }
      gt_all += cg;
      eq_all += ce;
    }
    s_base[0] = gt_before + (eq_before < need ? eq_before : need);
    s_base[1] = eq_before;
    s_base[2] = gt_all + (take_all ? 0 : (eq_all < need ? eq_all : need));
  }
  cluster_sync_all();       // the counts are read: a CTA may now finish and exit
  // ordered compaction of the slice, 16 consecutive candidates per thread: one block scan per
  // step of the packed counts (keys == T in the high half, keys > T in the low half)
  int out_base = s_base[0], tie_base = s_base[1];
  for (int base = lo; base < hi_c; base += kSelBlockKeys) {
    const int i0 = base + kSelPerThread * tid;
    uint4 v[kSelPerThread / 4];
#pragma unroll
    for (int r = 0; r < kSelPerThread / 4; ++r)
      v[r] = i0 + 4 * r < hi_c ? keys4[(i0 >> 2) + r] : make_uint4(0u, 0u, 0u, 0u);
    uint32_t gt, eq;
    classify(i0, v, gt, eq);
    const int ngt = __popc(gt), neq = __popc(eq);
    int total;
    const int excl = block_exclusive_scan((neq << 16) | ngt, total, s_warp);
    const int rem = need - tie_base > 0 ? need - tie_base : 0;   // ties still to keep
    if (gt | eq) {
      int e_seen = excl >> 16;
      int pos = out_base + (excl & 0xFFFF) + (e_seen < rem ? e_seen : rem);
      uint32_t m = gt | eq;
      while (m) {
        const int e = __ffs(m) - 1;
        m &= m - 1;
        bool take = true;
        if ((eq >> e) & 1u) take = e_seen++ < rem;
        if (take) {
          if (pos < p.n_sel) out[pos] = i0 + e;
          ++pos;
        }
      }
    }
    const int eq_total = total >> 16;
    out_base += (total & 0xFFFF) + (eq_total < rem ? eq_total : rem);
    tie_base += eq_total;
  }
  if (rank == 0)
    for (int j = s_base[2] + tid; j < p.n_sel; j += kSelThreads) out[j] = -1;   // too few candidates
}

}  // namespace mimo
