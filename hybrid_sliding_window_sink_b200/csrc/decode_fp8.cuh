// decode_fp8.cuh - split-KV decode (SWA ring pool, GA linear pool) and token-level sparse
// decode over FP8 KV caches, one warp per CTA, with the MMA operands built in registers
// straight from the cached bytes.
//
// Math ("MiMo-V2-Flash: Hybrid Sliding Window Attention Architecture", §4.4) as decode.cuh:
// for the query of sequence b and query head h, a_j = q.k_j * scale, m = max(sink, max_j a_j),
// o = sum_j exp(a_j - m) v_j / (exp(sink - m) + sum_j exp(a_j - m)). The key lists (ring,
// linear, sparse = recent window + selected tokens of "小米MiMo-V3的核心架构HySparse2" §四.3)
// and the chunk / combine split are those of decode.cuh. FP8 scheme: a cached K or V row is
// OCP E4M3 bytes with one fp32 scale per (token, KV head): k_j = e4m3(K8_j) ks_j and
// v_j = e4m3(V8_j) vs_j.
//
// Design. A CTA is one warp and owns one chunk of one (sequence, KV head) unit. The chunk is
// streamed in stages of 32 keys, NS in flight, copied as raw bytes by 16-byte cp.async (K 6 KB,
// V 4 KB and the 64 scales per stage) and tracked by cp.async groups. Nothing is rewritten in
// shared memory: every lane loads the bytes of its own MMA fragments and converts them in
// registers (E4M3 -> f16 is exact), one conversion per two cached bytes.
//  * S = Q K^T as m16n8k16 f16 MMAs. The sum over the 192 head dims may run in any order as
//    long as Q and K agree on it, so for the key of its n-tile column lane (gq, tq) loads the
//    48 consecutive bytes 48 tq .. 48 tq + 47 of the key's row (three 16-byte loads, free of
//    bank conflicts at the 192-byte row pitch), and k-step kk takes bytes 48 tq + 4 kk .. + 3
//    as the fragment's dims (2 tq, 2 tq + 1, 2 tq + 8, 2 tq + 9). Q is loaded once in the same
//    order and rounded to f16 (so it must lie inside the f16 range). The K scale multiplies
//    the fp32 score.
//  * O += P V as m16n8k16 f16 MMAs. For each of the 16 dv n-tiles, lane (gq, tq) needs the
//    bytes of keys 2 tq, 2 tq + 1, 2 tq + 8, 2 tq + 9 at the dv of its column gq. Letting
//    column gq of n-tile t stand for dv 16 gq + t turns those into one 16-byte load per key
//    row (rows XOR-swizzled in 16-byte units, so the loads are free of bank conflicts); byte
//    permutes pair the keys. The accumulator of lane (gq, tq) then holds dv 32 tq .. 32 tq + 31
//    of rows gq and gq + 8: n-tile t, column c is dv 16 c + t.
//  * The V scale goes into P: P' = P vs_j F, rounded to f16, where F is a power of two chosen
//    per stage so that every P' < 2 (F never grows along the chunk, so O, kept in units of F,
//    is only ever scaled down when F changes) and O is divided by F at the end. The
//    denominator sums the unscaled P in fp32.
#pragma once

#include "ptx.cuh"
#include "decode.cuh"

namespace mimo {

constexpr int kD8Keys = 32;                                        // keys per stage
constexpr int kD8KBytes = kD8Keys * kKRow8;                        // 6144
constexpr int kD8VBytes = kD8Keys * kVRow8;                        // 4096
constexpr int kD8StageBytes = kD8KBytes + kD8VBytes + 2 * kD8Keys * 4;   // + K and V scales: 10496

__host__ __device__ constexpr int d8_smem_bytes(int stages) { return stages * (kD8StageBytes + kD8Keys * 4); }

// The warp copies the K and V bytes and the two scales of 32 keys (tokens tk[0..31] of one
// sequence and KV head; a negative token is zero-filled) into a stage at sK: K rows as they
// are, V rows XOR-swizzled in 16-byte units, then ks[32] and vs[32]. Lane l serves rows
// 8 i + l / 4 (i = 0..3) and, in each, the 16-byte units 4 j + l % 4: every warp instruction
// reads 64 contiguous bytes from each of 8 rows, and a lane resolves each of its rows once.
// 22 cp.async per lane; the caller commits the group.
__device__ __forceinline__ void d8_gather(uint32_t sK, const int* tk, const uint8_t* kbase, const uint8_t* vbase,
                                          const float* ksbase, const float* vsbase, long long seq0,
                                          long long krow_stride, long long vrow_stride, int hkv) {
  const int lane = threadIdx.x & 31, lr = lane >> 2, lu = lane & 3;
  const uint32_t sV = sK + kD8KBytes, sS = sV + kD8VBytes;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = 8 * i + lr;
    const int t = tk[row];
    const uint32_t sz = t < 0 ? 0u : 16u;
    const long long tok = seq0 + (t < 0 ? 0 : t);
    const uint8_t* kg = kbase + tok * krow_stride + lu * 16;
    const uint8_t* vg = vbase + tok * vrow_stride + lu * 16;
    const uint32_t sk = sK + row * kKRow8 + lu * 16;
#pragma unroll
    for (int j = 0; j < kKRow8 / 64; ++j) cp_async16(sk + j * 64, kg + j * 64, sz);
#pragma unroll
    for (int j = 0; j < kVRow8 / 64; ++j)
      cp_async16(sV + row * kVRow8 + (((4 * j + lu) ^ (row & 7)) << 4), vg + j * 64, sz);
  }
  const int t = tk[lane];                          // the two scales of key `lane`
  const long long srow = (seq0 + (t < 0 ? 0 : t)) * hkv;
  cp_async4(sS + lane * 4, ksbase + srow, t < 0 ? 0u : 4u);
  cp_async4(sS + kD8Keys * 4 + lane * 4, vsbase + srow, t < 0 ? 0u : 4u);
}

// Query fragments of the group's G heads in f16, head dims in the order the K fragments take
// them: k-step kk of lane (gq, tq) holds dims 48 tq + 4 kk .. + 3 of rows gq and gq + 8
// (padding rows are zero).
template <int G>
__device__ __forceinline__ void d8_load_q(uint32_t (&qa)[12][4], const __nv_bfloat16* qg) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const bool r0ok = gq < G, r1ok = gq + 8 < G;
#pragma unroll
  for (int kk = 0; kk < 12; ++kk) {
    const int d0 = 48 * tq + 4 * kk;
    const uint2 x0 = r0ok ? __ldg(reinterpret_cast<const uint2*>(qg + gq * kDQK + d0)) : make_uint2(0u, 0u);
    const uint2 x1 = r1ok ? __ldg(reinterpret_cast<const uint2*>(qg + (gq + 8) * kDQK + d0)) : make_uint2(0u, 0u);
    qa[kk][0] = pack_f16(bf16_lo(x0.x), bf16_hi(x0.x));
    qa[kk][1] = pack_f16(bf16_lo(x1.x), bf16_hi(x1.x));
    qa[kk][2] = pack_f16(bf16_lo(x0.y), bf16_hi(x0.y));
    qa[kk][3] = pack_f16(bf16_lo(x1.y), bf16_hi(x1.y));
  }
}

__device__ __forceinline__ float2 ld_shared_f2(uint32_t addr) {
  float2 r;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(r.x), "=f"(r.y) : "r"(addr) : "memory");
  return r;
}

// One stage of 32 keys for one warp (laid out by d8_gather at sK): S = Q K^T with the K
// scales, the online softmax in the log2 domain (a key whose token tk[key] < 0 is masked), the
// stage's V-scale factor, and O += P' V. m0 / m1 and l0 / l1 are this thread's running max and
// partial sum of rows gq and gq + 8; O is kept in units of F.
__device__ __forceinline__ void d8_stage(uint32_t sK, const int* tk, const uint32_t (&qa)[12][4],
                                         float scale_log2, float (&o)[16][4], float& m0, float& m1,
                                         float& l0, float& l1, float& F) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  const uint32_t sV = sK + kD8KBytes, sS = sV + kD8VBytes;

  // S = Q K^T over four n-tiles of 8 keys; this lane's B column in n-tile nt is key 8 nt + gq.
  float sacc[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
    const uint32_t row = sK + (nt * 8 + gq) * kKRow8 + tq * 48;
    uint32_t w[12];
    ld_shared_v4(row, w[0], w[1], w[2], w[3]);
    ld_shared_v4(row + 16, w[4], w[5], w[6], w[7]);
    ld_shared_v4(row + 32, w[8], w[9], w[10], w[11]);
#pragma unroll
    for (int kk = 0; kk < 12; ++kk)
      mma_16816_f16(sacc[nt], qa[kk], e4m3x2_to_f16x2(static_cast<uint16_t>(w[kk] & 0xFFFFu)),
                    e4m3x2_to_f16x2(static_cast<uint16_t>(w[kk] >> 16)));
  }

  // K and V scales of this lane's score columns: keys 8 nt + 2 tq and 8 nt + 2 tq + 1.
  float2 ksc[4], vsc[4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    ksc[nt] = ld_shared_f2(sS + (nt * 8 + tq * 2) * 4);
    vsc[nt] = ld_shared_f2(sS + kD8Keys * 4 + (nt * 8 + tq * 2) * 4);
  }

  // Online softmax (log2 domain); masked keys contribute nothing.
  float s[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = nt * 8 + tq * 2 + (e & 1);
      const float ks = (e & 1) ? ksc[nt].y : ksc[nt].x;
      s[nt][e] = tk[key] >= 0 ? sacc[nt][e] * ks * scale_log2 : -INFINITY;
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

  // The stage's factor: 2^e with max_j |vs_j| 2^e in [1, 2) (lanes of equal tq hold the same
  // keys, so two shuffles cover all 32), never above the factor so far.
  float vm = 0.f;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) vm = fmaxf(vm, fmaxf(fabsf(vsc[nt].x), fabsf(vsc[nt].y)));
  vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, 1));
  vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, 2));
  const unsigned eb = min((__float_as_uint(vm) >> 23) & 0xFFu, 253u);
  const float Fn = fminf(F, __uint_as_float((254u - eb) << 23));
  const float ratio = Fn / F;                      // a power of two: exact
  F = Fn;
  const float oa0 = al0 * ratio, oa1 = al1 * ratio;
  if (__any_sync(0xffffffffu, oa0 != 1.f || oa1 != 1.f)) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      o[j][0] *= oa0; o[j][1] *= oa0;
      o[j][2] *= oa1; o[j][3] *= oa1;
    }
  }

  // O += P' V over two k-steps of 16 keys: keys 16 kb + 2 tq, + 1, + 8, + 9 for this lane.
#pragma unroll
  for (int kb = 0; kb < 2; ++kb) {
    const float2 va = vsc[2 * kb], vb = vsc[2 * kb + 1];
    uint32_t pa[4];
    pa[0] = pack_f16(pv[2 * kb][0] * (va.x * Fn), pv[2 * kb][1] * (va.y * Fn));
    pa[1] = pack_f16(pv[2 * kb][2] * (va.x * Fn), pv[2 * kb][3] * (va.y * Fn));
    pa[2] = pack_f16(pv[2 * kb + 1][0] * (vb.x * Fn), pv[2 * kb + 1][1] * (vb.y * Fn));
    pa[3] = pack_f16(pv[2 * kb + 1][2] * (vb.x * Fn), pv[2 * kb + 1][3] * (vb.y * Fn));
    const int k0 = kb * 16 + tq * 2, k2 = k0 + 8;
    uint32_t a[4], b[4], c[4], d[4];
    ld_shared_v4(sV + k0 * kVRow8 + ((gq ^ (k0 & 7)) << 4), a[0], a[1], a[2], a[3]);
    ld_shared_v4(sV + (k0 + 1) * kVRow8 + ((gq ^ ((k0 + 1) & 7)) << 4), b[0], b[1], b[2], b[3]);
    ld_shared_v4(sV + k2 * kVRow8 + ((gq ^ (k2 & 7)) << 4), c[0], c[1], c[2], c[3]);
    ld_shared_v4(sV + (k2 + 1) * kVRow8 + ((gq ^ ((k2 + 1) & 7)) << 4), d[0], d[1], d[2], d[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // word i holds dv 16 gq + 4 i .. + 3, i.e. n-tiles 4 i .. 4 i + 3 of this lane's column;
      // pair the keys byte by byte: (k0, k0 + 1) for b0 and (k2, k2 + 1) for b1
      const uint32_t x0 = __byte_perm(a[i], b[i], 0x5140), x1 = __byte_perm(a[i], b[i], 0x7362);
      const uint32_t y0 = __byte_perm(c[i], d[i], 0x5140), y1 = __byte_perm(c[i], d[i], 0x7362);
      mma_16816_f16(o[4 * i], pa, e4m3x2_to_f16x2(static_cast<uint16_t>(x0 & 0xFFFFu)),
                    e4m3x2_to_f16x2(static_cast<uint16_t>(y0 & 0xFFFFu)));
      mma_16816_f16(o[4 * i + 1], pa, e4m3x2_to_f16x2(static_cast<uint16_t>(x0 >> 16)),
                    e4m3x2_to_f16x2(static_cast<uint16_t>(y0 >> 16)));
      mma_16816_f16(o[4 * i + 2], pa, e4m3x2_to_f16x2(static_cast<uint16_t>(x1 & 0xFFFFu)),
                    e4m3x2_to_f16x2(static_cast<uint16_t>(y1 & 0xFFFFu)));
      mma_16816_f16(o[4 * i + 3], pa, e4m3x2_to_f16x2(static_cast<uint16_t>(x1 >> 16)),
                    e4m3x2_to_f16x2(static_cast<uint16_t>(y1 >> 16)));
    }
  }
}

template <int G, int NS>
__global__ void __launch_bounds__(32) decode_fp8_kernel(const DecodeParams p) {
  static_assert(G >= 1 && G <= 16, "group size");
  static_assert(NS >= 1 && NS <= 4, "stages in flight");
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
  int* s_tok = reinterpret_cast<int*>(smem + NS * kD8StageBytes);   // [NS][32]
  const int nst = (n_here + kD8Keys - 1) / kD8Keys;
  const long long seq0 = static_cast<long long>(b) * p.seq_stride;
  const uint8_t* kbase = p.k8 + g * kKRow8;
  const uint8_t* vbase = p.v8 + g * kVRow8;
  const float* ksbase = p.k_scale + g;
  const float* vsbase = p.v_scale + g;
  const long long krow_stride = static_cast<long long>(p.Hkv) * kKRow8;
  const long long vrow_stride = static_cast<long long>(p.Hkv) * kVRow8;

  // Gathers stage st (keys 32 st .. 32 st + 31 of the chunk) into buffer st % NS: each lane
  // resolves the token of its own key (-1 when masked), then the warp copies the 32 rows.
  auto issue = [&](int st, int tok) {
    const int buf = st % NS;
    int* tk = s_tok + buf * kD8Keys;
    tk[lane] = tok;
    __syncwarp();
    d8_gather(s_base + buf * kD8StageBytes, tk, kbase, vbase, ksbase, vsbase, seq0, krow_stride, vrow_stride,
              p.Hkv);
  };
  auto token = [&](int st) -> int {
    const int key = st * kD8Keys + lane;
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

  uint32_t qa[12][4];
  d8_load_q<G>(qa, p.q + (static_cast<long long>(b) * p.Hq + g * G) * kDQK);

  float o[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float F = 0x1p127f;                              // the first stage lowers it

  for (int st = 0; st < nst; ++st) {
    const int buf = st % NS;
    cp_async_wait<NS - 1>();                       // this lane's copies of stage st have landed
    __syncwarp();                                  // ... and every other lane's
    d8_stage(s_base + buf * kD8StageBytes, s_tok + buf * kD8Keys, qa, p.scale_log2, o, m0, m1, l0, l1, F);
    __syncwarp();                                  // every lane is done reading the buffer
    if (st + NS < nst) issue(st + NS, token(st + NS));
    cp_async_commit();
  }
  cp_async_wait<0>();

  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float invF = 1.f / F;                      // a power of two: exact

  // This lane holds dv 32 tq + t (o[t][2 half]) and 32 tq + 16 + t (o[t][2 half + 1]) of row
  // gq + 8 half, t = 0..15.
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = gq + 8 * half;
    if (r >= G) continue;
    const int h = g * G + r;
    const long long bh = static_cast<long long>(b) * p.Hq + h;
    const float m = half ? m1 : m0, l = half ? l1 : l0;
    const int c0 = 2 * half, c1 = 2 * half + 1;
    if (p.direct) {
      const float sk = p.sink ? p.sink[h] * 1.4426950408889634f : -INFINITY;
      const float M2 = fmaxf(m, sk);
      const float ref = M2 == -INFINITY ? 0.f : M2;
      const float sc = ex2(m - ref);
      const float Lt = l * sc + (p.sink ? ex2(sk - ref) : 0.f);
      const float inv = Lt > 0.f ? sc / Lt * invF : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(p.out + bh * kDV + 32 * tq);
#pragma unroll
      for (int q4 = 0; q4 < 2; ++q4) {
        const int t = 8 * q4;
        orow[q4] = make_uint4(pack_bf16(o[t][c0] * inv, o[t + 1][c0] * inv), pack_bf16(o[t + 2][c0] * inv, o[t + 3][c0] * inv),
                              pack_bf16(o[t + 4][c0] * inv, o[t + 5][c0] * inv), pack_bf16(o[t + 6][c0] * inv, o[t + 7][c0] * inv));
        orow[2 + q4] = make_uint4(pack_bf16(o[t][c1] * inv, o[t + 1][c1] * inv), pack_bf16(o[t + 2][c1] * inv, o[t + 3][c1] * inv),
                                  pack_bf16(o[t + 4][c1] * inv, o[t + 5][c1] * inv), pack_bf16(o[t + 6][c1] * inv, o[t + 7][c1] * inv));
      }
      if (tq == 0 && p.lse) p.lse[bh] = Lt > 0.f ? (ref + log2f(Lt)) * 0.6931471805599453f : -INFINITY;
    } else {
      const long long slot = bh * p.nchunks + c;
      float4* po = reinterpret_cast<float4*>(p.part_o + slot * kDV + 32 * tq);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        po[j] = make_float4(o[4 * j][c0] * invF, o[4 * j + 1][c0] * invF, o[4 * j + 2][c0] * invF, o[4 * j + 3][c0] * invF);
        po[4 + j] = make_float4(o[4 * j][c1] * invF, o[4 * j + 1][c1] * invF, o[4 * j + 2][c1] * invF, o[4 * j + 3][c1] * invF);
      }
      if (tq == 0) {
        p.part_ml[slot * 2 + 0] = m;
        p.part_ml[slot * 2 + 1] = l;
      }
    }
  }
}

}  // namespace mimo
