// mimo_attn.cu - the C ABI of libmimo_attn.so (declared in include/mimo_attn.h):
// host-side argument checks, tensor-map encoding, kernel selection and launches.
// One translation unit holds every kernel so that they share the device error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "mimo_attn.h"
#include "ptx.cuh"
#include "decode.cuh"
#include "decode_mq.cuh"
#include "decode_warp.cuh"
#include "decode_fp8.cuh"
#include "decode_mq_tma.cuh"
#include "select.cuh"
#include "prefill.cuh"
#include "prefill_swa.cuh"
#include "prefill_ga.cuh"

namespace mimo {

#ifdef MIMO_TEST_HOOKS
// Test builds only: one warp waits on an mbarrier that nothing ever arrives on, through the
// same bounded wait every kernel uses; the wait must give up and set the error word.
__global__ void stuck_wait_kernel(unsigned* err) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncwarp();
  const bool ok = mbar_wait(b, 0, &abort_flag, err);
  if (threadIdx.x == 0 && ok) atomicOr(err, 0x80000000u);   // would mean the wait "completed"
}
#endif
}

#ifdef MIMO_TEST_HOOKS
extern "C" int mimo_attn_test_stuck_wait(void* stream);
#endif

#ifdef MIMO_TRACE
// Debug builds only: device buffer that receives per-phase timestamps of the prefill kernels.
static unsigned long long* g_trace = nullptr;
extern "C" void mimo_attn_debug_set_trace(void* p) { g_trace = static_cast<unsigned long long*>(p); }
#endif

namespace {

using mimo::DecodeParams;
using mimo::PrefillParams;

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Current device and its SM count (148 on B200 when no device can be queried).
int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return dev;
}

int sm_count_for(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int v = g_sm_count[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Unique ID of the calling thread's current CUDA context (0 when there is none). IDs are
// never reused within a process, so a context created after a device reset gets a new one.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
    cudaGetLastError();
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx) get_id(ctx, &id);
  return id;
}

// Device address of a __device__ variable, looked up with cudaGetSymbolAddress once per
// (device, context) and cached: on the host the symbol names a stand-in, not device memory,
// and a context created after a device reset may place the module's variables elsewhere.
struct SymbolAddressCache {
  std::mutex mu;
  unsigned long long ctx_id[kMaxDevices] = {};
  void* addr[kMaxDevices] = {};
};

template <typename T>
void* cached_symbol_address(SymbolAddressCache& c, const T& symbol, int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(c.mu);
  const unsigned long long id = current_context_id();
  if (c.addr[dev] && id != 0 && c.ctx_id[dev] == id) return c.addr[dev];
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, symbol) != cudaSuccess || addr == nullptr) {
    cudaGetLastError();
    return nullptr;
  }
  c.addr[dev] = addr;
  c.ctx_id[dev] = current_context_id();   // the lookup made the primary context current
  return addr;
}

SymbolAddressCache g_err_cache;

unsigned* device_error_ptr(int dev) {
  return static_cast<unsigned*>(cached_symbol_address(g_err_cache, mimo::g_device_error, dev));
}

bool group_ok(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16; }

mimo_status check_heads(const mimo_shape* s) {
  if (!s) return MIMO_ERR_NULL;
  if (s->batch < 1 || s->n_q_heads < 1 || s->n_kv_heads < 1) return MIMO_ERR_SHAPE;
  if (s->n_q_heads % s->n_kv_heads) return MIMO_ERR_SHAPE;
  if (!(s->softmax_scale == s->softmax_scale) || std::isinf(s->softmax_scale)) return MIMO_ERR_SHAPE;
  if (s->head_dim_qk != mimo::kDQK || s->head_dim_v != mimo::kDV) return MIMO_ERR_UNSUPPORTED;
  if (!group_ok(s->n_q_heads / s->n_kv_heads)) return MIMO_ERR_UNSUPPORTED;
  if (s->batch > 65535) return MIMO_ERR_UNSUPPORTED;
  return MIMO_OK;
}

float scale_log2_of(const mimo_shape* s) {
  const float sc = s->softmax_scale > 0.f ? s->softmax_scale : 1.0f / std::sqrt(static_cast<float>(s->head_dim_qk));
  return sc * 1.4426950408889634f;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 4-D bf16 tensor [d3][d2][d1][d0] (d0 innermost), box {64, b1, b2, 1}, 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
               uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  cuuint32_t box[4] = {64, b1, b2, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- prefill
template <int G, int BN, int NKS>
mimo_status launch_prefill(const mimo_shape* s, const void* q, const void* k, const void* v,
                           PrefillParams prm, int sms, cudaStream_t st) {
  using C = mimo::PfCfg<G, BN, NKS>;
  CUtensorMap tq, tk, tv;
  const uint64_t n = static_cast<uint64_t>(s->seqlen), B = static_cast<uint64_t>(s->batch);
  const uint64_t nk = static_cast<uint64_t>(prm.nk);   // keys: n, or prefix + chunk
  if (!make_tmap(&tq, q, mimo::kDQK, s->n_q_heads, n, B, G, C::P) ||
      !make_tmap(&tk, k, mimo::kDQK, s->n_kv_heads, nk, B, 1, BN) ||
      !make_tmap(&tv, v, mimo::kDV, s->n_kv_heads, nk, B, 1, BN))
    return MIMO_ERR_CUDA;
  auto kern = mimo::prefill_kernel<G, BN, NKS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) {
    cudaGetLastError();
    return MIMO_ERR_CUDA;
  }
  prm.n_qtiles = (s->seqlen + C::P - 1) / C::P;
  const long long work = static_cast<long long>(s->batch) * s->n_kv_heads * prm.n_qtiles;
  if (work > 0x7fffffffLL) return MIMO_ERR_UNSUPPORTED;
  prm.num_work = static_cast<int>(work);
  const int grid = prm.num_work < sms ? prm.num_work : sms;
  kern<<<grid, mimo::kPfThreads, C::SMEM, st>>>(tq, tk, tv, prm);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

// SWA layer with 8 query heads per KV head, W <= 129, rot_dims <= 64: the ring kernel.
mimo_status launch_prefill_swa(const mimo_shape* s, const void* q, const void* k, const void* v,
                               PrefillParams prm, int sms, cudaStream_t st) {
  using L = mimo::SwaLayout;
  CUtensorMap tq, tk, tv;
  const uint64_t n = static_cast<uint64_t>(s->seqlen), B = static_cast<uint64_t>(s->batch);
  const uint64_t nk = static_cast<uint64_t>(prm.nk);   // keys: n, or prefix + chunk
  if (prm.q_off % mimo::kSwaP != 0) return MIMO_ERR_UNSUPPORTED;
  if (!make_tmap(&tq, q, mimo::kDQK, s->n_q_heads, n, B, mimo::kSwaG, mimo::kSwaP) ||
      !make_tmap(&tk, k, mimo::kDQK, s->n_kv_heads, nk, B, 1, 16) ||
      !make_tmap(&tv, v, mimo::kDV, s->n_kv_heads, nk, B, 1, 16))
    return MIMO_ERR_CUDA;
  if (cudaFuncSetAttribute(mimo::prefill_swa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           L::SMEM) != cudaSuccess) {
    cudaGetLastError();
    return MIMO_ERR_CUDA;
  }
  prm.n_qtiles = (s->seqlen + mimo::kSwaP - 1) / mimo::kSwaP;
  const long long work = static_cast<long long>(s->batch) * s->n_kv_heads * prm.n_qtiles;
  if (work > 0x7fffffffLL) return MIMO_ERR_UNSUPPORTED;
  prm.num_work = static_cast<int>(work);
  const int grid = prm.num_work < sms ? prm.num_work : sms;
  mimo::prefill_swa_kernel<<<grid, mimo::kSwaThreads, L::SMEM, st>>>(tq, tk, tv, prm);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

// Full causal prefix (GA layers) with 8 or 16 query heads per KV head, rot_dims <= 64:
// two row blocks per work item share every K/V tile.
template <int G>
mimo_status launch_prefill_ga(const mimo_shape* s, const void* q, const void* k, const void* v,
                              PrefillParams prm, int sms, cudaStream_t st) {
  using L = mimo::GaLayout<G>;
  CUtensorMap tq, tk, tv;
  const uint64_t n = static_cast<uint64_t>(s->seqlen), B = static_cast<uint64_t>(s->batch);
  const uint64_t nk = static_cast<uint64_t>(prm.nk);   // keys: n, or prefix + chunk
  if (!make_tmap(&tq, q, mimo::kDQK, s->n_q_heads, n, B, G, L::P) ||
      !make_tmap(&tk, k, mimo::kDQK, s->n_kv_heads, nk, B, 1, mimo::kGaBN) ||
      !make_tmap(&tv, v, mimo::kDV, s->n_kv_heads, nk, B, 1, mimo::kGaBN))
    return MIMO_ERR_CUDA;
  auto kern = mimo::prefill_ga_kernel<G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) != cudaSuccess) {
    cudaGetLastError();
    return MIMO_ERR_CUDA;
  }
  prm.n_qtiles = (s->seqlen + 2 * L::P - 1) / (2 * L::P);   // pairs of row blocks
  const long long work = static_cast<long long>(s->batch) * s->n_kv_heads * prm.n_qtiles;
  if (work > 0x7fffffffLL) return MIMO_ERR_UNSUPPORTED;
  prm.num_work = static_cast<int>(work);
  const int grid = prm.num_work < sms ? prm.num_work : sms;
  kern<<<grid, mimo::kGaThreads, L::SMEM, st>>>(tq, tk, tv, prm);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

template <int G>
mimo_status prefill_group(const mimo_shape* s, const void* q, const void* k, const void* v,
                          const PrefillParams& prm, int sms, cudaStream_t st) {
  constexpr int P = 128 / G;
  const bool swa = prm.window > 0 && prm.window < s->seqlen;
  if (G == mimo::kSwaG && swa && prm.window <= 129 && prm.rot_dims <= 64)
    return launch_prefill_swa(s, q, k, v, prm, sms, st);
  if constexpr (G == 8 || G == 16) {
    if (!swa && prm.rot_dims <= 64) return launch_prefill_ga<G>(s, q, k, v, prm, sms, st);
  }
  // one 144-key tile covers the whole window of a row block when P + W - 1 <= 144
  if (swa && P + prm.window - 1 <= 144) return launch_prefill<G, 144, 1>(s, q, k, v, prm, sms, st);
  return launch_prefill<G, 128, 2>(s, q, k, v, prm, sms, st);
}

// Chunked prefill: GA layers with 8 or 16 query heads per KV head on the pair kernel, SWA
// layers with 8 (W <= 129, chunk offset a multiple of 16) on the ring kernel, every other
// shape on the generic kernel (query positions offset, keys from a prefix + the chunk).
template <int G>
mimo_status prefill_chunk_group(const mimo_shape* s, const void* q, const void* k, const void* v,
                                const PrefillParams& prm, int sms, cudaStream_t st) {
  constexpr int P = 128 / G;
  const bool swa = prm.window > 0 && prm.window < prm.nk;
  if (G == mimo::kSwaG && swa && prm.window <= 129 && prm.rot_dims <= 64 && prm.q_off % mimo::kSwaP == 0)
    return launch_prefill_swa(s, q, k, v, prm, sms, st);
  if constexpr (G == 8 || G == 16) {   // full causal prefix: the pair kernel
    if (!swa && prm.rot_dims <= 64) return launch_prefill_ga<G>(s, q, k, v, prm, sms, st);
  }
  if (swa && P + prm.window - 1 <= 144) return launch_prefill<G, 144, 1>(s, q, k, v, prm, sms, st);
  return launch_prefill<G, 128, 2>(s, q, k, v, prm, sms, st);
}

// Launches a decode-side kernel, with programmatic stream serialization when `pdl` is set: its
// CTAs may then be scheduled while the previous kernel on the stream drains (each kernel's
// first statement is pdl_wait, so nothing is read before that kernel has completed). Used for
// the combine that follows a split-KV kernel and for the one-warp split kernels when a combine
// follows them (sparse call: 15.0 -> 14.5 us with the combine alone, 14.1 us with both); the
// one-kernel SWA ring layers measured slower launched this way (14.9 -> 16.8-17.3 us per layer)
// and the four-warp GA kernels no faster, so those are launched plainly (pdl_wait is then a
// no-op).
template <typename P>
cudaError_t launch_pdl(void (*kern)(P), dim3 grid, int threads, size_t smem, cudaStream_t st, const P& prm,
                       bool pdl = true) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, prm);
}

// ---------------------------------------------------------------- decode
struct DecodePlan {
  int chunk, nchunks, direct;
  size_t bytes;
};

int pow2_floor(long long x) {
  int r = 1;
  while (static_cast<long long>(r) * 2 <= x && r < (1 << 30)) r *= 2;
  return r;
}

DecodePlan plan_decode(const mimo_shape* s, int mode, int cap, int recent, int n_sel, int sms) {
  DecodePlan pl{};
  const long long units = static_cast<long long>(s->batch) * s->n_kv_heads;
  long long total = mode == mimo::kModeSparse ? static_cast<long long>(recent) + n_sel : cap;
  if (total < 1) total = 1;
  if (mode == mimo::kModeSparse) {
    // about one wave of two CTAs per SM
    long long c = (total * units + 2LL * sms - 1) / (2LL * sms);
    int ch = pow2_floor(c);
    if (ch < c) ch *= 2;
    pl.chunk = ch < 64 ? 64 : (ch > mimo::kDecMaxTokList ? mimo::kDecMaxTokList : ch);
  } else if (total <= 256) {
    pl.chunk = static_cast<int>((total + 63) / 64 * 64);
  } else {
    // several waves so that uneven lengths balance
    const long long c = total * units / (16LL * sms);
    const int ch = pow2_floor(c);
    pl.chunk = ch < 256 ? 256 : (ch > 4096 ? 4096 : ch);
  }
  pl.nchunks = static_cast<int>((total + pl.chunk - 1) / pl.chunk);
  pl.direct = pl.nchunks == 1;
  if (pl.direct) {
    pl.bytes = 0;
  } else {
    const size_t rows = static_cast<size_t>(s->batch) * s->n_q_heads * pl.nchunks;
    const size_t ml = (rows * 2 * sizeof(float) + 255) / 256 * 256;
    pl.bytes = ml + rows * mimo::kDV * sizeof(float);
  }
  return pl;
}

// Plan of the bf16 decode calls. Units of at most 256 keys (the SWA ring) and sparse key lists
// run on decode_warp_kernel (one warp per CTA): a ring unit is one chunk finalised in place,
// with two stages of 32 keys in flight; a sparse unit is cut into chunks of 64 keys (both
// stages in flight at once) merged by the combine. Longer units (GA linear caches) use the
// four-warp decode_split_kernel plan (*stages = 0).
DecodePlan plan_decode_warp(const mimo_shape* s, int mode, int cap, int recent, int n_sel, int sms,
                            int* stages) {
  long long total = mode == mimo::kModeSparse ? static_cast<long long>(recent) + n_sel : cap;
  if (total < 1) total = 1;
  if (mode != mimo::kModeSparse && total > 256) {
    *stages = 0;
    return plan_decode(s, mode, cap, recent, n_sel, sms);
  }
  DecodePlan pl{};
  *stages = 2;
  pl.chunk = mode == mimo::kModeSparse ? 64 : static_cast<int>((total + 31) / 32 * 32);
  if (pl.chunk > total) pl.chunk = static_cast<int>((total + 31) / 32 * 32);
  pl.nchunks = static_cast<int>((total + pl.chunk - 1) / pl.chunk);
  pl.direct = pl.nchunks == 1;
  if (pl.direct) {
    pl.bytes = 0;
  } else {
    const size_t rows = static_cast<size_t>(s->batch) * s->n_q_heads * pl.nchunks;
    const size_t ml = (rows * 2 * sizeof(float) + 255) / 256 * 256;
    pl.bytes = ml + rows * mimo::kDV * sizeof(float);
  }
  return pl;
}

// Plan of the FP8 decode calls (decode_fp8_kernel, one warp per CTA): a sparse unit in chunks
// of 64 keys (two stages, both in flight); a ring unit of at most 256 keys in one chunk,
// finalised in place, with four stages of 32 keys in flight; a longer (linear) unit in chunks
// of 256 .. 2048 keys, about 32 CTAs per SM in all so that uneven lengths balance, with two
// stages in flight: 21 KB of shared memory per CTA, so that registers (eight warps per SM)
// rather than shared memory bound the warps an SM holds (measured: 0.65 of HBM against 0.55
// with four stages and 0.63 with three on the 9 GA layers of the FP8 decode step).
DecodePlan plan_decode_fp8(const mimo_shape* s, int mode, int cap, int recent, int n_sel, int sms,
                           int* stages) {
  long long total = mode == mimo::kModeSparse ? static_cast<long long>(recent) + n_sel : cap;
  if (total < 1) total = 1;
  const long long units = static_cast<long long>(s->batch) * s->n_kv_heads;
  DecodePlan pl{};
  if (mode == mimo::kModeSparse) {
    *stages = 2;
    pl.chunk = 64;
  } else if (total <= 256) {
    *stages = 4;
    pl.chunk = static_cast<int>((total + 31) / 32 * 32);
  } else {
    *stages = 2;
    const int ch = pow2_floor(total * units / (32LL * sms));
    pl.chunk = ch < 256 ? 256 : (ch > 2048 ? 2048 : ch);
  }
  if (pl.chunk > total) pl.chunk = static_cast<int>((total + 31) / 32 * 32);
  pl.nchunks = static_cast<int>((total + pl.chunk - 1) / pl.chunk);
  pl.direct = pl.nchunks == 1;
  if (pl.direct) {
    pl.bytes = 0;
  } else {
    const size_t rows = static_cast<size_t>(s->batch) * s->n_q_heads * pl.nchunks;
    const size_t ml = (rows * 2 * sizeof(float) + 255) / 256 * 256;
    pl.bytes = ml + rows * mimo::kDV * sizeof(float);
  }
  return pl;
}

template <int G, int NS>
mimo_status launch_decode_fp8_g(DecodeParams prm, cudaStream_t st) {
  auto kern = mimo::decode_fp8_kernel<G, NS>;
  const int smem = mimo::d8_smem_bytes(NS);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return MIMO_ERR_CUDA;
  }
  dim3 grid(prm.nchunks, prm.Hkv, prm.B);
  if (launch_pdl(kern, grid, 32, smem, st, prm, !prm.direct) != cudaSuccess) return MIMO_ERR_CUDA;
  if (!prm.direct &&
      launch_pdl(mimo::decode_combine_kernel, dim3(prm.B * prm.Hq), mimo::kDV, 0, st, prm) != cudaSuccess)
    return MIMO_ERR_CUDA;
  return MIMO_OK;
}

template <int G>
mimo_status launch_decode_fp8_gs(DecodeParams prm, cudaStream_t st) {
  return prm.nstages == 2 ? launch_decode_fp8_g<G, 2>(prm, st) : launch_decode_fp8_g<G, 4>(prm, st);
}

template <int G>
mimo_status launch_decode_warp_g(DecodeParams prm, cudaStream_t st) {
  auto kern = mimo::decode_warp_kernel<G, 2>;
  const int smem = mimo::dw_smem_bytes(2);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return MIMO_ERR_CUDA;
  }
  dim3 grid(prm.nchunks, prm.Hkv, prm.B);
  if (launch_pdl(kern, grid, 32, smem, st, prm, !prm.direct) != cudaSuccess) return MIMO_ERR_CUDA;
  if (!prm.direct &&
      launch_pdl(mimo::decode_combine_kernel, dim3(prm.B * prm.Hq), mimo::kDV, 0, st, prm) != cudaSuccess)
    return MIMO_ERR_CUDA;
  return MIMO_OK;
}

template <int G>
mimo_status launch_decode_g(DecodeParams prm, cudaStream_t st) {
  auto kern = mimo::decode_split_kernel<G>;
  const int smem = mimo::kDecSmemBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return MIMO_ERR_CUDA;
  }
  dim3 grid(prm.nchunks, prm.Hkv, prm.B);
  if (launch_pdl(kern, grid, mimo::kDecThreads, smem, st, prm, false) != cudaSuccess) return MIMO_ERR_CUDA;
  if (!prm.direct &&
      launch_pdl(mimo::decode_combine_kernel, dim3(prm.B * prm.Hq), mimo::kDV, 0, st, prm) != cudaSuccess)
    return MIMO_ERR_CUDA;
  return MIMO_OK;
}

// FP8 caches: kc / vc are E4M3 bytes and ks / vs their per-(token, KV head) fp32 scales.
mimo_status run_decode(const mimo_shape* s, int mode, const void* q, const void* kc, const void* vc,
                       int cap, long long stride, const int* lengths, int recent, const int* sel,
                       int n_sel, const float* sink, void* out, float* lse, void* ws, size_t ws_bytes,
                       void* stream, bool fp8 = false, const float* ks = nullptr,
                       const float* vs = nullptr) {
  mimo_status e = check_heads(s);
  if (e != MIMO_OK) return e;
  if (!q || !kc || !vc || !lengths || !out) return MIMO_ERR_NULL;
  if (fp8 && (!ks || !vs)) return MIMO_ERR_NULL;
  if (fp8 && (!aligned(ks, 4) || !aligned(vs, 4))) return MIMO_ERR_ALIGN;
  if (mode == mimo::kModeSparse && n_sel > 0 && !sel) return MIMO_ERR_NULL;
  if (cap < 1 || stride < cap) return MIMO_ERR_SHAPE;
  if (mode == mimo::kModeSparse && (recent < 0 || n_sel < 0)) return MIMO_ERR_SHAPE;
  if (!aligned(q, 16) || !aligned(kc, 16) || !aligned(vc, 16) || !aligned(out, 16) ||
      !aligned(lengths, 4) || (sel && !aligned(sel, 4)) || (sink && !aligned(sink, 4)) ||
      (lse && !aligned(lse, 4)))
    return MIMO_ERR_ALIGN;
  const int dev = current_device();
  if (dev < 0) return MIMO_ERR_CUDA;
  const int sms = sm_count_for(dev);
  int stages = 2;
  const DecodePlan pl = fp8 ? plan_decode_fp8(s, mode, cap, recent, n_sel, sms, &stages)
                            : plan_decode_warp(s, mode, cap, recent, n_sel, sms, &stages);
  if (pl.bytes > 0 && (!ws || ws_bytes < pl.bytes)) return MIMO_ERR_WORKSPACE;
  if (ws && !aligned(ws, 16)) return MIMO_ERR_ALIGN;
  DecodeParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(q);
  if (fp8) {
    prm.k8 = static_cast<const uint8_t*>(kc);
    prm.v8 = static_cast<const uint8_t*>(vc);
    prm.k_scale = ks;
    prm.v_scale = vs;
  } else {
    prm.k = static_cast<const __nv_bfloat16*>(kc);
    prm.v = static_cast<const __nv_bfloat16*>(vc);
  }
  prm.lengths = lengths;
  prm.sel = sel;
  prm.sink = sink;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  if (pl.bytes > 0) {
    const size_t rows = static_cast<size_t>(s->batch) * s->n_q_heads * pl.nchunks;
    const size_t ml = (rows * 2 * sizeof(float) + 255) / 256 * 256;
    prm.part_ml = static_cast<float*>(ws);
    prm.part_o = reinterpret_cast<float*>(static_cast<char*>(ws) + ml);
  }
  prm.seq_stride = stride;
  prm.B = s->batch;
  prm.Hq = s->n_q_heads;
  prm.Hkv = s->n_kv_heads;
  prm.group = s->n_q_heads / s->n_kv_heads;
  prm.cap = cap;
  prm.mode = mode;
  prm.chunk = pl.chunk;
  prm.nchunks = pl.nchunks;
  prm.recent = recent;
  prm.n_sel = n_sel;
  prm.direct = pl.direct;
  prm.nstages = stages;
  prm.scale_log2 = scale_log2_of(s);
  prm.err = device_error_ptr(dev);
  if (!prm.err) return MIMO_ERR_CUDA;
  if (s->n_kv_heads > 65535) return MIMO_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!fp8 && stages > 0) {
    switch (prm.group) {
      case 1: return launch_decode_warp_g<1>(prm, st);
      case 2: return launch_decode_warp_g<2>(prm, st);
      case 4: return launch_decode_warp_g<4>(prm, st);
      case 8: return launch_decode_warp_g<8>(prm, st);
      default: return launch_decode_warp_g<16>(prm, st);
    }
  }
  if (fp8) {
    switch (prm.group) {
      case 1: return launch_decode_fp8_gs<1>(prm, st);
      case 2: return launch_decode_fp8_gs<2>(prm, st);
      case 4: return launch_decode_fp8_gs<4>(prm, st);
      case 8: return launch_decode_fp8_gs<8>(prm, st);
      default: return launch_decode_fp8_gs<16>(prm, st);
    }
  }
  switch (prm.group) {
    case 1: return launch_decode_g<1>(prm, st);
    case 2: return launch_decode_g<2>(prm, st);
    case 4: return launch_decode_g<4>(prm, st);
    case 8: return launch_decode_g<8>(prm, st);
    default: return launch_decode_g<16>(prm, st);
  }
}

// ---------------------------------------------------------------- multi-query decode
DecodePlan plan_decode_mq(const mimo_shape* s, int mode, int cap, int T, int W, int sms) {
  DecodePlan pl{};
  const long long units = static_cast<long long>(s->batch) * s->n_kv_heads;
  long long total = mode == mimo::kModeRing ? std::min<long long>(cap, static_cast<long long>(W) + T - 1) : cap;
  if (total < 1) total = 1;
  if (total <= 256) {
    pl.chunk = static_cast<int>((total + 63) / 64 * 64);
  } else {
    // linear caches: long chunks, since each CTA of the TMA kernel holds an SM and drains its
    // pipeline at the end (8192-key chunks measured 2% faster than 4096, 2048 slower)
    const long long c = total * units / (16LL * sms);
    const int ch = pow2_floor(c);
    pl.chunk = ch < 256 ? 256 : (ch > 8192 ? 8192 : ch);
  }
  pl.nchunks = static_cast<int>((total + pl.chunk - 1) / pl.chunk);
  pl.direct = pl.nchunks == 1;
  if (!pl.direct) {
    const size_t rows = static_cast<size_t>(s->batch) * T * s->n_q_heads * pl.nchunks;
    const size_t ml = (rows * 2 * sizeof(float) + 255) / 256 * 256;
    pl.bytes = ml + rows * mimo::kDV * sizeof(float);
  }
  return pl;
}

mimo_status check_mq(const mimo_shape* s, int cache_kind, int cap, int T, int W) {
  mimo_status e = check_heads(s);
  if (e != MIMO_OK) return e;
  if (cache_kind != MIMO_CACHE_RING && cache_kind != MIMO_CACHE_LINEAR) return MIMO_ERR_SHAPE;
  if (T < 1 || cap < 1) return MIMO_ERR_SHAPE;
  if (static_cast<long long>(T) * (s->n_q_heads / s->n_kv_heads) > mimo::kMqMaxRows) return MIMO_ERR_UNSUPPORTED;
  if (cache_kind == MIMO_CACHE_RING && (W < 1 || static_cast<long long>(W) + T - 1 > cap)) return MIMO_ERR_SHAPE;
  return MIMO_OK;
}

// Multi-query decode over a linear (GA) cache: decode_mq_tma_kernel (TMA-fed K/V subtiles,
// S and PV on tcgen05, O in TMEM, one CTA per SM). Ring caches, whose subtiles wrap around the
// ring, stay on decode_mq_kernel (cp.async gathers, mma.sync).
template <int G>
mimo_status launch_decode_mq_tma_g(const mimo::DecodeMqParams& prm, cudaStream_t st) {
  CUtensorMap tk, tv;
  if (!make_tmap(&tk, prm.k, mimo::kDQK, prm.Hkv, prm.seq_stride, prm.B, 1, mimo::kMtKeys) ||
      !make_tmap(&tv, prm.v, mimo::kDV, prm.Hkv, prm.seq_stride, prm.B, 1, mimo::kMtKeys))
    return MIMO_ERR_CUDA;
  auto kern = mimo::decode_mq_tma_kernel<G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mimo::kMtSmemBytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return MIMO_ERR_CUDA;
  }
  dim3 grid(prm.nchunks, prm.Hkv, prm.B);
#ifdef MIMO_TRACE
  const_cast<mimo::DecodeMqParams&>(prm).trace = g_trace;
#endif
  kern<<<grid, mimo::kMtThreads, mimo::kMtSmemBytes, st>>>(tk, tv, prm);
  if (cudaGetLastError() != cudaSuccess) return MIMO_ERR_CUDA;
  if (!prm.direct) {
    const long long rows = static_cast<long long>(prm.B) * prm.T * prm.Hq;
    if (rows > 0x7fffffffLL) return MIMO_ERR_UNSUPPORTED;
    if (launch_pdl(mimo::decode_mq_combine_kernel, dim3(static_cast<unsigned>(rows)), mimo::kDV, 0, st, prm) !=
        cudaSuccess)
      return MIMO_ERR_CUDA;
  }
  return MIMO_OK;
}

// Ring caches: decode_mq_kernel with 32-key subtiles (two stages: 40 KB of shared memory) and
// as many warps as 16-row tiles of the T * G rows (2 for the MTP step's SWA layers, 4 above 32
// rows), so the 131-slot units of a layer fit in one wave.
template <int G, int NW>
mimo_status launch_decode_mq_ring(const mimo::DecodeMqParams& prm, cudaStream_t st) {
  constexpr int kSub = 32;
  auto kern = mimo::decode_mq_kernel<G, NW, kSub>;
  const int smem = 2 * kSub * (mimo::kKRow + mimo::kVRow);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return MIMO_ERR_CUDA;
  }
  dim3 grid(prm.nchunks, prm.Hkv, prm.B);
  if (launch_pdl(kern, grid, NW * 32, smem, st, prm, false) != cudaSuccess) return MIMO_ERR_CUDA;
  if (!prm.direct) {
    const long long rows = static_cast<long long>(prm.B) * prm.T * prm.Hq;
    if (rows > 0x7fffffffLL) return MIMO_ERR_UNSUPPORTED;
    if (launch_pdl(mimo::decode_mq_combine_kernel, dim3(static_cast<unsigned>(rows)), mimo::kDV, 0, st, prm) !=
        cudaSuccess)
      return MIMO_ERR_CUDA;
  }
  return MIMO_OK;
}

template <int G>
mimo_status launch_decode_mq_g(const mimo::DecodeMqParams& prm, cudaStream_t st) {
  if (prm.mode == mimo::kModeLinear) return launch_decode_mq_tma_g<G>(prm, st);
  if (prm.T * G <= 32) return launch_decode_mq_ring<G, 2>(prm, st);
  return launch_decode_mq_ring<G, 4>(prm, st);
}

}  // namespace

// ============================================================== C ABI
extern "C" {

mimo_status mimo_attn_prefill(const mimo_shape* s, const void* q, const void* k, const void* v,
                              const float* sink, int window, float rope_theta, int rot_dims,
                              void* out, float* lse, void* stream) {
  mimo_status e = check_heads(s);
  if (e != MIMO_OK) return e;
  if (!q || !k || !v || !out) return MIMO_ERR_NULL;
  if (s->seqlen < 1) return MIMO_ERR_SHAPE;
  if (rot_dims < 0 || rot_dims > mimo::kDQK) return MIMO_ERR_SHAPE;
  if (rot_dims % 16) return MIMO_ERR_UNSUPPORTED;
  if (rot_dims > 0 && !(rope_theta > 0.f && std::isfinite(rope_theta))) return MIMO_ERR_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (sink && !aligned(sink, 4)) || (lse && !aligned(lse, 4)))
    return MIMO_ERR_ALIGN;
  const int dev = current_device();
  if (dev < 0) return MIMO_ERR_CUDA;
  PrefillParams prm{};
  prm.sink = sink;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.B = s->batch;
  prm.n = s->seqlen;
  prm.Hq = s->n_q_heads;
  prm.Hkv = s->n_kv_heads;
  prm.window = window;
  prm.rot_dims = rot_dims;
  prm.rope_theta = static_cast<double>(rope_theta);
  prm.scale_log2 = scale_log2_of(s);
  prm.q_off = 0;
  prm.nk = s->seqlen;
  prm.krot_from = 0;
  prm.err = device_error_ptr(dev);
  if (!prm.err) return MIMO_ERR_CUDA;
#ifdef MIMO_TRACE
  prm.trace = g_trace;
#endif
  const int sms = sm_count_for(dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (s->n_q_heads / s->n_kv_heads) {
    case 1: return prefill_group<1>(s, q, k, v, prm, sms, st);
    case 2: return prefill_group<2>(s, q, k, v, prm, sms, st);
    case 4: return prefill_group<4>(s, q, k, v, prm, sms, st);
    case 8: return prefill_group<8>(s, q, k, v, prm, sms, st);
    default: return prefill_group<16>(s, q, k, v, prm, sms, st);
  }
}

mimo_status mimo_attn_prefill_chunk(const mimo_shape* s, const void* q, const void* k, const void* v,
                                    int pos_offset, int k_prefix_rotated, const float* sink,
                                    int window, float rope_theta, int rot_dims, void* out,
                                    float* lse, void* stream) {
  mimo_status e = check_heads(s);
  if (e != MIMO_OK) return e;
  if (!q || !k || !v || !out) return MIMO_ERR_NULL;
  if (s->seqlen < 1 || pos_offset < 0) return MIMO_ERR_SHAPE;
  if (static_cast<long long>(pos_offset) + s->seqlen > 0x7fffffffLL) return MIMO_ERR_UNSUPPORTED;
  if (rot_dims < 0 || rot_dims > mimo::kDQK) return MIMO_ERR_SHAPE;
  if (rot_dims % 16) return MIMO_ERR_UNSUPPORTED;
  if (rot_dims > 0 && !(rope_theta > 0.f && std::isfinite(rope_theta))) return MIMO_ERR_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (sink && !aligned(sink, 4)) || (lse && !aligned(lse, 4)))
    return MIMO_ERR_ALIGN;
  const int dev = current_device();
  if (dev < 0) return MIMO_ERR_CUDA;
  PrefillParams prm{};
  prm.sink = sink;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.B = s->batch;
  prm.n = s->seqlen;
  prm.Hq = s->n_q_heads;
  prm.Hkv = s->n_kv_heads;
  prm.window = window;
  prm.rot_dims = rot_dims;
  prm.rope_theta = static_cast<double>(rope_theta);
  prm.scale_log2 = scale_log2_of(s);
  prm.q_off = pos_offset;
  prm.nk = pos_offset + s->seqlen;
  prm.krot_from = k_prefix_rotated ? pos_offset : 0;
  prm.err = device_error_ptr(dev);
  if (!prm.err) return MIMO_ERR_CUDA;
  const int sms = sm_count_for(dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (s->n_q_heads / s->n_kv_heads) {
    case 1: return prefill_chunk_group<1>(s, q, k, v, prm, sms, st);
    case 2: return prefill_chunk_group<2>(s, q, k, v, prm, sms, st);
    case 4: return prefill_chunk_group<4>(s, q, k, v, prm, sms, st);
    case 8: return prefill_chunk_group<8>(s, q, k, v, prm, sms, st);
    default: return prefill_chunk_group<16>(s, q, k, v, prm, sms, st);
  }
}

mimo_status mimo_attn_cache_append(const mimo_shape* s, const void* k_chunk, const void* v_chunk,
                                   int pos_offset, float rope_theta, int rot_dims, int cache_kind,
                                   void* k_cache, void* v_cache, int cache_capacity,
                                   long long seq_stride_tokens, void* stream) {
  mimo_status e = check_heads(s);
  if (e != MIMO_OK) return e;
  if (!k_chunk || !v_chunk || !k_cache || !v_cache) return MIMO_ERR_NULL;
  if (cache_kind != MIMO_CACHE_RING && cache_kind != MIMO_CACHE_LINEAR) return MIMO_ERR_SHAPE;
  if (s->seqlen < 1 || pos_offset < 0 || cache_capacity < 1 || seq_stride_tokens < cache_capacity)
    return MIMO_ERR_SHAPE;
  if (cache_kind == MIMO_CACHE_LINEAR && static_cast<long long>(pos_offset) + s->seqlen > cache_capacity)
    return MIMO_ERR_SHAPE;
  if (static_cast<long long>(pos_offset) + s->seqlen > 0x7fffffffLL) return MIMO_ERR_UNSUPPORTED;
  if (rot_dims < 0 || rot_dims > mimo::kDQK) return MIMO_ERR_SHAPE;
  if (rot_dims % 16) return MIMO_ERR_UNSUPPORTED;
  if (rot_dims > 0 && !(rope_theta > 0.f && std::isfinite(rope_theta))) return MIMO_ERR_SHAPE;
  if (!aligned(k_chunk, 16) || !aligned(v_chunk, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return MIMO_ERR_ALIGN;
  const int dev = current_device();
  if (dev < 0) return MIMO_ERR_CUDA;
  mimo::CacheAppendParams prm{};
  prm.k = static_cast<const __nv_bfloat16*>(k_chunk);
  prm.v = static_cast<const __nv_bfloat16*>(v_chunk);
  prm.kc = static_cast<__nv_bfloat16*>(k_cache);
  prm.vc = static_cast<__nv_bfloat16*>(v_cache);
  prm.stride = seq_stride_tokens;
  prm.B = s->batch;
  prm.n = s->seqlen;
  prm.Hkv = s->n_kv_heads;
  prm.off = pos_offset;
  prm.rot = rot_dims;
  prm.ring = cache_kind == MIMO_CACHE_RING;
  prm.cap = cache_capacity;
  prm.theta = static_cast<double>(rope_theta);
  const long long items = static_cast<long long>(s->batch) * s->seqlen * s->n_kv_heads * 40;
  const long long blocks = std::min<long long>((items + 255) / 256, 4LL * sm_count_for(dev));
  mimo::cache_append_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(prm);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

size_t mimo_attn_select_workspace_size(const mimo_shape* s, int cache_capacity) {
  if (check_heads(s) != MIMO_OK || cache_capacity < 1) return 0;
  // score keys [B, Hkv, round_up(cap, 4)] u32, then top-byte histograms [B, Hkv, chunks, 256] u16
  const size_t bg = static_cast<size_t>(s->batch) * s->n_kv_heads;
  const size_t keys = bg * ((static_cast<size_t>(cache_capacity) + 3) / 4 * 4) * sizeof(uint32_t);
  const size_t chunks = (static_cast<size_t>(cache_capacity) + mimo::kSelChunk - 1) / mimo::kSelChunk;
  const size_t n = keys + bg * chunks * 256 * sizeof(uint16_t);
  return (n + 255) / 256 * 256;
}

mimo_status mimo_attn_select_tokens(const mimo_shape* s, const void* q, const void* k_cache,
                                    int cache_capacity, long long seq_stride_tokens,
                                    const int* lengths, int recent, int n_sel, int* sel_idx,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  mimo_status e = check_heads(s);
  if (e != MIMO_OK) return e;
  if (!q || !k_cache || !lengths || (n_sel > 0 && !sel_idx)) return MIMO_ERR_NULL;
  if (cache_capacity < 1 || seq_stride_tokens < cache_capacity || recent < 0 || n_sel < 0)
    return MIMO_ERR_SHAPE;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(lengths, 4) || (sel_idx && !aligned(sel_idx, 4)))
    return MIMO_ERR_ALIGN;
  const size_t need = mimo_attn_select_workspace_size(s, cache_capacity);
  if (!workspace || workspace_bytes < need) return MIMO_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return MIMO_ERR_ALIGN;
  if (n_sel == 0) return MIMO_OK;
  if (s->n_kv_heads > 65535 || s->batch > 65535) return MIMO_ERR_UNSUPPORTED;
  if (current_device() < 0) return MIMO_ERR_CUDA;
  mimo::SelectParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k = static_cast<const __nv_bfloat16*>(k_cache);
  prm.lengths = lengths;
  prm.keys = static_cast<uint32_t*>(workspace);
  prm.key_stride = (cache_capacity + 3) / 4 * 4;
  prm.n_chunks = (cache_capacity + mimo::kSelChunk - 1) / mimo::kSelChunk;
  prm.hist = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) +
                                         static_cast<size_t>(s->batch) * s->n_kv_heads * prm.key_stride * 4);
  prm.sel = sel_idx;
  prm.seq_stride = seq_stride_tokens;
  prm.B = s->batch;
  prm.Hq = s->n_q_heads;
  prm.Hkv = s->n_kv_heads;
  prm.cap = cache_capacity;
  prm.recent = recent;
  prm.n_sel = n_sel;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int cand = std::max(1, cache_capacity - recent);
  const dim3 grid((cand + mimo::kSelChunk - 1) / mimo::kSelChunk, s->n_kv_heads, s->batch);
  auto launch = [&](auto kern) -> bool {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mimo::kSelScoreSmem) !=
        cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    kern<<<grid, mimo::kDecThreads, mimo::kSelScoreSmem, st>>>(prm);
    return true;
  };
  bool launched;
  switch (s->n_q_heads / s->n_kv_heads) {
    case 1: launched = launch(mimo::select_score_kernel<1>); break;
    case 2: launched = launch(mimo::select_score_kernel<2>); break;
    case 4: launched = launch(mimo::select_score_kernel<4>); break;
    case 8: launched = launch(mimo::select_score_kernel<8>); break;
    default: launched = launch(mimo::select_score_kernel<16>); break;
  }
  if (!launched) return MIMO_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return MIMO_ERR_CUDA;
  // top-k: a cluster of kSelCluster CTAs per (b, g) for long caches (each slice then holds
  // tens of thousands of keys), one CTA per (b, g) below that (small slices cost more in
  // cluster barriers and loop overhead than they save)
  if (cache_capacity >= mimo::kSelClusterMinCap) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(s->n_kv_heads * mimo::kSelCluster, s->batch);
    cfg.blockDim = dim3(mimo::kSelThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = mimo::kSelCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mimo::select_topk_kernel<mimo::kSelCluster>, prm) != cudaSuccess) return MIMO_ERR_CUDA;
  } else {
    mimo::select_topk_kernel<1><<<dim3(s->n_kv_heads, s->batch), mimo::kSelThreads, 0, st>>>(prm);
  }
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

mimo_status mimo_attn_decode(const mimo_shape* s, const void* q, const void* k_cache,
                             const void* v_cache, int cache_kind, int cache_capacity,
                             long long seq_stride_tokens, const int* lengths, const float* sink,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (cache_kind != MIMO_CACHE_RING && cache_kind != MIMO_CACHE_LINEAR) return MIMO_ERR_SHAPE;
  const int mode = cache_kind == MIMO_CACHE_RING ? mimo::kModeRing : mimo::kModeLinear;
  return run_decode(s, mode, q, k_cache, v_cache, cache_capacity, seq_stride_tokens, lengths, 0,
                    nullptr, 0, sink, out, lse, workspace, workspace_bytes, stream);
}

mimo_status mimo_attn_sparse(const mimo_shape* s, const void* q, const void* k_cache,
                             const void* v_cache, int cache_capacity, long long seq_stride_tokens,
                             const int* lengths, int recent, const int* sel_idx, int n_sel,
                             const float* sink, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream) {
  return run_decode(s, mimo::kModeSparse, q, k_cache, v_cache, cache_capacity, seq_stride_tokens,
                    lengths, recent, sel_idx, n_sel, sink, out, lse, workspace, workspace_bytes,
                    stream);
}

mimo_status mimo_attn_decode_mq(const mimo_shape* s, const void* q, const void* k_cache,
                                const void* v_cache, int cache_kind, int cache_capacity,
                                long long seq_stride_tokens, const int* lengths, int q_len,
                                int window, const float* sink, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream) {
  mimo_status e = check_mq(s, cache_kind, cache_capacity, q_len, window);
  if (e != MIMO_OK) return e;
  if (!q || !k_cache || !v_cache || !lengths || !out) return MIMO_ERR_NULL;
  if (seq_stride_tokens < cache_capacity) return MIMO_ERR_SHAPE;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(lengths, 4) || (sink && !aligned(sink, 4)) || (lse && !aligned(lse, 4)))
    return MIMO_ERR_ALIGN;
  const int dev = current_device();
  if (dev < 0) return MIMO_ERR_CUDA;
  const int mode = cache_kind == MIMO_CACHE_RING ? mimo::kModeRing : mimo::kModeLinear;
  const DecodePlan pl = plan_decode_mq(s, mode, cache_capacity, q_len, window, sm_count_for(dev));
  if (pl.bytes > 0 && (!workspace || workspace_bytes < pl.bytes)) return MIMO_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 16)) return MIMO_ERR_ALIGN;
  if (s->n_kv_heads > 65535) return MIMO_ERR_UNSUPPORTED;
  mimo::DecodeMqParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.k = static_cast<const __nv_bfloat16*>(k_cache);
  prm.v = static_cast<const __nv_bfloat16*>(v_cache);
  prm.lengths = lengths;
  prm.sink = sink;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  if (pl.bytes > 0) {
    const size_t rows = static_cast<size_t>(s->batch) * q_len * s->n_q_heads * pl.nchunks;
    const size_t ml = (rows * 2 * sizeof(float) + 255) / 256 * 256;
    prm.part_ml = static_cast<float*>(workspace);
    prm.part_o = reinterpret_cast<float*>(static_cast<char*>(workspace) + ml);
  }
  prm.seq_stride = seq_stride_tokens;
  prm.B = s->batch;
  prm.T = q_len;
  prm.Hq = s->n_q_heads;
  prm.Hkv = s->n_kv_heads;
  prm.cap = cache_capacity;
  prm.mode = mode;
  prm.window = window;
  prm.chunk = pl.chunk;
  prm.nchunks = pl.nchunks;
  prm.direct = pl.direct;
  prm.scale_log2 = scale_log2_of(s);
  prm.err = device_error_ptr(dev);
  if (!prm.err) return MIMO_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (s->n_q_heads / s->n_kv_heads) {
    case 1: return launch_decode_mq_g<1>(prm, st);
    case 2: return launch_decode_mq_g<2>(prm, st);
    case 4: return launch_decode_mq_g<4>(prm, st);
    case 8: return launch_decode_mq_g<8>(prm, st);
    default: return launch_decode_mq_g<16>(prm, st);
  }
}

size_t mimo_attn_decode_mq_workspace_size(const mimo_shape* s, int cache_kind, int cache_capacity,
                                          int q_len, int window) {
  if (check_mq(s, cache_kind, cache_capacity, q_len, window) != MIMO_OK) return 0;
  const int mode = cache_kind == MIMO_CACHE_RING ? mimo::kModeRing : mimo::kModeLinear;
  return plan_decode_mq(s, mode, cache_capacity, q_len, window, sm_count_for(current_device())).bytes;
}

mimo_status mimo_attn_decode_fp8(const mimo_shape* s, const void* q, const void* k_cache,
                                 const void* v_cache, const float* k_scale, const float* v_scale,
                                 int cache_kind, int cache_capacity, long long seq_stride_tokens,
                                 const int* lengths, const float* sink, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  if (cache_kind != MIMO_CACHE_RING && cache_kind != MIMO_CACHE_LINEAR) return MIMO_ERR_SHAPE;
  const int mode = cache_kind == MIMO_CACHE_RING ? mimo::kModeRing : mimo::kModeLinear;
  return run_decode(s, mode, q, k_cache, v_cache, cache_capacity, seq_stride_tokens, lengths, 0,
                    nullptr, 0, sink, out, lse, workspace, workspace_bytes, stream, true, k_scale,
                    v_scale);
}

mimo_status mimo_attn_sparse_fp8(const mimo_shape* s, const void* q, const void* k_cache,
                                 const void* v_cache, const float* k_scale, const float* v_scale,
                                 int cache_capacity, long long seq_stride_tokens, const int* lengths,
                                 int recent, const int* sel_idx, int n_sel, const float* sink,
                                 void* out, float* lse, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  return run_decode(s, mimo::kModeSparse, q, k_cache, v_cache, cache_capacity, seq_stride_tokens,
                    lengths, recent, sel_idx, n_sel, sink, out, lse, workspace, workspace_bytes,
                    stream, true, k_scale, v_scale);
}

size_t mimo_attn_workspace_size(const mimo_shape* s, int op, int cache_kind, int cache_capacity,
                                int recent, int n_sel) {
  if (check_heads(s) != MIMO_OK || cache_capacity < 1) return 0;
  int mode;
  if (op == MIMO_OP_SPARSE) {
    if (recent < 0 || n_sel < 0) return 0;
    mode = mimo::kModeSparse;
  } else if (op == MIMO_OP_DECODE) {
    if (cache_kind == MIMO_CACHE_RING) mode = mimo::kModeRing;
    else if (cache_kind == MIMO_CACHE_LINEAR) mode = mimo::kModeLinear;
    else return 0;
  } else {
    return 0;
  }
  // one size serves both the bf16 calls and the FP8 calls
  const int sms = sm_count_for(current_device());
  int stages = 2;
  return std::max(plan_decode_warp(s, mode, cache_capacity, recent, n_sel, sms, &stages).bytes,
                  plan_decode_fp8(s, mode, cache_capacity, recent, n_sel, sms, &stages).bytes);
}

mimo_status mimo_attn_check_indices(const mimo_shape* s, const int* lengths, const int* sel_idx,
                                    int n_sel, int recent, int cache_capacity,
                                    unsigned int* d_violations, void* stream) {
  if (!s) return MIMO_ERR_NULL;
  if (s->batch < 1 || s->n_kv_heads < 1 || n_sel < 0 || recent < 0 || cache_capacity < 1)
    return MIMO_ERR_SHAPE;
  if (!lengths || !d_violations || (n_sel > 0 && !sel_idx)) return MIMO_ERR_NULL;
  const int rows = s->batch * s->n_kv_heads;
  mimo::check_indices_kernel<<<(rows + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      lengths, sel_idx, s->batch, s->n_kv_heads, n_sel, recent, cache_capacity, d_violations);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}

unsigned int mimo_attn_last_device_error(void) {
  unsigned v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return 0xFFFFFFFFu;
  }
  if (cudaMemcpyFromSymbol(&v, mimo::g_device_error, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return 0xFFFFFFFFu;
  }
  const unsigned zero = 0;
  cudaMemcpyToSymbol(mimo::g_device_error, &zero, sizeof(zero));
  return v;
}

mimo_status mimo_attn_device_status(unsigned int* word) {
  const unsigned v = mimo_attn_last_device_error();
  if (word) *word = v;
  if (v == 0xFFFFFFFFu) return MIMO_ERR_CUDA;
  return v ? MIMO_ERR_DEVICE : MIMO_OK;
}

const char* mimo_status_string(mimo_status st) {
  switch (st) {
    case MIMO_OK: return "ok";
    case MIMO_ERR_NULL: return "a required pointer is NULL";
    case MIMO_ERR_SHAPE: return "sizes inconsistent or out of range";
    case MIMO_ERR_UNSUPPORTED: return "unsupported head dims, group size or rot_dims";
    case MIMO_ERR_ALIGN: return "misaligned data pointer";
    case MIMO_ERR_WORKSPACE: return "workspace missing or too small";
    case MIMO_ERR_CUDA: return "CUDA error";
    case MIMO_ERR_DEVICE: return "a kernel reported an error in the device error word";
  }
  return "unknown status";
}

int mimo_attn_version(void) { return 100; }

#ifdef MIMO_TEST_HOOKS
int mimo_attn_test_stuck_wait(void* stream) {
  const int dev = current_device();
  unsigned* err = dev < 0 ? nullptr : device_error_ptr(dev);
  if (!err) return MIMO_ERR_CUDA;
  mimo::stuck_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err);
  return cudaGetLastError() == cudaSuccess ? MIMO_OK : MIMO_ERR_CUDA;
}
#endif

}  // extern "C"

// ============================================================== allocation-free sparse decode
// The split-KV partials of mimo_attn_sparse_noalloc live in this library-owned array
// instead of a caller workspace. Host code must not pass the symbol itself to a kernel:
// on the host it names a stand-in, not device memory. The device address is looked up
// with cudaGetSymbolAddress (that device current) once per device and context, and cached.
static __device__ __align__(256) unsigned char g_sparse_noalloc_scratch[MIMO_SPARSE_NOALLOC_SCRATCH_BYTES];

namespace {
SymbolAddressCache g_noalloc_cache;

void* noalloc_scratch(int dev) {
  return cached_symbol_address(g_noalloc_cache, g_sparse_noalloc_scratch, dev);
}
}  // namespace

extern "C" mimo_status mimo_attn_sparse_noalloc(const mimo_shape* s, const void* q,
                                                const void* k_cache, const void* v_cache,
                                                int cache_capacity, long long seq_stride_tokens,
                                                const int* lengths, int recent, const int* sel_idx,
                                                int n_sel, const float* sink, void* out, float* lse,
                                                void* stream) {
  mimo_status e = check_heads(s);
  if (e != MIMO_OK) return e;
  if (cache_capacity < 1 || recent < 0 || n_sel < 0) return MIMO_ERR_SHAPE;
  const int dev = current_device();
  if (dev < 0) return MIMO_ERR_CUDA;
  int stages = 2;
  const size_t need =
      plan_decode_warp(s, mimo::kModeSparse, cache_capacity, recent, n_sel, sm_count_for(dev), &stages).bytes;
  if (need > MIMO_SPARSE_NOALLOC_SCRATCH_BYTES) return MIMO_ERR_WORKSPACE;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  if (need > 0) {
    ws = noalloc_scratch(dev);
    if (!ws) return MIMO_ERR_CUDA;
    ws_bytes = MIMO_SPARSE_NOALLOC_SCRATCH_BYTES;
  }
  return run_decode(s, mimo::kModeSparse, q, k_cache, v_cache, cache_capacity, seq_stride_tokens,
                    lengths, recent, sel_idx, n_sel, sink, out, lse, ws, ws_bytes, stream);
}
