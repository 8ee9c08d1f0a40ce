/*
 * mimo_attn.h - C ABI of libmimo_attn.so: attention-sink softmax attention for
 * hybrid sliding-window (SWA) / global (GA) decoder layers on NVIDIA B200 (sm_100a).
 *
 * What is computed ("MiMo-V2-Flash: Hybrid Sliding Window Attention
 * Architecture", §4.4 and §5 steps 2-5). For query i, query head h and its key
 * set J_i:
 *
 *   a_ij = (q_i . k_j) * scale                           (§1.2, scale = 1/sqrt(192))
 *   m_i  = max(sink_h, max_{j in J_i} a_ij)
 *   s_ij = exp(a_ij - m_i) / (exp(sink_h - m_i) + sum_{j' in J_i} exp(a_ij' - m_i))
 *   o_i  = sum_{j in J_i} s_ij v_j                        (the sink has no value vector)
 *   lse_i = m_i + ln(exp(sink_h - m_i) + sum_j exp(a_ij - m_i))   (natural log, sink included)
 *
 * J_i is the causal window W(i) = [max(0, i-W+1), i] on SWA layers (§2.1, 0-based)
 * or the causal prefix [0, i] on GA layers. A NULL sink means exp(sink) = 0.
 *
 * Conventions shared by every call:
 *  - bf16 tensors are passed as pointers to raw bf16 bits (__nv_bfloat16), row-major,
 *    contiguous in the layout stated per argument. fp32 tensors are float.
 *  - Every data pointer is a DEVICE pointer on the current CUDA device and must be
 *    16-byte aligned (MIMO_ERR_ALIGN otherwise). `stream` is a cudaStream_t
 *    (NULL = legacy default stream).
 *  - Ownership: the caller owns every buffer. The library never allocates, frees
 *    or synchronises; all work is enqueued on `stream` and the call returns
 *    immediately.
 *  - Errors: arguments are checked on the host before any launch; on error nothing
 *    is launched and a status other than MIMO_OK is returned. A failed launch maps
 *    to MIMO_ERR_CUDA. Contents of device arrays (lengths, indices) are not checked
 *    by the fast path; kernels clamp them so that no access leaves the caller's
 *    buffers, and mimo_attn_check_indices reports violations.
 *  - Supported head dims: head_dim_qk = 192, head_dim_v = 128. n_q_heads must be a
 *    multiple of n_kv_heads with group n_q_heads / n_kv_heads in {1, 2, 4, 8, 16};
 *    query head h reads KV head h / group (contiguous groups).
 *  - Precision: products of bf16 inputs are exact and accumulate in fp32. The RoPE-rotated
 *    Q/K dims (prefill) are carried in f16 for their MMAs, and the SWA prefill kernel keeps
 *    P and V in f16; inputs are therefore expected inside the f16 range (|x| <= 65504, and
 *    a rotated pair's norm too) - values outside it are clamped. The FP8 decode converts Q
 *    to f16 without clamping (a larger |q| becomes infinite). A build compiled with
 *    MIMO_DEBUG records every such value in the device error word (bit 16, see
 *    mimo_attn_last_device_error). Outputs are rounded to bf16, lse is fp32.
 *  - Thread safety: calls may be made from several host threads; the shared mutable
 *    state is the device error word read by mimo_attn_last_device_error and the scratch
 *    array of mimo_attn_sparse_noalloc (see there).
 */
#ifndef MIMO_ATTN_H
#define MIMO_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mimo_status {
  MIMO_OK = 0,
  MIMO_ERR_NULL = 1,        /* a required pointer is NULL */
  MIMO_ERR_SHAPE = 2,       /* sizes inconsistent or out of range */
  MIMO_ERR_UNSUPPORTED = 3, /* well-formed but not implemented (head dims, group size, rot_dims) */
  MIMO_ERR_ALIGN = 4,       /* a data pointer is not 16-byte aligned */
  MIMO_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than mimo_attn_workspace_size() */
  MIMO_ERR_CUDA = 6,        /* a CUDA call failed (no device, launch failure, ...) */
  MIMO_ERR_DEVICE = 7       /* a kernel set the device error word (see mimo_attn_device_status) */
} mimo_status;

/* Problem sizes. softmax_scale <= 0 selects 1/sqrt(head_dim_qk). */
typedef struct mimo_shape {
  int batch;        /* B */
  int seqlen;       /* n (prefill only; ignored by decode / sparse) */
  int n_q_heads;    /* Hq */
  int n_kv_heads;   /* Hkv */
  int head_dim_qk;  /* 192 */
  int head_dim_v;   /* 128 */
  float softmax_scale;
} mimo_shape;

enum { MIMO_CACHE_RING = 0, MIMO_CACHE_LINEAR = 1 };
enum { MIMO_OP_DECODE = 0, MIMO_OP_SPARSE = 1 };

/*
 * Prefill of one layer over whole sequences ("MiMo-V2-Flash ..." §5 steps 2-5;
 * partial RoPE from "...MiMo-V2.6-Flash-MOPD混合SWA设计原理" §5).
 *
 *  q    [B, n, Hq, 192]  bf16, un-rotated
 *  k    [B, n, Hkv, 192] bf16, un-rotated
 *  v    [B, n, Hkv, 128] bf16
 *  sink [Hq] fp32, or NULL (no sink term)
 *  window     W > 0 and W < n: SWA with J_i = [max(0, i-W+1), i]; W <= 0 or W >= n: GA (causal prefix)
 *  rope_theta RoPE base (1e4 for SWA, 1e7 for GA); must be > 0 when rot_dims > 0
 *  rot_dims   number of leading QK dims rotated at positions 0..n-1 with the rotate-half
 *             pairing (d, d + rot_dims/2) and inverse frequency theta^(-2k/rot_dims);
 *             0 or a multiple of 16 up to 192 (64 = 0.334 * 192 on MiMo)
 *  out  [B, n, Hq, 128] bf16 (written)
 *  lse  [B, Hq, n] fp32 natural-log LSE including the sink (written), or NULL
 *
 * Runs the sm_100a tensor-core kernel (TMA-staged tiles, tcgen05 MMAs with TMEM
 * accumulators). Tiles fully outside the window or the causal prefix are skipped.
 */
mimo_status mimo_attn_prefill(const mimo_shape* shape, const void* q, const void* k,
                              const void* v, const float* sink, int window,
                              float rope_theta, int rot_dims, void* out, float* lse,
                              void* stream);

/*
 * One-token decode over a KV cache (SWA ring pool of O(W) slots, or GA linear pool;
 * "...MiMo-V2.5..." dual-pool KV cache; math as above with i = L_b - 1).
 *
 *  q        [B, Hq, 192] bf16, already rotated at position L_b - 1
 *  k_cache  [B, seq_stride_tokens, Hkv, 192] bf16, rotated K
 *  v_cache  [B, seq_stride_tokens, Hkv, 128] bf16
 *  cache_kind MIMO_CACHE_RING: token p of sequence b lives in slot p mod cache_capacity and
 *             the query attends slots [0, min(L_b, cache_capacity)) (the last
 *             cache_capacity tokens, i.e. the window when capacity = W);
 *             MIMO_CACHE_LINEAR: slot t holds token t; the query attends [0, L_b)
 *  cache_capacity     slots per sequence (>= 1, <= seq_stride_tokens)
 *  seq_stride_tokens  distance between sequences in tokens
 *  lengths  [B] int32 device: L_b >= 0 tokens so far including the query's own token
 *           (linear: L_b <= cache_capacity; values are clamped to the cache). L_b = 0 (an
 *           empty cache) is an empty key set: the formula with an empty sum gives o = 0
 *           and lse = sink (-inf without a sink)
 *  sink     [Hq] fp32 or NULL
 *  out      [B, Hq, 128] bf16 (written); lse [B, Hq] fp32 or NULL
 *  workspace  device scratch of at least mimo_attn_workspace_size(shape, MIMO_OP_DECODE, cache_kind,
 *             cache_capacity, 0, 0) bytes (may be NULL when that size is 0)
 *
 * Split-KV: partial (m, l, o) per chunk of keys without the sink, then one combine
 * that adds the sink term once.
 */
mimo_status mimo_attn_decode(const mimo_shape* shape, const void* q, const void* k_cache,
                             const void* v_cache, int cache_kind, int cache_capacity,
                             long long seq_stride_tokens, const int* lengths,
                             const float* sink, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * Token-level sparse decode ("小米MiMo-V3的核心架构HySparse2" §四.3): one merged sink
 * softmax over the most recent `recent` tokens {L_b-recent, ..., L_b-1} plus `n_sel`
 * selected tokens, read from one linear cache.
 *
 *  q, k_cache, v_cache, lengths, sink, out, lse: as in mimo_attn_decode (linear cache)
 *  cache_capacity   slots per sequence; lengths and indices are clamped to it
 *  recent           size of the forced recent window (128 on MiMo), >= 0
 *  sel_idx [B, Hkv, n_sel] int32 device: per (sequence, KV head) sorted unique token
 *          indices in [0, L_b - recent), shared by the group's query heads, optionally
 *          followed by -1 entries that name no token (the padding mimo_attn_select_tokens
 *          writes when a sequence has fewer candidates than n_sel); a -1 entry is skipped
 *  n_sel            number of selected tokens (1024 on MiMo), >= 0
 *  workspace        at least mimo_attn_workspace_size(shape, MIMO_OP_SPARSE, MIMO_CACHE_LINEAR,
 *                   cache_capacity, recent, n_sel) bytes
 *
 * The index list drives a row gather; no dense mask is formed. Duplicates or indices
 * inside the recent window are a precondition violation (counted by
 * mimo_attn_check_indices), not an error of this call.
 */
mimo_status mimo_attn_sparse(const mimo_shape* shape, const void* q, const void* k_cache,
                             const void* v_cache, int cache_capacity,
                             long long seq_stride_tokens, const int* lengths, int recent,
                             const int* sel_idx, int n_sel, const float* sink, void* out,
                             float* lse, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * Chunked prefill over a KV prefix (youngju.dev "mimo-v25-inference-optimization", serving
 * section: long prompts are prefilled in chunks). A chunk of n = shape->seqlen query tokens
 * at positions pos_offset .. pos_offset + n - 1 attends the keys of positions
 * 0 .. pos_offset + n - 1, exactly as those rows of mimo_attn_prefill over the whole sequence.
 *
 *  q    [B, n, Hq, 192] bf16 device, un-rotated (rotated here at their positions)
 *  k, v [B, pos_offset + n, Hkv, 192 | 128] bf16 device: every key position. The chunk's
 *       rows (positions >= pos_offset) are un-rotated; the prefix rows are taken as stored
 *       when k_prefix_rotated != 0 (as a KV cache holds them) and rotated here otherwise
 *  pos_offset >= 0; sink, window (<= 0 or >= pos_offset + n: full causal), rope_theta,
 *       rot_dims: as mimo_attn_prefill
 *  out  [B, n, Hq, 128] bf16 device; lse [B, Hq, n] fp32 device or NULL
 *
 * Full-causal chunks with 8 or 16 query heads per KV head run on the GA pair kernel; SWA
 * chunks with 8 query heads per KV head, window <= 129, rot_dims <= 64 and pos_offset a
 * multiple of 16 on the K/V-ring kernel (the fast path for SWA layers: choose chunk
 * boundaries on multiples of 16); all other shapes on the generic prefill kernel. Errors as
 * mimo_attn_prefill; MIMO_ERR_SHAPE also for pos_offset < 0.
 */
mimo_status mimo_attn_prefill_chunk(const mimo_shape* shape, const void* q, const void* k,
                                    const void* v, int pos_offset, int k_prefix_rotated,
                                    const float* sink, int window, float rope_theta, int rot_dims,
                                    void* out, float* lse, void* stream);

/*
 * Writes a chunk of n = shape->seqlen tokens (positions pos_offset .. pos_offset + n - 1) into
 * a KV cache, as the decode calls read it: K rotated at its position (first rot_dims dims,
 * rotate-half pairing, theta rope_theta) and rounded to bf16, V copied; token p goes to slot
 * p mod cache_capacity (MIMO_CACHE_RING, only the chunk's last cache_capacity tokens are
 * written) or slot p (MIMO_CACHE_LINEAR, pos_offset + n <= cache_capacity).
 *
 *  k_chunk [B, n, Hkv, 192], v_chunk [B, n, Hkv, 128] bf16 device (un-rotated K)
 *  k_cache [B, seq_stride_tokens, Hkv, 192], v_cache [.., 128] bf16 device, written in place
 *
 * Errors: MIMO_ERR_NULL, MIMO_ERR_SHAPE (bad kind, sizes, a linear cache too small),
 * MIMO_ERR_UNSUPPORTED (rot_dims not a multiple of 16), MIMO_ERR_ALIGN, MIMO_ERR_CUDA.
 */
mimo_status mimo_attn_cache_append(const mimo_shape* shape, const void* k_chunk,
                                   const void* v_chunk, int pos_offset, float rope_theta,
                                   int rot_dims, int cache_kind, void* k_cache, void* v_cache,
                                   int cache_capacity, long long seq_stride_tokens, void* stream);

/*
 * Multi-query decode: MTP draft verification (syt-nju.github.io "mimo-mtp-swa-not-mla",
 * MTP section: the main model checks the draft tokens in one forward pass). The q_len
 * newest tokens of each sequence, at positions L_b - q_len .. L_b - 1 and already written
 * to the cache, are attended together; draft token t (position p = L_b - q_len + t) sees
 *   MIMO_CACHE_RING   (SWA pool; token p in slot p mod cache_capacity): tokens
 *                     [max(0, p - window + 1), p]; needs cache_capacity >= window + q_len - 1
 *                     so that no draft token's window has been overwritten;
 *   MIMO_CACHE_LINEAR (GA pool): tokens [0, p] (window ignored).
 * With q_len = 1 on a ring of window slots this is mimo_attn_decode.
 *
 *  shape            batch, n_q_heads, n_kv_heads, head dims (192 / 128), softmax_scale;
 *                   seqlen is ignored
 *  q       [B, q_len, Hq, 192] bf16 device, already rotated, contiguous
 *  k_cache, v_cache, cache_kind, cache_capacity, seq_stride_tokens, sink: as in
 *                   mimo_attn_decode (K stored rotated)
 *  lengths [B] int32 device: tokens in the cache per sequence including the draft tokens;
 *                   precondition q_len <= L_b (draft tokens before position 0 have no keys)
 *  q_len            draft tokens per sequence, 1 <= q_len and q_len * Hq/Hkv <= 64
 *  window           SWA window W >= 1 (ring only)
 *  out     [B, q_len, Hq, 128] bf16 device; lse [B, q_len, Hq] fp32 device or NULL
 *  workspace        at least mimo_attn_decode_mq_workspace_size(...) bytes (may be NULL
 *                   when that is 0)
 *
 * Each (sequence, KV head) unit reads its key range [min_t window start, L_b) once for all
 * q_len * Hq/Hkv query rows. Errors as mimo_attn_decode; MIMO_ERR_SHAPE also when the ring
 * is smaller than window + q_len - 1 or window < 1; MIMO_ERR_UNSUPPORTED when
 * q_len * Hq/Hkv > 64.
 */
mimo_status mimo_attn_decode_mq(const mimo_shape* shape, const void* q, const void* k_cache,
                                const void* v_cache, int cache_kind, int cache_capacity,
                                long long seq_stride_tokens, const int* lengths, int q_len,
                                int window, const float* sink, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace mimo_attn_decode_mq needs for these sizes on the current device
 * (0 when none is needed or the arguments are invalid). */
size_t mimo_attn_decode_mq_workspace_size(const mimo_shape* shape, int cache_kind,
                                          int cache_capacity, int q_len, int window);

/*
 * Decode and token-level sparse decode over FP8 KV caches. The pages size their KV caches
 * in FP8 but state no scaling scheme; this library's scheme: K and V hold OCP FP8 E4M3
 * bytes (bias 7, no infinities, S.1111.111 is NaN) and each (token, KV head) row has one
 * fp32 scale per tensor; the cached value is e4m3(byte) * scale. Attention is that of
 * mimo_attn_decode / mimo_attn_sparse on those values.
 *
 *  k_cache [B, seq_stride_tokens, Hkv, 192] uint8 device (E4M3), rows 16-byte aligned
 *  v_cache [B, seq_stride_tokens, Hkv, 128] uint8 device (E4M3)
 *  k_scale, v_scale [B, seq_stride_tokens, Hkv] fp32 device, 4-byte aligned
 *  every other argument, the workspace size (mimo_attn_workspace_size with the same op,
 *  kind and sizes) and the errors: as mimo_attn_decode / mimo_attn_sparse; MIMO_ERR_NULL
 *  also for a missing scale array.
 *
 * The E4M3 bytes are converted exactly to f16 (K and V); the K scale multiplies the fp32
 * score and the V scale multiplies P, which is rounded to f16 after a power-of-two factor per
 * 32 keys that keeps it below 2 (the factor is divided out of the output). q must lie inside
 * the f16 range (|q| <= 65504) because S = Q K^T runs as an f16 MMA.
 */
mimo_status mimo_attn_decode_fp8(const mimo_shape* shape, const void* q, const void* k_cache,
                                 const void* v_cache, const float* k_scale, const float* v_scale,
                                 int cache_kind, int cache_capacity, long long seq_stride_tokens,
                                 const int* lengths, const float* sink, void* out, float* lse,
                                 void* workspace, size_t workspace_bytes, void* stream);
mimo_status mimo_attn_sparse_fp8(const mimo_shape* shape, const void* q, const void* k_cache,
                                 const void* v_cache, const float* k_scale, const float* v_scale,
                                 int cache_capacity, long long seq_stride_tokens, const int* lengths,
                                 int recent, const int* sel_idx, int n_sel, const float* sink,
                                 void* out, float* lse, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * Token selection for mimo_attn_sparse ("小米MiMo-V3的核心架构HySparse2" §二.2 / §四.3: token
 * level, reused from the preceding full-attention layer, no trained retrieval module; the
 * pages give no scoring rule - this is the library's). For sequence b and KV head g, every
 * token t in [0, L_b - recent) scores max over the group's query heads of q_h . k_t; the
 * n_sel best are kept (equal scores: lower t first) and written in increasing t, which is
 * the sel_idx layout mimo_attn_sparse reads.
 *
 *  q        [B, Hq, 192] bf16 device (rotated), e.g. the query of the preceding GA layer
 *  k_cache  [B, seq_stride_tokens, Hkv, 192] bf16 device, linear cache of rotated K
 *  lengths  [B] int32 device (clamped to cache_capacity)
 *  sel_idx  [B, Hkv, n_sel] int32 device (written); rows with fewer than n_sel candidates
 *           hold all of them followed by -1, which mimo_attn_sparse skips, so selection
 *           followed by the sparse decode attends every token of such a sequence
 *  workspace  at least mimo_attn_select_workspace_size(shape, cache_capacity) bytes
 *
 * Two launches: a score pass (1,024 candidates per CTA; q . k on the tensor cores with fp32
 * accumulation, writing an order-preserving key per candidate and a histogram of its top
 * byte) and one CTA per (b, g) doing a radix select and an ordered compaction. The
 * workspace holds the keys, [B, Hkv, cache_capacity rounded up to 4] uint32, followed by
 * the histograms, [B, Hkv, ceil(cache_capacity / 1024), 256] uint16. Errors: MIMO_ERR_NULL,
 * MIMO_ERR_SHAPE (capacity, stride, recent or n_sel out of range), MIMO_ERR_ALIGN,
 * MIMO_ERR_WORKSPACE, MIMO_ERR_UNSUPPORTED (batch or Hkv above 65535), MIMO_ERR_CUDA.
 */
mimo_status mimo_attn_select_tokens(const mimo_shape* shape, const void* q, const void* k_cache,
                                    int cache_capacity, long long seq_stride_tokens,
                                    const int* lengths, int recent, int n_sel, int* sel_idx,
                                    void* workspace, size_t workspace_bytes, void* stream);
size_t mimo_attn_select_workspace_size(const mimo_shape* shape, int cache_capacity);

/* Bytes of device workspace mimo_attn_decode / mimo_attn_sparse need for these sizes
 * on the current device (0 when none is needed). Returns 0 for invalid arguments. */
size_t mimo_attn_workspace_size(const mimo_shape* shape, int op, int cache_kind,
                                int cache_capacity, int recent, int n_sel);

/* Fixed size of the library-owned scratch array used by mimo_attn_sparse_noalloc (8 MiB). */
#define MIMO_SPARSE_NOALLOC_SCRATCH_BYTES 8388608u

/*
 * Allocation-free variant of mimo_attn_sparse. The paper has no counterpart: this is a
 * deployment convenience of this library.
 *
 * Who needs it: callers that cannot allocate device memory when they call attention,
 * e.g. a serving loop whose KV-cache pools reserve nearly all of HBM up front (a late
 * cudaMalloc would fail or force evictions), or a plug-in inside a host framework that
 * owns every device allocation and forbids direct cudaMalloc / cudaFree (cudaFree also
 * synchronises the whole device). They pass inputs and outputs only; the split-KV
 * partials go to a static device array of MIMO_SPARSE_NOALLOC_SCRATCH_BYTES that the
 * library holds on every GPU that loads it, until the process exits.
 *
 * Arguments and results are those of mimo_attn_sparse without workspace. Returns
 * MIMO_ERR_WORKSPACE, with nothing launched, when these sizes need more scratch than
 * the array holds (mimo_attn_workspace_size(shape, MIMO_OP_SPARSE, ...) larger than
 * MIMO_SPARSE_NOALLOC_SCRATCH_BYTES). The first call on a device, and the first after a
 * device reset (a new CUDA context), looks up the array's device address with that device
 * current (a host-side query, no allocation); make that first call before any stream
 * capture. All calls share the one array: two calls whose
 * kernels overlap on the GPU (different streams, no ordering between them) race on it
 * and give wrong results; order them on one stream. No part of the array needs to start
 * at zero: each call writes every partial it later reads.
 */
mimo_status mimo_attn_sparse_noalloc(const mimo_shape* shape, const void* q, const void* k_cache,
                                     const void* v_cache, int cache_capacity,
                                     long long seq_stride_tokens, const int* lengths, int recent,
                                     const int* sel_idx, int n_sel, const float* sink, void* out,
                                     float* lse, void* stream);

/* Debug check of sparse-decode preconditions, on `stream`: counts, into the device
 * word *d_violations (which the caller zeroes first), every (b, g) row that is not a
 * strictly increasing run of indices in [0, L_b - recent) followed by zero or more -1
 * entries, or whose L_b is outside [0, cache_capacity]. Never traps. */
mimo_status mimo_attn_check_indices(const mimo_shape* shape, const int* lengths,
                                    const int* sel_idx, int n_sel, int recent,
                                    int cache_capacity, unsigned int* d_violations,
                                    void* stream);

/* Synchronises the current device, then returns and clears the device error word
 * (0 = none). Kernels OR bits into it instead of trapping: 1 = a wait on work in progress
 * gave up (2 s; the kernel then left its loops, waited for its own copies and MMAs in flight,
 * freed its tensor memory and returned without finishing its output), 2 = one of those
 * exit-path waits gave up too, and in builds compiled with MIMO_DEBUG 4 = a sequence length
 * outside [0, capacity], 8 = a selected index outside [0, L - recent) or not increasing
 * (both clamped, so no access leaves the caller's buffers) and 16 = an operand carried in
 * f16 (see Precision) beyond +-65504 or NaN (converted as in the product build).
 * Host-blocking; for tests and debugging. Returns 0xFFFFFFFF if the device could not be
 * synchronised. */
unsigned int mimo_attn_last_device_error(void);

/* mimo_attn_last_device_error as a status: MIMO_OK when the word was 0, MIMO_ERR_DEVICE
 * when a kernel set it (the word is stored in *word when word is not NULL, then cleared),
 * MIMO_ERR_CUDA when the device could not be synchronised. Host-blocking. */
mimo_status mimo_attn_device_status(unsigned int* word);

/* Static description of a status code. */
const char* mimo_status_string(mimo_status status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int mimo_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MIMO_ATTN_H */
