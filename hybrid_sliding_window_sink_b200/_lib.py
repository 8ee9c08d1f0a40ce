"""ctypes binding of libmimo_attn.so (include/mimo_attn.h): argument marshalling only.

Each function takes torch tensors, checks dtype / device / contiguity / shape,
passes raw device pointers and the current CUDA stream to the C entry point of
the same name, and raises ``MimoError`` on any status other than MIMO_OK. All
arithmetic happens in the library's CUDA kernels. The library must be built
(``python -m hybrid_sliding_window_sink_b200.build``); there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmimo_attn.so")

MIMO_CACHE_RING = 0
MIMO_CACHE_LINEAR = 1
MIMO_OP_DECODE = 0
MIMO_OP_SPARSE = 1
STATUS = {0: "MIMO_OK", 1: "MIMO_ERR_NULL", 2: "MIMO_ERR_SHAPE", 3: "MIMO_ERR_UNSUPPORTED",
          4: "MIMO_ERR_ALIGN", 5: "MIMO_ERR_WORKSPACE", 6: "MIMO_ERR_CUDA", 7: "MIMO_ERR_DEVICE"}

#: Every symbol include/mimo_attn.h declares.
EXPORTS = ("mimo_attn_prefill", "mimo_attn_decode", "mimo_attn_sparse", "mimo_attn_sparse_noalloc",
           "mimo_attn_decode_mq", "mimo_attn_decode_mq_workspace_size", "mimo_attn_workspace_size",
           "mimo_attn_decode_fp8", "mimo_attn_sparse_fp8", "mimo_attn_prefill_chunk",
           "mimo_attn_cache_append", "mimo_attn_select_tokens", "mimo_attn_select_workspace_size",
           "mimo_attn_check_indices", "mimo_attn_last_device_error", "mimo_attn_device_status",
           "mimo_status_string", "mimo_attn_version")


class MimoError(RuntimeError):
    def __init__(self, fn, status, lib=None):
        msg = STATUS.get(status, str(status))
        if lib is not None:
            msg += ": " + lib.mimo_status_string(status).decode()
        super().__init__(f"{fn} failed with {msg}")
        self.status = status


class MimoShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim_qk", ctypes.c_int),
                ("head_dim_v", ctypes.c_int), ("softmax_scale", ctypes.c_float)]


_LIB = None


def lib():
    """Load libmimo_attn.so once; raise if it has not been built."""
    global _LIB
    if _LIB is None:
        _LIB = load(LIB_PATH)
    return _LIB


def load(path):
    """Load one build of the library (the product build, or a test build such as the one
    with a short wait limit) and declare the argument types of every entry point."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m hybrid_sliding_window_sink_b200.build`")
    L = ctypes.CDLL(path)
    P, I, F, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong, ctypes.c_size_t
    SP = ctypes.POINTER(MimoShape)
    L.mimo_attn_prefill.argtypes = [SP, P, P, P, P, I, F, I, P, P, P]
    L.mimo_attn_decode.argtypes = [SP, P, P, P, I, I, LL, P, P, P, P, P, SZ, P]
    L.mimo_attn_sparse.argtypes = [SP, P, P, P, I, LL, P, I, P, I, P, P, P, P, SZ, P]
    L.mimo_attn_sparse_noalloc.argtypes = [SP, P, P, P, I, LL, P, I, P, I, P, P, P, P]
    L.mimo_attn_decode_mq.argtypes = [SP, P, P, P, I, I, LL, P, I, I, P, P, P, P, SZ, P]
    L.mimo_attn_decode_mq_workspace_size.argtypes = [SP, I, I, I, I]
    L.mimo_attn_decode_mq_workspace_size.restype = SZ
    L.mimo_attn_prefill_chunk.argtypes = [SP, P, P, P, I, I, P, I, F, I, P, P, P]
    L.mimo_attn_cache_append.argtypes = [SP, P, P, I, F, I, I, P, P, I, LL, P]
    L.mimo_attn_select_tokens.argtypes = [SP, P, P, I, LL, P, I, I, P, P, SZ, P]
    L.mimo_attn_select_workspace_size.argtypes = [SP, I]
    L.mimo_attn_select_workspace_size.restype = SZ
    L.mimo_attn_decode_fp8.argtypes = [SP, P, P, P, P, P, I, I, LL, P, P, P, P, P, SZ, P]
    L.mimo_attn_sparse_fp8.argtypes = [SP, P, P, P, P, P, I, LL, P, I, P, I, P, P, P, P, SZ, P]
    L.mimo_attn_workspace_size.argtypes = [SP, I, I, I, I, I]
    L.mimo_attn_workspace_size.restype = SZ
    L.mimo_attn_check_indices.argtypes = [SP, P, P, I, I, I, P, P]
    L.mimo_attn_last_device_error.argtypes = []
    L.mimo_attn_last_device_error.restype = ctypes.c_uint
    L.mimo_attn_device_status.argtypes = [P]
    L.mimo_attn_device_status.restype = I
    L.mimo_status_string.argtypes = [I]
    L.mimo_status_string.restype = ctypes.c_char_p
    L.mimo_attn_version.argtypes = []
    L.mimo_attn_version.restype = I
    for fn in ("mimo_attn_prefill", "mimo_attn_decode", "mimo_attn_sparse", "mimo_attn_sparse_noalloc",
               "mimo_attn_check_indices"):
        getattr(L, fn).restype = I
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, status):
    if status != 0:
        raise MimoError(fn, status, _LIB)


def _need(t, name, dtype, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def make_shape(batch, seqlen, hq, hkv, dqk=192, dv=128, softmax_scale=0.0):
    return MimoShape(int(batch), int(seqlen), int(hq), int(hkv), int(dqk), int(dv),
                     float(softmax_scale))


def prefill(q, k, v, sink=None, *, window=128, rope_theta=1.0e4, rot_dims=64,
            softmax_scale=0.0, out=None, lse=None, want_lse=True, stream=None):
    """mimo_attn_prefill. q [B,n,Hq,192], k [B,n,Hkv,192], v [B,n,Hkv,128] bf16,
    sink [Hq] fp32 or None. Returns (out [B,n,Hq,128] bf16, lse [B,Hq,n] fp32 or None)."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, n, hq, dqk = q.shape
    hkv = k.shape[2]
    if k.shape[:2] != (B, n) or v.shape[:3] != (B, n, hkv):
        raise ValueError("q, k, v batch / sequence / head shapes disagree")
    if sink is not None:
        _need(sink, "sink", torch.float32, 1)
        if sink.shape[0] != hq:
            raise ValueError("sink must have Hq entries")
    if out is None:
        out = torch.empty(B, n, hq, v.shape[3], dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    if lse is None and want_lse:
        lse = torch.empty(B, hq, n, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, 3)
    shape = make_shape(B, n, hq, hkv, dqk, v.shape[3], softmax_scale)
    st = lib().mimo_attn_prefill(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(sink),
                                 int(window), float(rope_theta), int(rot_dims), _ptr(out),
                                 _ptr(lse), _stream(stream))
    _check("mimo_attn_prefill", st)
    return out, lse


def workspace_size(batch, hq, hkv, *, op, kind=MIMO_CACHE_LINEAR, capacity=1, recent=0, n_sel=0):
    shape = make_shape(batch, 1, hq, hkv)
    return int(lib().mimo_attn_workspace_size(ctypes.byref(shape), int(op), int(kind),
                                              int(capacity), int(recent), int(n_sel)))


def _workspace(ws, nbytes, device):
    if nbytes == 0:
        return ws
    if ws is None:
        return torch.empty(nbytes, dtype=torch.uint8, device=device)
    if ws.numel() * ws.element_size() < nbytes:
        raise ValueError("workspace too small")
    return ws


def decode(q, k_cache, v_cache, lengths, sink=None, *, kind="ring", capacity=None,
           softmax_scale=0.0, out=None, lse=None, want_lse=True, workspace=None, stream=None):
    """mimo_attn_decode. q [B,Hq,192]; caches [B,stride,Hkv,192/128] bf16 (rotated K);
    lengths [B] int32. kind "ring" (slot p mod capacity) or "linear"."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(lengths, "lengths", torch.int32, 1)
    B, hq, dqk = q.shape
    _, stride, hkv, _ = k_cache.shape
    if v_cache.shape[:3] != (B, stride, hkv) or k_cache.shape[0] != B or lengths.shape[0] != B:
        raise ValueError("cache / lengths shapes disagree with q")
    cap = stride if capacity is None else int(capacity)
    kind_id = {"ring": MIMO_CACHE_RING, "linear": MIMO_CACHE_LINEAR}[kind]
    if sink is not None:
        _need(sink, "sink", torch.float32, 1)
    if out is None:
        out = torch.empty(B, hq, v_cache.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, hq, dtype=torch.float32, device=q.device)
    shape = make_shape(B, 1, hq, hkv, dqk, v_cache.shape[3], softmax_scale)
    nbytes = int(lib().mimo_attn_workspace_size(ctypes.byref(shape), MIMO_OP_DECODE, kind_id, cap, 0, 0))
    ws = _workspace(workspace, nbytes, q.device)
    st = lib().mimo_attn_decode(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), kind_id,
                                cap, stride, _ptr(lengths), _ptr(sink), _ptr(out), _ptr(lse),
                                _ptr(ws), nbytes, _stream(stream))
    _check("mimo_attn_decode", st)
    return out, lse


def prefill_chunk(q, k, v, sink=None, *, pos_offset, k_prefix_rotated=True, window=0,
                  rope_theta=1e4, rot_dims=64, softmax_scale=0.0, out=None, lse=None,
                  want_lse=True, stream=None):
    """mimo_attn_prefill_chunk. q [B,n,Hq,192] (the chunk); k, v [B,pos_offset+n,Hkv,·] (every
    key position; prefix K rotated when k_prefix_rotated). Returns (out [B,n,Hq,128],
    lse [B,Hq,n])."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, n, hq, dqk = q.shape
    _, nk, hkv, _ = k.shape
    if nk != pos_offset + n or v.shape[:3] != (B, nk, hkv):
        raise ValueError("k / v must hold positions 0 .. pos_offset + n - 1")
    if sink is not None:
        _need(sink, "sink", torch.float32, 1)
    if out is None:
        out = torch.empty(B, n, hq, v.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, hq, n, dtype=torch.float32, device=q.device)
    shape = make_shape(B, n, hq, hkv, dqk, v.shape[3], softmax_scale)
    st = lib().mimo_attn_prefill_chunk(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), int(pos_offset),
                                       1 if k_prefix_rotated else 0, _ptr(sink), int(window),
                                       float(rope_theta), int(rot_dims), _ptr(out), _ptr(lse),
                                       _stream(stream))
    _check("mimo_attn_prefill_chunk", st)
    return out, lse


def cache_append(k_chunk, v_chunk, k_cache, v_cache, *, pos_offset, rope_theta=1e4, rot_dims=64,
                 kind="ring", capacity=None, stream=None):
    """mimo_attn_cache_append: writes the chunk's rotated K and its V into the caches in place."""
    _need(k_chunk, "k_chunk", torch.bfloat16, 4)
    _need(v_chunk, "v_chunk", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    B, n, hkv, dqk = k_chunk.shape
    stride = k_cache.shape[1]
    cap = stride if capacity is None else int(capacity)
    kind_id = {"ring": MIMO_CACHE_RING, "linear": MIMO_CACHE_LINEAR}[kind]
    shape = make_shape(B, n, hkv, hkv, dqk, v_chunk.shape[3])
    st = lib().mimo_attn_cache_append(ctypes.byref(shape), _ptr(k_chunk), _ptr(v_chunk), int(pos_offset),
                                      float(rope_theta), int(rot_dims), kind_id, _ptr(k_cache),
                                      _ptr(v_cache), cap, stride, _stream(stream))
    _check("mimo_attn_cache_append", st)
    return k_cache, v_cache


def select_tokens(q, k_cache, lengths, *, recent=128, n_sel=1024, capacity=None, out=None,
                  workspace=None, stream=None):
    """mimo_attn_select_tokens. q [B,Hq,192]; linear k_cache [B,stride,Hkv,192] (rotated K);
    lengths [B] int32. Returns sel_idx [B,Hkv,n_sel] int32 (sorted, as sparse() reads it)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(lengths, "lengths", torch.int32, 1)
    B, hq, dqk = q.shape
    _, stride, hkv, _ = k_cache.shape
    cap = stride if capacity is None else int(capacity)
    if out is None:
        out = torch.empty(B, hkv, n_sel, dtype=torch.int32, device=q.device)
    shape = make_shape(B, 1, hq, hkv, dqk)
    nbytes = int(lib().mimo_attn_select_workspace_size(ctypes.byref(shape), cap))
    ws = _workspace(workspace, nbytes, q.device)
    st = lib().mimo_attn_select_tokens(ctypes.byref(shape), _ptr(q), _ptr(k_cache), cap, stride,
                                       _ptr(lengths), int(recent), int(n_sel), _ptr(out), _ptr(ws),
                                       nbytes, _stream(stream))
    _check("mimo_attn_select_tokens", st)
    return out


def decode_mq(q, k_cache, v_cache, lengths, sink=None, *, kind="ring", window=128, capacity=None,
              softmax_scale=0.0, out=None, lse=None, want_lse=True, workspace=None, stream=None):
    """mimo_attn_decode_mq. q [B,T,Hq,192] (the T newest tokens of each sequence, rotated);
    caches [B,stride,Hkv,192/128] bf16 holding them; lengths [B] int32 including them.
    kind "ring" (slot p mod capacity, needs capacity >= window + T - 1) or "linear"."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(lengths, "lengths", torch.int32, 1)
    B, T, hq, dqk = q.shape
    _, stride, hkv, _ = k_cache.shape
    if v_cache.shape[:3] != (B, stride, hkv) or k_cache.shape[0] != B or lengths.shape[0] != B:
        raise ValueError("cache / lengths shapes disagree with q")
    cap = stride if capacity is None else int(capacity)
    kind_id = {"ring": MIMO_CACHE_RING, "linear": MIMO_CACHE_LINEAR}[kind]
    if sink is not None:
        _need(sink, "sink", torch.float32, 1)
    if out is None:
        out = torch.empty(B, T, hq, v_cache.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, T, hq, dtype=torch.float32, device=q.device)
    shape = make_shape(B, 1, hq, hkv, dqk, v_cache.shape[3], softmax_scale)
    nbytes = int(lib().mimo_attn_decode_mq_workspace_size(ctypes.byref(shape), kind_id, cap, T,
                                                          int(window)))
    ws = _workspace(workspace, nbytes, q.device)
    st = lib().mimo_attn_decode_mq(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), kind_id,
                                   cap, stride, _ptr(lengths), T, int(window), _ptr(sink), _ptr(out),
                                   _ptr(lse), _ptr(ws), nbytes, _stream(stream))
    _check("mimo_attn_decode_mq", st)
    return out, lse


def _need_fp8(k8, v8, ks, vs):
    _need(k8, "k_cache", torch.uint8, 4)
    _need(v8, "v_cache", torch.uint8, 4)
    _need(ks, "k_scale", torch.float32, 3)
    _need(vs, "v_scale", torch.float32, 3)
    if ks.shape != k8.shape[:3] or vs.shape != v8.shape[:3] or k8.shape[:3] != v8.shape[:3]:
        raise ValueError("FP8 caches and scales disagree in shape")


def decode_fp8(q, k8, v8, k_scale, v_scale, lengths, sink=None, *, kind="ring", capacity=None,
               softmax_scale=0.0, out=None, lse=None, want_lse=True, workspace=None, stream=None):
    """mimo_attn_decode_fp8. q [B,Hq,192] bf16; k8/v8 [B,stride,Hkv,192/128] uint8 E4M3;
    k_scale/v_scale [B,stride,Hkv] fp32; value = e4m3(byte) * scale."""
    _need(q, "q", torch.bfloat16, 3)
    _need_fp8(k8, v8, k_scale, v_scale)
    _need(lengths, "lengths", torch.int32, 1)
    B, hq, dqk = q.shape
    _, stride, hkv, _ = k8.shape
    cap = stride if capacity is None else int(capacity)
    kind_id = {"ring": MIMO_CACHE_RING, "linear": MIMO_CACHE_LINEAR}[kind]
    if sink is not None:
        _need(sink, "sink", torch.float32, 1)
    if out is None:
        out = torch.empty(B, hq, v8.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, hq, dtype=torch.float32, device=q.device)
    shape = make_shape(B, 1, hq, hkv, dqk, v8.shape[3], softmax_scale)
    nbytes = int(lib().mimo_attn_workspace_size(ctypes.byref(shape), MIMO_OP_DECODE, kind_id, cap, 0, 0))
    ws = _workspace(workspace, nbytes, q.device)
    st = lib().mimo_attn_decode_fp8(ctypes.byref(shape), _ptr(q), _ptr(k8), _ptr(v8), _ptr(k_scale),
                                    _ptr(v_scale), kind_id, cap, stride, _ptr(lengths), _ptr(sink),
                                    _ptr(out), _ptr(lse), _ptr(ws), nbytes, _stream(stream))
    _check("mimo_attn_decode_fp8", st)
    return out, lse


def sparse_fp8(q, k8, v8, k_scale, v_scale, lengths, sel_idx, sink=None, *, recent=128,
               capacity=None, softmax_scale=0.0, out=None, lse=None, want_lse=True, workspace=None,
               stream=None):
    """mimo_attn_sparse_fp8: sparse() over FP8 linear caches with per-row scales."""
    _need(q, "q", torch.bfloat16, 3)
    _need_fp8(k8, v8, k_scale, v_scale)
    _need(lengths, "lengths", torch.int32, 1)
    _need(sel_idx, "sel_idx", torch.int32, 3)
    B, hq, dqk = q.shape
    _, stride, hkv, _ = k8.shape
    n_sel = sel_idx.shape[2]
    cap = stride if capacity is None else int(capacity)
    if sink is not None:
        _need(sink, "sink", torch.float32, 1)
    if out is None:
        out = torch.empty(B, hq, v8.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, hq, dtype=torch.float32, device=q.device)
    shape = make_shape(B, 1, hq, hkv, dqk, v8.shape[3], softmax_scale)
    nbytes = int(lib().mimo_attn_workspace_size(ctypes.byref(shape), MIMO_OP_SPARSE,
                                                MIMO_CACHE_LINEAR, cap, int(recent), n_sel))
    ws = _workspace(workspace, nbytes, q.device)
    st = lib().mimo_attn_sparse_fp8(ctypes.byref(shape), _ptr(q), _ptr(k8), _ptr(v8), _ptr(k_scale),
                                    _ptr(v_scale), cap, stride, _ptr(lengths), int(recent),
                                    _ptr(sel_idx), n_sel, _ptr(sink), _ptr(out), _ptr(lse), _ptr(ws),
                                    nbytes, _stream(stream))
    _check("mimo_attn_sparse_fp8", st)
    return out, lse


def sparse(q, k_cache, v_cache, lengths, sel_idx, sink=None, *, recent=128, capacity=None,
           softmax_scale=0.0, out=None, lse=None, want_lse=True, workspace=None, stream=None):
    """mimo_attn_sparse. q [B,Hq,192]; linear caches [B,stride,Hkv,·]; lengths [B] int32;
    sel_idx [B,Hkv,n_sel] int32 sorted unique in [0, L-recent)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(lengths, "lengths", torch.int32, 1)
    _need(sel_idx, "sel_idx", torch.int32, 3)
    B, hq, dqk = q.shape
    _, stride, hkv, _ = k_cache.shape
    if sel_idx.shape[:2] != (B, hkv):
        raise ValueError("sel_idx must be [B, Hkv, n_sel]")
    n_sel = sel_idx.shape[2]
    cap = stride if capacity is None else int(capacity)
    if sink is not None:
        _need(sink, "sink", torch.float32, 1)
    if out is None:
        out = torch.empty(B, hq, v_cache.shape[3], dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, hq, dtype=torch.float32, device=q.device)
    shape = make_shape(B, 1, hq, hkv, dqk, v_cache.shape[3], softmax_scale)
    nbytes = int(lib().mimo_attn_workspace_size(ctypes.byref(shape), MIMO_OP_SPARSE,
                                                MIMO_CACHE_LINEAR, cap, int(recent), n_sel))
    ws = _workspace(workspace, nbytes, q.device)
    st = lib().mimo_attn_sparse(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache), cap,
                                stride, _ptr(lengths), int(recent), _ptr(sel_idx), n_sel, _ptr(sink),
                                _ptr(out), _ptr(lse), _ptr(ws), nbytes, _stream(stream))
    _check("mimo_attn_sparse", st)
    return out, lse


def check_indices(lengths, sel_idx, *, hq, recent=128, capacity, stream=None):
    """mimo_attn_check_indices: number of (b, g) rows violating the sparse preconditions."""
    _need(lengths, "lengths", torch.int32, 1)
    _need(sel_idx, "sel_idx", torch.int32, 3)
    B, hkv, n_sel = sel_idx.shape
    shape = make_shape(B, 1, hq, hkv)
    cnt = torch.zeros(1, dtype=torch.int32, device=lengths.device)
    st = lib().mimo_attn_check_indices(ctypes.byref(shape), _ptr(lengths), _ptr(sel_idx), n_sel,
                                       int(recent), int(capacity), _ptr(cnt), _stream(stream))
    _check("mimo_attn_check_indices", st)
    return int(cnt.item())


def last_device_error():
    return int(lib().mimo_attn_last_device_error())
