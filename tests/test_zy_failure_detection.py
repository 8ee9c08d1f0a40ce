"""Failure detection, exercised without faulting, trapping or hanging the GPU.

Every wait inside a kernel is bounded: when it gives up, the kernel leaves its loops, waits
(with a separate 2 s limit) for its own copies and MMAs in flight, frees its tensor memory,
ORs a bit into the device error word and returns. Two test builds of the same source
(hybrid_sliding_window_sink_b200.build.VARIANTS) are loaded next to the product build:

* shortwait: waits on work in progress give up after 1 ns, so the abort paths of the real
  kernels run; it also has a hook that waits on a barrier nothing ever arrives on.
* debug: kernels record lengths and selected indices outside their ranges in the error word
  (and still clamp them, so no access leaves the caller's buffers), and every operand they
  carry in f16 that lies beyond +-65504.

After each, the product build runs on the same CUDA context and must give correct results.
"""

import contextlib
import ctypes

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, build, workloads as wl
from oracle import ref
from parity_util import compare

pytestmark = pytest.mark.gpu

MIMO_OK, MIMO_ERR_DEVICE = 0, 7
WAIT_TIMEOUT, DRAIN_TIMEOUT, BAD_LENGTH, BAD_INDEX, F16_RANGE = 1, 2, 4, 8, 16


@contextlib.contextmanager
def _library(name):
    """Routes the binding's calls to a test build of the library for the duration."""
    lib = _lib.load(build.build(variant=name))
    saved = _lib._LIB
    _lib._LIB = lib
    try:
        yield lib
    finally:
        _lib._LIB = saved


def _status(lib):
    word = ctypes.c_uint(0)
    st = lib.mimo_attn_device_status(ctypes.byref(word))
    return st, word.value


def test_wait_on_a_barrier_nothing_arrives_on(cuda_device):
    """The bounded wait every kernel uses gives up on a barrier nothing ever completes, sets
    the wait-timeout bit and returns; the status call reports MIMO_ERR_DEVICE once."""
    with _library("shortwait") as lib:
        assert _status(lib) == (MIMO_OK, 0)
        lib.mimo_attn_test_stuck_wait.argtypes = [ctypes.c_void_p]
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        assert lib.mimo_attn_test_stuck_wait(stream) == MIMO_OK
        assert _status(lib) == (MIMO_ERR_DEVICE, WAIT_TIMEOUT)
        assert _status(lib) == (MIMO_OK, 0)          # read and cleared


def test_kernels_give_up_and_the_context_stays_usable(cuda_device):
    """Under the 1 ns wait limit the persistent SWA-ring and GA-pair prefill kernels give up
    (wait-timeout bit) and the generic prefill, decode and multi-query decode kernels may (their
    waits are short); no exit-path wait ever gives up. Afterwards the product build, on the same context,
    matches the oracle and leaves the word clear."""
    dev = cuda_device
    cases = [(wl.prefill_inputs(1, 640, 64, 8, seed=61), 128, 1e4),             # SWA ring kernel
             (wl.prefill_inputs(1, 384, 64, 4, seed=62, k_scale=0.5), 0, 1e7),  # GA pair kernel
             (wl.prefill_inputs(1, 300, 16, 4, seed=63), 64, 1e4)]              # generic kernel
    lengths = [4096, 100, 3000, 1, 4096, 2048, 7, 999]
    d = wl.decode_inputs(len(lengths), 64, 4, 4096, lengths, seed=64)
    dd = {k: v.to(dev) for k, v in d.items()}
    mq_lengths = [3000, 4, 1500]    # multi-query decode over a linear cache: the TMA / tcgen05 kernel
    mq = wl.decode_mq_inputs(len(mq_lengths), 4, 64, 4, 3000, mq_lengths, seed=66)
    mqd = {k: v.to(dev) for k, v in mq.items()}
    with _library("shortwait") as lib:
        for i, (x, window, theta) in enumerate(cases):
            _lib.prefill(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), x["sink"].to(dev),
                         window=window, rope_theta=theta, rot_dims=64)
            st, word = _status(lib)
            assert st == (MIMO_ERR_DEVICE if word else MIMO_OK) and not word & DRAIN_TIMEOUT, (window, word)
            if i < 2:   # persistent kernels: every CTA waits on work in progress many times
                assert word == WAIT_TIMEOUT, (window, word)
        _lib.decode(dd["q"], dd["k_cache"], dd["v_cache"], dd["lengths"], dd["sink"], kind="linear")
        st, word = _status(lib)
        assert not word & DRAIN_TIMEOUT, word
        _lib.decode_mq(mqd["q_mq"], mqd["k_cache"], mqd["v_cache"], mqd["lengths"], mqd["sink"], kind="linear",
                       window=0)
        st, word = _status(lib)
        assert not word & DRAIN_TIMEOUT, word
    for x, window, theta in cases:
        out, lse = _lib.prefill(x["q"].to(dev), x["k"].to(dev), x["v"].to(dev), x["sink"].to(dev),
                                window=window, rope_theta=theta, rot_dims=64)
        torch.cuda.synchronize()
        o_ref, l_ref = ref.prefill(wl.to_f64(x["q"]), wl.to_f64(x["k"]), wl.to_f64(x["v"]),
                                   wl.to_f64(x["sink"]), window, theta, 64)
        compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, f"after abort: prefill W={window}")
    out, lse = _lib.decode(dd["q"], dd["k_cache"], dd["v_cache"], dd["lengths"], dd["sink"], kind="linear")
    torch.cuda.synchronize()
    o_ref, l_ref = ref.decode(wl.to_f64(d["q"]), wl.to_f64(d["k_cache"]), wl.to_f64(d["v_cache"]), "linear",
                              lengths, wl.to_f64(d["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "after abort: decode")
    out, lse = _lib.decode_mq(mqd["q_mq"], mqd["k_cache"], mqd["v_cache"], mqd["lengths"], mqd["sink"],
                              kind="linear", window=0)
    torch.cuda.synchronize()
    o_ref, l_ref = ref.decode_multi(wl.to_f64(mq["q_mq"]), wl.to_f64(mq["k_cache"]), wl.to_f64(mq["v_cache"]),
                                    "linear", mq_lengths, 0, wl.to_f64(mq["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "after abort: multi-query decode")
    assert _status(_lib.lib()) == (MIMO_OK, 0)


def test_debug_build_reports_bad_lengths_and_indices(cuda_device):
    """The debug build records a selected index inside the recent window, one beyond the
    cache and an unsorted pair (bad-index bit), and a length beyond a linear cache
    (bad-length bit); it still clamps them, so outputs stay finite. Valid calls leave the
    word clear and match the oracle."""
    dev = cuda_device
    B, hq, hkv, cap, recent, n_sel = 2, 64, 4, 3000, 128, 64
    lengths = [3000, 700]
    d = wl.decode_inputs(B, hq, hkv, cap, lengths, seed=65)
    sel = wl.sorted_unique_indices(B, hkv, n_sel, [x - recent for x in lengths], seed=65)
    dd = {k: v.to(dev) for k, v in d.items()}
    with _library("debug") as lib:
        out, lse = _lib.sparse(dd["q"], dd["k_cache"], dd["v_cache"], dd["lengths"], sel.to(dev), dd["sink"],
                               recent=recent)
        torch.cuda.synchronize()
        assert _status(lib) == (MIMO_OK, 0)
        o_ref, l_ref = ref.sparse_decode(wl.to_f64(d["q"]), wl.to_f64(d["k_cache"]), wl.to_f64(d["v_cache"]),
                                         lengths, recent, sel.numpy(), wl.to_f64(d["sink"]))
        compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "debug build, valid sparse call")
        bad = sel.clone()
        bad[0, 0, -1] = lengths[0] - 5           # inside the recent window
        bad[1, 2, -1] = cap + 100                 # beyond the cache (clamped)
        bad[1, 3, 10], bad[1, 3, 11] = bad[1, 3, 11].item(), bad[1, 3, 10].item()   # unsorted
        out, lse = _lib.sparse(dd["q"], dd["k_cache"], dd["v_cache"], dd["lengths"], bad.to(dev), dd["sink"],
                               recent=recent)
        torch.cuda.synchronize()
        st, word = _status(lib)
        assert st == MIMO_ERR_DEVICE and word == BAD_INDEX, word
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        long_l = torch.tensor([cap + 50, 10], dtype=torch.int32, device=dev)
        out, lse = _lib.decode(dd["q"], dd["k_cache"], dd["v_cache"], long_l, dd["sink"], kind="linear")
        torch.cuda.synchronize()
        st, word = _status(lib)
        assert st == MIMO_ERR_DEVICE and word == BAD_LENGTH, word
        assert torch.isfinite(out).all()
        # the clamped length reads the whole cache: the same result as L = capacity
        o_ref, l_ref = ref.decode(wl.to_f64(d["q"]), wl.to_f64(d["k_cache"]), wl.to_f64(d["v_cache"]), "linear",
                                  [cap, 10], wl.to_f64(d["sink"]))
        compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "debug build, clamped length")


def _bf16(x, s):
    return (x.float() * s).to(torch.bfloat16)


@pytest.mark.parametrize("n, hq, hkv, window, theta", [
    (640, 64, 8, 128, 1e4),      # SWA ring kernel: rotated Q/K, P and V in f16
    (384, 64, 4, 0, 1e7),        # GA pair kernel: rotated Q/K in f16
    (300, 16, 4, 64, 1e4),       # generic kernel: rotated Q/K in f16
])
def test_debug_build_reports_operands_beyond_the_f16_range(cuda_device, n, hq, hkv, window, theta):
    """In the debug build, K and V in the thousands (inside the f16 range) leave the word clear
    and match the oracle; one K entry of 1e5 in a rotated dim sets the f16-range bit, the same
    entry in a dim carried in bf16 does not; a V entry of 1e5 sets it in the SWA ring kernel,
    the one kernel that carries V in f16."""
    dev = cuda_device
    x = wl.prefill_inputs(1, n, hq, hkv, seed=66 + n)
    q, k, v = _bf16(x["q"], 1e-3), _bf16(x["k"], 1e3), _bf16(x["v"], 2e3)
    sink = x["sink"].to(dev)

    def run(kk, vv):
        out, lse = _lib.prefill(q.to(dev), kk.to(dev), vv.to(dev), sink, window=window,
                                rope_theta=theta, rot_dims=64)
        torch.cuda.synchronize()
        return out, lse

    with _library("debug") as lib:
        out, lse = run(k, v)
        assert _status(lib) == (MIMO_OK, 0)
        o_ref, l_ref = ref.prefill(wl.to_f64(q), wl.to_f64(k), wl.to_f64(v), wl.to_f64(x["sink"]), window,
                                   theta, 64)
        compare(wl.to_f64(out) / 2e3, o_ref / 2e3, wl.to_f64(lse), l_ref, f"debug build, W={window}")
        k_rot = k.clone()
        k_rot[0, n // 2, 0, 5] = 1e5             # dims 0..63 are rotated
        run(k_rot, v)
        assert _status(lib) == (MIMO_ERR_DEVICE, F16_RANGE)
        k_plain = k.clone()
        k_plain[0, n // 2, 0, 150] = 1e5         # an unrotated dim, multiplied in bf16
        out, _ = run(k_plain, v)
        assert _status(lib) == (MIMO_OK, 0)
        assert torch.isfinite(out).all()
        v_big = v.clone()
        v_big[0, n // 2, 0, 9] = 1e5
        run(k, v_big)
        assert _status(lib) == ((MIMO_ERR_DEVICE, F16_RANGE) if (window, hkv) == (128, 8) else (MIMO_OK, 0))


def test_debug_build_reports_an_fp8_decode_query_beyond_the_f16_range(cuda_device):
    """The FP8 decode multiplies Q in f16: a query entry of 1e5 sets the f16-range bit in the
    debug build; the same call with the query in range leaves it clear."""
    dev = cuda_device
    lengths = [700, 4096]
    inp = wl.decode_fp8_inputs(2, 64, 4, 4096, lengths, seed=69)
    d = {k: v.to(dev) for k, v in inp.items() if v is not None}
    with _library("debug") as lib:
        _lib.decode_fp8(d["q"], d["k8"], d["v8"], d["k_scale"], d["v_scale"], d["lengths"], d["sink"],
                        kind="linear")
        torch.cuda.synchronize()
        assert _status(lib) == (MIMO_OK, 0)
        q = d["q"].clone()
        q[1, 3, 17] = 1e5
        _lib.decode_fp8(q, d["k8"], d["v8"], d["k_scale"], d["v_scale"], d["lengths"], d["sink"], kind="linear")
        torch.cuda.synchronize()
        assert _status(lib) == (MIMO_ERR_DEVICE, F16_RANGE)
