"""The allocation-free sparse decode against the regular one.

mimo_attn_sparse_noalloc is for callers that cannot allocate device memory when
they call attention (for example a serving loop whose KV pools already hold nearly
all of HBM, or a plug-in whose host framework owns every allocation). It keeps its
split-KV partials in a fixed 8 MiB array inside the library. This test calls it
through the C ABI twice in a row, on different inputs, and then a third time with a
smaller plan, and checks each result against mimo_attn_sparse with a caller-provided
workspace, so stale contents left in the shared array by an earlier call cannot leak
into a later one. It also checks
that sizes needing more scratch than the array holds are refused before any launch.
This file sorts last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from parity_util import compare

pytestmark = pytest.mark.gpu


def _case(seed, dev, B=4, hq=64, hkv=4, L=20000, recent=128, n_sel=1024):
    lengths = [L - 17 * b for b in range(B)]
    inp = wl.decode_inputs(B, hq, hkv, L, lengths, seed=seed, device=dev)
    inp["sel"] = wl.sorted_unique_indices(B, hkv, n_sel, [x - recent for x in lengths],
                                          seed=seed).to(dev)
    return inp


def _noalloc(inp, recent, cap):
    B, hq, _ = inp["q"].shape
    hkv = inp["k_cache"].shape[2]
    n_sel = inp["sel"].shape[2]
    shape = _lib.make_shape(B, 1, hq, hkv)
    out = torch.empty(B, hq, 128, dtype=torch.bfloat16, device=inp["q"].device)
    lse = torch.empty(B, hq, dtype=torch.float32, device=inp["q"].device)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = _lib.lib().mimo_attn_sparse_noalloc(
        ctypes.byref(shape), p(inp["q"]), p(inp["k_cache"]), p(inp["v_cache"]), cap,
        inp["k_cache"].shape[1], p(inp["lengths"]), recent, p(inp["sel"]), n_sel, p(inp["sink"]),
        p(out), p(lse), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out, lse


def test_noalloc_matches_workspace_version_twice(cuda_device):
    recent, cap = 128, 20000
    a = _case(501, cuda_device)
    b = _case(502, cuda_device)
    # a third call with a smaller batch and fewer selected tokens: fewer chunks per
    # (sequence, KV head) and a different slot layout in the array than the calls before it
    c = _case(503, cuda_device, B=2, n_sel=300)
    need = _lib.workspace_size(4, 64, 4, op=_lib.MIMO_OP_SPARSE, capacity=cap, recent=recent,
                               n_sel=1024)
    need_c = _lib.workspace_size(2, 64, 4, op=_lib.MIMO_OP_SPARSE, capacity=cap, recent=recent,
                                 n_sel=300)
    assert 0 < need <= 8 * 1024 * 1024, need      # the case really uses the scratch array
    assert 0 < need_c < need, need_c
    for inp in (a, b, c):                          # calls in a row, different inputs and plans
        st, out, lse = _noalloc(inp, recent, cap)
        assert st == 0, _lib.STATUS.get(st)
        ref_out, ref_lse = _lib.sparse(inp["q"], inp["k_cache"], inp["v_cache"], inp["lengths"],
                                       inp["sel"], inp["sink"], recent=recent, capacity=cap)
        torch.cuda.synchronize()
        compare(out.double().cpu().numpy(), ref_out.double().cpu().numpy(),
                lse.double().cpu().numpy(), ref_lse.double().cpu().numpy(), "noalloc vs workspace")
    assert _lib.last_device_error() == 0


def test_noalloc_rejects_sizes_beyond_the_array(cuda_device):
    # B=64, 64 heads, 1152 keys per (b, g): the partials need more than 8 MiB
    B, hq, hkv, recent, n_sel, cap = 64, 64, 4, 128, 4096, 8192
    need = _lib.workspace_size(B, hq, hkv, op=_lib.MIMO_OP_SPARSE, capacity=cap, recent=recent,
                               n_sel=n_sel)
    assert need > 8 * 1024 * 1024
    shape = _lib.make_shape(B, 1, hq, hkv)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    ptr = ctypes.c_void_p(dummy.data_ptr())
    st = _lib.lib().mimo_attn_sparse_noalloc(ctypes.byref(shape), ptr, ptr, ptr, cap, cap, ptr,
                                             recent, ptr, n_sel, None, ptr, None, None)
    assert st == 5   # MIMO_ERR_WORKSPACE, nothing launched
    torch.cuda.synchronize()
