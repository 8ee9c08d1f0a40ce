"""Multi-query decode (MTP draft verification) parity: the C ABI against the oracle."""

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from oracle import ref
from parity_util import compare

pytestmark = pytest.mark.gpu


def _check(B, T, hq, hkv, kind, cap, lengths, window, dev, seed, sink=True):
    inp = wl.decode_mq_inputs(B, T, hq, hkv, cap, lengths, seed=seed)
    s = inp["sink"] if sink else None
    out, lse = _lib.decode_mq(inp["q_mq"].to(dev), inp["k_cache"].to(dev), inp["v_cache"].to(dev),
                              inp["lengths"].to(dev), None if s is None else s.to(dev), kind=kind,
                              window=window)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.decode_multi(wl.to_f64(inp["q_mq"]), wl.to_f64(inp["k_cache"]),
                                    wl.to_f64(inp["v_cache"]), kind, lengths, window,
                                    None if s is None else wl.to_f64(s))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, f"mq {kind} T={T} {hq}/{hkv} L={lengths}")
    return inp, out, lse


@pytest.mark.parametrize("B,T,hq,hkv,cap,lengths", [
    (3, 4, 64, 8, 131, [4, 131, 5000]),         # MiMo SWA: 8 heads per KV head, ring of W + 3
    (2, 1, 64, 8, 128, [60, 300]),              # one token: plain decode
    (2, 2, 16, 4, 140, [139, 1000]),            # 4 per KV head, ring larger than needed
    (1, 8, 16, 2, 135, [777]),                  # 8 draft tokens x 8 heads = 64 rows
    (2, 16, 8, 2, 143, [16, 2000]),             # 16 draft tokens x 4 heads
])
def test_ring(cuda_device, B, T, hq, hkv, cap, lengths):
    _check(B, T, hq, hkv, "ring", cap, lengths, 128, cuda_device, seed=600 + T + cap)


@pytest.mark.parametrize("B,T,hq,hkv,cap,lengths", [
    (2, 4, 64, 4, 3000, [3000, 1289]),          # MiMo GA: 16 heads per KV head, several chunks
    (3, 4, 64, 4, 200, [4, 64, 200]),           # one chunk
    (1, 1, 64, 4, 2500, [2500]),
    (2, 3, 32, 4, 1500, [700, 1500]),           # 3 draft tokens x 8 heads
    (2, 4, 64, 4, 200, [100, 130]),             # one chunk of two and of three 64-key subtiles
    (2, 4, 64, 4, 1200, [612, 1200]),           # last chunk of two subtiles after full ones
])
def test_linear(cuda_device, B, T, hq, hkv, cap, lengths):
    _check(B, T, hq, hkv, "linear", cap, lengths, 0, cuda_device, seed=700 + T + cap)


def test_ring_small_window_and_no_sink(cuda_device):
    _check(2, 3, 16, 2, "ring", 9, [9, 50], 7, cuda_device, seed=801, sink=False)


def test_one_token_matches_decode(cuda_device):
    """q_len = 1 on a ring of W slots and on a linear cache agrees with mimo_attn_decode."""
    lengths = [100, 128, 4000]
    inp = wl.decode_mq_inputs(3, 1, 64, 8, 128, lengths, seed=900, device=cuda_device)
    a, la = _lib.decode_mq(inp["q_mq"], inp["k_cache"], inp["v_cache"], inp["lengths"], inp["sink"],
                           kind="ring", window=128)
    b, lb = _lib.decode(inp["q_mq"][:, 0].contiguous(), inp["k_cache"], inp["v_cache"], inp["lengths"],
                        inp["sink"], kind="ring")
    torch.cuda.synchronize()
    o_ref, l_ref = ref.decode(wl.to_f64(inp["q_mq"][:, 0]), wl.to_f64(inp["k_cache"]),
                              wl.to_f64(inp["v_cache"]), "ring", lengths, wl.to_f64(inp["sink"]))
    compare(wl.to_f64(a[:, 0]), o_ref, wl.to_f64(la[:, 0]), l_ref, "mq T=1 vs oracle decode")
    compare(wl.to_f64(b), o_ref, wl.to_f64(lb), l_ref, "decode vs oracle")
    compare(wl.to_f64(a[:, 0]), wl.to_f64(b), wl.to_f64(la[:, 0]), wl.to_f64(lb), "mq T=1 vs decode")
