"""Chunked prefill over a KV prefix and KV-cache append: C ABI against the oracle."""

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from oracle import ref
from parity_util import compare

pytestmark = pytest.mark.gpu


def _rotated_prefix(k, off, theta, rot):
    """k with rows [0, off) replaced by their rotation (the oracle's, rounded to bf16), as a
    KV cache would hold them."""
    kk = k.clone()
    if off > 0:
        pos = np.arange(off, dtype=np.float64)
        kr = np.stack([ref.rope(wl.to_f64(k[b, :off]), pos, theta, rot) for b in range(k.shape[0])])
        kk[:, :off] = torch.from_numpy(kr).to(torch.bfloat16)
    return kk


@pytest.mark.parametrize("B,n,off,hq,hkv,window,rotated", [
    (1, 300, 1000, 64, 8, 128, True),      # SWA layer layout, chunk after a 1000-token prefix
    (1, 257, 600, 64, 4, 0, True),         # GA layer layout
    (2, 130, 1, 16, 2, 128, False),        # prefix of one token, raw prefix
    (1, 200, 0, 64, 4, 0, True),           # no prefix: plain prefill
    (1, 64, 4097, 16, 1, 7, True),         # tiny window far into the sequence
    (1, 100, 150, 32, 8, 300, False),      # window longer than the chunk, shorter than the keys
    # SWA ring kernel (8 heads per KV head, W <= 129, offset a multiple of 16)
    (1, 300, 1024, 64, 8, 128, True),      # SWA layer layout, stored-rotated prefix
    (2, 130, 16, 16, 2, 128, False),       # one raw prefix unit
    (1, 97, 4096, 16, 2, 129, True),       # W = 129, ragged last block
    (2, 1536, 2048, 64, 8, 128, True),     # long runs per CTA: ring units reused across blocks
])
def test_prefill_chunk(cuda_device, B, n, off, hq, hkv, window, rotated):
    theta = wl.SWA_THETA if window > 0 else wl.GA_THETA
    inp = wl.prefill_inputs(B, off + n, hq, hkv, seed=1300 + n + off, k_scale=0.5 if window == 0 else 1.0)
    k = _rotated_prefix(inp["k"], off, theta, 64) if rotated else inp["k"]
    q = inp["q"][:, off:].contiguous()
    dev = cuda_device
    out, lse = _lib.prefill_chunk(q.to(dev), k.to(dev), inp["v"].to(dev), inp["sink"].to(dev),
                                  pos_offset=off, k_prefix_rotated=rotated, window=window,
                                  rope_theta=theta, rot_dims=64)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.prefill_chunk(wl.to_f64(q), wl.to_f64(k), wl.to_f64(inp["v"]), off, rotated,
                                     wl.to_f64(inp["sink"]), window, theta, 64)
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, f"chunk off={off} n={n} W={window}")


@pytest.mark.parametrize("cuts", [(0, 250, 511, 700), (0, 256, 512, 700)])
def test_chunks_match_whole_prefill(cuda_device, cuts):
    """Three chunks (each reading the raw prefix) and one whole-sequence call both match the
    oracle's whole-sequence rows (chunks at offsets that are multiples of 16 run on the SWA
    ring kernel like the whole call, the others on the generic kernel)."""
    n, hq, hkv = 700, 16, 2
    inp = wl.prefill_inputs(1, n, hq, hkv, seed=1400)
    d = {k: v.to(cuda_device) for k, v in inp.items()}
    o_ref, l_ref = ref.prefill(wl.to_f64(inp["q"]), wl.to_f64(inp["k"]), wl.to_f64(inp["v"]),
                               wl.to_f64(inp["sink"]), 128, 1e4, 64)
    whole, lw = _lib.prefill(d["q"], d["k"], d["v"], d["sink"], window=128, rope_theta=1e4, rot_dims=64)
    torch.cuda.synchronize()
    compare(wl.to_f64(whole), o_ref, wl.to_f64(lw), l_ref, "whole")
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = _lib.prefill_chunk(d["q"][:, a:b].contiguous(), d["k"][:, :b].contiguous(),
                                  d["v"][:, :b].contiguous(), d["sink"], pos_offset=a,
                                  k_prefix_rotated=False, window=128, rope_theta=1e4, rot_dims=64)
        torch.cuda.synchronize()
        compare(wl.to_f64(o), o_ref[:, a:b], wl.to_f64(l), l_ref[:, :, a:b], f"chunk [{a},{b})")


@pytest.mark.parametrize("kind,cap,off,n", [
    ("ring", 128, 0, 300),      # chunk longer than the ring: only its last 128 tokens land
    ("ring", 131, 4000, 50),    # wrap-around in the middle of the chunk
    ("linear", 2048, 1000, 600),
])
def test_cache_append(cuda_device, kind, cap, off, n):
    B, hkv = 2, 4
    g = torch.Generator().manual_seed(1500 + n)
    kch = torch.randn(B, n, hkv, 192, generator=g).to(torch.bfloat16)
    vch = torch.randn(B, n, hkv, 128, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, cap, hkv, 192, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, cap, hkv, 128, generator=g).to(torch.bfloat16)
    dev = cuda_device
    kd, vd = kc.to(dev), vc.to(dev)
    _lib.cache_append(kch.to(dev), vch.to(dev), kd, vd, pos_offset=off, rope_theta=1e4, rot_dims=64,
                      kind=kind)
    torch.cuda.synchronize()
    k_ref, v_ref = ref.cache_append(wl.to_f64(kch), wl.to_f64(vch), off, 1e4, 64, kind,
                                    wl.to_f64(kc), wl.to_f64(vc))
    # V and untouched slots: bit-exact; rotated K: the bf16 rounding (2^-9 relative) of the
    # rotation, which the GPU forms in fp32 (about 1e-7 of |x| + |y| for inputs of order 1)
    assert torch.equal(vd.cpu().double(), torch.from_numpy(v_ref))
    got = wl.to_f64(kd)
    want = k_ref
    tol = np.abs(want) * 2.0 ** -8 + 1e-5
    assert np.all(np.abs(got - want) <= tol), float(np.max(np.abs(got - want) - tol))


def test_append_then_decode_matches_prefill(cuda_device):
    """Append a prompt to a ring cache in two chunks, then decode the last prompt token as
    the next step would see it. The oracle side appends with ref.cache_append and stores
    the values as bf16 (what the cache holds), then runs ref.decode; the GPU's decode also
    agrees with its own prefill row of that token."""
    n, hq, hkv = 400, 64, 8
    inp = wl.prefill_inputs(1, n, hq, hkv, seed=1600, device=cuda_device)
    whole, lw = _lib.prefill(inp["q"], inp["k"], inp["v"], inp["sink"], window=128,
                             rope_theta=1e4, rot_dims=64)
    ring_k = torch.zeros(1, 128, hkv, 192, dtype=torch.bfloat16, device=cuda_device)
    ring_v = torch.zeros(1, 128, hkv, 128, dtype=torch.bfloat16, device=cuda_device)
    kc_ref, vc_ref = np.zeros((1, 128, hkv, 192)), np.zeros((1, 128, hkv, 128))
    for a, b in ((0, 333), (333, 400)):
        _lib.cache_append(inp["k"][:, a:b].contiguous(), inp["v"][:, a:b].contiguous(), ring_k, ring_v,
                          pos_offset=a, rope_theta=1e4, rot_dims=64, kind="ring")
        kc_ref, vc_ref = ref.cache_append(wl.to_f64(inp["k"][:, a:b]), wl.to_f64(inp["v"][:, a:b]), a,
                                          1e4, 64, "ring", kc_ref, vc_ref)
    as_bf16 = lambda x: torch.from_numpy(x).to(torch.bfloat16)  # noqa: E731
    # the decode query is the rotated q of position n-1 (rotated by the oracle, held as bf16)
    qr = ref.rope(wl.to_f64(inp["q"][0, n - 1:n]), np.array([n - 1.0]), 1e4, 64)
    qd = as_bf16(qr)
    o, l = _lib.decode(qd.to(cuda_device), ring_k, ring_v,
                       torch.tensor([n], dtype=torch.int32, device=cuda_device), inp["sink"], kind="ring")
    torch.cuda.synchronize()
    o_ref, l_ref = ref.decode(wl.to_f64(qd), wl.to_f64(as_bf16(kc_ref)), wl.to_f64(as_bf16(vc_ref)), "ring",
                              [n], wl.to_f64(inp["sink"]))
    compare(wl.to_f64(o), o_ref, wl.to_f64(l), l_ref, "append + decode vs oracle")
    compare(wl.to_f64(o[0]), wl.to_f64(whole[0, n - 1]), wl.to_f64(l[0]), wl.to_f64(lw[0, :, n - 1]),
            "append + decode vs prefill row")
