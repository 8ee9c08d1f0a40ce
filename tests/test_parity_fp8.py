"""FP8 (E4M3, per-(token, KV head) scales) decode and sparse decode: C ABI against the oracle,
which decodes the same bytes and scales in float64."""

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from oracle import ref
from parity_util import compare

pytestmark = pytest.mark.gpu


def _f(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("B,hq,hkv,kind,cap,lengths", [
    (3, 64, 8, "ring", 128, [50, 128, 7000]),        # SWA layer layout, ring of 128
    (2, 64, 4, "linear", 3000, [3000, 1289]),        # GA layer layout, several chunks
    (2, 16, 4, "linear", 200, [1, 200]),             # one chunk, a one-token sequence
    (1, 8, 8, "ring", 128, [300]),                   # one query head per KV head
])
def test_decode_fp8(cuda_device, B, hq, hkv, kind, cap, lengths):
    inp = wl.decode_fp8_inputs(B, hq, hkv, cap, lengths, seed=1100 + cap + B)
    d = {k: (v.to(cuda_device) if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, lse = _lib.decode_fp8(d["q"], d["k8"], d["v8"], d["k_scale"], d["v_scale"], d["lengths"],
                               d["sink"], kind=kind)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.decode_fp8(wl.to_f64(inp["q"]), _f(inp["k8"]), _f(inp["v8"]),
                                  _f(inp["k_scale"]), _f(inp["v_scale"]), kind, lengths,
                                  wl.to_f64(inp["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, f"fp8 decode {kind} {hq}/{hkv}")


def test_decode_fp8_extreme_bytes(cuda_device):
    """Subnormal, zero, negative-zero and largest E4M3 bytes, and scales far from 1."""
    B, hq, hkv, cap = 2, 16, 2, 96
    r = np.random.default_rng(3)
    pool = np.array([0x00, 0x80, 0x01, 0x81, 0x07, 0x08, 0x7E, 0xFE, 0x38, 0xB8, 0x30, 0x44],
                    dtype=np.uint8)
    k8 = torch.from_numpy(r.choice(pool, size=(B, cap, hkv, 192)))
    v8 = torch.from_numpy(r.choice(pool, size=(B, cap, hkv, 128)))
    ks = torch.from_numpy(r.uniform(1e-4, 4e-3, size=(B, cap, hkv)).astype(np.float32))
    vs = torch.from_numpy(r.uniform(1e-3, 1e-2, size=(B, cap, hkv)).astype(np.float32))   # |v| <= 4.5
    base = wl.decode_inputs(B, hq, hkv, cap, [96, 40], seed=5)
    q, sink, L = base["q"], base["sink"], base["lengths"]
    dev = cuda_device
    out, lse = _lib.decode_fp8(q.to(dev), k8.to(dev), v8.to(dev), ks.to(dev), vs.to(dev), L.to(dev),
                               sink.to(dev), kind="linear")
    torch.cuda.synchronize()
    o_ref, l_ref = ref.decode_fp8(wl.to_f64(q), _f(k8), _f(v8), _f(ks), _f(vs), "linear", [96, 40],
                                  wl.to_f64(sink))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "fp8 extreme bytes")


@pytest.mark.parametrize("B,hq,hkv,cap,L,recent,n_sel", [
    (2, 64, 4, 4096, [3000, 1500], 128, 1024),
    (3, 16, 2, 600, [600, 300, 129], 128, 1),
])
def test_sparse_fp8(cuda_device, B, hq, hkv, cap, L, recent, n_sel):
    inp = wl.decode_fp8_inputs(B, hq, hkv, cap, L, seed=1200 + n_sel)
    sel = wl.sorted_unique_indices(B, hkv, n_sel, [x - recent for x in L], seed=1200 + n_sel)
    dev = cuda_device
    out, lse = _lib.sparse_fp8(inp["q"].to(dev), inp["k8"].to(dev), inp["v8"].to(dev),
                               inp["k_scale"].to(dev), inp["v_scale"].to(dev),
                               inp["lengths"].to(dev), sel.to(dev), inp["sink"].to(dev), recent=recent)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.sparse_decode_fp8(wl.to_f64(inp["q"]), _f(inp["k8"]), _f(inp["v8"]),
                                         _f(inp["k_scale"]), _f(inp["v_scale"]), L, recent,
                                         sel.numpy(), wl.to_f64(inp["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, f"fp8 sparse n_sel={n_sel}")


def test_sparse_fp8_short_selection_rows(cuda_device):
    """A sequence with fewer candidates than n_sel (L - recent < n_sel) has selection rows
    ending in -1 entries, as the token selection writes them; the FP8 sparse kernel skips those
    entries, and the result matches the oracle on the valid indices."""
    B, hq, hkv, cap, recent, n_sel = 2, 16, 2, 512, 64, 200
    L = [512, 150]                                   # the second sequence has 86 candidates
    inp = wl.decode_fp8_inputs(B, hq, hkv, cap, L, seed=1300)
    sel = torch.full((B, hkv, n_sel), -1, dtype=torch.int32)
    sel[0] = wl.sorted_unique_indices(1, hkv, n_sel, [L[0] - recent], seed=1301)[0]
    sel[1, :, :L[1] - recent] = torch.arange(L[1] - recent, dtype=torch.int32)
    dev = cuda_device
    out, lse = _lib.sparse_fp8(inp["q"].to(dev), inp["k8"].to(dev), inp["v8"].to(dev),
                               inp["k_scale"].to(dev), inp["v_scale"].to(dev),
                               inp["lengths"].to(dev), sel.to(dev), inp["sink"].to(dev), recent=recent)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.sparse_decode_fp8(wl.to_f64(inp["q"]), _f(inp["k8"]), _f(inp["v8"]),
                                         _f(inp["k_scale"]), _f(inp["v_scale"]), L, recent,
                                         sel.numpy(), wl.to_f64(inp["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "fp8 sparse, -1 padded rows")


def test_decode_fp8_scales_over_many_orders(cuda_device):
    """V scales spread over seven orders of magnitude (1e-7 .. 1, every 17th row exactly 0) and
    K scales over three: the kernel folds each key's V scale into P with a power-of-two factor
    per 32 keys, so P * vs stays inside f16 for the large scales without losing the small ones.
    The outputs reach a few hundred (E4M3 bytes up to 448 times scales up to 1; bf16 rounds them
    to about 2^-9 of their size), so both sides are compared after dividing by 1000; the lse does
    not depend on V."""
    B, hq, hkv, cap = 2, 64, 4, 1000
    L = [1000, 333]
    inp = wl.decode_fp8_inputs(B, hq, hkv, cap, L, seed=1310)
    r = np.random.default_rng(1311)
    vs = torch.from_numpy((10.0 ** r.uniform(-7, 0, size=(B, cap, hkv))).astype(np.float32))
    vs[:, ::17] = 0.0
    ks = torch.from_numpy((10.0 ** r.uniform(-4, -1, size=(B, cap, hkv))).astype(np.float32))
    dev = cuda_device
    out, lse = _lib.decode_fp8(inp["q"].to(dev), inp["k8"].to(dev), inp["v8"].to(dev), ks.to(dev), vs.to(dev),
                               inp["lengths"].to(dev), inp["sink"].to(dev), kind="linear")
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.decode_fp8(wl.to_f64(inp["q"]), _f(inp["k8"]), _f(inp["v8"]), _f(ks), _f(vs), "linear",
                                  L, wl.to_f64(inp["sink"]))
    assert np.abs(o_ref).max() > 10.0                # the large scales do reach the output
    compare(wl.to_f64(out) / 1000.0, o_ref / 1000.0, wl.to_f64(lse), l_ref, "fp8 scales over seven orders")
