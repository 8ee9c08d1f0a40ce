"""Prefill parity: the sm_100a kernel through the C ABI against the float64 oracle."""

import math

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from oracle import ref
from parity_util import compare

pytestmark = pytest.mark.gpu


def _run_and_compare(inp, window, theta, rot, dev, what, scale=0.0):
    q, k, v, sink = (inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev),
                     None if inp["sink"] is None else inp["sink"].to(dev))
    out, lse = _lib.prefill(q, k, v, sink, window=window, rope_theta=theta, rot_dims=rot,
                            softmax_scale=scale)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.prefill(wl.to_f64(inp["q"]), wl.to_f64(inp["k"]), wl.to_f64(inp["v"]),
                               None if inp["sink"] is None else wl.to_f64(inp["sink"]),
                               window, theta, rot, scale=scale or None)
    return compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, what)


def test_tiny_swa_config(cuda_device):
    """Tiny SWA+sink prefill: n=1024, 8 Q / 1 KV heads, W=128, RoPE 64 dims theta 1e4."""
    c = wl.TINY_SWA_PREFILL
    inp = wl.case_prefill_inputs(c)
    _run_and_compare(inp, c.window, c.theta, wl.ROT_DIMS, cuda_device, c.name)


@pytest.mark.parametrize("n,hq,hkv,window,sink,rot", [
    (16, 8, 1, 128, False, 0),        # one tile, no RoPE, no sink
    (16, 8, 1, 128, True, 64),
    (1, 8, 1, 128, True, 64),         # single row
    (37, 8, 1, 5, True, 64),          # ragged, tiny window
    (300, 8, 1, 128, True, 64),       # several row blocks, ragged tail
    (300, 16, 1, 128, True, 64),      # group 16 (8 positions per block)
    (300, 8, 2, 1, True, 64),         # window 1: only the diagonal
    (300, 8, 2, 299, True, 64),       # window n-1
    (200, 4, 1, 128, True, 64),       # group 4: P + W - 1 > 144, multi-tile SWA
    (200, 2, 2, 17, True, 16),        # group 1, 128 positions per block
])
def test_swa_shapes(cuda_device, n, hq, hkv, window, sink, rot):
    inp = wl.prefill_inputs(1, n, hq, hkv, seed=100 + n + hq + window, with_sink=sink)
    _run_and_compare(inp, window, wl.SWA_THETA, rot, cuda_device, f"swa n={n} {hq}/{hkv} W={window}")


@pytest.mark.parametrize("B,n,hq,hkv,window,rot", [
    (2, 3000, 16, 2, 128, 64),        # runs of row blocks crossing (b, kv-head) boundaries
    (1, 5000, 8, 1, 129, 64),         # widest window of the ring kernel
    (1, 2100, 64, 8, 100, 32),        # MiMo head layout, partial window, 32 rotated dims
    (3, 700, 8, 1, 128, 0),           # no RoPE
    (1, 2500, 16, 2, 7, 16),
])
def test_swa_ring_kernel(cuda_device, B, n, hq, hkv, window, rot):
    """SWA layers with 8 query heads per KV head and W <= 129 (the K/V ring kernel)."""
    inp = wl.prefill_inputs(B, n, hq, hkv, seed=150 + n + window)
    _run_and_compare(inp, window, wl.SWA_THETA, rot, cuda_device, f"swa-ring B={B} n={n} W={window}")


@pytest.mark.parametrize("B,n,hq,hkv,window,rot,period", [
    (1, 2000, 16, 2, 128, 64, 400),
    (2, 1500, 8, 1, 129, 32, 333),
    (1, 1200, 64, 8, 128, 64, 64),
])
def test_swa_ring_kernel_steep_scores(cuda_device, B, n, hq, hkv, window, rot, period):
    """Scores that climb by ~2.5 (log2 units) per 16 keys inside a window, resetting every
    `period` keys: the ring kernel's single-pass softmax must move its reference (and scale
    the P blocks already written) several times per row, and keep it where the row max comes
    first."""
    inp = wl.prefill_inputs(B, n, hq, hkv, seed=170 + n + period)
    # unrotated dims: q += 1, k += 4.7 (t mod period) / period, i.e. about 128 * 4.7 / period
    # added to every score per key of the saw tooth
    t = torch.arange(n, dtype=torch.float32)
    shift = 4.7 * torch.remainder(t, period) / period
    k = inp["k"].float()
    k[..., 64:] += shift[None, :, None, None]
    q = inp["q"].float()
    q[..., 64:] += 1.0
    inp["k"], inp["q"] = k.to(torch.bfloat16), q.to(torch.bfloat16)
    _run_and_compare(inp, window, wl.SWA_THETA, rot, cuda_device,
                     f"swa-ring steep B={B} n={n} W={window} period={period}")


@pytest.mark.parametrize("B,n,hq,hkv,rot,k_scale", [
    (1, 129, 8, 1, 64, 0.5),
    (1, 600, 16, 1, 64, 0.5),         # GA heads 16 per KV head, several key tiles
    (2, 300, 8, 2, 64, 1.0),          # batch 2
    (1, 257, 4, 1, 128, 1.0),         # group 4
    (1, 130, 2, 2, 192, 1.0),         # group 1, full-width RoPE
    (1, 200, 8, 1, 0, 1.0),           # no RoPE
])
def test_ga_shapes(cuda_device, B, n, hq, hkv, rot, k_scale):
    inp = wl.prefill_inputs(B, n, hq, hkv, seed=200 + n + hq, k_scale=k_scale)
    _run_and_compare(inp, 0, wl.GA_THETA, rot, cuda_device, f"ga B={B} n={n} {hq}/{hkv}")


@pytest.mark.parametrize("B,n,hq,hkv,rot,k_scale,ramp", [
    (2, 3000, 32, 2, 64, 0.5, False),  # 16 heads per KV head, more work items than SMs
    (1, 1000, 64, 8, 64, 1.0, False),  # 8 heads per KV head
    (1, 9, 16, 1, 64, 1.0, False),     # second row block wholly past the end, one key tile
    (1, 24, 16, 1, 32, 1.0, False),    # second row block partly past the end
    (3, 515, 16, 4, 0, 2.0, False),    # no RoPE, (b, kv-head) crossings
    (1, 700, 16, 1, 64, 1.0, True),    # scores grow along the sequence: running max moves often
    (1, 2049, 8, 1, 16, 1.0, True),
])
def test_ga_pair_kernel(cuda_device, B, n, hq, hkv, rot, k_scale, ramp):
    """Full causal prefix with 8 or 16 query heads per KV head: the kernel that pairs two
    row blocks per work item and rescales its output only when the running max jumps."""
    inp = wl.prefill_inputs(B, n, hq, hkv, seed=250 + n + hq, k_scale=k_scale)
    if ramp:
        # A shared offset on the unrotated dims of q (+1) and k (+2 t / n) adds about
        # 128 * 2 t / (n sqrt(192)) ~ 18 t / n to every score of key t, so the row max keeps
        # climbing from tile to tile while the values stay small enough for f16 rounding.
        shift = 2.0 * torch.arange(n, dtype=torch.float32) / n
        k = inp["k"].float()
        k[..., 64:] += shift[None, :, None, None]
        q = inp["q"].float()
        q[..., 64:] += 1.0
        inp["k"], inp["q"] = k.to(torch.bfloat16), q.to(torch.bfloat16)
    _run_and_compare(inp, 0, wl.GA_THETA, rot, cuda_device, f"ga-pair B={B} n={n} {hq}/{hkv}")


def test_window_ge_n_equals_ga(cuda_device):
    """W >= n is full causal attention: same result as window = 0, bit for bit."""
    inp = wl.prefill_inputs(1, 200, 8, 1, seed=7)
    q, k, v, s = (inp[x].to(cuda_device) for x in ("q", "k", "v", "sink"))
    a, la = _lib.prefill(q, k, v, s, window=200, rope_theta=1e4, rot_dims=64)
    b, lb = _lib.prefill(q, k, v, s, window=0, rope_theta=1e4, rot_dims=64)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_sink_closed_form_on_gpu(cuda_device):
    """V = 1 makes o the total weight S/(e^sink + S) = 1 - exp(sink - lse) (no oracle)."""
    inp = wl.prefill_inputs(1, 300, 8, 1, seed=9)
    v1 = torch.ones_like(inp["v"]).to(cuda_device)
    q, k, s = (inp[x].to(cuda_device) for x in ("q", "k", "sink"))
    out, lse = _lib.prefill(q, k, v1, s, window=128, rope_theta=1e4, rot_dims=64)
    torch.cuda.synchronize()
    want = 1.0 - torch.exp(s.double()[None, :, None] - lse.double())      # [1, Hq, n]
    got = out.double()[..., 0].permute(0, 2, 1)
    assert float((got - want).abs().max()) < 1e-2


def test_large_and_missing_sink(cuda_device):
    inp = wl.prefill_inputs(1, 150, 8, 1, seed=11)
    inp["sink"] = torch.full((8,), 30.0)
    _run_and_compare(inp, 128, 1e4, 64, cuda_device, "sink 30")
    inp["sink"] = torch.full((8,), -1e4)
    _run_and_compare(inp, 128, 1e4, 64, cuda_device, "sink -1e4")
    inp["sink"] = None
    _run_and_compare(inp, 0, 1e7, 64, cuda_device, "GA no sink")


def test_deterministic_and_guarded(cuda_device):
    """Two runs give identical bits; writes stay inside out / lse (guard bands)."""
    inp = wl.prefill_inputs(1, 333, 16, 1, seed=12)
    q, k, v, s = (inp[x].to(cuda_device) for x in ("q", "k", "v", "sink"))
    guard = 4096
    o_buf = torch.full((guard * 2 + 333 * 16 * 128,), 7.0, dtype=torch.bfloat16, device=cuda_device)
    l_buf = torch.full((guard * 2 + 16 * 333,), 7.0, dtype=torch.float32, device=cuda_device)
    out = o_buf[guard:guard + 333 * 16 * 128].view(1, 333, 16, 128)
    lse = l_buf[guard:guard + 16 * 333].view(1, 16, 333)
    _lib.prefill(q, k, v, s, window=128, rope_theta=1e4, rot_dims=64, out=out, lse=lse)
    first = (out.clone(), lse.clone())
    _lib.prefill(q, k, v, s, window=0, rope_theta=1e7, rot_dims=64, out=out, lse=lse)
    _lib.prefill(q, k, v, s, window=128, rope_theta=1e4, rot_dims=64, out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(first[0], out) and torch.equal(first[1], lse)
    assert bool((o_buf[:guard] == 7.0).all()) and bool((o_buf[-guard:] == 7.0).all())
    assert bool((l_buf[:guard] == 7.0).all()) and bool((l_buf[-guard:] == 7.0).all())


def _sample_rows(n, nrand, seed, ends=256):
    """The first and last ``ends`` rows, rows around the window and tile boundaries
    (127/128/129, 143-145, 255/256) and at 64 multiples of 16 spread over the sequence,
    and ``nrand`` seeded random rows."""
    r = np.random.default_rng(seed)
    rows = set(range(0, ends)) | set(range(n - ends, n))
    for t in (127, 128, 129, 143, 144, 145, 255, 256):
        rows |= {t - 1, t, t + 1}
    rows |= {16 * k for k in range(1, n // 16, max(1, n // (16 * 64)))}
    rows |= set(r.choice(n, nrand, replace=False).tolist())
    return sorted(x for x in rows if 0 <= x < n)


@pytest.mark.parametrize("case,nrand,heads", [
    (wl.SWA_PREFILL, 1024, None),
    (wl.GA_PREFILL, 1024, 4),
])
def test_full_size_sampled(cuda_device, case, nrand, heads):
    """Full-size configurations, exactly as the benchmark launches them, against the
    oracle on sampled rows: the first and last 256 rows, window and tile boundaries and
    1,024 seeded random rows. SWA: all 64 heads of every sampled row; GA: 4 heads per row
    (one per KV head), rotating so that every head is checked on a quarter of the rows."""
    inp = wl.case_prefill_inputs(case, device=cuda_device)
    out, lse = _lib.prefill(inp["q"], inp["k"], inp["v"], inp["sink"], window=case.window,
                            rope_theta=case.theta, rot_dims=wl.ROT_DIMS)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    n = case.seqlen
    pos = _sample_rows(n, nrand, case.seed)
    G = case.hq // case.hkv
    if heads is None:
        head_sets = [list(range(case.hq))] * len(pos)
    else:   # one head per KV head, shifted by one within the group from row to row
        head_sets = [[g * G + (a + g) % G for g in range(case.hkv)] for a in range(len(pos))]
    # the oracle receives the exact bf16 values: the sampled query rows and all of K, V
    qs = wl.to_f64(inp["q"][0, pos])                                  # [len(pos), Hq, 192]
    rows = [(0, h, i) for a, i in enumerate(pos) for h in head_sets[a]]
    q_rows = np.stack([qs[a, h] for a in range(len(pos)) for h in head_sets[a]])
    o_ref, l_ref = ref.prefill_rows(q_rows, wl.to_f64(inp["k"]), wl.to_f64(inp["v"]),
                                    wl.to_f64(inp["sink"]), case.window, case.theta, wl.ROT_DIMS,
                                    rows, case.hq)
    og = wl.to_f64(out[0, pos])                                       # [len(pos), Hq, 128]
    lg = wl.to_f64(lse[0][:, pos])                                    # [Hq, len(pos)]
    o_gpu = np.stack([og[a, h] for a in range(len(pos)) for h in head_sets[a]])
    l_gpu = np.array([lg[h, a] for a in range(len(pos)) for h in head_sets[a]])
    compare(o_gpu, o_ref, l_gpu, l_ref, case.name)
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    del inp, out, lse
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,n,hq,hkv,window,theta", [
    (1, 700, 64, 8, 128, 1e4),     # SWA ring kernel: rotated K and V carried in f16
    (1, 600, 64, 4, 0, 1e7),       # GA pair kernel: rotated K in f16
    (1, 300, 16, 4, 64, 1e4),      # generic kernel
])
def test_large_magnitudes_inside_the_f16_range(cuda_device, B, n, hq, hkv, window, theta):
    """K and V of magnitude in the thousands (Q scaled down so the logits keep their usual
    size) pass through the kernels' f16 operands without clamping: the outputs, divided by
    the V scale, and the lse match the oracle at the usual tolerances."""
    inp = wl.prefill_inputs(B, n, hq, hkv, seed=77 + n)
    q = (inp["q"].float() * 1e-3).to(torch.bfloat16)
    k = (inp["k"].float() * 1e3).to(torch.bfloat16)
    v = (inp["v"].float() * 2e3).to(torch.bfloat16)
    assert float(k.float().abs().max()) > 3000 and float(v.float().abs().max()) > 6000
    dev = cuda_device
    out, lse = _lib.prefill(q.to(dev), k.to(dev), v.to(dev), inp["sink"].to(dev), window=window,
                            rope_theta=theta, rot_dims=64)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.prefill(wl.to_f64(q), wl.to_f64(k), wl.to_f64(v), wl.to_f64(inp["sink"]), window, theta, 64)
    compare(wl.to_f64(out) / 2e3, o_ref / 2e3, wl.to_f64(lse), l_ref, f"large magnitudes W={window}")
