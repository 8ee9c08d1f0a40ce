"""Parity at the exact shapes the benchmark times, for the widened rows.

Each test launches the library with the benchmark's sizes (so the same chunk plans, grids
and scheduling rounds run) and compares against the float64 oracle on sampled units that
the oracle finishes in seconds: whole (sequence, KV head) units for decode-side calls (all
their query heads and draft tokens), and sampled query rows for the chunked prefill. The
oracle functions are called as they stand, on slices of the inputs.
"""

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from oracle import ref
from parity_util import compare

pytestmark = pytest.mark.gpu


def _sampled_sequences(lengths, extra, seed):
    """Indices of the shortest and longest sequences plus ``extra`` seeded others."""
    order = np.argsort(lengths, kind="stable")
    r = np.random.default_rng(seed)
    pick = {int(order[0]), int(order[1]), int(order[-1]), int(order[-2])}
    pick |= set(r.choice(len(lengths), extra, replace=False).tolist())
    return sorted(pick)


def _q_and_sink(batch, rows, hq, seed, dev):
    g = torch.Generator(device=dev).manual_seed(seed)
    q = torch.randn(batch, *rows, hq, wl.DQK, generator=g, device=dev).to(torch.bfloat16)
    sink = torch.randn(hq, generator=g, device=dev)
    return q, sink


def test_mtp_ga_layer_bench_shape(cuda_device):
    """MTP verification (1 + 3 draft tokens) on one GA layer as the benchmark runs it: B=64,
    lengths uniform in [4096, 131072], one linear cache of 131072 slots, 64 Q / 4 KV heads
    (the multi-chunk plan with its combine). Oracle on 6+ whole sequences x 2 KV heads."""
    c, T, dev = wl.HYBRID_DECODE_GA, 4, cuda_device
    L = wl.lengths_uniform(c.batch, c.min_len, c.max_len, seed=c.seed)
    inp = wl.decode_mq_inputs(c.batch, T, c.hq, c.hkv, c.capacity, L, seed=c.seed + 5, device=dev)
    out, lse = _lib.decode_mq(inp["q_mq"], inp["k_cache"], inp["v_cache"], inp["lengths"], inp["sink"],
                              kind="linear", window=0)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    Ls = L.tolist()
    G = c.hq // c.hkv
    sink = wl.to_f64(inp["sink"])
    got_o, got_l, want_o, want_l = [], [], [], []
    for i, b in enumerate(_sampled_sequences(Ls, 3, c.seed)):
        Lb = Ls[b]
        for g in ((0, 3), (1, 2))[i % 2]:
            hs = slice(g * G, (g + 1) * G)
            o, l = ref.decode_multi(wl.to_f64(inp["q_mq"][b:b + 1, :, hs]),
                                    wl.to_f64(inp["k_cache"][b:b + 1, :Lb, g:g + 1]),
                                    wl.to_f64(inp["v_cache"][b:b + 1, :Lb, g:g + 1]),
                                    "linear", [Lb], 0, sink[hs])
            want_o.append(o[0]); want_l.append(l[0])
            got_o.append(wl.to_f64(out[b, :, hs])); got_l.append(wl.to_f64(lse[b, :, hs]))
    compare(np.stack(got_o), np.stack(want_o), np.stack(got_l), np.stack(want_l), "MTP GA layer")
    assert torch.isfinite(out).all()
    del inp, out, lse
    torch.cuda.empty_cache()


def test_mtp_swa_layer_bench_shape(cuda_device):
    """MTP verification on one SWA layer as the benchmark runs it (B=64, rings of
    W + 3 = 131 slots, 64 Q / 8 KV): every output against the oracle."""
    c, T, dev = wl.HYBRID_DECODE_SWA, 4, cuda_device
    cap = wl.SWA_WINDOW + T - 1
    L = wl.lengths_uniform(c.batch, c.min_len, c.max_len, seed=c.seed)
    inp = wl.decode_mq_inputs(c.batch, T, c.hq, c.hkv, cap, L, seed=c.seed + 6, device=dev)
    out, lse = _lib.decode_mq(inp["q_mq"], inp["k_cache"], inp["v_cache"], inp["lengths"], inp["sink"],
                              kind="ring", window=wl.SWA_WINDOW)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.decode_multi(wl.to_f64(inp["q_mq"]), wl.to_f64(inp["k_cache"]),
                                    wl.to_f64(inp["v_cache"]), "ring", L.tolist(), wl.SWA_WINDOW,
                                    wl.to_f64(inp["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "MTP SWA layer")


def test_fp8_ga_layer_bench_shape(cuda_device):
    """FP8-cache decode on one GA layer as the benchmark runs it: B=64, lengths uniform in
    [4096, 131072], one linear cache of 131072 slots of random E4M3 bytes with per-row
    scales in [0.002, 0.01], 64 Q / 4 KV. Oracle on 6+ whole sequences x 2 KV heads."""
    c, dev = wl.HYBRID_DECODE_GA, cuda_device
    L = wl.lengths_uniform(c.batch, c.min_len, c.max_len, seed=c.seed)
    k8, v8, ks, vs = wl.random_fp8_cache(c.batch, c.capacity, c.hkv, seed=c.seed + 9, device=dev)
    q, sink = _q_and_sink(c.batch, (), c.hq, c.seed + 10, dev)
    out, lse = _lib.decode_fp8(q, k8, v8, ks, vs, L.to(dev), sink, kind="linear")
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    Ls = L.tolist()
    G = c.hq // c.hkv
    sk = wl.to_f64(sink)
    got_o, got_l, want_o, want_l = [], [], [], []
    f = lambda t: t.cpu().numpy()  # noqa: E731
    for i, b in enumerate(_sampled_sequences(Ls, 3, c.seed + 1)):
        Lb = Ls[b]
        for g in ((0, 3), (1, 2))[i % 2]:
            hs = slice(g * G, (g + 1) * G)
            sl = (slice(b, b + 1), slice(0, Lb), slice(g, g + 1))
            o, l = ref.decode_fp8(wl.to_f64(q[b:b + 1, hs]), f(k8[sl]), f(v8[sl]), f(ks[sl]), f(vs[sl]),
                                  "linear", [Lb], sk[hs])
            want_o.append(o[0]); want_l.append(l[0])
            got_o.append(wl.to_f64(out[b, hs])); got_l.append(wl.to_f64(lse[b, hs]))
    compare(np.stack(got_o), np.stack(want_o), np.stack(got_l), np.stack(want_l), "FP8 GA layer")
    assert torch.isfinite(out).all()
    del k8, v8, ks, vs, out, lse
    torch.cuda.empty_cache()


def test_fp8_swa_layer_bench_shape(cuda_device):
    """FP8-cache decode on one SWA layer as the benchmark runs it (B=64, rings of 128
    slots, 64 Q / 8 KV): every output against the oracle."""
    c, dev = wl.HYBRID_DECODE_SWA, cuda_device
    L = wl.lengths_uniform(c.batch, c.min_len, c.max_len, seed=c.seed)
    k8, v8, ks, vs = wl.random_fp8_cache(c.batch, c.capacity, c.hkv, seed=c.seed + 11, device=dev)
    q, sink = _q_and_sink(c.batch, (), c.hq, c.seed + 12, dev)
    out, lse = _lib.decode_fp8(q, k8, v8, ks, vs, L.to(dev), sink, kind="ring")
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.decode_fp8(wl.to_f64(q), k8.cpu().numpy(), v8.cpu().numpy(), ks.cpu().numpy(),
                                  vs.cpu().numpy(), "ring", L.tolist(), wl.to_f64(sink))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "FP8 SWA layer")


def _chunk_rows(n, nrand, seed, block):
    """Rows of a chunk to check: both ends, around multiples of ``block`` and of 128,
    and seeded random rows."""
    r = np.random.default_rng(seed)
    rows = set(range(0, 48)) | set(range(n - 48, n))
    for t in list(range(block, n, block * max(1, n // (24 * block)))) + [127, 128, 255, 256, n // 2]:
        rows |= {t - 1, t, t + 1}
    rows |= set(r.choice(n, nrand, replace=False).tolist())
    return sorted(x for x in rows if 0 <= x < n)


@pytest.mark.parametrize("layer", ["swa", "ga"])
def test_chunk_prefill_bench_shape(cuda_device, layer):
    """Chunked prefill as the benchmark runs it: a 16384-token chunk after a 16384-token
    prefix whose K is stored rotated, B=1; SWA layer (64 Q / 8 KV, W=128, the K/V-ring
    kernel) and GA layer (64 Q / 4 KV, the pair kernel's multi-round schedule at an
    offset). Oracle on sampled rows; SWA all 64 heads, GA 4 heads per row that rotate
    through all 64."""
    prefix = chunk = 16384
    hq, hkv, window, theta = ((64, 8, wl.SWA_WINDOW, wl.SWA_THETA) if layer == "swa"
                              else (64, 4, 0, wl.GA_THETA))
    dev = cuda_device
    inp = wl.prefill_inputs(1, prefix + chunk, hq, hkv, seed=1700, device=dev,
                            k_scale=0.5 if window == 0 else 1.0)
    q = inp["q"][:, prefix:].contiguous()
    out, lse = _lib.prefill_chunk(q, inp["k"], inp["v"], inp["sink"], pos_offset=prefix,
                                  k_prefix_rotated=True, window=window, rope_theta=theta, rot_dims=wl.ROT_DIMS)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    pos = _chunk_rows(chunk, 256 if layer == "swa" else 96, 1701, 16 if layer == "swa" else 8)
    if layer == "swa":
        rows = [(0, h, i) for i in pos for h in range(hq)]
    else:
        rows = [(0, (4 * a + j * 16 + a // 16) % hq, i) for a, i in enumerate(pos) for j in range(4)]
    k = wl.to_f64(inp["k"])
    v = wl.to_f64(inp["v"])
    o_ref, l_ref = ref.prefill_chunk(wl.to_f64(q), k, v, prefix, True, wl.to_f64(inp["sink"]), window,
                                     theta, wl.ROT_DIMS, rows=rows)
    og = out[0]
    o_gpu = np.stack([wl.to_f64(og[i, h]) for (_, h, i) in rows])
    l_gpu = np.array([float(lse[0, h, i]) for (_, h, i) in rows])
    compare(o_gpu, o_ref, l_gpu, l_ref, f"chunked prefill {layer} 16K after 16K")
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    del inp, q, out, lse
    torch.cuda.empty_cache()


def test_select_bench_shape(cuda_device):
    """Token selection as the benchmark runs it (B=8, L=262144, 64 Q / 4 KV, recent 128,
    n_sel 1024: 16 compaction blocks per row) on small-integer q and K, whose scores are
    exact integers in fp32 and float64 with many ties at the threshold. Six whole
    (sequence, KV head) rows must equal the oracle's bit for bit."""
    c, dev = wl.SPARSE_DECODE, cuda_device
    q, k = wl.integer_qk(c.batch, c.hq, c.hkv, c.context, seed=c.seed, device=dev)
    lengths = [c.context] * c.batch
    L = torch.tensor(lengths, dtype=torch.int32, device=dev)
    sel = _lib.select_tokens(q, k, L, recent=c.recent, n_sel=c.n_sel)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    got = sel.cpu().numpy().astype(np.int64)
    G = c.hq // c.hkv
    for b, g in ((0, 0), (1, 3), (3, 1), (4, 2), (6, 0), (7, 3)):
        want = ref.select_tokens(wl.to_f64(q[b:b + 1, g * G:(g + 1) * G]), wl.to_f64(k[b:b + 1, :, g:g + 1]),
                                 [c.context], c.recent, c.n_sel)
        assert np.array_equal(got[b, g], want[0, 0]), (b, g)
    del q, k, sel
    torch.cuda.empty_cache()
