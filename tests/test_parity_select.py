"""Token selection for the sparse decode: C ABI against the oracle.

With small-integer queries and keys every score is an exact integer in fp32 and float64,
so the selected indices must agree bit for bit (ties included: lower index first). With
N(0,1) inputs the fp32 and float64 scores can order near-ties differently; there the check
is that every disagreement lies within rounding of the selection threshold."""

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from oracle import ref

pytestmark = pytest.mark.gpu


def _int_inputs(B, hq, hkv, cap, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randint(-2, 3, (B, hq, 192), generator=g).to(torch.bfloat16)
    k = torch.randint(-2, 3, (B, cap, hkv, 192), generator=g).to(torch.bfloat16)
    return q, k


@pytest.mark.parametrize("B,hq,hkv,cap,lengths,recent,n_sel", [
    (2, 64, 4, 8192, [8192, 3000], 128, 1024),    # MiMo GA layout (16 heads per KV head)
    (3, 16, 2, 2000, [2000, 1153, 600], 128, 64),
    (1, 8, 8, 700, [700], 0, 572),                # one head per KV head, no recent window
    (2, 4, 1, 300, [300, 140], 128, 12),          # exactly as many candidates as selected
])
def test_select_exact_on_integer_scores(cuda_device, B, hq, hkv, cap, lengths, recent, n_sel):
    q, k = _int_inputs(B, hq, hkv, cap, seed=1800 + cap)
    L = torch.tensor(lengths, dtype=torch.int32)
    sel = _lib.select_tokens(q.to(cuda_device), k.to(cuda_device), L.to(cuda_device), recent=recent,
                             n_sel=n_sel)
    torch.cuda.synchronize()
    want = ref.select_tokens(wl.to_f64(q), wl.to_f64(k), lengths, recent, n_sel)
    assert np.array_equal(sel.cpu().numpy().astype(np.int64), want)


@pytest.mark.parametrize("lengths", [[140, 2000, 128, 0], [129, 1153]])
def test_select_short_rows_against_oracle(cuda_device, lengths):
    """Sequences with fewer candidates than n_sel keep all of them, then -1 (the oracle's
    rule), next to sequences with enough candidates."""
    B, cap = len(lengths), max(lengths)
    q, k = _int_inputs(B, 16, 2, cap, seed=5 + cap)
    sel = _lib.select_tokens(q.to(cuda_device), k.to(cuda_device),
                             torch.tensor(lengths, dtype=torch.int32, device=cuda_device),
                             recent=128, n_sel=20)
    torch.cuda.synchronize()
    want = ref.select_tokens(wl.to_f64(q), wl.to_f64(k), lengths, 128, 20)
    assert np.array_equal(sel.cpu().numpy().astype(np.int64), want)


def test_select_then_sparse_short_sequences(cuda_device):
    """Select, then sparse decode, on a batch where some sequences have fewer candidates than
    n_sel (their rows end in -1): the sparse decode skips the padding and matches the oracle,
    which here equals the dense decode of those sequences."""
    B, hq, hkv, cap, recent, n_sel = 4, 64, 4, 3000, 128, 1024
    lengths = [3000, 700, 128, 5]
    q, k = _int_inputs(B, hq, hkv, cap, seed=9)
    d = wl.decode_inputs(B, hq, hkv, cap, lengths, seed=10)
    dev = cuda_device
    L = d["lengths"].to(dev)
    sel = _lib.select_tokens(q.to(dev), k.to(dev), L, recent=recent, n_sel=n_sel)
    out, lse = _lib.sparse(d["q"].to(dev), k.to(dev), d["v_cache"].to(dev), L, sel, d["sink"].to(dev),
                           recent=recent)
    assert _lib.check_indices(L, sel, hq=hq, recent=recent, capacity=cap) == 0
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    want_sel = ref.select_tokens(wl.to_f64(q), wl.to_f64(k), lengths, recent, n_sel)
    assert np.array_equal(sel.cpu().numpy().astype(np.int64), want_sel)
    o_ref, l_ref = ref.sparse_decode(wl.to_f64(d["q"]), wl.to_f64(k), wl.to_f64(d["v_cache"]), lengths,
                                     recent, want_sel, wl.to_f64(d["sink"]))
    from parity_util import compare
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "select -> sparse, short sequences")
    o_d, l_d = ref.decode(wl.to_f64(d["q"][1:]), wl.to_f64(k[1:]), wl.to_f64(d["v_cache"][1:]), "linear",
                          lengths[1:], wl.to_f64(d["sink"]))
    compare(wl.to_f64(out[1:]), o_d, wl.to_f64(lse[1:]), l_d, "short sequences = dense decode")


def test_select_random_scores_within_rounding(cuda_device):
    B, hq, hkv, cap, recent, n_sel = 2, 64, 4, 20000, 128, 1024
    lengths = [20000, 9000]
    d = wl.decode_inputs(B, hq, hkv, cap, lengths, seed=1900)
    sel = _lib.select_tokens(d["q"].to(cuda_device), d["k_cache"].to(cuda_device),
                             d["lengths"].to(cuda_device), recent=recent, n_sel=n_sel)
    torch.cuda.synchronize()
    got = sel.cpu().numpy()
    q, k = wl.to_f64(d["q"]), wl.to_f64(d["k_cache"])
    want = ref.select_tokens(q, k, lengths, recent, n_sel)
    G = hq // hkv
    for b in range(B):
        hi = lengths[b] - recent
        for g in range(hkv):
            s = got[b, g]
            assert np.all(np.diff(s) > 0) and s[0] >= 0 and s[-1] < hi
            score = (k[b, :hi, g] @ q[b, g * G:(g + 1) * G].T).max(axis=1)
            thr = np.sort(score)[::-1][n_sel - 1]
            diff = set(s.tolist()) ^ set(want[b, g].tolist())
            # fp32 dot products of 192 terms: relative error well under 1e-5 of the magnitudes
            tol = 1e-4 * max(1.0, abs(thr))
            assert all(abs(score[t] - thr) <= tol for t in diff), sorted(diff)[:8]


def test_select_then_sparse(cuda_device):
    """The selected indices drive mimo_attn_sparse exactly as the oracle's do."""
    B, hq, hkv, cap = 2, 64, 4, 4096
    lengths = [4096, 2500]
    q, k = _int_inputs(B, hq, hkv, cap, seed=7)
    d = wl.decode_inputs(B, hq, hkv, cap, lengths, seed=8)
    dev = cuda_device
    L = d["lengths"].to(dev)
    sel = _lib.select_tokens(q.to(dev), k.to(dev), L, recent=128, n_sel=512)
    out, lse = _lib.sparse(d["q"].to(dev), k.to(dev), d["v_cache"].to(dev), L, sel, d["sink"].to(dev),
                           recent=128)
    torch.cuda.synchronize()
    want_sel = ref.select_tokens(wl.to_f64(q), wl.to_f64(k), lengths, 128, 512)
    assert np.array_equal(sel.cpu().numpy().astype(np.int64), want_sel)
    o_ref, l_ref = ref.sparse_decode(wl.to_f64(d["q"]), wl.to_f64(k), wl.to_f64(d["v_cache"]), lengths,
                                     128, want_sel, wl.to_f64(d["sink"]))
    from parity_util import compare
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "select -> sparse")
