"""Token-level sparse decode parity (recent window + selected indices, one softmax)."""

import numpy as np
import pytest
import torch

from hybrid_sliding_window_sink_b200 import _lib, workloads as wl
from oracle import ref
from parity_util import compare

pytestmark = pytest.mark.gpu


def _inputs(B, hq, hkv, cap, lengths, recent, n_sel, seed, device="cpu"):
    inp = wl.decode_inputs(B, hq, hkv, cap, lengths, seed=seed, device=device)
    hi = [max(0, L - recent) for L in lengths]
    inp["sel"] = wl.sorted_unique_indices(B, hkv, n_sel, hi, seed=seed).to(device)
    return inp


def _run(inp, recent, dev, sink=True):
    return _lib.sparse(inp["q"].to(dev), inp["k_cache"].to(dev), inp["v_cache"].to(dev),
                       inp["lengths"].to(dev), inp["sel"].to(dev),
                       inp["sink"].to(dev) if sink else None, recent=recent)


@pytest.mark.parametrize("B,hq,hkv,cap,lengths,recent,n_sel", [
    (2, 64, 4, 4096, [3000, 700], 128, 200),
    (3, 64, 4, 1024, [1024, 300, 129], 128, 1),
    (2, 16, 2, 2048, [2048, 1200], 128, 1024),
    (1, 8, 8, 512, [400], 16, 300),
    (2, 64, 4, 256, [50, 200], 128, 0),      # window only, one sequence shorter than it
])
def test_sparse_small(cuda_device, B, hq, hkv, cap, lengths, recent, n_sel):
    inp = _inputs(B, hq, hkv, cap, lengths, recent, n_sel, seed=400 + cap + n_sel)
    out, lse = _run(inp, recent, cuda_device)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.sparse_decode(wl.to_f64(inp["q"]), wl.to_f64(inp["k_cache"]),
                                     wl.to_f64(inp["v_cache"]), lengths, recent,
                                     inp["sel"].numpy(), wl.to_f64(inp["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, f"sparse {lengths}")


@pytest.mark.parametrize("B,hq,hkv,n_sel", [
    (15, 64, 4, 300),     # 60 (b, g) units of 428 keys, 16 heads per KV head
    (40, 32, 4, 100),     # 160 units, 8 heads per KV head
    (80, 16, 4, 64),      # 320 units (more than two per SM), 4 heads per KV head
])
def test_sparse_many_units(cuda_device, B, hq, hkv, n_sel):
    """Sparse calls over many (b, g) units with ragged lengths per sequence (different
    chunk plans and group sizes)."""
    r = np.random.default_rng(B + n_sel)
    cap = 512
    recent = 128
    lengths = [int(x) for x in r.integers(recent + n_sel, cap + 1, size=B)]
    inp = _inputs(B, hq, hkv, cap, lengths, recent, n_sel, seed=500 + B)
    out, lse = _run(inp, recent, cuda_device)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    o_ref, l_ref = ref.sparse_decode(wl.to_f64(inp["q"]), wl.to_f64(inp["k_cache"]),
                                     wl.to_f64(inp["v_cache"]), lengths, recent,
                                     inp["sel"].numpy(), wl.to_f64(inp["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, f"sparse B={B} n_sel={n_sel}")


def test_sparse_full_config(cuda_device):
    """B=8, L=262144, 64/4, recent 128 + 1,024 sorted unique indices: every output."""
    c = wl.SPARSE_DECODE
    lengths = [c.context] * c.batch
    inp = wl.decode_inputs(c.batch, c.hq, c.hkv, c.context, lengths, seed=c.seed, device=cuda_device)
    sel = wl.sorted_unique_indices(c.batch, c.hkv, c.n_sel, [c.context - c.recent] * c.batch,
                                   seed=c.seed)
    out, lse = _lib.sparse(inp["q"], inp["k_cache"], inp["v_cache"], inp["lengths"],
                           sel.to(cuda_device), inp["sink"], recent=c.recent)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    assert _lib.check_indices(inp["lengths"], sel.to(cuda_device), hq=c.hq, recent=c.recent,
                              capacity=c.context) == 0
    # oracle on exactly the rows the key sets touch
    o_ref = np.zeros((c.batch, c.hq, 128)); l_ref = np.zeros((c.batch, c.hq))
    sink = wl.to_f64(inp["sink"])
    group = c.hq // c.hkv
    for b in range(c.batch):
        for g in range(c.hkv):
            keys = ref.sparse_key_set(c.context, c.recent, sel[b, g].numpy())
            idx = torch.as_tensor(keys, device=cuda_device)
            K = wl.to_f64(inp["k_cache"][b, :, g].index_select(0, idx))
            V = wl.to_f64(inp["v_cache"][b, :, g].index_select(0, idx))
            for h in range(g * group, (g + 1) * group):
                o_ref[b, h], l_ref[b, h] = ref.attend_row(wl.to_f64(inp["q"][b, h]), K, V,
                                                          np.arange(len(keys)), sink[h],
                                                          1.0 / np.sqrt(192.0))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, c.name)
    del inp, out, lse
    torch.cuda.empty_cache()


def test_index_membership_bit_exact(cuda_device):
    """Q = 0 and one-hot values: output column d is non-zero exactly when the probe
    token carrying e_d is in the merged key set (recent window or selected)."""
    L, cap, recent, hkv, hq = 1000, 1024, 128, 2, 4
    r = np.random.default_rng(5)
    sel = np.stack([np.sort(r.choice(L - recent, 64, replace=False)) for _ in range(hkv)])
    probes = set()
    for g in range(hkv):
        s = sel[g]
        probes |= set(s[:20].tolist()) | set((s[:20] + 1).tolist()) | set((s[:20] - 1).tolist())
    probes |= {L - recent - 2, L - recent - 1, L - recent, L - recent + 1, L - 1, 0}
    probes = sorted(p for p in probes if 0 <= p < L)[:128]
    q = torch.zeros(1, hq, 192, dtype=torch.bfloat16)
    kc = torch.zeros(1, cap, hkv, 192, dtype=torch.bfloat16)
    vc = torch.zeros(1, cap, hkv, 128, dtype=torch.bfloat16)
    for d, t in enumerate(probes):
        vc[0, t, :, d] = 1.0
    inp = {"q": q, "k_cache": kc, "v_cache": vc, "lengths": torch.tensor([L], dtype=torch.int32),
           "sel": torch.from_numpy(sel[None].astype(np.int32)), "sink": torch.zeros(hq)}
    out, _ = _run(inp, recent, cuda_device)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    for h in range(hq):
        g = h // (hq // hkv)
        keyset = set(ref.sparse_key_set(L, recent, sel[g]).tolist())
        want = {d for d, t in enumerate(probes) if t in keyset}
        have = set(np.nonzero(o[0, h] != 0)[0].tolist())
        assert have == want, (h, sorted(have ^ want))


def test_sparse_padding_and_empty_cache(cuda_device):
    """Rows padded with -1 (fewer selected tokens than n_sel) and an empty cache (L = 0):
    the padding names no token and L = 0 gives o = 0, lse = sink, as the oracle says."""
    B, hq, hkv, cap, recent, n_sel = 4, 64, 4, 2048, 128, 300
    lengths = [2048, 300, 0, 129]
    inp = wl.decode_inputs(B, hq, hkv, cap, lengths, seed=450)
    sel = np.full((B, hkv, n_sel), -1, dtype=np.int32)
    r = np.random.default_rng(450)
    for b, L in enumerate(lengths):
        hi = max(0, L - recent)
        for g in range(hkv):
            m = min(hi, n_sel - 7 * g)     # a different number of real entries per row
            sel[b, g, :m] = np.sort(r.choice(hi, m, replace=False))
    inp["sel"] = torch.from_numpy(sel)
    out, lse = _run(inp, recent, cuda_device)
    torch.cuda.synchronize()
    assert _lib.last_device_error() == 0
    assert _lib.check_indices(inp["lengths"].to(cuda_device), inp["sel"].to(cuda_device), hq=hq,
                              recent=recent, capacity=cap) == 0
    o_ref, l_ref = ref.sparse_decode(wl.to_f64(inp["q"]), wl.to_f64(inp["k_cache"]),
                                     wl.to_f64(inp["v_cache"]), lengths, recent, sel,
                                     wl.to_f64(inp["sink"]))
    compare(wl.to_f64(out), o_ref, wl.to_f64(lse), l_ref, "sparse with -1 padding and L = 0")


def test_check_indices_counts_violations(cuda_device):
    L = torch.tensor([500, 500, 0], dtype=torch.int32, device=cuda_device)
    good = np.arange(0, 300, 3, dtype=np.int32)
    sel = np.stack([good, good, good, good[::-1].copy(), good, good])
    sel[4, 5] = sel[4, 4]                    # duplicate
    sel = torch.from_numpy(sel.reshape(3, 2, -1)).to(cuda_device)
    # rows: (0,0) ok, (0,1) ok, (1,0) ok, (1,1) unsorted, (2,*) indices beyond L - recent
    # (L = 0 itself is allowed), and (2,0) also a duplicate
    n = _lib.check_indices(L, sel, hq=4, recent=128, capacity=1000)
    assert n == 3
    # -1 padding after the real entries is valid; a -1 before a real entry is not
    pad = sel.clone()
    pad[0, 0, 50:] = -1
    pad[0, 1, 10:20] = -1
    n2 = _lib.check_indices(L, pad, hq=4, recent=128, capacity=1000)
    assert n2 == 4
