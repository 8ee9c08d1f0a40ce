"""Checks that pin the oracle to facts outside itself.

Each ``check_*`` takes the oracle module and raises AssertionError on a
mismatch. ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` plants mistakes in a copy of the oracle and requires
that some check fails for each one.

What each check compares against (pages: "MiMo-V2-Flash: Hybrid Sliding Window
Attention Architecture" = rslog.cc; "...MiMo-V2.6-Flash-MOPD混合SWA设计原理" =
pwwt.cn; "小米MiMo-V3的核心架构HySparse2" = aideepthink.cn):

* closed forms of the sink softmax (rslog.cc §4.2, §4.3);
* torch's scaled_dot_product_attention in float64 (an independent library
  routine for softmax attention) with the sink as one extra zero-valued key
  whose logit is the sink (rslog.cc §4.2: a virtual denominator term with no V);
* HF transformers' rotary embedding and rotate_half (pwwt.cn §5: partial
  rotary, two bases);
* brute-force set definitions (rslog.cc §2.1 window, §2.6 receptive field,
  aideepthink.cn §四.3 sparse key set);
* hand-derived golden fixtures under tests/golden/.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_values(x):
    """Round float64 samples to bf16 values (so inputs look like the GPU's)."""
    return torch.from_numpy(np.asarray(x)).to(torch.bfloat16).to(torch.float64).numpy()


def _rand_prefill(seed, B=1, n=40, hq=4, hkv=2, d=16, dv=8, scale_k=1.0):
    r = _rng(seed)
    q = _bf16_values(r.standard_normal((B, n, hq, d)))
    k = _bf16_values(r.standard_normal((B, n, hkv, d)) * scale_k)
    v = _bf16_values(r.standard_normal((B, n, hkv, dv)))
    sink = r.standard_normal(hq)
    return q, k, v, sink


def _sdpa_reference(q, k, v, sink, window, scale):
    """softmax attention by torch SDPA (float64) with the sink as an extra key.

    The extra key has K = 0, V = 0 and additive logit ``sink_h``; masked
    positions get -inf; the library applies the GQA head map itself.
    """
    B, n, hq, d = q.shape
    hkv = k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)           # [B, hq, n, d]
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)           # [B, hkv, n, d]
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    kz = torch.zeros(B, hkv, 1, d, dtype=torch.float64)
    vz = torch.zeros(B, hkv, 1, v.shape[-1], dtype=torch.float64)
    kt = torch.cat([kt, kz], dim=2)
    vt = torch.cat([vt, vz], dim=2)
    i = torch.arange(n)[:, None]
    j = torch.arange(n)[None, :]
    keep = j <= i
    if 0 < window < n:
        keep &= j > i - window
    mask = torch.full((hq, n, n + 1), -math.inf, dtype=torch.float64)
    mask[:, :, :n] = torch.where(keep, 0.0, -math.inf).to(torch.float64)
    if sink is None:
        mask[:, :, n] = -math.inf
    else:
        mask[:, :, n] = torch.from_numpy(np.asarray(sink, dtype=np.float64))[:, None]
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask[None], scale=scale,
                                       enable_gqa=(hq != hkv))
    return o.permute(0, 2, 1, 3).numpy()


def _hf_rope(x, positions, theta, rot_dims):
    """Rotate the first rot_dims dims with HF transformers' Llama rotary path."""
    from transformers import LlamaConfig
    from transformers.models.llama import modeling_llama as ml
    cfg = LlamaConfig(hidden_size=rot_dims, num_attention_heads=1, head_dim=rot_dims,
                      rope_theta=theta, max_position_embeddings=4096)
    emb = ml.LlamaRotaryEmbedding(cfg)
    xt = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float32)  # [n, H, D]
    pos = torch.as_tensor(positions, dtype=torch.int64)[None, :]
    cos, sin = emb(xt, pos)                                       # [1, n, rot]
    rot = xt[..., :rot_dims].unsqueeze(0)                          # [1, n, H, rot]
    r, _ = ml.apply_rotary_pos_emb(rot, rot, cos, sin, unsqueeze_dim=2)
    out = xt.clone()
    out[..., :rot_dims] = r[0]
    return out.to(torch.float64).numpy()


# ---------------------------------------------------------------------------
# rslog.cc §4.2-§4.4: the sink softmax
# ---------------------------------------------------------------------------

def check_sink_mass_closed_form(ref):
    """With V = 1 the output is the total weight sum_j s_ij = S/(e^sink + S)
    (§4.2), and lse = ln(e^sink + S), so o_i = 1 - exp(sink - lse_i).
    With Q = 0 every a_ij = 0 and o_i = |J_i| / (e^sink + |J_i|) where
    |J_i| = min(i + 1, W) (§2.1: W tokens including i)."""
    q, k, v, sink = _rand_prefill(11, n=37, hq=4, hkv=2)
    ones = np.ones_like(v)
    for window in (5, 0):
        o, lse = ref.prefill(q, k, ones, sink, window, 1e4, 8)
        for h in range(4):
            want = 1.0 - np.exp(sink[h] - lse[0, h])
            np.testing.assert_allclose(o[0, :, h, 0], want, rtol=0, atol=1e-12)
    qz = np.zeros_like(q)
    for window, n in ((5, 37), (0, 37), (64, 37)):
        o, _ = ref.prefill(qz, k, ones, sink, window, 1e4, 8)
        sizes = np.array([min(i + 1, window) if 0 < window < n else i + 1 for i in range(n)],
                         dtype=np.float64)
        for h in range(4):
            want = sizes / (math.exp(sink[h]) + sizes)
            np.testing.assert_allclose(o[0, :, h, 0], want, rtol=0, atol=1e-12)


def check_sink_limits(ref):
    """§4.3: sink -> -inf recovers the standard softmax (weights sum to 1);
    a very large sink absorbs almost all mass (output -> 0)."""
    q, k, v, _ = _rand_prefill(12, n=20, hq=2, hkv=1)
    ones = np.ones_like(v)
    o, _ = ref.prefill(q, k, ones, None, 6, 1e4, 8)
    np.testing.assert_allclose(o, 1.0, atol=1e-12)
    o2, _ = ref.prefill(q, k, ones, np.array([-800.0, -800.0]), 6, 1e4, 8)
    np.testing.assert_allclose(o2, 1.0, atol=1e-12)
    o3, _ = ref.prefill(q, k, ones, np.array([60.0, 60.0]), 6, 1e4, 8)
    assert np.all(o3 < 1e-20)
    # §4.4: the max includes the sink so exp never overflows; with a sink far
    # above every score, lse = sink + ln(1 + S e^-sink) = sink to double precision
    o4, lse4 = ref.prefill(q, k, ones, np.array([800.0, 800.0]), 6, 1e4, 8)
    assert np.all(np.isfinite(lse4)) and np.all(np.abs(lse4 - 800.0) < 1e-9)
    assert np.all(o4 == 0.0)


def check_against_sdpa(ref):
    """Whole layer (no RoPE) against torch SDPA with the sink as a zero-valued
    extra key: SWA windows, GA causal, GQA head sharing, with and without sink."""
    q, k, v, sink = _rand_prefill(13, B=2, n=33, hq=4, hkv=2, d=16, dv=8)
    scale = 1.0 / math.sqrt(16)
    for window in (1, 3, 8, 32, 33, 0):
        for s in (sink, None):
            o, _ = ref.prefill(q, k, v, s, window, 1e4, 0)
            want = _sdpa_reference(q, k, v, s, window, scale)
            np.testing.assert_allclose(o, want, rtol=1e-11, atol=1e-12)


def check_rows_match_full(ref):
    """Row-sampled prefill gives exactly the full-layer result at those rows."""
    q, k, v, sink = _rand_prefill(21, B=2, n=30, hq=4, hkv=2)
    for window in (7, 0):
        o, lse = ref.prefill(q, k, v, sink, window, 1e7, 8)
        rows = [(1, 3, 29), (0, 0, 0), (0, 2, 17), (1, 1, 6)]
        o2, l2 = ref.prefill(q, k, v, sink, window, 1e7, 8, rows=rows)
        for r, (b, h, i) in enumerate(rows):
            np.testing.assert_array_equal(o2[r], o[b, i, h])
            assert l2[r] == lse[b, h, i]


def check_window_ge_n_is_causal(ref):
    """§2: SWA differs from global attention only in the range of j, so a
    window >= n gives full causal attention (torch SDPA is_causal)."""
    q, k, v, _ = _rand_prefill(14, n=25, hq=2, hkv=2, d=8, dv=8)
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    want = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True).permute(0, 2, 1, 3).numpy()
    for window in (25, 26, 1000, 0, -3):
        o, _ = ref.prefill(q, k, v, None, window, 1e4, 0)
        np.testing.assert_allclose(o, want, rtol=1e-11, atol=1e-12)


def _support(ref, n, window, sink=None):
    """Membership matrix via one-hot values: V[j] = e_j, Q = 0, so
    o_i[j] = s_ij > 0 exactly when j is in J_i."""
    q = np.zeros((1, n, 1, 4))
    k = np.zeros((1, n, 1, 4))
    v = np.eye(n)[None, :, None, :]
    o, _ = ref.prefill(q, k, v, sink, window, 1e4, 0)
    return o[0, :, 0, :] > 0


def check_window_membership(ref):
    """§2.1 brute force: W(i) = {j : max(1, i-W+1) <= j <= i} (1-based)."""
    for n in (1, 2, 9, 40):
        for window in (1, 2, 3, 8, 39, 40, 41, 0):
            got = _support(ref, n, window, sink=np.array([0.3]))
            for i1 in range(1, n + 1):
                if 0 < window < n:
                    want = {j1 for j1 in range(1, n + 1) if max(1, i1 - window + 1) <= j1 <= i1}
                else:
                    want = {j1 for j1 in range(1, n + 1) if j1 <= i1}
                have = {j + 1 for j in np.nonzero(got[i1 - 1])[0]}
                assert have == want, (n, window, i1)


def check_receptive_field(ref):
    """§2.6: after L stacked windows, token i reaches [max(1, i-LW+L), i]
    (1-based). Reachability is the boolean L-th power of the one-layer
    membership matrix taken from the oracle's outputs."""
    n = 48
    for window in (2, 3, 5, 8):
        one = _support(ref, n, window).astype(np.int64)
        reach = np.eye(n, dtype=np.int64)
        for L in range(1, 6):
            reach = ((one @ reach) > 0).astype(np.int64)
            for i1 in range(1, n + 1):
                lo1 = max(1, i1 - L * window + L)
                have = {j + 1 for j in np.nonzero(reach[i1 - 1])[0]}
                assert have == set(range(lo1, i1 + 1)), (window, L, i1)
                assert ref.receptive_field(i1 - 1, L, window) == (lo1 - 1, i1 - 1)


def check_rope_against_hf(ref):
    """pwwt.cn §5 partial rotary: the first rot_dims dims rotate with HF's
    rotary embedding (rotate_half pairing, base theta); the rest pass through."""
    r = _rng(15)
    x = r.standard_normal((50, 3, 24))
    pos = np.arange(50) + 7
    for theta, rot in ((1e4, 8), (1e7, 16), (1e4, 24)):
        got = ref.rope(x, pos, theta, rot)
        want = _hf_rope(x, pos, theta, rot)
        np.testing.assert_allclose(got, want, rtol=0, atol=5e-5)
        np.testing.assert_array_equal(got[..., rot:], x[..., rot:])
    np.testing.assert_array_equal(ref.rope(x, pos, 1e4, 0), x)


def check_rope_relative(ref):
    """RoPE makes q.k depend on positions only through their difference, and
    equals multiplication of (x_k + i x_{k+half}) by exp(i * pos * theta^(-2k/r))."""
    r = _rng(16)
    q = r.standard_normal((1, 1, 32))
    k = r.standard_normal((1, 1, 32))
    for theta in (1e4, 1e7):
        d = []
        for shift in (0, 5, 1000, 30000):
            qr = ref.rope(q, np.array([shift + 40.0]), theta, 16)
            kr = ref.rope(k, np.array([shift + 3.0]), theta, 16)
            d.append(float(qr.ravel() @ kr.ravel()))
        assert max(d) - min(d) < 1e-9, d
    x = r.standard_normal((3, 1, 20))
    pos = np.array([0.0, 1.0, 12345.0])
    got = ref.rope(x, pos, 1e4, 12)
    z = x[..., :6] + 1j * x[..., 6:12]
    w = np.exp(1j * pos[:, None, None] * (1e4 ** (-np.arange(6) / 6.0)))[:, :, :]
    zz = z * w
    np.testing.assert_allclose(got[..., :6], zz.real, atol=1e-9)
    np.testing.assert_allclose(got[..., 6:12], zz.imag, atol=1e-9)


def check_split_combine(ref):
    """Splitting the sum over j into chunks and merging (m_c, l_c, o_c) with the
    sink counted once reproduces the one-shot §4.4 result."""
    r = _rng(17)
    K = r.standard_normal((300, 16))
    V = r.standard_normal((300, 8))
    q = r.standard_normal(16) * 2.0
    keys = np.sort(r.choice(300, 211, replace=False))
    for sink in (1.7, -40.0, None):
        o1, l1 = ref.attend_row(q, K, V, keys, sink, 0.25)
        for cuts in ((211,), (1, 210), (64, 64, 64, 19), tuple([7] * 30 + [1])):
            parts, s = [], 0
            for c in cuts:
                parts.append(ref.partial_state(q, K, V, keys[s:s + c], 0.25))
                s += c
            o2, l2 = ref.combine_partials(parts, sink)
            np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
            assert abs(l2 - l1) < 1e-12


def check_decode_matches_prefill(ref):
    """A decode query at position L-1 over a cache holding the rotated K of the
    same sequence gives the last prefill row: ring (slot p mod 128 holds token
    p; W(L-1) is the last 128 tokens) for SWA, linear prefix for GA."""
    n, hq, hkv, d, dv, cap = 150, 4, 2, 16, 8, 128
    q, k, v, sink = _rand_prefill(18, n=n, hq=hq, hkv=hkv, d=d, dv=dv)
    for L in (1, 2, 127, 128, 129, 150):
        pos = np.arange(L, dtype=np.float64)
        kr = ref.rope(k[0, :L], pos, 1e4, 8)
        qr = ref.rope(q[0, L - 1:L], pos[L - 1:], 1e4, 8)[0]
        o_pf, lse_pf = ref.prefill(q[:, :L], k[:, :L], v[:, :L], sink, 128, 1e4, 8)
        ring_k = np.zeros((1, cap, hkv, d))
        ring_v = np.zeros((1, cap, hkv, dv))
        for p in range(L):
            ring_k[0, p % cap] = kr[p]
            ring_v[0, p % cap] = v[0, p]
        o, lse = ref.decode(qr[None], ring_k, ring_v, "ring", [L], sink)
        np.testing.assert_allclose(o[0], o_pf[0, L - 1], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[0], lse_pf[0, :, L - 1], rtol=0, atol=1e-11)
        o_ga, lse_ga = ref.prefill(q[:, :L], k[:, :L], v[:, :L], sink, 0, 1e4, 8)
        o2, lse2 = ref.decode(qr[None], kr[None], v[:, :L], "linear", [L], sink)
        np.testing.assert_allclose(o2[0], o_ga[0, L - 1], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse2[0], lse_ga[0, :, L - 1], rtol=0, atol=1e-11)


def check_multi_decode_matches_prefill(ref):
    """MTP verification (syt-nju "mimo-mtp-swa-not-mla", MTP section): the T newest
    tokens of a sequence, verified together against the cache, give the last T rows of
    a prefill of the same sequence: on a ring of capacity >= W + T - 1 (token p in slot
    p mod capacity, with wrap-around) for SWA, on a linear cache for GA. T = 1 is the
    one-token decode. A ring that has lost part of a draft token's window is refused."""
    n, hq, hkv, d, dv, W = 90, 4, 2, 16, 8, 12
    q, k, v, sink = _rand_prefill(23, n=n, hq=hq, hkv=hkv, d=d, dv=dv)
    for T, cap in ((1, 12), (3, 14), (4, 16), (4, 21)):
        for L in (T, T + 1, W, W + T, 40, 90):
            if L < T or L > n:
                continue
            pos = np.arange(L, dtype=np.float64)
            kr = ref.rope(k[0, :L], pos, 1e4, 8)
            qr = ref.rope(q[0, L - T:L], pos[L - T:], 1e4, 8)
            o_pf, lse_pf = ref.prefill(q[:, :L], k[:, :L], v[:, :L], sink, W, 1e4, 8)
            ring_k = np.zeros((1, cap, hkv, d))
            ring_v = np.zeros((1, cap, hkv, dv))
            for p in range(L):
                ring_k[0, p % cap] = kr[p]
                ring_v[0, p % cap] = v[0, p]
            o, lse = ref.decode_multi(qr[None], ring_k, ring_v, "ring", [L], W, sink)
            np.testing.assert_allclose(o[0], o_pf[0, L - T:L], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(lse[0], lse_pf[0, :, L - T:L].T, rtol=0, atol=1e-11)
            o_ga, lse_ga = ref.prefill(q[:, :L], k[:, :L], v[:, :L], sink, 0, 1e4, 8)
            o2, lse2 = ref.decode_multi(qr[None], kr[None], v[:, :L], "linear", [L], 0, sink)
            np.testing.assert_allclose(o2[0], o_ga[0, L - T:L], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(lse2[0], lse_ga[0, :, L - T:L].T, rtol=0, atol=1e-11)
            if T == 1:
                o1, l1 = ref.decode(qr, ring_k, ring_v, "ring", [L], sink)
                np.testing.assert_allclose(o[0, 0], o1[0], rtol=1e-13, atol=1e-14)
                np.testing.assert_allclose(lse[0, 0], l1[0], rtol=0, atol=1e-13)
    try:
        ring = np.zeros((1, W + 1, hkv, d))
        ref.decode_multi(q[:, :3], ring, ring[..., :dv], "ring", [40], W, sink)
    except ValueError:
        pass
    else:
        raise AssertionError("a ring without room for every draft token's window must be refused")


def check_chunked_prefill_matches_whole(ref):
    """Chunked prefill (youngju.dev "mimo-v25-inference-optimization", serving section):
    cutting a sequence into chunks, each chunk attending the prefix (from a cache holding
    rotated K, or un-rotated) plus itself, reproduces the whole-sequence prefill row for row
    (SWA and GA), and appending each chunk to a ring or linear cache leaves exactly the
    rotated K / V that make a following decode equal the next prefill row."""
    n, hq, hkv, d, dv = 61, 4, 2, 16, 8
    q, k, v, sink = _rand_prefill(31, n=n, hq=hq, hkv=hkv, d=d, dv=dv)
    pos = np.arange(n, dtype=np.float64)
    kr = ref.rope(k[0], pos, 1e4, 8)[None]
    for window in (9, 0):
        o_full, l_full = ref.prefill(q, k, v, sink, window, 1e4, 8)
        for cuts in ((0, 61), (0, 20, 41, 61), (0, 1, 2, 60, 61), (0, 33, 61)):
            for a, b in zip(cuts[:-1], cuts[1:]):
                for rotated in (True, False):
                    kk = k[:, :b].copy()
                    if rotated:
                        kk[:, :a] = kr[:, :a]
                    o, l = ref.prefill_chunk(q[:, a:b], kk, v[:, :b], a, rotated, sink, window, 1e4, 8)
                    np.testing.assert_allclose(o, o_full[:, a:b], rtol=1e-11, atol=1e-12)
                    np.testing.assert_allclose(l, l_full[:, :, a:b], rtol=0, atol=1e-11)
                    # the row-sampled form gives exactly the full form's rows
                    rows = [(0, h, i) for i in sorted({0, (b - a) // 2, b - a - 1}) for h in (0, 3)]
                    o_r, l_r = ref.prefill_chunk(q[:, a:b], kk, v[:, :b], a, rotated, sink, window,
                                                 1e4, 8, rows=rows)
                    for r, (_, h, i) in enumerate(rows):
                        np.testing.assert_array_equal(o_r[r], o[0, i, h])
                        assert l_r[r] == l[0, h, i]
    # cache write-back: chunks appended to a ring of 12 slots and to a linear cache
    for kind, cap in (("ring", 12), ("linear", 64)):
        kc = np.zeros((1, cap, hkv, d))
        vc = np.zeros((1, cap, hkv, dv))
        for a, b in ((0, 20), (20, 41), (41, 50)):
            kc, vc = ref.cache_append(k[:, a:b], v[:, a:b], a, 1e4, 8, kind, kc, vc)
        L = 50
        for p in range(max(0, L - cap), L):
            slot = p % cap if kind == "ring" else p
            np.testing.assert_allclose(kc[0, slot], kr[0, p], rtol=0, atol=1e-15)
            np.testing.assert_array_equal(vc[0, slot], v[0, p])
        qr = ref.rope(q[0, L - 1:L], pos[L - 1:L], 1e4, 8)
        W = cap if kind == "ring" else 0
        o_pf, l_pf = ref.prefill(q[:, :L], k[:, :L], v[:, :L], sink, W, 1e4, 8)
        o, l = ref.decode(qr, kc, vc, kind, [L], sink)
        np.testing.assert_allclose(o[0], o_pf[0, L - 1], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(l[0], l_pf[0, :, L - 1], rtol=0, atol=1e-11)


def check_select_tokens(ref):
    """Token selection (aideepthink.cn §四.3 key set; scoring rule taken as the largest
    group logit): against a direct per-token scan, the kept set is exactly the n_sel best
    (every kept score >= every dropped one), ties go to the lower index, the order is
    increasing, heads of a group commute, positive scalings of q do not change the choice,
    and with n_sel = all candidates the sparse decode over the chosen set equals decode over
    the whole cache."""
    r = _rng(37)
    B, Hq, Hkv, D, cap = 2, 8, 2, 16, 60
    q = r.integers(-2, 3, size=(B, Hq, D)).astype(np.float64)
    k = r.integers(-2, 3, size=(B, cap, Hkv, D)).astype(np.float64)
    lengths, recent, n_sel = [60, 45], 8, 10
    sel = ref.select_tokens(q, k, lengths, recent, n_sel)
    group = Hq // Hkv
    for b in range(B):
        hi = lengths[b] - recent
        for g in range(Hkv):
            s = sel[b, g]
            assert len(s) == n_sel and np.all(np.diff(s) > 0) and s[0] >= 0 and s[-1] < hi
            score = np.array([max(float(q[b, h] @ k[b, t, g]) for h in range(g * group, (g + 1) * group))
                              for t in range(hi)])
            kept = set(s.tolist())
            dropped = [t for t in range(hi) if t not in kept]
            assert min(score[list(kept)]) >= max(score[dropped])
            thr = min(score[list(kept)])
            # ties at the threshold: the kept ones are the lowest indices among them
            tied = [t for t in range(hi) if score[t] == thr]
            n_tied_kept = sum(1 for t in tied if t in kept)
            assert [t for t in tied if t in kept] == tied[:n_tied_kept]
    # a constructed tie: equal scores everywhere -> the first n_sel candidates
    qz = np.zeros((1, 4, D))
    kz = r.standard_normal((1, 30, 1, D))
    assert np.array_equal(ref.select_tokens(qz, kz, [30], 5, 7)[0, 0], np.arange(7))
    # heads of a group commute; positive scaling of q keeps the choice
    perm = np.arange(Hq).reshape(Hkv, group)[:, ::-1].ravel()
    assert np.array_equal(ref.select_tokens(q[:, perm], k, lengths, recent, n_sel), sel)
    assert np.array_equal(ref.select_tokens(q * 3.5, k, lengths, recent, n_sel), sel)
    # n_sel = every candidate: sparse decode over it is decode over the whole cache
    v = r.standard_normal((B, cap, Hkv, 8))
    sink = r.standard_normal(Hq)
    L = [60, 60]
    full_sel = ref.select_tokens(q, k, L, recent, 60 - recent)
    o1, l1 = ref.sparse_decode(q, k, v, L, recent, full_sel, sink)
    o2, l2 = ref.decode(q, k, v, "linear", L, sink)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)
    # real-valued scores (distinct almost surely): the kept set is a library top-k of the
    # group-max logits, computed here with numpy's argpartition on an explicit product
    qr = r.standard_normal((1, 8, 24))
    kr = r.standard_normal((1, 300, 2, 24))
    got = ref.select_tokens(qr, kr, [300], 20, 37)
    for g in range(2):
        logits = np.einsum("td,hd->th", kr[0, :280, g], qr[0, 4 * g:4 * g + 4])
        best = np.argpartition(-logits.max(axis=1), 37)[:37]
        assert np.array_equal(got[0, g], np.sort(best))


def check_empty_key_set(ref):
    """A decode query over a cache that holds no token yet (L = 0) has an empty key set.
    rslog.cc §4.4 with an empty sum leaves only the sink term, so the weights are empty,
    o = 0 and lse = sink; this equals torch SDPA over the sink alone (one zero-valued
    extra key, §4.2) and torch.logsumexp of the sink, and the V = 1 closed form
    o = 1 - exp(sink - lse) gives 0. Without a sink lse = -inf. The other sequences of
    the batch are unaffected, in ring, linear and sparse decode."""
    r = _rng(41)
    B, hq, hkv, d, dv, cap = 3, 4, 2, 16, 8, 24
    q = r.standard_normal((B, hq, d))
    kc = r.standard_normal((B, cap, hkv, d))
    vc = r.standard_normal((B, cap, hkv, dv))
    sink = r.standard_normal(hq)
    lengths = [0, 7, 24]
    # the sink alone through SDPA: one key with K = 0, V = 0 and additive logit sink_h
    qt = torch.zeros(1, hq, 1, d, dtype=torch.float64)
    kz = torch.zeros(1, hq, 1, d, dtype=torch.float64)
    vz = torch.zeros(1, hq, 1, dv, dtype=torch.float64)
    mask = torch.from_numpy(sink).reshape(1, hq, 1, 1)
    o_sdpa = F.scaled_dot_product_attention(qt, kz, vz, attn_mask=mask)[0, :, 0].numpy()
    lse_sdpa = torch.logsumexp(torch.from_numpy(sink)[:, None], dim=1).numpy()
    for kind in ("ring", "linear"):
        o, lse = ref.decode(q, kc, vc, kind, lengths, sink)
        np.testing.assert_array_equal(o[0], o_sdpa)
        np.testing.assert_array_equal(lse[0], lse_sdpa)
        o1, l1 = ref.decode(q, kc, np.ones_like(vc), kind, lengths, sink)
        np.testing.assert_allclose(o1[0, :, 0], 1.0 - np.exp(sink - l1[0]), atol=1e-15)
        o2, l2 = ref.decode(q[1:], kc[1:], vc[1:], kind, lengths[1:], sink)
        np.testing.assert_array_equal(o[1:], o2)
        np.testing.assert_array_equal(lse[1:], l2)
        o3, l3 = ref.decode(q, kc, vc, kind, lengths, None)
        assert np.all(o3[0] == 0.0) and np.all(np.isneginf(l3[0]))
        assert np.all(np.isfinite(l3[1:]))
    sel = np.full((B, hkv, 3), -1)
    sel[2] = [[0, 5, 9], [1, 2, 3]]
    o, lse = ref.sparse_decode(q, kc, vc, [0, 7, 24], 8, sel, sink)
    np.testing.assert_array_equal(o[0], o_sdpa)
    np.testing.assert_array_equal(lse[0], lse_sdpa)


def check_select_short_rows(ref):
    """aideepthink.cn §四.3 selects n_sel tokens outside the recent window; a sequence
    with fewer candidates than that keeps every candidate (brute force: the row is
    0, 1, ..., hi-1), and the rest of its row is -1, which names no token. So selecting
    and then running the sparse decode over such a sequence attends the whole cache: it
    equals the dense decode over the linear cache (also for L <= recent, where nothing is
    selected and the window alone covers the sequence)."""
    r = _rng(43)
    B, Hq, Hkv, D, cap, recent, n_sel = 4, 8, 2, 16, 70, 10, 12
    q = r.standard_normal((B, Hq, D))
    k = r.standard_normal((B, cap, Hkv, D))
    v = r.standard_normal((B, cap, Hkv, 8))
    sink = r.standard_normal(Hq)
    lengths = [70, 15, 10, 4]           # 60, 5, 0 and 0 candidates
    sel = ref.select_tokens(q, k, lengths, recent, n_sel)
    assert sel.shape == (B, Hkv, n_sel)
    for b, L in enumerate(lengths):
        hi = max(0, L - recent)
        for g in range(Hkv):
            if hi < n_sel:
                assert list(sel[b, g, :hi]) == list(range(hi))
                assert np.all(sel[b, g, hi:] == -1)
            else:
                assert np.all(sel[b, g] >= 0) and np.all(np.diff(sel[b, g]) > 0)
    full = ref.select_tokens(q[:1], k[:1], lengths[:1], recent, n_sel)
    np.testing.assert_array_equal(sel[:1], full)
    o1, l1 = ref.sparse_decode(q[1:], k[1:], v[1:], lengths[1:], recent, sel[1:], sink)
    o2, l2 = ref.decode(q[1:], k[1:], v[1:], "linear", lengths[1:], sink)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def check_e4m3_decoding(ref):
    """OCP FP8 E4M3: every one of the 256 byte patterns decodes as torch.float8_e4m3fn
    does, and the landmarks of the format hold (1.0, the largest 448, the smallest
    normal 2^-6 and subnormal 2^-9, signed zero, the two NaNs)."""
    import torch
    bits = np.arange(256)
    got = ref.e4m3_to_float(bits)
    want = torch.from_numpy(bits.astype(np.uint8)).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.array_equal(got[~np.isnan(got)], want[~np.isnan(want)])
    assert got[0x38] == 1.0 and got[0x7E] == 448.0 and got[0xFE] == -448.0
    assert got[0x08] == 2.0 ** -6 and got[0x01] == 2.0 ** -9 and got[0x07] == 7 * 2.0 ** -9
    assert got[0x00] == 0.0 and got[0x80] == 0.0 and np.signbit(got[0x80])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and int(np.isnan(got).sum()) == 2
    assert got[0x40] == 2.0 and got[0x39] == 1.125 and got[0xB8] == -1.0


def check_fp8_decode_reduces_to_bf16(ref):
    """With power-of-two scales, e4m3(b) * s is exact in bf16: FP8 decode and sparse
    decode over the bytes equal decode / sparse_decode over those bf16 values."""
    r = _rng(29)
    B, cap, hq, hkv, d, dv = 2, 40, 4, 2, 16, 8
    kb = r.integers(0, 256, size=(B, cap, hkv, d))
    vb = r.integers(0, 256, size=(B, cap, hkv, dv))
    kb[(kb & 0x7F) == 0x7F] = 0x3C                     # no NaN patterns in a cache
    vb[(vb & 0x7F) == 0x7F] = 0x3C
    ks = np.exp2(r.integers(-4, 3, size=(B, cap, hkv))).astype(np.float64)
    vs = np.exp2(r.integers(-4, 3, size=(B, cap, hkv))).astype(np.float64)
    kf = ref.e4m3_to_float(kb) * ks[..., None]
    vf = ref.e4m3_to_float(vb) * vs[..., None]
    q = r.standard_normal((B, hq, d))
    sink = r.standard_normal(hq)
    for kind, L in (("ring", [30, 40]), ("linear", [17, 40])):
        o1, l1 = ref.decode_fp8(q, kb, vb, ks, vs, kind, L, sink)
        o2, l2 = ref.decode(q, kf, vf, kind, L, sink)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)
    sel = np.stack([np.stack([np.sort(r.choice(20, 6, replace=False)) for _ in range(hkv)])
                    for _ in range(B)])
    o1, l1 = ref.sparse_decode_fp8(q, kb, vb, ks, vs, [40, 36], 8, sel, sink)
    o2, l2 = ref.sparse_decode(q, kf, vf, [40, 36], 8, sel, sink)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # the scale applies per (token, KV head) row: with all scores equal (K bytes 0), doubling
    # one row's V scale moves exactly the query heads of that KV head in that sequence, by
    # that row's share of the output
    k0 = np.zeros_like(kb)
    vs2 = vs.copy()
    vs2[0, 5, 1] *= 2.0
    o3, _ = ref.decode_fp8(q, k0, vb, ks, vs2, "linear", [40, 40], sink)
    o4, _ = ref.decode_fp8(q, k0, vb, ks, vs, "linear", [40, 40], sink)
    assert np.array_equal(o3[1], o4[1]) and np.array_equal(o3[0, :2], o4[0, :2])
    for h in (2, 3):
        share = 1.0 / (40.0 + np.exp(sink[h]))        # weight of each key, all scores 0
        np.testing.assert_allclose(o3[0, h] - o4[0, h], share * vf[0, 5, 1], rtol=1e-12, atol=1e-14)


def check_sparse_membership(ref):
    """aideepthink.cn §四.3: the key set is the most recent ``recent`` tokens
    plus the selected ones, in one softmax. One-hot values expose membership."""
    L, recent, hkv, hq = 300, 16, 2, 4
    r = _rng(19)
    sel = np.stack([np.sort(r.choice(L - recent, 20, replace=False)) for _ in range(hkv)])[None]
    q = np.zeros((1, hq, 4))
    kc = np.zeros((1, L, hkv, 4))
    vc = np.zeros((1, L, hkv, L))
    for g in range(hkv):
        vc[0, :, g, :] = np.eye(L)
    o, _ = ref.sparse_decode(q, kc, vc, [L], recent, sel, np.zeros(hq))
    for h in range(hq):
        g = h // (hq // hkv)
        have = set(np.nonzero(o[0, h] > 0)[0].tolist())
        want = set(range(L - recent, L)) | set(sel[0, g].tolist())
        assert have == want, h
        assert (L - recent - 1) not in have or (L - recent - 1) in sel[0, g]
    # selecting every token outside the window gives dense causal decode
    q2, k2, v2, sink = _rand_prefill(20, n=L, hq=hq, hkv=hkv, d=16, dv=8)
    allsel = np.broadcast_to(np.arange(L - recent), (1, hkv, L - recent))
    o1, l1 = ref.sparse_decode(q2[:, -1], k2, v2, [L], recent, allsel, sink)
    o2, l2 = ref.decode(q2[:, -1], k2, v2, "linear", [L], sink)
    np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-11)


def check_golden(ref):
    """Hand-derived fixtures under tests/golden/ (each file states its source)."""
    with open(os.path.join(GOLDEN, "sink_two_keys.json")) as f:
        g = json.load(f)
    K = np.array(g["K"], dtype=np.float64)
    V = np.array(g["V"], dtype=np.float64)
    o, lse = ref.attend_row(np.array(g["q"], dtype=np.float64), K, V, np.arange(len(K)),
                            g["sink"], g["scale"])
    np.testing.assert_allclose(o, g["o"], rtol=1e-14)
    assert abs(lse - math.log(g["exp_lse"])) < 1e-14
    s, _ = ref.sink_softmax(np.array(g["a"]), g["sink"])
    np.testing.assert_allclose(s, g["s"], rtol=1e-14)

    with open(os.path.join(GOLDEN, "window_sizes.json")) as f:
        g = json.load(f)
    for i1, size in g["sizes"]:
        assert len(ref.window_keys(i1 - 1, g["W"], g["n"])) == size

    with open(os.path.join(GOLDEN, "receptive_field.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        lo, hi = ref.receptive_field(case["i"] - 1, case["L"], case["W"])
        assert (lo + 1, hi + 1) == tuple(case["range_1based"])

    with open(os.path.join(GOLDEN, "pair_ratio.json")) as f:
        g = json.load(f)
    n, W = g["n"], g["W"]
    swa_pairs = sum(len(ref.window_keys(i, W, n)) for i in range(0, n, 1))
    ratio = n * n / swa_pairs
    assert abs(ratio - g["approx_ratio"]) / g["approx_ratio"] < g["rel_tol"], ratio

    with open(os.path.join(GOLDEN, "rope_hand.json")) as f:
        g = json.load(f)
    x = np.array(g["x"], dtype=np.float64)[None, None, :]
    got = ref.rope(x, np.array([g["pos"]], dtype=np.float64), g["theta"], g["rot_dims"])
    np.testing.assert_allclose(got.ravel(), g["out"], rtol=0, atol=1e-15)


ALL_CHECKS = [
    check_sink_mass_closed_form,
    check_sink_limits,
    check_against_sdpa,
    check_window_ge_n_is_causal,
    check_rows_match_full,
    check_window_membership,
    check_receptive_field,
    check_rope_against_hf,
    check_rope_relative,
    check_split_combine,
    check_decode_matches_prefill,
    check_multi_decode_matches_prefill,
    check_chunked_prefill_matches_whole,
    check_select_tokens,
    check_select_short_rows,
    check_empty_key_set,
    check_sparse_membership,
    check_e4m3_decoding,
    check_fp8_decode_reduces_to_bf16,
    check_golden,
]
