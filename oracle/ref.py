"""Float64 CPU oracle for attention-sink softmax attention in a hybrid SWA/GA decoder.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The CUDA library never calls it, and this module imports nothing from the
CUDA package: the two share no code.

Every function is the plain definition written out in float64 NumPy, with no
tiling, fusion or reordering beyond what the definition states. Inputs are the
exact values of the bf16 tensors the GPU receives, upcast to float64.

Sources (page title and section):

* "MiMo-V2-Flash: Hybrid Sliding Window Attention Architecture" (rslog.cc):
  §1.2 scores a_ij = q_i.k_j / sqrt(d); §2.1 causal window
  W(i) = {j : max(1, i-W+1) <= j <= i}; §2.6 multi-layer receptive field
  [max(1, i-LW+L), i]; §4.2 sink softmax; §4.4 the stable form with
  m_i = max(max_j a_ij, sink); §5 steps 2-5 of the single-layer forward.
* "39层滑窗+9层全局注意力：一文看懂MiMo-V2.6-Flash-MOPD混合SWA设计原理" (pwwt.cn):
  §3-§4 head layout (SWA 64 Q / 8 KV, GA 64 Q / 4 KV, head_dim 192 / v 128);
  §5 two RoPE bases (1e4 SWA, 1e7 GA) and partial_rotary_factor 0.334.
* "小米MiMo-V3的核心架构HySparse2" (aideepthink.cn): §二.2 / §四.3 token-level
  selection, most recent 128 tokens plus 1,024 selected tokens in one merged
  sparse attention over one shared KV cache.
* syt-nju.github.io visual reading "mimo-mtp-swa-not-mla", MTP section: three draft
  tokens verified in one forward pass of the main model (speculative decoding).
* youngju.dev "mimo-v25-inference-optimization", KV-cache section: a dual pool, the
  SWA pool holding O(W) slots per sequence.

Readings where the pages are silent (each also listed in the design notes):

* Positions are 0-based: W(i) = [max(0, i-W+1), i].
* GA scope is the causal prefix [0, i] (a decoder); window <= 0 or >= n means GA.
* The sink is in the scaled logit space of a_ij and is taken on every layer
  type when given; ``sink=None`` (exp(sink) = 0) is the GA form of §5.
* lse = ln(exp(sink) + sum_j exp(a_ij)), the log of the full denominator.
* RoPE rotates the first ``rot_dims`` dims with the rotate-half pairing
  (d, d + rot_dims/2) and inverse frequency theta**(-2k/rot_dims).
* GQA: query head h reads KV head h // (Hq // Hkv).
* Ring cache: token p of a sequence lives in slot p mod capacity.
* Multi-query decode: the T newest tokens of a sequence (positions L-T .. L-1, all
  already written to the cache) are verified together; each has its own window
  (SWA) or causal prefix (GA), exactly as the same rows of a prefill would.
* Chunked prefill (youngju.dev "mimo-v25-inference-optimization", serving section: long
  prompts are prefilled in chunks): a chunk of n tokens at positions off .. off+n-1 attends
  the keys 0 .. off+n-1 exactly as those rows of a whole-sequence prefill would; the prefix
  keys may come from a KV cache (already rotated) or un-rotated; the chunk's own keys are
  un-rotated. Appending a chunk to a cache stores its rotated K and its V at slot
  p mod capacity (ring) or p (linear) for each of its positions p.
* Token selection (aideepthink.cn §二.2 / §四.3: token-level, reused from the preceding
  full-attention layer, no separately trained retrieval module; the scoring rule itself
  is not given): for a sequence and KV head, every token outside the recent window is
  scored by its largest attention logit over the group's query heads; the n_sel best
  are kept (equal scores: lower index first) and returned in increasing order. With
  fewer candidates than n_sel all of them are kept and the row is padded with -1; a
  negative index in a sparse key list names no token.
* Empty key set (a decode query over a cache that holds nothing yet): the §4.4 formula
  with an empty sum, o = 0 and lse = sink (lse = -inf without a sink).
* FP8 KV cache (the pages size their KV caches in FP8 but give no scaling scheme):
  K and V bytes are OCP FP8 E4M3 (bias 7, no infinities, S.1111.111 is NaN), each
  (token, KV head) row carries one fp32 scale per tensor, and the cached value is
  e4m3(byte) * scale. Attention then runs on those values exactly as on bf16 ones.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "window_keys",
    "receptive_field",
    "rope",
    "sink_softmax",
    "attend_row",
    "prefill",
    "prefill_rows",
    "decode",
    "decode_multi",
    "sparse_decode",
    "sparse_key_set",
    "prefill_chunk",
    "cache_append",
    "select_tokens",
    "e4m3_to_float",
    "dequant_fp8",
    "decode_fp8",
    "sparse_decode_fp8",
    "partial_state",
    "combine_partials",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Scopes (rslog.cc §2.1, §2.6, §5 step 2)
# --------------------------------------------------------------------------

def window_keys(i: int, window: int, n: int) -> np.ndarray:
    """Key positions J_i of query i (0-based).

    SWA (§2.1): W(i) = {j : max(0, i - W + 1) <= j <= i}, i.e. W tokens
    including i itself once i >= W - 1. GA (§5 step 2, causal reading):
    [0, i]. ``window <= 0`` or ``window >= n`` selects GA.
    """
    if i < 0 or i >= n:
        raise ValueError("query position out of range")
    if window <= 0 or window >= n:
        lo = 0
    else:
        lo = max(0, i - window + 1)
    return np.arange(lo, i + 1, dtype=np.int64)


def receptive_field(i: int, layers: int, window: int) -> tuple[int, int]:
    """Theoretical receptive field after ``layers`` stacked SWA layers (§2.6).

    The page gives [max(1, i - L*W + L), i] for 1-based i; in 0-based
    positions this is [max(0, i - L*(W - 1)), i].
    """
    return max(0, i - layers * (window - 1)), i


# --------------------------------------------------------------------------
# Partial RoPE (pwwt.cn §5)
# --------------------------------------------------------------------------

def rope(x, positions, theta: float, rot_dims: int) -> np.ndarray:
    """Rotate the first ``rot_dims`` dims of ``x`` by position (rotate-half pairing).

    x: [..., n, H, D] float64, positions: [n]. For k in [0, rot_dims/2):
    angle = pos * theta**(-2k/rot_dims);
    out[k]        = x[k] cos - x[k + half] sin
    out[k + half] = x[k + half] cos + x[k] sin.
    Dims >= rot_dims pass through unchanged. All arithmetic in float64.
    """
    x = _f64(x)
    if rot_dims == 0:
        return x.copy()
    if rot_dims % 2 or rot_dims > x.shape[-1]:
        raise ValueError("rot_dims must be even and <= head dim")
    half = rot_dims // 2
    k = np.arange(half, dtype=np.float64)
    inv_freq = np.power(float(theta), -2.0 * k / rot_dims)
    ang = _f64(positions)[:, None] * inv_freq[None, :]          # [n, half]
    cos = np.cos(ang)[:, None, :]                                # [n, 1, half]
    sin = np.sin(ang)[:, None, :]
    out = x.copy()
    x1 = x[..., :half]
    x2 = x[..., half:rot_dims]
    out[..., :half] = x1 * cos - x2 * sin
    out[..., half:rot_dims] = x2 * cos + x1 * sin
    return out


# --------------------------------------------------------------------------
# Sink softmax (rslog.cc §4.2, §4.4) and one attention row (§5 steps 3-5)
# --------------------------------------------------------------------------

def sink_softmax(a, sink: float | None):
    """Stable sink softmax of one row of scores (§4.4).

    m = max(max_j a_j, sink); den = exp(sink - m) + sum_j exp(a_j - m);
    s_j = exp(a_j - m) / den. Returns (s, lse) with lse = m + ln(den).
    ``sink=None`` drops the sink term (exp(sink) = 0). An empty row is the
    formula with an empty sum: den = exp(sink - m) with m = sink, so lse = sink
    and there are no weights; with no sink either, lse = -inf.
    """
    a = _f64(a)
    m = a.max() if a.size else -math.inf
    if sink is not None:
        m = max(m, float(sink))
    if m == -math.inf:
        # no key and no sink: the denominator is an empty sum (reading of an empty key set)
        return np.zeros_like(a), -math.inf
    e = np.exp(a - m)
    den = e.sum()
    if sink is not None:
        den += math.exp(float(sink) - m)
    return e / den, m + math.log(den)


def attend_row(q_i, K, V, keys, sink, scale):
    """o_i and lse_i for one query over the key set ``keys`` (§5 steps 3-5).

    a_ij = (q_i . k_j) * scale for j in keys; s = sink_softmax(a, sink);
    o_i = sum_j s_ij v_j (the sink carries no value vector, §4.2).
    """
    keys = np.asarray(keys, dtype=np.int64)
    if keys.size and keys[-1] - keys[0] + 1 == keys.size and np.all(np.diff(keys) == 1):
        Kj, Vj = K[keys[0]:keys[-1] + 1], V[keys[0]:keys[-1] + 1]   # contiguous: a view
    else:
        Kj, Vj = K[keys], V[keys]
    a = (Kj @ _f64(q_i)) * scale
    s, lse = sink_softmax(a, sink)
    o = s @ Vj
    return o, lse


def _scale(scale, d):
    return 1.0 / math.sqrt(d) if not scale else float(scale)


# --------------------------------------------------------------------------
# Prefill: SWA or GA layer over a whole sequence
# --------------------------------------------------------------------------

def prefill(q, k, v, sink, window: int, rope_theta: float, rot_dims: int,
            scale: float | None = None, rows=None):
    """Sink attention of one layer over full sequences.

    q: [B, n, Hq, Dqk], k: [B, n, Hkv, Dqk], v: [B, n, Hkv, Dv] (values of the
    bf16 inputs), sink: [Hq] or None. Q and K are rotated with ``rope`` at
    positions 0..n-1 before the scores (pwwt.cn §5). Query head h reads KV head
    h // (Hq // Hkv).

    ``rows=None`` computes every row and returns (o [B, n, Hq, Dv],
    lse [B, Hq, n]). Otherwise ``rows`` is an iterable of (b, h, i) and the
    result is (o [len, Dv], lse [len]) in that order.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, n, Hq, D = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    sc = _scale(scale, D)
    pos = np.arange(n, dtype=np.float64)
    kr = np.stack([rope(k[b], pos, rope_theta, rot_dims) for b in range(B)])
    sinks = None if sink is None else _f64(sink)

    def one(b, h, i, qr_row):
        g = h // group
        keys = window_keys(i, window, n)
        return attend_row(qr_row, kr[b, :, g, :], v[b, :, g, :], keys,
                          None if sinks is None else sinks[h], sc)

    if rows is None:
        qr = np.stack([rope(q[b], pos, rope_theta, rot_dims) for b in range(B)])
        o = np.zeros((B, n, Hq, v.shape[-1]))
        lse = np.zeros((B, Hq, n))
        for b in range(B):
            for h in range(Hq):
                for i in range(n):
                    o[b, i, h], lse[b, h, i] = one(b, h, i, qr[b, i, h])
        return o, lse
    rows = list(rows)
    q_rows = np.stack([q[b, i, h] for (b, h, i) in rows]) if rows else np.zeros((0, D))
    return prefill_rows(q_rows, k, v, sink, window, rope_theta, rot_dims, rows, Hq, scale)


def prefill_rows(q_rows, k, v, sink, window: int, rope_theta: float, rot_dims: int, rows,
                 n_q_heads: int, scale: float | None = None):
    """``prefill`` for selected rows only, without materialising all of Q.

    q_rows[r] is the un-rotated query of rows[r] = (b, h, i); k, v are the full
    [B, n, Hkv, D] tensors; query head h reads KV head h // (n_q_heads // Hkv).
    Returns (o [len(rows), Dv], lse [len(rows)]).
    """
    k, v = _f64(k), _f64(v)
    B, n, Hkv, D = k.shape
    if n_q_heads % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = n_q_heads // Hkv
    sc = _scale(scale, D)
    pos = np.arange(n, dtype=np.float64)
    kr = np.stack([rope(k[b], pos, rope_theta, rot_dims) for b in range(B)])
    sinks = None if sink is None else _f64(sink)
    rows = list(rows)
    o = np.zeros((len(rows), v.shape[-1]))
    lse = np.zeros(len(rows))
    for r, (b, h, i) in enumerate(rows):
        g = h // group
        qrow = rope(_f64(q_rows[r])[None, None, :], pos[i:i + 1], rope_theta, rot_dims)[0, 0]
        keys = window_keys(i, window, n)
        o[r], lse[r] = attend_row(qrow, kr[b, :, g, :], v[b, :, g, :], keys,
                                  None if sinks is None else sinks[h], sc)
    return o, lse


# --------------------------------------------------------------------------
# Decode over a KV cache (one query token per sequence)
# --------------------------------------------------------------------------

def _cache_rows(kind: str, L: int, capacity: int) -> np.ndarray:
    """Cache slots a decode query at position L-1 attends.

    ring (SWA pool of O(W) slots): token p lives in slot p mod capacity, so
    the window W(L-1) occupies slots 0..min(L, capacity)-1; linear (GA pool):
    slots 0..L-1 hold tokens 0..L-1. L = 0 (nothing cached yet) attends no
    slot: the key set is empty, so o = 0 and lse = sink (§4.4 with an empty sum).
    """
    if L < 0:
        raise ValueError("negative cache length")
    if kind == "ring":
        return np.arange(min(L, capacity), dtype=np.int64)
    if kind == "linear":
        if L > capacity:
            raise ValueError("length exceeds linear cache capacity")
        return np.arange(L, dtype=np.int64)
    raise ValueError(kind)


def decode(q, k_cache, v_cache, kind: str, lengths, sink, scale=None):
    """One-token decode. q: [B, Hq, Dqk]; caches: [B, cap, Hkv, D] holding
    already-rotated K. Returns (o [B, Hq, Dv], lse [B, Hq])."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, D = q.shape
    cap, Hkv = kc.shape[1], kc.shape[2]
    group = Hq // Hkv
    sc = _scale(scale, D)
    o = np.zeros((B, Hq, vc.shape[-1]))
    lse = np.zeros((B, Hq))
    for b in range(B):
        slots = _cache_rows(kind, int(lengths[b]), cap)
        for h in range(Hq):
            g = h // group
            o[b, h], lse[b, h] = attend_row(q[b, h], kc[b, :, g, :], vc[b, :, g, :], slots,
                                            None if sink is None else float(sink[h]), sc)
    return o, lse


def _multi_rows(kind: str, L: int, T: int, t: int, capacity: int, window: int) -> np.ndarray:
    """Cache slots draft token t (position p = L - T + t) attends in multi-query decode.

    ring: the tokens of its window [max(0, p-W+1), p], at slots token mod capacity; the
    ring must still hold all of them (capacity >= W + T - 1 covers every t); linear:
    tokens 0..p at slots 0..p.
    """
    if not 1 <= T <= L:
        raise ValueError("multi-query decode needs 1 <= T <= L")
    p = L - T + t
    if kind == "ring":
        lo = max(0, p - window + 1)
        if lo < L - capacity:
            raise ValueError("ring too small: part of the window was overwritten")
        return np.arange(lo, p + 1, dtype=np.int64) % capacity
    if kind == "linear":
        if L > capacity:
            raise ValueError("length exceeds linear cache capacity")
        return np.arange(p + 1, dtype=np.int64)
    raise ValueError(kind)


def decode_multi(q, k_cache, v_cache, kind: str, lengths, window: int, sink, scale=None):
    """Multi-query decode (MTP draft verification). q: [B, T, Hq, Dqk], the already
    rotated queries of the T newest tokens of each sequence; caches as in decode().
    Returns (o [B, T, Hq, Dv], lse [B, T, Hq])."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, T, Hq, D = q.shape
    cap, Hkv = kc.shape[1], kc.shape[2]
    group = Hq // Hkv
    sc = _scale(scale, D)
    o = np.zeros((B, T, Hq, vc.shape[-1]))
    lse = np.zeros((B, T, Hq))
    for b in range(B):
        for t in range(T):
            slots = _multi_rows(kind, int(lengths[b]), T, t, cap, window)
            for h in range(Hq):
                g = h // group
                o[b, t, h], lse[b, t, h] = attend_row(q[b, t, h], kc[b, :, g, :], vc[b, :, g, :],
                                                      slots, None if sink is None else float(sink[h]), sc)
    return o, lse


def sparse_key_set(L: int, recent: int, sel) -> np.ndarray:
    """Merged key set of token-level sparse attention (aideepthink.cn §四.3).

    The most recent ``recent`` tokens {L-recent, ..., L-1} together with the
    selected token indices ``sel`` (drawn from outside the window, so the two
    parts are disjoint), in one set. Negative entries of ``sel`` name no token:
    they are the padding ``select_tokens`` writes when a sequence has fewer
    candidates than n_sel, and they are left out.
    """
    win = np.arange(max(0, L - recent), L, dtype=np.int64)
    sel = np.asarray(sel, dtype=np.int64)
    return np.concatenate([win, sel[sel >= 0]])


def sparse_decode(q, k_cache, v_cache, lengths, recent: int, sel_idx, sink, scale=None):
    """Token-level sparse decode: one merged sink softmax over recent + selected.

    q: [B, Hq, Dqk]; caches: [B, cap, Hkv, D] (linear, rotated K);
    sel_idx: [B, Hkv, n_sel] shared by all query heads of a KV group.
    Returns (o [B, Hq, Dv], lse [B, Hq]).
    """
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    group = Hq // Hkv
    sc = _scale(scale, D)
    sel_idx = np.asarray(sel_idx)
    o = np.zeros((B, Hq, vc.shape[-1]))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            g = h // group
            keys = sparse_key_set(int(lengths[b]), recent, sel_idx[b, g])
            o[b, h], lse[b, h] = attend_row(q[b, h], kc[b, :, g, :], vc[b, :, g, :], keys,
                                            None if sink is None else float(sink[h]), sc)
    return o, lse


# --------------------------------------------------------------------------
# Split-KV algebra (the sum over j of §4.4 broken into chunks)
# --------------------------------------------------------------------------

def partial_state(q_i, K, V, keys, scale):
    """Unnormalised state of one chunk of keys, without the sink:
    m_c = max_j a_j, l_c = sum_j exp(a_j - m_c), o_c = sum_j exp(a_j - m_c) v_j."""
    keys = np.asarray(keys, dtype=np.int64)
    a = (K[keys] @ _f64(q_i)) * scale
    m = a.max()
    e = np.exp(a - m)
    return m, e.sum(), e @ V[keys]


def combine_partials(parts, sink):
    """Merge chunk states into the §4.4 result, counting the sink once.

    M = max(sink, max_c m_c); L = exp(sink - M) + sum_c l_c exp(m_c - M);
    o = sum_c o_c exp(m_c - M) / L; lse = M + ln L.
    """
    M = max(m for m, _, _ in parts)
    if sink is not None:
        M = max(M, float(sink))
    L = sum(l * math.exp(m - M) for m, l, _ in parts)
    if sink is not None:
        L += math.exp(float(sink) - M)
    o = sum(oc * math.exp(m - M) for m, _, oc in parts) / L
    return o, M + math.log(L)


# --------------------------------------------------------------------------
# Token selection for the sparse decode
# --------------------------------------------------------------------------

def select_tokens(q, k_cache, lengths, recent: int, n_sel: int, scale=None) -> np.ndarray:
    """sel [B, Hkv, n_sel] int64: per sequence b and KV head g, the n_sel tokens t in
    [0, L_b - recent) with the largest score max_{h in group g} (q_h . k_t) * scale, equal
    scores taken in increasing t, listed in increasing t. q: [B, Hq, Dqk] (rotated);
    k_cache: [B, cap, Hkv, Dqk] linear (rotated K). A sequence with fewer candidates
    than n_sel keeps all of them (in increasing t) and fills the rest of its row with -1,
    which the sparse key set skips."""
    q, kc = _f64(q), _f64(k_cache)
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    group = Hq // Hkv
    sc = _scale(scale, D)
    out = np.full((B, Hkv, n_sel), -1, dtype=np.int64)
    for b in range(B):
        hi = max(0, int(lengths[b]) - recent)
        keep = min(hi, n_sel)
        for g in range(Hkv):
            logits = (kc[b, :hi, g, :] @ q[b, g * group:(g + 1) * group, :].T) * sc   # [hi, group]
            score = logits.max(axis=1)
            order = sorted(range(hi), key=lambda t: (-score[t], t))
            out[b, g, :keep] = np.sort(np.asarray(order[:keep], dtype=np.int64))
    return out


# --------------------------------------------------------------------------
# Chunked prefill over a KV prefix, and appending a chunk to a cache
# --------------------------------------------------------------------------

def prefill_chunk(q, k, v, pos_offset: int, k_prefix_rotated: bool, sink, window: int,
                  rope_theta: float, rot_dims: int, scale: float | None = None, rows=None):
    """Sink attention of a chunk of n query tokens at positions off .. off+n-1.

    q: [B, n, Hq, Dqk] (un-rotated); k: [B, off+n, Hkv, Dqk], v: [B, off+n, Hkv, Dv] hold
    every key position 0 .. off+n-1. Key rows at positions < off are used as stored when
    ``k_prefix_rotated`` (a cache holds rotated K) and rotated otherwise; the chunk's key
    rows (positions >= off) are rotated. Query i of the chunk is rotated at position
    off + i and attends window_keys(off + i, window, off + n).
    Returns (o [B, n, Hq, Dv], lse [B, Hq, n]); with ``rows``, an iterable of (b, h, i)
    (i counted within the chunk), only those rows: (o [len, Dv], lse [len]) in that order.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, n, Hq, D = q.shape
    nk, Hkv = k.shape[1], k.shape[2]
    off = int(pos_offset)
    if nk != off + n or v.shape[1] != nk:
        raise ValueError("keys must cover positions 0 .. pos_offset + n - 1")
    group = Hq // Hkv
    sc = _scale(scale, D)
    kpos = np.arange(nk, dtype=np.float64)
    kr = np.stack([rope(k[b], kpos, rope_theta, rot_dims) for b in range(B)])
    if k_prefix_rotated:
        kr[:, :off] = k[:, :off]
    if rows is not None:
        rows = list(rows)
        o = np.zeros((len(rows), v.shape[-1]))
        lse = np.zeros(len(rows))
        for r, (b, h, i) in enumerate(rows):
            g = h // group
            qrow = rope(q[b, i:i + 1, h:h + 1], np.array([off + i], dtype=np.float64),
                        rope_theta, rot_dims)[0, 0]
            keys = window_keys(off + i, window, nk)
            o[r], lse[r] = attend_row(qrow, kr[b, :, g, :], v[b, :, g, :], keys,
                                      None if sink is None else float(_f64(sink)[h]), sc)
        return o, lse
    qpos = off + np.arange(n, dtype=np.float64)
    qr = np.stack([rope(q[b], qpos, rope_theta, rot_dims) for b in range(B)])
    o = np.zeros((B, n, Hq, v.shape[-1]))
    lse = np.zeros((B, Hq, n))
    for b in range(B):
        for h in range(Hq):
            g = h // group
            for i in range(n):
                keys = window_keys(off + i, window, nk)
                o[b, i, h], lse[b, h, i] = attend_row(qr[b, i, h], kr[b, :, g, :], v[b, :, g, :],
                                                      keys, None if sink is None else float(_f64(sink)[h]), sc)
    return o, lse


def cache_append(k_chunk, v_chunk, pos_offset: int, rope_theta: float, rot_dims: int, kind: str,
                 k_cache, v_cache):
    """Copies of the caches [B, cap, Hkv, D] after appending a chunk of n tokens at
    positions off .. off+n-1: K rotated at its position, V as is, at slot p mod cap
    (ring) or p (linear; needs off + n <= cap). Returns (k_cache', v_cache')."""
    kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
    kn, vn = _f64(k_chunk), _f64(v_chunk)
    B, n = kn.shape[0], kn.shape[1]
    cap = kc.shape[1]
    off = int(pos_offset)
    if kind == "linear" and off + n > cap:
        raise ValueError("linear cache too small")
    if kind not in ("ring", "linear"):
        raise ValueError(kind)
    pos = off + np.arange(n, dtype=np.float64)
    for b in range(B):
        kr = rope(kn[b], pos, rope_theta, rot_dims)
        for i in range(n):
            p = off + i
            slot = p % cap if kind == "ring" else p
            kc[b, slot] = kr[i]
            vc[b, slot] = vn[b, i]
    return kc, vc


# --------------------------------------------------------------------------
# FP8 (E4M3) KV cache
# --------------------------------------------------------------------------

def e4m3_to_float(bits) -> np.ndarray:
    """Value of each OCP FP8 E4M3 byte: sign bit 7, exponent bits 6-3 (bias 7),
    mantissa bits 2-0; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN;
    there are no infinities (the largest finite magnitude is 448)."""
    b = np.asarray(bits, dtype=np.int64) & 0xFF
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = sign * val
    return np.where((e == 15) & (m == 7), np.nan, val)


def dequant_fp8(bits, scale) -> np.ndarray:
    """Cached values of an FP8 cache: bits [B, S, Hkv, D] uint8, scale [B, S, Hkv] fp32;
    value = e4m3(bits) * scale of its (token, KV head) row."""
    return e4m3_to_float(bits) * _f64(scale)[..., None]


def decode_fp8(q, k_bits, v_bits, k_scale, v_scale, kind: str, lengths, sink, scale=None):
    """One-token decode over an FP8 cache: decode() on the dequantized values."""
    return decode(q, dequant_fp8(k_bits, k_scale), dequant_fp8(v_bits, v_scale), kind, lengths,
                  sink, scale)


def sparse_decode_fp8(q, k_bits, v_bits, k_scale, v_scale, lengths, recent: int, sel_idx, sink,
                      scale=None):
    """Token-level sparse decode over an FP8 cache: sparse_decode() on the dequantized values."""
    return sparse_decode(q, dequant_fp8(k_bits, k_scale), dequant_fp8(v_bits, v_scale), lengths,
                         recent, sel_idx, sink, scale)
