"""Plant plausible mistakes in a copy of the oracle; some pin must catch each.

The mutated copy is executed from source in a fresh module object; the real
oracle module is never modified.
"""

import os
import types

import pytest

import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "ref.py")

MUTANTS = {
    "sink term dropped from denominator": ("den += math.exp(float(sink) - m)", "den += 0.0"),
    "sink exponent sign flipped": ("den += math.exp(float(sink) - m)", "den += math.exp(m - float(sink))"),
    "sink left out of the running max": ("m = max(m, float(sink))", "m = m"),
    "lse without the max": ("return e / den, m + math.log(den)", "return e / den, math.log(den)"),
    "window one too wide": ("lo = max(0, i - window + 1)", "lo = max(0, i - window)"),
    "window one too narrow": ("lo = max(0, i - window + 1)", "lo = max(0, i - window + 2)"),
    "query excluded from its own window": ("return np.arange(lo, i + 1, dtype=np.int64)",
                                           "return np.arange(lo, max(lo + 1, i), dtype=np.int64)"),
    "rope sin sign": ("out[..., :half] = x1 * cos - x2 * sin", "out[..., :half] = x1 * cos + x2 * sin"),
    "rope frequency exponent": ("-2.0 * k / rot_dims", "-1.0 * k / rot_dims"),
    "rope interleaved partner": ("x2 = x[..., half:rot_dims]", "x2 = np.roll(x[..., :rot_dims], -1, axis=-1)[..., :half]"),
    "scale ignored": ("return 1.0 / math.sqrt(d) if not scale else float(scale)", "return 1.0"),
    "gqa map modulo": ("        g = h // group\n        keys = window_keys", "        g = h % Hkv\n        keys = window_keys"),
    "scores on a truncated dot product": ("a = (Kj @ _f64(q_i)) * scale", "a = (Kj[:, :1] @ _f64(q_i)[:1]) * scale"),
    "values gathered from keys": ("o = s @ Vj", "o = s @ Kj[:, :Vj.shape[1]]"),
    "ring slots off by one": ("return np.arange(min(L, capacity), dtype=np.int64)",
                              "return np.arange(min(L, capacity) - 1, dtype=np.int64)"),
    "sparse window misses newest": ("win = np.arange(max(0, L - recent), L, dtype=np.int64)",
                                    "win = np.arange(max(0, L - recent - 1), L - 1, dtype=np.int64)"),
    "combine counts sink per chunk": ("L += math.exp(float(sink) - M)", "L += len(parts) * math.exp(float(sink) - M)"),
    "combine without rescale": ("o = sum(oc * math.exp(m - M) for m, _, oc in parts) / L",
                                "o = sum(oc for m, _, oc in parts) / L"),
    "draft tokens all at the last position": ("    p = L - T + t\n", "    p = L - 1\n"),
    "draft window one too wide": ("lo = max(0, p - window + 1)", "lo = max(0, p - window)"),
    "draft ring slot without modulo": ("return np.arange(lo, p + 1, dtype=np.int64) % capacity",
                                       "return np.arange(lo, p + 1, dtype=np.int64) - max(0, L - capacity)"),
    "draft causal prefix excludes itself": ("        return np.arange(p + 1, dtype=np.int64)\n",
                                            "        return np.arange(p, dtype=np.int64)\n"),
    "chunk queries at chunk-relative positions": ("    qpos = off + np.arange(n, dtype=np.float64)\n",
                                                  "    qpos = np.arange(n, dtype=np.float64)\n"),
    "chunk window measured on the chunk only": ("                keys = window_keys(off + i, window, nk)\n",
                                                "                keys = window_keys(off + i, window, nk)[-(i + 1):]\n"),
    "sampled chunk rows at chunk-relative positions": (
        "            qrow = rope(q[b, i:i + 1, h:h + 1], np.array([off + i], dtype=np.float64),\n",
        "            qrow = rope(q[b, i:i + 1, h:h + 1], np.array([i], dtype=np.float64),\n"),
    "cached prefix rotated twice": ("    if k_prefix_rotated:\n        kr[:, :off] = k[:, :off]\n",
                                    "    if False:\n        kr[:, :off] = k[:, :off]\n"),
    "appended K left un-rotated": ("            kc[b, slot] = kr[i]\n", "            kc[b, slot] = kn[b, i]\n"),
    "ring append without modulo": ("            slot = p % cap if kind == \"ring\" else p\n",
                                   "            slot = min(p, cap - 1)\n"),
    "selection keeps the worst": ("            order = sorted(range(hi), key=lambda t: (-score[t], t))\n",
                                  "            order = sorted(range(hi), key=lambda t: (score[t], t))\n"),
    "selection ties to the higher index": ("            order = sorted(range(hi), key=lambda t: (-score[t], t))\n",
                                           "            order = sorted(range(hi), key=lambda t: (-score[t], -t))\n"),
    "selection by the group's mean logit": ("            score = logits.max(axis=1)\n", "            score = logits.mean(axis=1)\n"),
    "selection reaches into the window": ("        hi = max(0, int(lengths[b]) - recent)\n",
                                          "        hi = max(0, int(lengths[b]) - recent + 1)\n"),
    "selection pads short rows with token 0": ("    out = np.full((B, Hkv, n_sel), -1, dtype=np.int64)\n",
                                               "    out = np.zeros((B, Hkv, n_sel), dtype=np.int64)\n"),
    "selection of a short row drops its last candidate": ("        keep = min(hi, n_sel)\n",
                                                          "        keep = min(hi - 1, n_sel) if hi < n_sel else n_sel\n"),
    "sparse key set keeps the -1 padding": ("    return np.concatenate([win, sel[sel >= 0]])",
                                            "    return np.concatenate([win, sel])"),
    "empty cache attends slot 0": ("    if L < 0:\n        raise ValueError(\"negative cache length\")\n",
                                   "    L = max(L, 1)\n"),
    "empty key set without the sink": ("    m = a.max() if a.size else -math.inf\n",
                                       "    if not a.size:\n        return np.zeros_like(a), -math.inf\n    m = a.max()\n"),
    "e4m3 exponent bias 8": ("np.exp2(e.astype(np.float64) - 7.0)", "np.exp2(e.astype(np.float64) - 8.0)"),
    "e4m3 subnormal scale": ("m / 8.0 * 2.0 ** -6", "m / 8.0 * 2.0 ** -7"),
    "e4m3 without NaN": ("np.where((e == 15) & (m == 7), np.nan, val)", "val"),
    "fp8 scale per token only": ("e4m3_to_float(bits) * _f64(scale)[..., None]",
                                 "e4m3_to_float(bits) * _f64(scale)[..., :1, None]"),
}


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique or missing: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mod = _mutant(*MUTANTS[name])
    failures = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(mod)
        except Exception as e:  # AssertionError or a crash both count
            failures.append(check.__name__)
            break
    assert failures, f"no pin caught mutant: {name}"
