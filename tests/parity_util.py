"""Comparison helpers for GPU-vs-oracle parity tests.

Tolerances (floating point): bf16 output max-abs error <= 1e-2 and relative L2
error <= 5e-3 against the float64 oracle; fp32 LSE within 1e-3 absolute.
Index handling (which tokens enter a key set) is compared exactly.
"""

from __future__ import annotations

import numpy as np

OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 5e-3
LSE_ABS = 1e-3


def compare(out_gpu, out_ref, lse_gpu=None, lse_ref=None, what=""):
    """out_gpu / lse_gpu: float64 arrays of the GPU results; *_ref: oracle results."""
    og = np.asarray(out_gpu, dtype=np.float64)
    orf = np.asarray(out_ref, dtype=np.float64)
    assert og.shape == orf.shape, (what, og.shape, orf.shape)
    assert np.all(np.isfinite(og)), f"{what}: non-finite output"
    err = np.abs(og - orf)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(orf))
    rel = float(np.linalg.norm(og - orf) / denom) if denom > 0 else float(np.linalg.norm(og))
    stats = {"max_abs": max_abs, "rel_l2": rel}
    if lse_gpu is not None:
        lg = np.asarray(lse_gpu, dtype=np.float64)
        lr = np.asarray(lse_ref, dtype=np.float64)
        assert lg.shape == lr.shape
        both_inf = np.isneginf(lg) & np.isneginf(lr)
        d = np.where(both_inf, 0.0, np.abs(lg - lr))
        stats["lse_max_abs"] = float(d.max()) if d.size else 0.0
    assert max_abs <= OUT_MAX_ABS, f"{what}: out max-abs {max_abs:.3g} > {OUT_MAX_ABS} ({stats})"
    assert rel <= OUT_REL_L2, f"{what}: out rel-L2 {rel:.3g} > {OUT_REL_L2} ({stats})"
    if lse_gpu is not None:
        assert stats["lse_max_abs"] <= LSE_ABS, f"{what}: lse error {stats['lse_max_abs']:.3g} ({stats})"
    return stats
