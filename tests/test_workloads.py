"""Synthetic input recipes: shapes, seeds and structural facts of the pages."""

import torch

from hybrid_sliding_window_sink_b200 import workloads as wl


def test_layer_pattern_39_swa_9_ga():
    """pwwt.cn §2: 48 layers, GA at 0, 6, ..., 42, 47 -> 9 GA + 39 SWA."""
    pat = wl.layer_pattern()
    assert len(pat) == 48 and pat.count(0) == 9 and pat.count(1) == 39
    assert [i for i, x in enumerate(pat) if x == 0] == [0, 6, 12, 18, 24, 30, 36, 42, 47]


def test_inputs_are_seeded_and_shaped():
    a = wl.prefill_inputs(1, 40, 8, 1, seed=5)
    b = wl.prefill_inputs(1, 40, 8, 1, seed=5)
    assert all(torch.equal(a[x], b[x]) for x in ("q", "k", "v", "sink"))
    assert a["q"].shape == (1, 40, 8, 192) and a["v"].shape == (1, 40, 1, 128)
    assert a["q"].dtype == torch.bfloat16 and a["sink"].dtype == torch.float32
    k5 = wl.prefill_inputs(1, 2000, 4, 4, seed=6, k_scale=0.5)["k"].float()
    assert 0.45 < float(k5.std()) < 0.55


def test_sorted_unique_indices():
    idx = wl.sorted_unique_indices(3, 4, 1024, [262144 - 128, 5000, 1100], seed=1)
    for b, hi in enumerate([262144 - 128, 5000, 1100]):
        for g in range(4):
            row = idx[b, g]
            assert bool((row[1:] > row[:-1]).all())
            assert int(row[0]) >= 0 and int(row[-1]) < hi


def test_lengths_uniform_range():
    L = wl.lengths_uniform(64, 4096, 131072, seed=1004)
    assert L.dtype == torch.int32 and int(L.min()) >= 4096 and int(L.max()) <= 131072


def test_integer_qk_is_seeded_and_small_integers():
    q, k = wl.integer_qk(2, 8, 2, 50, seed=3)
    q2, k2 = wl.integer_qk(2, 8, 2, 50, seed=3)
    assert torch.equal(q, q2) and torch.equal(k, k2)
    assert q.shape == (2, 8, 192) and k.shape == (2, 50, 2, 192)
    for t in (q.float(), k.float()):
        assert torch.equal(t, t.round()) and t.min() >= -2 and t.max() <= 2
