"""The seeded generators: exact per-column counts, determinism, order independence."""
from fractions import Fraction

import numpy as np

import synth


def test_nnz_per_column_matches_floor_rule():
    for k in (128, 2048, 3072, 11008):
        for rho in (0.2, 0.25, 0.3, 0.4, 0.5, 1.0):
            removed = int((1 - Fraction(str(rho))) * k // 1)
            assert synth.nnz_per_column(k, rho) == k - removed


def test_llama_counts():
    assert synth.nnz_per_column(2048, 0.3) == 615
    assert synth.nnz_per_column(3072, 0.25) == 768
    assert synth.nnz_per_column(128, 0.5) == 64


def test_support_uniform_sorted_and_deterministic():
    s1 = synth.gen_support(1, 0, 0, 0, 2048, 64, 615)
    s2 = synth.gen_support(1, 0, 0, 0, 2048, 64, 615)
    assert np.array_equal(s1, s2)
    assert s1.shape == (64, 615)
    assert np.all(np.diff(s1, axis=1) > 0) and s1.min() >= 0 and s1.max() < 2048
    big = synth.gen_support(1, 0, 0, 1, 256, 4000, 64)
    hist = np.bincount(big.reshape(-1), minlength=256) / big.size
    assert np.all(np.abs(hist - 1 / 256) < 0.25 / 256)  # roughly uniform


def test_order_independent_streams():
    a = synth.gen_dictionary(3, 2, 1, 64, 32)
    _ = synth.gen_dictionary(3, 0, 0, 64, 32)
    b = synth.gen_dictionary(3, 2, 1, 64, 32)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, synth.gen_dictionary(3, 2, 2, 64, 32))


def test_outlier_channels():
    x = synth.gen_activations(4, 0, 0, 64, 4096, outlier_frac=0.01)
    base = synth.gen_activations(4, 0, 0, 64, 4096)
    ratio = np.abs(x.astype(np.float32)).mean(0) / np.abs(base.astype(np.float32)).mean(0)
    assert np.count_nonzero(ratio > 10) == round(0.01 * 4096)


def test_workloads_shapes():
    w = synth.full_step()
    assert len(w.projections) == 224
    assert len(w.groups()) == 112
    assert all(0.2 <= p.rho < 0.4 for p in w.projections)
    assert [p.name for p in w.projections[:7]] == list(synth.PROJ_TYPES)
