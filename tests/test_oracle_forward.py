"""Pins for the oracle's forward: brute force, associativity, linearity, the
D = I and density-1 special cases, and the worked refit example of the
technical review (section 'Method III', after Eq. (9))."""
import json
import os

import numpy as np
import pytest
import scipy.sparse as sp

import synth
from oracle import forward as F
from oracle.pack import pack_coeff, pack_dictionary


def _tiny_case(M=2, d_in=32, k=16, d_out=24, rho=0.5, seed=0):
    D = synth.gen_dictionary(8, seed, 0, d_in, k)
    C = synth.gen_coeff(8, seed, 0, 0, k, d_out, rho)
    X = synth.gen_activations(8, seed, 0, M, d_in)
    pd = pack_dictionary(D)
    pc = pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    return X, pd, pc


def test_brute_force_agrees():
    X, pd, pc = _tiny_case()
    Dh, Ch = F.decode_dictionary(pd), F.decode_coeff_dense(pc)
    yb = F.forward_brute(X, Dh, Ch)
    assert np.allclose(F.forward_reference(X, pd, pc), yb, rtol=1e-12, atol=1e-12)
    assert np.allclose(F.forward_factored(X, pd, pc), yb, rtol=1e-12, atol=1e-12)


def test_tiny_workload_dense_equals_factored():
    w = synth.tiny()
    for p in w.projections:
        D, C = synth.projection_inputs(p)
        pd = pack_dictionary(D)
        pc = pack_coeff(C.col_ptr, C.atom_idx, C.vals, p.k, p.d_out)
        for M in w.tokens:
            X = synth.gen_activations(0, p.layer, p.site, M, p.d_in)
            y1 = F.forward_reference(X, pd, pc)
            y2 = F.forward_factored(X, pd, pc)
            assert np.allclose(y1, y2, rtol=1e-11, atol=1e-11)
            assert F.within_tolerance(y2, y1)[0]


def test_pre_decoded_forward_is_the_same():
    X, pd, pc = _tiny_case(M=3)
    dec = F.decode_projection(pd, pc)
    assert np.array_equal(F.forward_factored_decoded(X, dec), F.forward_factored(X, pd, pc))


def test_linearity_in_x():
    X, pd, pc = _tiny_case(M=3)
    X2, _, _ = _tiny_case(M=3, seed=5)
    a, b = 0.75, -2.0
    combo = (a * X.astype(np.float64) + b * X2.astype(np.float64))
    # forward_factored accepts any float array for X
    lhs = F.forward_factored(combo, pd, pc)
    rhs = a * F.forward_factored(X, pd, pc) + b * F.forward_factored(X2, pd, pc)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def _identity_dictionary(n):
    """Packed D = I exactly: code 2 (1.0), scale 0x38 (1.0), s_D = 1."""
    codes = np.zeros((n, n), np.uint8)
    np.fill_diagonal(codes, 2)
    flat = codes.reshape(-1)  # atom-major = row j of D^T = column j of I
    packed = (flat[0::2] | (flat[1::2] << 4)).astype(np.uint8)
    return {"d_in": n, "k": n, "codes": packed,
            "scales": np.full(n * n // 16, 0x38, np.uint8), "s": np.float32(1.0)}


def test_identity_dictionary_reduces_to_csc_spmm():
    k, d_out = 64, 40
    C = synth.gen_coeff(8, 1, 0, 0, k, d_out, 0.3)
    pc = pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    pd = _identity_dictionary(k)
    assert np.array_equal(F.decode_dictionary(pd), np.eye(k))
    X = synth.gen_activations(8, 1, 0, 5, k)
    atoms, vals = F.decode_coeff_entries(pc)
    ptr = pc["col_ptr"].astype(np.int64)
    Cs = sp.csc_matrix((vals, atoms, ptr), shape=(k, d_out))
    want = Cs.T.dot(X.astype(np.float64).T).T  # scipy CSC product
    got = F.forward_factored(X, pd, pc)
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


def test_density_one_reduces_to_matmul():
    X, pd, pc = _tiny_case(rho=1.0, k=16)
    Dh, Ch = F.decode_dictionary(pd), F.decode_coeff_dense(pc)
    assert np.count_nonzero(pc["nnz"] == 16) == pc["d_out"]
    want = np.matmul(np.matmul(X.astype(np.float64), Dh), Ch)
    assert np.allclose(F.forward_factored(X, pd, pc), want, rtol=1e-12, atol=1e-12)


def test_refit_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "refit_example.json")))
    W = np.array(g["W"], float)
    Ct = np.array(g["C_tilde"], float)
    Dr = np.array(g["D_refit_columns"], float).T  # columns (2.5,1), (0.5,1)
    prod = F.expand_weight(Dr, Ct)
    assert np.array_equal(prod, np.array(g["D_refit_times_C_tilde"], float))
    assert np.sum((W - prod) ** 2) == g["squared_error_refit"]
    assert np.sum((W - F.expand_weight(np.eye(2), Ct)) ** 2) == g["squared_error_identity"]
    assert np.array_equal(Ct @ Ct.T, np.array(g["coefficient_gram"], float))
    assert np.array_equal(W @ Ct.T, np.array(g["W_Ct"], float))
    # The same product through the oracle's packed sparse path: C~ packed by
    # hand with exact NVFP4 codes (1.0 -> code 2, 2.0 -> code 4, scale 1.0).
    codes = np.array([2] + [0] * 15 + [4] + [0] * 15 + [2] + [0] * 15, np.uint8)
    pc = {"k": 2, "d_out": 3, "nseg": 1,
          "col_ptr": np.array([0, 16, 32, 48], np.uint32), "nnz": np.array([1, 1, 1], np.uint32),
          "codes": (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8),
          "scales": np.full(3, 0x38, np.uint8),
          "idx": np.array([0] + [0] * 15 + [1] + [0] * 15 + [0] + [0] * 15, np.uint8),
          "seg_start": np.zeros(3, np.uint16), "s": np.float32(1.0)}
    assert np.array_equal(F.decode_coeff_dense(pc), Ct)
    # rows of Z = I @ D_refit give D_refit C~ through the sparse columns product
    assert np.array_equal(F.sparse_columns_product(Dr, pc), prod)


def test_sampled_outputs_match_full():
    X, pd, pc = _tiny_case(M=3, d_in=48, k=32, d_out=20, rho=0.3)
    y = F.forward_reference(X, pd, pc)
    rows = [0, 1, 2, 2, 0]
    cols = [0, 5, 19, 7, 13]
    got = F.sampled_outputs(X, pd, pc, rows, cols)
    assert np.allclose(got, y[rows, cols], rtol=1e-12, atol=1e-12)


def test_sampled_outputs_by_rows_match_dense_product():
    # pinned to the dense X (D C) product, a different association of Eq. (1),
    # with repeated rows, an out-of-order row list and more than one segment
    X, pd, pc = _tiny_case(M=5, d_in=64, k=288, d_out=24, rho=0.4)
    y = F.forward_reference(X, pd, pc)
    rows = [4, 0, 1, 4, 2, 3, 0, 4]
    cols = [23, 0, 5, 7, 19, 11, 13, 0]
    got = F.sampled_outputs_rows(X, pd, pc, rows, cols)
    assert np.allclose(got, y[rows, cols], rtol=1e-12, atol=1e-12)


def test_tolerance_helper_flags_errors():
    y = np.linspace(-3, 3, 100)
    assert F.within_tolerance(y * (1 + 1e-4), y)[0]
    assert not F.within_tolerance(y * 1.02, y)[0]
    bad = y.copy()
    bad[10] += 0.5
    assert not F.within_tolerance(bad, y)[0]
    assert not F.within_tolerance(np.full_like(y, np.nan), y)[0]


def test_planted_mistakes_are_caught():
    """A wrong sign, a transposed factor or a dropped scale in the oracle would
    fail the brute-force comparison above; check that the comparison is sharp."""
    X, pd, pc = _tiny_case()
    Dh, Ch = F.decode_dictionary(pd), F.decode_coeff_dense(pc)
    ref = F.forward_brute(X, Dh, Ch)
    wrong_scale = dict(pd, s=np.float32(float(pd["s"]) * 1.01))
    assert not np.allclose(F.forward_factored(X, wrong_scale, pc), ref, rtol=1e-6)
    flipped = dict(pc, codes=(pc["codes"] ^ 0x88).astype(np.uint8))
    assert not np.allclose(F.forward_factored(X, pd, flipped), ref, rtol=1e-6)
    shifted = dict(pc, idx=((pc["idx"].astype(np.int64) + 1) % pc["k"]).astype(np.uint8))
    assert not np.allclose(F.forward_factored(X, pd, shifted), ref, rtol=1e-6)


# ------------------------------------------------------------------ exactly representable factors
from exact_factors import exact_case  # noqa: E402


def test_exactly_representable_factors_give_the_exact_product():
    from oracle.pack import pack_coeff_bitmap
    X, D, col_ptr, atoms, vals, k, d_out, exact = exact_case()
    pd = pack_dictionary(D)
    assert pd["s"] == 1.0 and np.all(pd["scales"] == 0x7E)
    assert np.array_equal(F.decode_dictionary(pd), D.astype(np.float64))
    pc = pack_coeff(col_ptr, atoms, vals, k, d_out)
    assert pc["s"] == 1.0 and pc["nseg"] == 2
    assert np.array_equal(F.forward_factored(X, pd, pc), exact.astype(np.float64))
    assert np.array_equal(F.forward_reference(X, pd, pc), exact.astype(np.float64))
    pb = pack_coeff_bitmap(col_ptr, atoms, vals, k, d_out)
    assert np.array_equal(F.forward_factored_bitmap(X, pd, pb), exact.astype(np.float64))


def test_exactly_representable_block_supports_give_the_exact_product():
    from oracle.pack import pack_coeff_blocks
    X, D, col_ptr, atoms, vals, k, d_out, exact = exact_case(seed=1, blocks=True)
    pd = pack_dictionary(D)
    pk = pack_coeff_blocks(col_ptr, atoms, vals, k, d_out)
    assert np.array_equal(F.forward_factored_blocks(X, pd, pk), exact.astype(np.float64))
