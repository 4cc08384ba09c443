"""Pins of the oracle's bitmap-indexed coefficient layout (Eq. (12) of the
technical review, a = 0, h = 1: one bit per logical position)."""
import json
import os

import numpy as np

import synth
from oracle import forward as F
from oracle.accounting import eq12_breakeven
from oracle.pack import bitmap_entry_atoms, coeff_entry_atoms, pack_coeff, pack_coeff_bitmap


def test_hand_derived_example(golden_dir):
    with open(os.path.join(golden_dir, "bitmap_example.json")) as f:
        g = json.load(f)
    cols = [np.array(c, np.int64) for c in g["columns"]]
    ptr = np.zeros(g["d_out"] + 1, np.int64)
    ptr[1:] = np.cumsum([c.size for c in cols])
    atoms = np.concatenate(cols)
    vals = np.linspace(-1, 1, atoms.size).astype(np.float32)
    pb = pack_coeff_bitmap(ptr, atoms, vals, g["k"], g["d_out"])
    assert pb["words"] == 2
    assert pb["bitmap"].reshape(g["d_out"], 2).tolist() == g["bitmap_words"]
    assert np.diff(pb["col_ptr"].astype(np.int64)).tolist() == g["padded_entries"]
    got = bitmap_entry_atoms(pb)
    assert got.tolist() == [0, 5, 31] + [-1] * 13 + [32, 39] + [-1] * 14


def _layer(k, d_out, rho, seed=0):
    C = synth.gen_coeff(50, seed, 0, 0, k, d_out, rho)
    return C, pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out), pack_coeff_bitmap(C.col_ptr, C.atom_idx, C.vals,
                                                                                  k, d_out)


def test_same_values_as_the_u8_layout_and_one_bit_per_retained_atom():
    for k, d_out, rho in [(40, 7, 0.5), (2048, 96, 0.3), (3000, 33, 0.25), (16, 5, 1.0), (300, 12, 0.01)]:
        C, pc, pb = _layer(k, d_out, rho)
        for n in ("col_ptr", "nnz", "codes", "scales"):
            assert np.array_equal(pc[n], pb[n]), n
        assert pc["s"] == pb["s"]
        bm = pb["bitmap"].reshape(d_out, pb["words"])
        pop = np.array([sum(bin(int(w)).count("1") for w in row) for row in bm])
        assert np.array_equal(pop, np.diff(C.col_ptr))
        # no bit at or beyond k
        if k % 32:
            assert np.all(bm[:, -1] >> np.uint32(k % 32) == 0)
        # the stored entries' atoms from the bitmap are the input support, and the u8 index agrees
        a_bm = bitmap_entry_atoms(pb)
        a_u8 = coeff_entry_atoms(pc)
        ptr = pb["col_ptr"].astype(np.int64)
        for o in range(d_out):
            n = int(C.col_ptr[o + 1] - C.col_ptr[o])
            want = C.atom_idx[C.col_ptr[o]:C.col_ptr[o + 1]]
            assert np.array_equal(a_bm[ptr[o]:ptr[o] + n], want)
            assert np.array_equal(a_u8[ptr[o]:ptr[o] + n], want)
            assert np.all(a_bm[ptr[o] + n:ptr[o + 1]] == -1)


def test_bitmap_forward_matches_u8_and_dense_forwards():
    k, d_in, d_out = 288, 64, 40
    D = synth.gen_dictionary(50, 1, 0, d_in, k)
    C = synth.gen_coeff(50, 1, 0, 0, k, d_out, 0.35)
    X = synth.gen_activations(50, 1, 0, 3, d_in)
    from oracle.pack import pack_dictionary
    pd = pack_dictionary(D)
    pc = pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    pb = pack_coeff_bitmap(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    yb = F.forward_factored_bitmap(X, pd, pb)
    assert np.allclose(yb, F.forward_factored(X, pd, pc), rtol=1e-12, atol=1e-12)
    assert np.allclose(yb, F.forward_reference(X, pd, pc), rtol=1e-10, atol=1e-12)
    # a planted mistake (one bit moved) changes the result
    bad = dict(pb, bitmap=pb["bitmap"].copy())
    w = bad["bitmap"]
    j = int(np.flatnonzero(w)[0])
    low = int(w[j]) & -int(w[j])
    w[j] = np.uint32((int(w[j]) ^ low) | (low << 1 if low < (1 << 31) else 1))
    assert not np.allclose(F.forward_factored_bitmap(X, pd, bad), yb, rtol=1e-6)


def test_byte_break_even_against_dense_nvfp4_is_the_printed_22_percent():
    """Eq. (12) with b = 4.5 bits (NVFP4 value plus scale share), a = 0, h = 1: a
    bitmap-indexed array saves bytes over the dense array iff the pruned fraction p
    exceeds 1/4.5 = 22.2%, the figure the review prints. Checked on actual packed
    sizes: values + scales at 4.5 bits per retained value plus one bit per logical
    position, against 4.5 bits per logical position dense."""
    assert abs(eq12_breakeven(0.0, 4.5, 1.0) - 1 / 4.5) < 1e-15
    k, d_out = 4096, 64
    for p, saves in [(0.20, False), (0.25, True)]:
        rho = 1.0 - p
        _, _, pb = _layer(k, d_out, rho, seed=3)
        n = int(np.diff(pb["col_ptr"].astype(np.int64)).max())
        nnz = np.diff(synth.gen_coeff(50, 3, 0, 0, k, d_out, rho).col_ptr)
        bits_sparse = float(np.sum(4.5 * nnz)) + pb["bitmap"].size * 32
        bits_dense = 4.5 * k * d_out
        assert (bits_sparse < bits_dense) == saves, (p, bits_sparse, bits_dense, n)
