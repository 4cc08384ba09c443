"""Pins for the oracle's packed layouts (the bit-exact contract the library must meet)."""
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import nvfp4
from oracle.pack import (PAD, SEG, coeff_entry_atoms, pack_coeff, pack_dictionary,
                         pack_nibbles, unpack_nibbles)


def test_nibble_order_low_first():
    assert pack_nibbles(np.array([1, 2, 15, 0], np.uint8)).tolist() == [0x21, 0x0F]
    assert unpack_nibbles(np.array([0x21, 0x0F], np.uint8)).tolist() == [1, 2, 15, 0]


def test_dictionary_layout_positions():
    # atom j, element i carries the E2M1 value whose code is (i + j) % 8, scaled
    # per block so that every block has the same amax 6 -> scale 448 * s_T = 1... .
    d_in, k = 64, 3
    D = np.zeros((d_in, k), np.float32)
    for j in range(k):
        for i in range(d_in):
            D[i, j] = nvfp4.E2M1_TABLE[(i + j) % 8]
    for j in range(k):  # make each block's amax exactly 6 so codes are exact
        for b in range(d_in // 16):
            D[16 * b, j] = 6.0
    pd = pack_dictionary(D)
    codes = unpack_nibbles(pd["codes"])
    assert codes.size == k * d_in
    for j in range(k):
        for i in range(d_in):
            c = codes[j * d_in + i]
            assert nvfp4.E2M1_TABLE[c] * nvfp4.E4M3_TABLE[pd["scales"][j * (d_in // 16) + i // 16]] \
                * float(pd["s"]) == pytest.approx(float(D[i, j]), rel=1e-6, abs=1e-12)
    # byte j*d_in/2 + i/2 holds element i of atom j, even i in the low nibble
    raw = pd["codes"]
    assert raw[0] & 0xF == codes[0] and raw[0] >> 4 == codes[1]
    assert raw[d_in // 2] & 0xF == codes[d_in]


def _small_coeff(k, d_out, rho, seed=0):
    C = synth.gen_coeff(9, seed, 0, 0, k, d_out, rho)
    return C, pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out)


@pytest.mark.parametrize("k,rho", [(128, 0.5), (600, 0.3), (700, 0.05), (512, 1.0), (300, 0.0)])
def test_coeff_layout_invariants(k, rho):
    d_out = 37
    C, pc = _small_coeff(k, d_out, rho)
    nnz_expected = k - int(Fraction(1) * ((1 - Fraction(str(rho))) * k).__floor__())
    assert np.all(pc["nnz"] == nnz_expected)
    ptr = pc["col_ptr"].astype(np.int64)
    assert ptr[0] == 0 and np.all(np.diff(ptr) % PAD == 0)
    assert np.all(np.diff(ptr) == -(-pc["nnz"].astype(np.int64) // PAD) * PAD)
    total = int(ptr[-1])
    assert pc["idx"].size == total and pc["codes"].size == total // 2 and pc["scales"].size == total // 16
    nseg = -(-k // SEG)
    assert pc["seg_start"].size == d_out * nseg
    atoms = coeff_entry_atoms(pc)
    codes = unpack_nibbles(pc["codes"])
    for o in range(d_out):
        n = int(pc["nnz"][o])
        a = atoms[ptr[o]:ptr[o] + n]
        assert np.array_equal(a, C.atom_idx[C.col_ptr[o]:C.col_ptr[o + 1]])  # support recovered
        assert np.all(np.diff(a) > 0) and (n == 0 or (a[0] >= 0 and a[-1] < k))
        pad = slice(ptr[o] + n, ptr[o + 1])
        assert not codes[pad].any() and not pc["idx"][pad].any()  # padding is zero
        assert np.all(atoms[pad] == SEG * (nseg - 1))  # padding sits in the last segment
        ss = pc["seg_start"].reshape(d_out, nseg)[o].astype(np.int64)
        assert ss[0] == 0 and np.all(np.diff(ss) >= 0)
        for s in range(nseg):
            assert ss[s] == np.count_nonzero(a < SEG * s)


def test_coeff_blocks_follow_stored_entries():
    # a column of 20 entries: block 0 = entries 0..15, block 1 = entries 16..19 + 12 pads
    k = 64
    atoms = np.arange(0, 40, 2)
    vals = np.linspace(-1, 1, 20).astype(np.float32)
    vals[17] = 3.0
    pc = pack_coeff(np.array([0, 20]), atoms, vals, k, 1)
    s = float(pc["s"])
    sc = pc["scales"]
    assert sc.size == 2
    assert nvfp4.E4M3_TABLE[sc[1]] * s * 6 == pytest.approx(3.0, rel=1 / 16)
    assert nvfp4.E4M3_TABLE[sc[0]] * s * 6 == pytest.approx(1.0, rel=1 / 16)


def test_pack_rejects_bad_input():
    with pytest.raises(ValueError):
        pack_coeff(np.array([0, 2]), np.array([3, 3]), np.ones(2, np.float32), 8, 1)
    with pytest.raises(ValueError):
        pack_coeff(np.array([0, 1]), np.array([8]), np.ones(1, np.float32), 8, 1)
    with pytest.raises(ValueError):
        pack_dictionary(np.ones((24, 4), np.float32))
