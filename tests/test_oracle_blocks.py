"""Pins of the oracle's block-structured coefficient layout (support = whole
aligned 16-atom blocks; one NVFP4 block and one uint16 index per kept block)."""
import json
import os

import numpy as np
import pytest

import synth
from oracle import forward as F
from oracle.accounting import eq12_breakeven
from oracle.pack import pack_coeff, pack_coeff_blocks, pack_dictionary


def test_hand_built_example(golden_dir):
    with open(os.path.join(golden_dir, "block_support_example.json")) as f:
        g = json.load(f)
    cols = [np.concatenate([np.arange(16 * b, 16 * b + 16) for b in bl]) if bl else np.zeros(0, np.int64)
            for bl in g["blocks"]]
    ptr = np.zeros(g["d_out"] + 1, np.int64)
    ptr[1:] = np.cumsum([c.size for c in cols])
    atoms = np.concatenate(cols)
    vals = np.linspace(-1, 1, atoms.size).astype(np.float32)
    pk = pack_coeff_blocks(ptr, atoms, vals, g["k"], g["d_out"])
    assert pk["blk_ptr"].tolist() == g["blk_ptr"]
    assert pk["blk_idx"].tolist() == g["blk_idx"]
    assert pk["codes"].size == 8 * 3 and pk["scales"].size == 3
    at, _ = F.decode_coeff_block_entries(pk)
    assert at.tolist() == atoms.tolist()


def test_rejects_supports_that_are_not_aligned_blocks():
    with pytest.raises(ValueError):
        pack_coeff_blocks(np.array([0, 16]), np.arange(1, 17), np.ones(16, np.float32), 32, 1)
    with pytest.raises(ValueError):
        pack_coeff_blocks(np.array([0, 8]), np.arange(8), np.ones(8, np.float32), 32, 1)


@pytest.mark.parametrize("k,d_out,rho", [(2048, 64, 0.3), (3072, 40, 0.25), (64, 9, 1.0), (512, 33, 0.0)])
def test_same_values_as_the_u8_layout_and_the_input_support(k, d_out, rho):
    C = synth.gen_coeff_blocks(52, 0, 0, 0, k, d_out, rho)
    pc = pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    pk = pack_coeff_blocks(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    # block-aligned supports need no padding: the NVFP4 blocks coincide
    assert np.array_equal(pc["col_ptr"].astype(np.int64), pk["blk_ptr"].astype(np.int64) * 16)
    assert np.array_equal(pc["codes"], pk["codes"]) and np.array_equal(pc["scales"], pk["scales"])
    assert pc["s"] == pk["s"]
    at, _ = F.decode_coeff_block_entries(pk)
    assert np.array_equal(at, C.atom_idx.astype(np.int64))
    kb = k // 16
    nb = kb - int(np.floor((1 - rho) * kb))
    assert np.all(np.diff(pk["blk_ptr"].astype(np.int64)) == nb)


def test_block_forward_matches_the_dense_product():
    k, d_in, d_out = 256, 64, 21
    D = synth.gen_dictionary(52, 1, 0, d_in, k)
    C = synth.gen_coeff_blocks(52, 1, 0, 0, k, d_out, 0.4)
    X = synth.gen_activations(52, 1, 0, 4, d_in)
    pd = pack_dictionary(D)
    pk = pack_coeff_blocks(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    pc = pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    y = F.forward_factored_blocks(X, pd, pk)
    assert np.allclose(y, F.forward_reference(X, pd, pc), rtol=1e-10, atol=1e-12)
    bad = dict(pk, blk_idx=pk["blk_idx"].copy())
    bad["blk_idx"][0] ^= 1  # one block moved
    assert not np.allclose(F.forward_factored_blocks(X, pd, bad), y, rtol=1e-6)


def test_index_cost_and_break_even(golden_dir):
    # 16 index bits per 16 values: Eq. (12) with a = 1, h = 0 against dense NVFP4 (b = 4.5)
    assert abs(eq12_breakeven(1.0, 4.5, 0.0) - 1 / 5.5) < 1e-15
    k, d_out = 2048, 64
    for p, saves in [(0.15, False), (0.21, True)]:
        C = synth.gen_coeff_blocks(52, 2, 0, 0, k, d_out, 1 - p)
        pk = pack_coeff_blocks(C.col_ptr, C.atom_idx, C.vals, k, d_out)
        bits = 4.5 * C.atom_idx.size + 16 * pk["blk_idx"].size
        assert (bits < 4.5 * k * d_out) == saves
