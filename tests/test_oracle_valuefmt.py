"""Pins of the oracle's coefficient value formats (Table 4: FP16, FP8, INT8 C
with an NVFP4 dictionary)."""
import json
import os

import numpy as np
import pytest

import synth
from oracle import forward as F
from oracle import valuefmt as VF
from oracle.nvfp4 import E4M3_TABLE
from oracle.pack import pack_coeff, pack_coeff_fmt, pack_dictionary


def test_table4_gains_follow_from_the_bits_per_value(golden_dir):
    """The NVFP4 / FP16 row fixes the dictionary's share r of the factorised
    model's values; the FP8, INT8 and NVFP4 rows then follow from 8, 8 and 4.5
    bits per coefficient value (no block scale for the 8-bit formats)."""
    with open(os.path.join(golden_dir, "table4_formats.json")) as f:
        rows = {(r["D"], r["C"]): r["gain"] for r in json.load(f)["rows"]}
    r = VF.table4_dictionary_fraction(rows[("nvfp4", "fp16")])
    assert 0.5 < r < 0.56
    for c in ("fp8", "int8", "nvfp4"):
        assert abs(VF.table4_gain(c, r) - rows[("nvfp4", c)]) < 0.006, c
    # an 8-bit format with a 16-value block scale (8.5 bits) would not give 2.60
    assert abs(16.0 / (4.5 * r + 8.5 * (1 - r)) - 2.60) > 0.07


def test_fp8_codes_are_the_nearest_e4m3_values_brute_force():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(4000) * np.exp(rng.uniform(-6, 3, 4000))).astype(np.float32)
    x[:5] = [0.0, -0.0, 1e-30, -1e-30, 0.0]
    s = VF.fp8_scale(x)
    codes = VF.fp8_encode(x, s)
    q = (x / s).astype(np.float64)
    finite = np.arange(256)[np.isfinite(E4M3_TABLE)]
    for qi, c in zip(q, codes):
        d = np.abs(E4M3_TABLE[finite] - qi)
        best = finite[d == d.min()]
        assert c in best, (qi, c, best)
        if best.size > 1:  # a tie between two codes goes to the even code (same sign)
            assert c % 2 == 0
    assert np.max(np.abs(x)) / s == pytest.approx(448.0, rel=1e-6)
    assert codes[1] == 0  # -0 written as 0


def test_int8_rounding_ties_and_clamp():
    s = np.float32(1.0)
    v = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, 127.49, 200.0, -300.0, 0.49999997], np.float32)
    assert VF.int8_encode(v, s).tolist() == [0, 2, 2, 0, -2, -2, 126, 127, 127, -127, 0]
    rng = np.random.default_rng(2)
    x = rng.standard_normal(5000).astype(np.float32)
    sc = VF.int8_scale(x)
    c = VF.int8_encode(x, sc).astype(np.float64)
    assert np.all(np.abs((x / sc).astype(np.float64) - c) <= 0.5 + 1e-6)
    assert np.max(np.abs(c)) == 127


def test_fp16_encoding_agrees_with_torch_half():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(3000) * np.exp(rng.uniform(-20, 10, 3000))).astype(np.float32)
    bits = VF.fp16_encode(x)
    t = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, t)
    with pytest.raises(ValueError):
        VF.fp16_encode(np.array([1e6], np.float32))


@pytest.mark.parametrize("fmt", ["fp16", "fp8", "int8"])
def test_formats_share_the_index_and_match_the_dense_forward(fmt):
    k, d_in, d_out = 300, 64, 29
    D = synth.gen_dictionary(51, 0, 0, d_in, k)
    C = synth.gen_coeff(51, 0, 0, 0, k, d_out, 0.4)
    X = synth.gen_activations(51, 0, 0, 3, d_in)
    pd = pack_dictionary(D)
    pc = pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    pf = pack_coeff_fmt(C.col_ptr, C.atom_idx, C.vals, k, d_out, fmt)
    for n in ("col_ptr", "nnz", "idx", "seg_start"):
        assert np.array_equal(pf[n], pc[n]), n
    assert pf["values"].size == int(pc["col_ptr"][-1])
    assert pf["values"].dtype == (np.uint16 if fmt == "fp16" else np.uint8)
    # dense expansion of the same decoded values, a different association of Eq. (1)
    atoms, vals = F.decode_coeff_fmt_entries(pf)
    Cd = np.zeros((k, d_out))
    cols = np.repeat(np.arange(d_out), np.diff(pf["col_ptr"].astype(np.int64)))
    np.add.at(Cd, (atoms, cols), vals)
    ref = F.forward_dense(X, F.decode_dictionary(pd) @ Cd)
    y = F.forward_factored_fmt(X, pd, pf)
    assert np.allclose(y, ref, rtol=1e-10, atol=1e-12)
    # and the decoded values are the inputs within the format's error bound
    ptr = pf["col_ptr"].astype(np.int64)
    got = np.concatenate([vals[ptr[o]:ptr[o] + (C.col_ptr[o + 1] - C.col_ptr[o])] for o in range(d_out)])
    err = np.abs(got - C.vals.astype(np.float64))
    amax = float(np.max(np.abs(C.vals)))
    bound = {"fp16": np.abs(C.vals) * 2.0 ** -11 + 2.0 ** -25,
             "fp8": np.abs(C.vals) * 2.0 ** -4 + float(pf["s"]) * 2.0 ** -10,
             "int8": np.full(C.vals.shape, 0.5 * amax / 127 * (1 + 1e-6))}[fmt]
    assert np.all(err <= bound)
