"""Pins for the oracle's NVFP4 codec (E2M1 / E4M3 tables, encoders, quantiser).

The E2M1 and E4M3 tables are checked exhaustively against the public format
tables (tests/golden/format_values.json) and against PyTorch's float8_e4m3fn
conversion, a library routine independent of the oracle.  The quantiser is
checked against hand-derived blocks (tests/golden/nvfp4_blocks.json) and
round-to-nearest invariants.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4
from oracle.pack import pack_coeff, pack_dictionary, unpack_nibbles


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def test_e2m1_table_matches_spec(golden_dir):
    g = _golden(golden_dir, "format_values.json")["e2m1"]
    for code in range(16):
        want = g[str(code)]
        got = nvfp4.E2M1_TABLE[code]
        assert got == want, (code, got, want)
        assert np.signbit(got) == np.signbit(want) or want == 0.0


def test_e4m3_table_matches_spec_spots(golden_dir):
    g = _golden(golden_dir, "format_values.json")
    for code, want in g["e4m3_spot"].items():
        assert nvfp4.E4M3_TABLE[int(code)] == want, code
    for code in g["e4m3_nan_codes"]:
        assert np.isnan(nvfp4.E4M3_TABLE[code])


def test_e4m3_table_matches_torch_float8():
    raw = torch.arange(256, dtype=torch.uint8)
    ref = raw.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = nvfp4.E4M3_TABLE
    nan_ref = np.isnan(ref)
    assert np.array_equal(nan_ref, np.isnan(ours))
    assert np.array_equal(ref[~nan_ref], ours[~nan_ref])


def test_e4m3_encoder_matches_torch_rne():
    # torch's fp32 -> float8_e4m3fn cast rounds to nearest even; compare on
    # values inside the finite range, including every exact midpoint.
    pos = nvfp4.E4M3_TABLE[:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2.0
    rng = np.random.default_rng(1)
    rnd = rng.uniform(0, 448, 20000)
    tiny = rng.uniform(0, 0.03, 20000)
    vals = np.concatenate([pos, mids, rnd, tiny]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = nvfp4.e4m3_encode(vals)
    assert np.array_equal(ref, ours)


def test_e4m3_encoder_saturates():
    assert nvfp4.e4m3_encode(np.array([448.0, 460.0, 1e6], np.float32)).tolist() == [0x7E] * 3


def test_e2m1_roundtrip_and_ties():
    for c in range(16):
        v = nvfp4.E2M1_TABLE[c]
        want = 0 if c == 8 else c  # -0 is written as +0
        assert nvfp4.e2m1_encode(np.array([v], np.float32))[0] == want
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in ties.items():
        for sgn in (1, -1):
            c = nvfp4.e2m1_encode(np.array([sgn * x], np.float32))[0]
            assert nvfp4.E2M1_TABLE[c] == sgn * want or (want == 0 and c == 0)
    assert nvfp4.e2m1_encode(np.array([7.0, -100.0], np.float32)).tolist() == [7, 15]


def test_e2m1_encoder_is_nearest():
    rng = np.random.default_rng(2)
    q = rng.uniform(-7, 7, 50000).astype(np.float32)
    c = nvfp4.e2m1_encode(q)
    dec = nvfp4.E2M1_TABLE[c]
    clipped = np.clip(q, -6, 6).astype(np.float64)
    best = np.min(np.abs(clipped[:, None] - nvfp4.E2M1_TABLE[None, :]), axis=1)
    assert np.all(np.abs(clipped - dec) <= best + 0.0)


def test_hand_derived_blocks(golden_dir):
    g = _golden(golden_dir, "nvfp4_blocks.json")
    x = np.concatenate([np.array(b["x"], np.float32) for b in g["blocks"]])
    s = nvfp4.tensor_scale(x)
    assert s == np.float32(g["tensor_scale"])
    codes, sc = nvfp4.quantize_blocks(x.reshape(-1, 16), s)
    for i, b in enumerate(g["blocks"]):
        assert sc[i] == b["scale_code"], b["name"]
        assert codes[i].tolist() == b["codes"], b["name"]


def test_hand_derived_blocks_through_both_packers(golden_dir):
    g = _golden(golden_dir, "nvfp4_blocks.json")
    x = np.concatenate([np.array(b["x"], np.float32) for b in g["blocks"]])
    want_codes = np.concatenate([b["codes"] for b in g["blocks"]]).astype(np.uint8)
    want_sc = np.array([b["scale_code"] for b in g["blocks"]], np.uint8)
    # as one dictionary atom (blocks run along d_in)
    pd = pack_dictionary(x.reshape(-1, 1))
    assert np.array_equal(unpack_nibbles(pd["codes"]), want_codes)
    assert np.array_equal(pd["scales"], want_sc)
    # as one coefficient column over atoms 0..95 (blocks run along stored entries)
    n = x.size
    pc = pack_coeff(np.array([0, n]), np.arange(n), x, k=n, d_out=1)
    assert np.array_equal(unpack_nibbles(pc["codes"]), want_codes)
    assert np.array_equal(pc["scales"], want_sc)
    assert pc["s"] == np.float32(g["tensor_scale"])


def test_quantiser_error_bound_and_idempotence():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(16 * 4000) * np.exp(rng.uniform(-6, 3, 16 * 4000))).astype(np.float32)
    s = nvfp4.tensor_scale(x)
    codes, sc = nvfp4.quantize_blocks(x.reshape(-1, 16), s)
    xh = nvfp4.dequantize(codes, sc, float(s))
    scale = nvfp4.E4M3_TABLE[sc] * float(s)
    # per element: error <= half the E2M1 spacing at that magnitude, times the
    # block scale (spacing 0.5 below 2, 1 in [2,4), 2 in [4,6]); saturation
    # when the block amax rounds the scale down adds at most 1/16 of amax_b.
    xb = x.reshape(-1, 16).astype(np.float64)
    q = np.abs(xb) / np.where(scale[:, None] > 0, scale[:, None], 1)
    half = np.where(q < 2, 0.25, np.where(q < 4, 0.5, 1.0)) * scale[:, None]
    sat = np.maximum(np.abs(xb) - 6 * scale[:, None], 0)
    amaxb = np.max(np.abs(xb), axis=1, keepdims=True)
    live = scale[:, None] > 0
    err = np.abs(xb - xh)
    assert np.all(err[live.repeat(16, 1)] <= (half + sat + 1e-12 * amaxb)[live.repeat(16, 1)])
    assert np.all(sat <= amaxb / 16 + 1e-30)
    # quantising the decoded values again gives the same codes
    codes2, sc2 = nvfp4.quantize_blocks(xh.astype(np.float32).reshape(-1, 16), s)
    live_b = sc != 0
    assert np.array_equal(codes2[live_b], codes[live_b])


def test_all_zero_tensor():
    s = nvfp4.tensor_scale(np.zeros(32, np.float32))
    assert s == 1.0
    codes, sc = nvfp4.quantize_blocks(np.zeros((2, 16), np.float32), s)
    assert not codes.any() and not sc.any()


def test_rejects_non_finite():
    with pytest.raises(ValueError):
        nvfp4.quantize_blocks(np.full((1, 16), np.inf, np.float32), np.float32(1.0))
