"""Pins for the oracle's accounting against the numbers the technical review prints
(tests/golden/budget_pins.json)."""
import json
import os

import pytest

from oracle import accounting as A


@pytest.fixture(scope="module")
def pins(golden_dir):
    return json.load(open(os.path.join(golden_dir, "budget_pins.json")))


def test_eq3_ranks(pins):
    for c in pins["eq3_rank"]:
        assert A.eq3_rank(c["rho_fac"], c["n"], c["d_in"], c["d_out"]) == c["k"], c["what"]


def test_retained_fraction(pins):
    r = pins["retained_fraction"]
    f = A.retained_fraction(r["rho_fac"], r["n"], r["d"], r["d"], r["p"])
    assert round(f, r["digits"]) == r["value"]
    assert round(100 * (1 - f), pins["removed_percent"]["digits"]) == pins["removed_percent"]["value"]
    # the closed form the review gives: 0.8 (1 - 2p/3)
    assert f == pytest.approx(0.8 * (1 - 2 * r["p"] / 3), rel=1e-12)


def test_dictionary_shares(pins):
    k = A.eq3_rank_real(0.2, 2, 4096, 4096)
    b = A.eq2_budget(2, 4096, 4096, k, 0.0)
    d_share = 4096 * k / b["Np"]
    assert round(d_share, 4) == round(pins["dictionary_share_of_factored"]["value"], 4)
    assert round(A.dictionary_share(0.2, 2, 4096, 4096), 4) == pins["dictionary_share_of_original"]["value"]


def test_mac_fraction(pins):
    m = pins["mac_fraction"]
    assert round(A.mac_fraction(m["n"], m["k"], m["d"], m["d"], m["p"]), m["digits"]) == m["value"]


def test_nvfp4_bits_and_gains(pins):
    assert A.nvfp4_bits() == pins["nvfp4_bits_per_value"]
    g = 16 / A.nvfp4_bits()
    assert round(g, 2) == pins["nvfp4_gain_vs_fp16"]["value"]
    assert round(round(g, 2) * 1.43, 2) == pins["gain_times_1_43"]["value"]
    assert round(round(g, 2) * 2, 2) == pins["gain_times_2"]["value"]


def test_eq12(pins):
    for c in pins["eq12_breakeven"]:
        assert round(A.eq12_breakeven(c["a"], c["b"], c["h"]), c["digits"]) == c["p"], c["what"]
    n = pins["eq12_no_help"]
    assert A.eq12_saves(n["p"], n["a"], n["b"], n["h"]) is n["saves"]
    assert A.eq12_saves(0.7, 8, 4.5, 0) is True
    assert A.eq12_saves(0.3, 0, 4.5, 1) is True


def test_call_bytes_attention_projection():
    # 4096 -> 4096, k = 2048, 615 atoms per column (density 0.3), M = 1
    b = A.call_bytes(1, 4096, 4096, 2048, 615)
    assert b["D"] == 4096 * 2048 // 2 + 4096 * 2048 // 16 + 4
    assert b["C"] == 4 + 4096 * (308 + 39 + 615 + 16 + 4)
    assert round(b["total"] / 1e6, 3) == 8.757


def test_call_flops():
    f = A.call_flops(2048, 4096, 2048, 4096 * 615)
    assert round(f["dict"] / 1e9, 1) == 34.4
    assert round(f["coeff"] / 1e9, 1) == 10.3
