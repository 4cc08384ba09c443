"""Host-only helpers of the C ABI: the Eq. (3) rank and Eq. (2) counts of the
DictLLM technical review ("The budget: trading shared rank against sparsity"),
checked against the review's printed ranks and against the oracle's own
restatement; and the packed-file export / import (review Algorithm 2, export
step), checked for bit-exact round trips and for rejecting damaged files."""
import json
import os

import numpy as np
import pytest

import synth
import dictionary_compressed_linear_b200 as dp
from dictionary_compressed_linear_b200.binding import DictprojError
from oracle import accounting as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "budget_pins.json")


def test_rank_matches_the_review_printed_values():
    pins = json.load(open(GOLDEN))["eq3_rank"]
    for p in pins:
        assert dp.dictproj_rank_for_budget(p["rho_fac"], p["n"], p["d_in"], p["d_out"]) == p["k"], p["what"]


def test_rank_and_budget_agree_with_the_oracle():
    rng = np.random.default_rng(5)
    for _ in range(200):
        rho = float(rng.uniform(0, 0.95))
        n, d_in, d_out = int(rng.integers(1, 9)), int(rng.integers(64, 20000)), int(rng.integers(64, 20000))
        k = dp.dictproj_rank_for_budget(rho, n, d_in, d_out)
        assert k == A.eq3_rank(rho, n, d_in, d_out)
        p = float(rng.uniform(0, 1))
        got = dp.dictproj_budget(n, d_in, d_out, k, p)
        ref = A.eq2_budget(n, d_in, d_out, k, p)
        for key in ("N0", "Np", "rho", "G"):
            assert got[key] == pytest.approx(ref[key], rel=1e-12), key


def test_rank_alignment_rounds_down_and_rejects_empty_budgets():
    assert dp.dictproj_rank_for_budget(0.2, 2, 4096, 4096, 16) == 2176  # 2184 rounded down to 16
    with pytest.raises(DictprojError):
        dp.dictproj_rank_for_budget(0.999999, 1, 16, 16, 16)
    with pytest.raises(DictprojError):
        dp.dictproj_rank_for_budget(1.0, 1, 4096, 4096)


@pytest.fixture(scope="module")
def packed():
    D = synth.gen_dictionary(0, 0, 0, 256, 128)
    C = synth.gen_coeff(0, 0, 0, 0, 128, 256, 0.5)
    return dp.dictproj_pack_group_host(D), dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, 128, 256)


def test_group_file_round_trip_is_bit_exact(tmp_path, packed):
    pg, _ = packed
    path = str(tmp_path / "g.dpj")
    dp.dictproj_group_file_write(path, pg)
    back = dp.dictproj_group_file_read(path)
    assert back["d_in"] == pg["d_in"] and back["k"] == pg["k"]
    assert np.float32(back["s"]).tobytes() == np.float32(pg["s"]).tobytes()
    for n in ("codes", "scales"):
        assert np.array_equal(back[n], pg[n])
    assert os.path.getsize(path) == 64 + 256 * 128 // 2 + 256 * 128 // 16


def test_layer_file_round_trip_is_bit_exact(tmp_path, packed):
    _, pc = packed
    path = str(tmp_path / "l.dpj")
    dp.dictproj_layer_file_write(path, pc)
    back = dp.dictproj_layer_file_read(path)
    assert back["k"] == 128 and back["d_out"] == 256
    assert np.float32(back["s"]).tobytes() == np.float32(pc["s"]).tobytes()
    for n in ("col_ptr", "codes", "scales", "idx", "seg_start"):
        assert np.array_equal(back[n], pc[n]), n


def test_damaged_files_are_rejected(tmp_path, packed):
    pg, pc = packed
    g, l = str(tmp_path / "g.dpj"), str(tmp_path / "l.dpj")
    dp.dictproj_group_file_write(g, pg)
    dp.dictproj_layer_file_write(l, pc)
    raw = open(g, "rb").read()
    bad = bytearray(raw)
    bad[64 + 100] ^= 0x10                     # one payload bit
    open(str(tmp_path / "flip.dpj"), "wb").write(bytes(bad))
    open(str(tmp_path / "short.dpj"), "wb").write(raw[:-7])
    open(str(tmp_path / "long.dpj"), "wb").write(raw + b"\0")
    for name, status in (("flip.dpj", -10), ("short.dpj", -10), ("long.dpj", -10)):
        with pytest.raises(DictprojError) as e:
            dp.dictproj_group_file_read(str(tmp_path / name))
        assert e.value.status == status, name
    with pytest.raises(DictprojError) as e:        # a layer file is not a group file
        dp.dictproj_group_file_read(l)
    assert e.value.status == -10
    with pytest.raises(DictprojError) as e:
        dp.dictproj_group_file_read(str(tmp_path / "missing.dpj"))
    assert e.value.status == -11


def test_read_checks_the_callers_buffer_shapes(tmp_path, packed):
    pg, _ = packed
    path = str(tmp_path / "g.dpj")
    dp.dictproj_group_file_write(path, pg)
    L = dp.lib()
    import ctypes as C
    codes = np.zeros(256 * 64 // 2, np.uint8)
    scales = np.zeros(256 * 64 // 16, np.uint8)
    s = C.c_float()
    st = L.dictproj_group_file_read(path.encode(), codes.ctypes.data_as(C.POINTER(C.c_uint8)),
                                    scales.ctypes.data_as(C.POINTER(C.c_uint8)), C.byref(s), 256, 64)
    assert st == -4  # MISMATCH: the file holds k = 128
