"""CPU tests of the C-ABI library: it loads, exports every declared symbol, its
host packer matches the oracle's packed layouts bit for bit, and its host-side
validation returns the documented status codes. No compute call needs a GPU here."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from oracle.pack import pack_coeff, pack_dictionary

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dp():
    import dictionary_compressed_linear_b200 as m
    from dictionary_compressed_linear_b200 import build
    build.build()
    return m


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(dictproj_[a-z0-9_]+)\s*\(", txt))
    return names


def test_library_exports_every_declared_symbol(dp):
    lib = ctypes.CDLL(dp.LIB_PATH)
    declared = _declared_symbols()
    assert len(declared) >= 20
    for name in sorted(declared):
        assert hasattr(lib, name), name
    bound = {n for n, _, _ in dp.SIGNATURES}
    assert declared == bound, declared ^ bound


def test_version_and_status_strings(dp):
    assert dp.dictproj_version() >= 10000
    assert dp.dictproj_status_string(0) == "DICTPROJ_OK"
    assert dp.dictproj_status_string(-8) == "DICTPROJ_ERR_TIMEOUT"
    from dictionary_compressed_linear_b200.binding import STATUS
    for code, name in STATUS.items():
        assert dp.dictproj_status_string(code) == name


def _same_layer(a, b):
    for n in ("col_ptr", "nnz", "codes", "scales", "idx", "seg_start"):
        assert np.array_equal(a[n], b[n]), n
    assert a["s"] == b["s"]


@pytest.mark.parametrize("d_in,k", [(256, 128), (4096, 2048), (11008, 3072), (32, 16), (96, 272)])
def test_group_packer_bit_exact(dp, d_in, k):
    D = synth.gen_dictionary(7, d_in, k, d_in, k)
    a = dp.dictproj_pack_group_host(D)
    b = pack_dictionary(D)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scales"], b["scales"])
    assert a["s"] == b["s"]


@pytest.mark.parametrize("k,d_out,rho", [(128, 256, 0.5), (2048, 512, 0.3), (3072, 300, 0.25),
                                         (272, 45, 0.05), (16, 7, 1.0), (512, 33, 0.0)])
def test_layer_packer_bit_exact(dp, k, d_out, rho):
    C = synth.gen_coeff(7, k, d_out, 1, k, d_out, rho)
    a = dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    b = pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    _same_layer(a, b)


def test_layer_packer_bit_exact_ragged_columns(dp):
    # columns of different lengths, including empty and full ones, atoms in sparse segments
    rng = np.random.default_rng(11)
    k, d_out = 1000, 20
    cols = []
    for o in range(d_out):
        n = [0, k, 1, 17, 255, 256, 3][o % 7]
        cols.append(np.sort(rng.choice(k, size=n, replace=False)))
    cols[5] = np.array([3, 700, 999])  # segments 1 and 2 empty
    ptr = np.zeros(d_out + 1, np.int32)
    ptr[1:] = np.cumsum([c.size for c in cols])
    atoms = np.concatenate(cols).astype(np.int32)
    vals = (rng.standard_normal(atoms.size) * np.exp(rng.uniform(-8, 4, atoms.size))).astype(np.float32)
    vals[::7] = 0.0
    a = dp.dictproj_pack_layer_host(ptr, atoms, vals, k, d_out)
    b = pack_coeff(ptr, atoms, vals, k, d_out)
    _same_layer(a, b)


def test_group_packer_extreme_values(dp):
    rng = np.random.default_rng(5)
    D = (rng.standard_normal((64, 32)) * np.exp(rng.uniform(-30, 30, (64, 32)))).astype(np.float32)
    D[:16, 0] = 0.0
    D[16:32, 1] = 1e-38
    a = dp.dictproj_pack_group_host(D)
    b = pack_dictionary(D)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


def test_host_validation(dp):
    from dictionary_compressed_linear_b200 import DictprojError
    with pytest.raises(DictprojError) as e:
        dp.dictproj_pack_group_host(np.ones((24, 4), np.float32))
    assert e.value.status == -2
    bad = np.ones((32, 4), np.float32)
    bad[3, 1] = np.nan
    with pytest.raises(DictprojError) as e:
        dp.dictproj_pack_group_host(bad)
    assert e.value.status == -10
    with pytest.raises(DictprojError) as e:  # unsorted atoms
        dp.dictproj_pack_layer_host(np.array([0, 2]), np.array([5, 1]), np.ones(2), 16, 1)
    assert e.value.status == -5
    with pytest.raises(DictprojError) as e:  # atom out of range
        dp.dictproj_pack_layer_host(np.array([0, 1]), np.array([16]), np.ones(1), 16, 1)
    assert e.value.status == -5
    with pytest.raises(DictprojError) as e:  # column longer than k
        dp.dictproj_layer_packed_entries(np.array([0, 20]), 16, 1)
    assert e.value.status == -5
    lib = dp.lib()
    assert lib.dictproj_pack_group_host(None, 32, 16, None, None, None) == -1
    assert dp.dictproj_forward_status(0, 1, None, None, 0) == -1
    assert "NULL" in dp.dictproj_last_error()
    # the prefill entry points and the host helpers validate before touching a device
    import ctypes as C
    assert lib.dictproj_dictionary_stage_prefill(None, 16, None, None, None) == -1
    assert lib.dictproj_group_reserve_prefill(None, 4096) == -1
    assert lib.dictproj_forward_noalloc(None, None, None, 1, None, None) == -1
    k = C.c_int()
    assert lib.dictproj_rank_for_budget(0.2, 0, 4096, 4096, 1, C.byref(k)) == -2
    assert lib.dictproj_rank_for_budget(-0.1, 1, 4096, 4096, 1, C.byref(k)) == -5
    assert lib.dictproj_rank_for_budget(0.2, 1, 4096, 4096, 1, None) == -1
    assert lib.dictproj_budget(1, 4096, 4096, 16, 1.5, None, None, None, None) == -5
    assert lib.dictproj_group_file_write(None, None, None, 1.0, 64, 16) == -1
    codes = np.zeros(64 * 16 // 2, np.uint8)
    scales = np.zeros(64 * 16 // 16, np.uint8)
    u8 = C.POINTER(C.c_uint8)
    assert lib.dictproj_group_file_write(b"/nonexistent-dir/x.dpj", codes.ctypes.data_as(u8),
                                         scales.ctypes.data_as(u8), 1.0, 64, 16) == -11
    assert lib.dictproj_group_file_write(b"x.dpj", codes.ctypes.data_as(u8), scales.ctypes.data_as(u8),
                                         float("nan"), 64, 16) == -10
    assert lib.dictproj_group_file_write(b"x.dpj", codes.ctypes.data_as(u8), scales.ctypes.data_as(u8),
                                         1.0, 48, 16) == -2


def test_device_calls_fail_loudly_without_gpu(dp):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    from dictionary_compressed_linear_b200 import DictprojError
    with pytest.raises(DictprojError) as e:
        dp.dictproj_pack_group(np.ones((32, 16), np.float32), 1)
    assert e.value.status == -6


def test_noalloc_and_selftest_validate_before_any_device_call(dp):
    # fake (never dereferenced) device addresses: validation rejects the call on
    # the host, before any CUDA call, so this runs without a GPU
    base = 1 << 40
    g = dp.DeviceGroup(base, base + 4096, 1.0, 64, 32)
    l = dp.DeviceLayer(base + 8192, base + 12288, base + 16384, base + 20480, base + 24576, 1.0, 32, 16)
    for field in ("codes", "scales"):
        gg = dp.DeviceGroup(base, base + 4096, 1.0, 64, 32)
        setattr(gg, field, getattr(gg, field) + 8)
        assert dp.dictproj_forward_noalloc_status(gg, l, base + 28672, 1, base + 32768, 0) == -3
        assert "16-byte aligned" in dp.dictproj_last_error()
    for field in ("col_ptr", "codes", "scales", "idx", "seg_start"):
        ll = dp.DeviceLayer(base + 8192, base + 12288, base + 16384, base + 20480, base + 24576, 1.0, 32, 16)
        setattr(ll, field, getattr(ll, field) + 2)
        assert dp.dictproj_forward_noalloc_status(g, ll, base + 28672, 1, base + 32768, 0) == -3
        assert field in dp.dictproj_last_error()
    lib = dp.lib()
    assert lib.dictproj_selftest_wait_timeout(0, None) == -5
    assert lib.dictproj_selftest_wait_timeout((1 << 31) + 1, None) == -5


@pytest.mark.parametrize("k,d_out,rho", [(128, 256, 0.5), (2048, 512, 0.3), (3072, 300, 0.25),
                                         (272, 45, 0.05), (16, 7, 1.0), (40, 33, 0.0), (8448, 9, 0.1)])
def test_bitmap_layer_packer_bit_exact(dp, k, d_out, rho):
    from oracle.pack import pack_coeff_bitmap
    C = synth.gen_coeff(7, k, d_out, 2, k, d_out, rho)
    a = dp.dictproj_pack_layer_bitmap_host(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    b = pack_coeff_bitmap(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    for n in ("col_ptr", "nnz", "codes", "scales", "bitmap"):
        assert np.array_equal(a[n], b[n]), n
    assert a["s"] == b["s"] and a["words"] == b["words"]


@pytest.mark.parametrize("fmt", ["fp16", "fp8", "int8"])
@pytest.mark.parametrize("k,d_out,rho", [(128, 64, 0.5), (2048, 300, 0.3), (272, 45, 0.05), (16, 7, 1.0)])
def test_value_format_packer_bit_exact(dp, fmt, k, d_out, rho):
    from oracle.pack import pack_coeff_fmt
    C = synth.gen_coeff(8, k, d_out, 3, k, d_out, rho)
    vals = C.vals.copy()
    if vals.size > 8:  # exercise ties, zeros, tiny and large magnitudes
        vals[0] = 0.0
        vals[1] = -0.0
        vals[2] = 1e-30
        vals[3] = float(np.max(np.abs(vals))) * 1.0
        vals[4] = 3.0517578125e-05 * 1.5  # between fp16 subnormals
    a = dp.dictproj_pack_layer_fmt_host(C.col_ptr, C.atom_idx, vals, k, d_out, fmt)
    b = pack_coeff_fmt(C.col_ptr, C.atom_idx, vals, k, d_out, fmt)
    for n in ("col_ptr", "nnz", "values", "idx", "seg_start"):
        assert np.array_equal(a[n], b[n]), n
    assert a["s"] == b["s"]


def test_fp16_value_packer_matches_the_binary16_definition_everywhere(dp):
    # magnitudes across the whole binary16 range, including subnormals and the
    # rounding boundary at the top; compared with numpy's float16 cast
    rng = np.random.default_rng(12)
    e = rng.uniform(-27, 15.99, 20000)
    x = (np.sign(rng.standard_normal(20000)) * 2.0 ** e).astype(np.float32)
    x[:4] = [65504.0, -65504.0, 65519.0, 2.0 ** -25]
    n = x.size
    ptr = np.array([0, n], np.int32)
    atoms = np.arange(n, dtype=np.int32)
    a = dp.dictproj_pack_layer_fmt_host(ptr, atoms, x, n + (-n) % 16, 1, "fp16")
    want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(a["values"][:n], want)
    from dictionary_compressed_linear_b200 import DictprojError
    with pytest.raises(DictprojError) as e:
        dp.dictproj_pack_layer_fmt_host(np.array([0, 1], np.int32), atoms[:1], np.array([65520.0], np.float32), 16, 1,
                                        "fp16")
    assert e.value.status == -10


@pytest.mark.parametrize("k,d_out,rho", [(2048, 64, 0.3), (3072, 40, 0.25), (64, 9, 1.0), (512, 33, 0.0)])
def test_block_layer_packer_bit_exact(dp, k, d_out, rho):
    from oracle.pack import pack_coeff_blocks
    C = synth.gen_coeff_blocks(9, k, d_out, 1, k, d_out, rho)
    a = dp.dictproj_pack_layer_blocks_host(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    b = pack_coeff_blocks(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    for n in ("blk_ptr", "blk_idx", "codes", "scales"):
        assert np.array_equal(a[n], b[n]), n
    assert a["s"] == b["s"]


def test_block_layer_packer_rejects_unaligned_supports(dp):
    from dictionary_compressed_linear_b200 import DictprojError
    with pytest.raises(DictprojError) as e:
        dp.dictproj_pack_layer_blocks_host(np.array([0, 16]), np.arange(1, 17), np.ones(16), 32, 1)
    assert e.value.status == -5
    with pytest.raises(DictprojError) as e:
        dp.dictproj_pack_layer_blocks_host(np.array([0, 8]), np.arange(8), np.ones(8), 32, 1)
    assert e.value.status == -5


def test_decode_kernel_choice_is_validated_and_kept(dp):
    assert dp.dictproj_get_decode_kernels() == dp.DECODE_AUTO
    for which in (dp.DECODE_FUSED, dp.DECODE_SPLIT, dp.DECODE_AUTO):
        dp.dictproj_set_decode_kernels(which)
        assert dp.dictproj_get_decode_kernels() == which
    for bad in (-1, 3):
        with pytest.raises(dp.DictprojError) as err:
            dp.dictproj_set_decode_kernels(bad)
        assert err.value.status == -5
    assert dp.dictproj_get_decode_kernels() == dp.DECODE_AUTO


def test_index_format_uploads_validate_before_touching_a_device(dp):
    """Bitmap and block uploads check their arrays first (no device is needed to
    be refused)."""
    import numpy as np
    k, d_out = 48, 2
    good = {"col_ptr": np.array([0, 16, 32], np.uint32), "codes": np.zeros(16, np.uint8),
            "scales": np.zeros(2, np.uint8), "bitmap": np.array([0xF, 0, 0x1, 0], np.uint32),
            "s": np.float32(1.0), "k": k, "d_out": d_out}
    bad_bit = dict(good, bitmap=np.array([0xF, 1 << 20, 0x1, 0], np.uint32))  # atom 52 >= k
    too_many = dict(good, bitmap=np.array([0xFFFFFFFF, 0, 0x1, 0], np.uint32))  # 32 bits for 16 entries
    for packed, status in ((bad_bit, -5), (too_many, -5), (dict(good, s=np.float32(0.0)), -10)):
        with pytest.raises(dp.DictprojError) as err:
            dp.dictproj_layer_upload_bitmap(packed)
        assert err.value.status == status
    blocks = {"blk_ptr": np.array([0, 2, 3], np.uint32), "blk_idx": np.array([2, 1, 0], np.uint16),
              "codes": np.zeros(24, np.uint8), "scales": np.zeros(3, np.uint8), "s": np.float32(1.0), "k": k,
              "d_out": d_out}
    with pytest.raises(dp.DictprojError) as err:  # column 0's blocks not ascending
        dp.dictproj_layer_upload_blocks(blocks)
    assert err.value.status == -5
    with pytest.raises(dp.DictprojError) as err:  # block 3 of a k = 48 layer
        dp.dictproj_layer_upload_blocks(dict(blocks, blk_idx=np.array([0, 1, 3], np.uint16)))
    assert err.value.status == -5
    with pytest.raises(dp.DictprojError) as err:  # not a union of aligned 16-atom blocks
        dp.dictproj_pack_layer_blocks(np.array([0, 3], np.int32), np.array([0, 1, 2], np.int32),
                                      np.ones(3, np.float32), 48, 1)
    assert err.value.status < 0


def test_batched_decode_grid_follows_each_projections_bytes(dp):
    # the dictionary grid takes the J of least modelled time (waves x (fixed +
    # rows per CTA)); on the LLaMA-7B shapes that is the fastest J measured: one
    # slice for the q/k/v and gate/up batches, J = 1 for o alone, three slices for
    # down. A mixed batch streams about the same rows per CTA in every projection,
    # and the coefficient kernel's CTAs go where the batch would otherwise finish last.
    n_sm = 148
    qkv = (4096, 2048, 4096, 4096 * 624)
    gate = (4096, 3072, 11008, 11008 * 784)
    down = (11008, 3072, 4096, 4096 * 784)
    assert dp.dictproj_decode_batch_plan([qkv], 1, n_sm)[0]["dict_slices"] == 4
    assert all(b["dict_slices"] == 1 and b["dict_ctas"] == 128 for b in dp.dictproj_decode_batch_plan([qkv] * 3, 1, n_sm))
    assert all(b["dict_slices"] == 1 for b in dp.dictproj_decode_batch_plan([gate] * 2, 1, n_sm))
    assert dp.dictproj_decode_batch_plan([down], 1, n_sm)[0]["dict_slices"] == 3
    batch = dp.dictproj_decode_batch_plan([qkv] * 3, 1, n_sm)
    assert sorted(b["coeff_ctas"] for b in batch) == [49, 49, 50]
    lone = dp.dictproj_decode_batch_plan([qkv], 1, n_sm)[0]
    assert n_sm - 2 <= lone["coeff_ctas"] <= n_sm  # columns per CTA rounded up
    mixed = [qkv, down, gate]
    plan = dp.dictproj_decode_batch_plan(mixed, 1, n_sm)
    rows = [d / p["dict_slices"] for (d, _, _, _), p in zip(mixed, plan)]
    assert max(rows) / min(rows) < 1.15  # per-CTA dictionary bytes within rounding of one slice
    for (d_in, k, _, _), p in zip(mixed, plan):
        assert p["dict_ctas"] == (k // 16) * p["dict_slices"]
        assert p["dict_slices"] <= -(-d_in // 1024)  # at most the J = 1 slices the group's Z scratch holds
    assert sum(p["coeff_ctas"] for p in plan) <= n_sm and all(p["coeff_ctas"] >= 1 for p in plan)
    # the gather's CTAs go one at a time to the projection that would finish last
    # (whole columns per warp; a column costs two 256-entry windows plus its
    # windows): at densities 0.2 / 0.3 / 0.4 over 32768 columns the sparser
    # projections get more CTAs per stored entry than a split by entries would give
    wide = [(4096, 2048, 32768, 32768 * e) for e in (416, 624, 832)]
    shares = [p["coeff_ctas"] for p in dp.dictproj_decode_batch_plan(wide, 1, n_sm)]
    assert shares == [40, 49, 59], shares
    assert sum(shares) == n_sm
    tiny = dp.dictproj_decode_batch_plan([(64, 32, 8, 16), (4096, 2048, 4096, 10 ** 7)], 1, n_sm)
    assert tiny[0]["coeff_ctas"] >= 1 and tiny[0]["dict_slices"] == 1
    with pytest.raises(dp.DictprojError):
        dp.dictproj_decode_batch_plan([qkv], 9, n_sm)
    with pytest.raises(dp.DictprojError):
        dp.dictproj_decode_batch_plan([(4096, 2047, 16, 0)], 1, n_sm)


def test_stage_mask_and_diagnostic_calls_validate_on_the_host(dp):
    # the stage mask and the timestamp buffer are checked before any device call,
    # so these run without a GPU
    import ctypes as C
    lib = C.CDLL(dp.LIB_PATH)
    lib.dictproj_forward_batch_stages.restype = C.c_int
    lib.dictproj_forward_batch_stages.argtypes = [C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                                                  C.c_void_p, C.c_int]
    for bad in (0, 4, -1):
        assert lib.dictproj_forward_batch_stages(1, None, 1, None, None, None, None, bad) == -5
    assert lib.dictproj_forward_batch_stages(1, None, 1, None, None, None, None, 3) == -1  # NULL arrays
    lib.dictproj_diag_gather_times.restype = C.c_int
    lib.dictproj_diag_gather_times.argtypes = [C.c_void_p, C.c_int]
    assert lib.dictproj_diag_gather_times(C.c_void_p(1 << 40), 0) == -5   # a buffer with no CTAs
    assert lib.dictproj_diag_gather_times(C.c_void_p((1 << 40) + 4), 8) == -3  # not 8-byte aligned


def test_host_packers_on_exactly_representable_factors(dp):
    # the factors of the oracle's exact-product pin (every NVFP4 block holds an
    # entry of magnitude 6 x 448): the library's host packers give the oracle's
    # bytes, tensor scale 1 and block scale 448 throughout, so the device path is
    # tied to the exact integer product through the same bytes
    from exact_factors import exact_case
    X, D, col_ptr, atoms, vals, k, d_out, exact = exact_case()
    a = dp.dictproj_pack_group_host(D)
    b = pack_dictionary(D)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    assert a["s"] == b["s"] == 1.0 and np.all(a["scales"] == 0x7E)
    _same_layer(dp.dictproj_pack_layer_host(col_ptr, atoms, vals, k, d_out), pack_coeff(col_ptr, atoms, vals, k, d_out))
