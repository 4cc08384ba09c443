"""ctypes binding of libdictproj.so: argument marshalling only.

Every function here has the name of the C entry point it calls (include/dictproj.h)
and does nothing but convert Python / NumPy arguments to C types and raise on a
non-zero status. All arithmetic of the forward pass runs in the library's CUDA
kernels. Device buffers are passed as integer addresses (e.g. a torch tensor's
``data_ptr()``); streams as integer handles (e.g. ``torch.cuda.current_stream().cuda_stream``).
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdictproj.so")

STATUS = {
    0: "DICTPROJ_OK", -1: "DICTPROJ_ERR_NULL", -2: "DICTPROJ_ERR_SHAPE", -3: "DICTPROJ_ERR_ALIGN",
    -4: "DICTPROJ_ERR_MISMATCH", -5: "DICTPROJ_ERR_RANGE", -6: "DICTPROJ_ERR_CUDA",
    -7: "DICTPROJ_ERR_OOM", -8: "DICTPROJ_ERR_TIMEOUT", -9: "DICTPROJ_ERR_UNSUPPORTED",
    -10: "DICTPROJ_ERR_VALUE", -11: "DICTPROJ_ERR_IO",
}
PATH_AUTO, PATH_DECODE, PATH_PREFILL = 0, 1, 2
DECODE_AUTO, DECODE_FUSED, DECODE_SPLIT = 0, 1, 2
IFMT = {"u8": 0, "bitmap": 1, "blocks": 2}
CFMT = {"nvfp4": 0, "fp16": 1, "fp8": 2, "int8": 3}  # DICTPROJ_CFMT_*


class DictprojError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_u8p = C.POINTER(C.c_uint8)
_u16p = C.POINTER(C.c_uint16)
_u32p = C.POINTER(C.c_uint32)
_i32p = C.POINTER(C.c_int32)
_f32p = C.POINTER(C.c_float)
_szp = C.POINTER(C.c_size_t)
_intp = C.POINTER(C.c_int)

class DeviceGroup(C.Structure):
    """dictproj_device_group: caller-owned device copies of a packed D_g."""
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("s", C.c_float), ("d_in", C.c_int),
                ("k", C.c_int)]


class DeviceLayer(C.Structure):
    """dictproj_device_layer: caller-owned device copies of a packed C_l."""
    _fields_ = [("col_ptr", C.c_void_p), ("codes", C.c_void_p), ("scales", C.c_void_p), ("idx", C.c_void_p),
                ("seg_start", C.c_void_p), ("s", C.c_float), ("k", C.c_int), ("d_out", C.c_int)]


# (name, restype, argtypes) for every entry point declared in include/dictproj.h
SIGNATURES = [
    ("dictproj_group_packed_sizes", C.c_int, [C.c_int, C.c_int, _szp, _szp]),
    ("dictproj_pack_group_host", C.c_int, [_f32p, C.c_int, C.c_int, _u8p, _u8p, _f32p]),
    ("dictproj_layer_packed_entries", C.c_int, [_i32p, C.c_int, C.c_int, _szp]),
    ("dictproj_pack_layer_host", C.c_int,
     [_i32p, _i32p, _f32p, C.c_int, C.c_int, _u32p, _u32p, _u8p, _u8p, _u8p, _u16p, _f32p]),
    ("dictproj_pack_layer_bitmap_host", C.c_int,
     [_i32p, _i32p, _f32p, C.c_int, C.c_int, _u32p, _u32p, _u8p, _u8p, _u32p, _f32p]),
    ("dictproj_pack_layer_blocks_host", C.c_int,
     [_i32p, _i32p, _f32p, C.c_int, C.c_int, _u32p, _u16p, _u8p, _u8p, _f32p]),
    ("dictproj_cfmt_value_bytes", C.c_int, [C.c_int]),
    ("dictproj_layer_upload_fmt", C.c_int,
     [_u32p, C.c_void_p, _u8p, _u16p, C.c_float, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_pack_layer_fmt", C.c_int,
     [_i32p, _i32p, _f32p, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_layer_format", C.c_int, [C.c_void_p, _intp]),
    ("dictproj_layer_export_fmt", C.c_int, [C.c_void_p, _u32p, C.c_void_p, _u8p, _u16p, _f32p]),
    ("dictproj_pack_layer_fmt_host", C.c_int,
     [_i32p, _i32p, _f32p, C.c_int, C.c_int, C.c_int, _u32p, _u32p, C.c_void_p, _u8p, _u16p, _f32p]),
    ("dictproj_group_upload", C.c_int,
     [_u8p, _u8p, C.c_float, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_pack_group", C.c_int, [_f32p, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_group_reserve_prefill", C.c_int, [C.c_void_p, C.c_int]),
    ("dictproj_layer_upload", C.c_int,
     [_u32p, _u8p, _u8p, _u8p, _u16p, C.c_float, C.c_int, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_pack_layer", C.c_int, [_i32p, _i32p, _f32p, C.c_int, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_pack", C.c_int,
     [_f32p, C.c_int, C.c_int, C.c_int, C.c_int, C.POINTER(_i32p), C.POINTER(_i32p),
      C.POINTER(_f32p), _intp, C.POINTER(C.c_void_p), C.POINTER(C.c_void_p)]),
    ("dictproj_group_export", C.c_int, [C.c_void_p, _u8p, _u8p, _f32p]),
    ("dictproj_layer_export", C.c_int, [C.c_void_p, _u32p, _u8p, _u8p, _u8p, _u16p, _f32p]),
    ("dictproj_group_info", C.c_int, [C.c_void_p, _intp, _intp, _intp]),
    ("dictproj_layer_info", C.c_int, [C.c_void_p, _intp, _intp, _szp, _szp]),
    ("dictproj_free_group", None, [C.c_void_p]),
    ("dictproj_free_layer", None, [C.c_void_p]),
    ("dictproj_forward", C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    ("dictproj_layer_upload_bitmap", C.c_int,
     [C.POINTER(C.c_uint32), C.POINTER(C.c_uint8), C.POINTER(C.c_uint8), C.POINTER(C.c_uint32), C.c_float, C.c_int,
      C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_pack_layer_bitmap", C.c_int,
     [C.POINTER(C.c_int32), C.POINTER(C.c_int32), C.POINTER(C.c_float), C.c_int, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_layer_upload_blocks", C.c_int,
     [C.POINTER(C.c_uint32), C.POINTER(C.c_uint16), C.POINTER(C.c_uint8), C.POINTER(C.c_uint8), C.c_float, C.c_int,
      C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_pack_layer_blocks", C.c_int,
     [C.POINTER(C.c_int32), C.POINTER(C.c_int32), C.POINTER(C.c_float), C.c_int, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_layer_index_format", C.c_int, [C.c_void_p, _intp]),
    ("dictproj_layer_export_bitmap", C.c_int,
     [C.c_void_p, C.POINTER(C.c_uint32), C.POINTER(C.c_uint8), C.POINTER(C.c_uint8), C.POINTER(C.c_uint32),
      C.POINTER(C.c_float)]),
    ("dictproj_layer_export_blocks", C.c_int,
     [C.c_void_p, C.POINTER(C.c_uint32), C.POINTER(C.c_uint16), C.POINTER(C.c_uint8), C.POINTER(C.c_uint8),
      C.POINTER(C.c_float)]),
    ("dictproj_set_decode_kernels", C.c_int, [C.c_int]),
    ("dictproj_get_decode_kernels", C.c_int, []),
    ("dictproj_forward_path", C.c_int,
     [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int]),
    ("dictproj_forward_batch", C.c_int,
     [C.c_int, C.POINTER(C.c_void_p), C.c_int, C.POINTER(C.c_void_p), C.POINTER(C.c_void_p),
      C.POINTER(C.c_void_p), C.c_void_p]),
    ("dictproj_forward_batch_stages", C.c_int,
     [C.c_int, C.POINTER(C.c_void_p), C.c_int, C.POINTER(C.c_void_p), C.POINTER(C.c_void_p),
      C.POINTER(C.c_void_p), C.c_void_p, C.c_int]),
    ("dictproj_decode_batch_plan", C.c_int,
     [C.c_int, _intp, _intp, _intp, C.POINTER(C.c_longlong), C.c_int, C.c_int, _intp, _intp, _intp]),
    ("dictproj_launch_count", C.c_int,
     [C.c_int, C.POINTER(C.c_void_p), C.c_int, C.POINTER(C.c_void_p), C.POINTER(C.c_void_p), _intp]),
    ("dictproj_dictionary_stage", C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]),
    ("dictproj_coefficient_stage", C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]),
    ("dictproj_dictionary_stage_prefill", C.c_int, [C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]),
    ("dictproj_forward_noalloc", C.c_int,
     [C.POINTER(DeviceGroup), C.POINTER(DeviceLayer), C.c_void_p, C.c_int, C.c_void_p, C.c_void_p]),
    ("dictproj_rank_for_budget", C.c_int, [C.c_double, C.c_int, C.c_int, C.c_int, C.c_int, _intp]),
    ("dictproj_budget", C.c_int, [C.c_int, C.c_int, C.c_int, C.c_int, C.c_double, C.POINTER(C.c_double),
                                  C.POINTER(C.c_double), C.POINTER(C.c_double), C.POINTER(C.c_double)]),
    ("dictproj_group_file_write", C.c_int, [C.c_char_p, _u8p, _u8p, C.c_float, C.c_int, C.c_int]),
    ("dictproj_group_file_info", C.c_int, [C.c_char_p, _intp, _intp]),
    ("dictproj_group_file_read", C.c_int, [C.c_char_p, _u8p, _u8p, _f32p, C.c_int, C.c_int]),
    ("dictproj_layer_file_write", C.c_int, [C.c_char_p, _u32p, _u8p, _u8p, _u8p, _u16p, C.c_float, C.c_int, C.c_int]),
    ("dictproj_layer_file_info", C.c_int, [C.c_char_p, _intp, _intp, _szp]),
    ("dictproj_layer_file_read", C.c_int,
     [C.c_char_p, _u32p, _u8p, _u8p, _u8p, _u16p, _f32p, C.c_int, C.c_int, C.c_size_t]),
    ("dictproj_group_save", C.c_int, [C.c_void_p, C.c_char_p]),
    ("dictproj_group_load", C.c_int, [C.c_char_p, C.c_int, C.POINTER(C.c_void_p)]),
    ("dictproj_layer_save", C.c_int, [C.c_void_p, C.c_char_p]),
    ("dictproj_layer_load", C.c_int, [C.c_char_p, C.POINTER(C.c_void_p)]),
    ("dictproj_check", C.c_int, [C.c_void_p]),
    ("dictproj_selftest_wait_timeout", C.c_int, [C.c_longlong, C.c_void_p]),
    ("dictproj_diag_phase_times", C.c_int, [C.POINTER(C.c_ulonglong), C.c_int, _intp]),
    ("dictproj_diag_gather_times", C.c_int, [C.c_void_p, C.c_int]),
    ("dictproj_last_error", C.c_char_p, []),
    ("dictproj_status_string", C.c_char_p, [C.c_int]),
    ("dictproj_version", C.c_int, []),
]

_lib = None


def lib():
    """Load libdictproj.so (built in-tree). Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m dictionary_compressed_linear_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def dictproj_last_error() -> str:
    return lib().dictproj_last_error().decode()


def dictproj_status_string(status: int) -> str:
    return lib().dictproj_status_string(int(status)).decode()


def dictproj_version() -> int:
    return lib().dictproj_version()


def _check(status: int):
    if status != 0:
        raise DictprojError(status, dictproj_last_error())


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(C.POINTER(ctype))


# ---------------------------------------------------------------- host packing
def dictproj_group_packed_sizes(d_in: int, k: int):
    a, b = C.c_size_t(), C.c_size_t()
    _check(lib().dictproj_group_packed_sizes(d_in, k, C.byref(a), C.byref(b)))
    return a.value, b.value


def dictproj_pack_group_host(D: np.ndarray) -> dict:
    """D: fp32 (d_in, k) C-contiguous. Returns {'codes','scales','s'}."""
    D = np.ascontiguousarray(D, dtype=np.float32)
    d_in, k = D.shape
    nc, ns = dictproj_group_packed_sizes(d_in, k)
    codes = np.zeros(nc, np.uint8)
    scales = np.zeros(ns, np.uint8)
    s = C.c_float()
    _check(lib().dictproj_pack_group_host(_ptr(D, C.c_float), d_in, k, _ptr(codes, C.c_uint8),
                                          _ptr(scales, C.c_uint8), C.byref(s)))
    return {"d_in": d_in, "k": k, "codes": codes, "scales": scales, "s": np.float32(s.value)}


def dictproj_layer_packed_entries(col_ptr: np.ndarray, k: int, d_out: int) -> int:
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    t = C.c_size_t()
    _check(lib().dictproj_layer_packed_entries(_ptr(col_ptr, C.c_int32), k, d_out, C.byref(t)))
    return t.value


def dictproj_pack_layer_host(col_ptr, atom_idx, vals, k: int, d_out: int) -> dict:
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    atom_idx = np.ascontiguousarray(atom_idx, dtype=np.int32)
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    total = dictproj_layer_packed_entries(col_ptr, k, d_out)
    nseg = -(-k // 256)
    out = {
        "col_ptr": np.zeros(d_out + 1, np.uint32), "nnz": np.zeros(d_out, np.uint32),
        "codes": np.zeros(total // 2, np.uint8), "scales": np.zeros(total // 16, np.uint8),
        "idx": np.zeros(total, np.uint8), "seg_start": np.zeros(d_out * nseg, np.uint16),
    }
    s = C.c_float()
    _check(lib().dictproj_pack_layer_host(
        _ptr(col_ptr, C.c_int32), _ptr(atom_idx, C.c_int32), _ptr(vals, C.c_float), k, d_out,
        _ptr(out["col_ptr"], C.c_uint32), _ptr(out["nnz"], C.c_uint32), _ptr(out["codes"], C.c_uint8),
        _ptr(out["scales"], C.c_uint8), _ptr(out["idx"], C.c_uint8), _ptr(out["seg_start"], C.c_uint16),
        C.byref(s)))
    out.update(k=k, d_out=d_out, nseg=nseg, s=np.float32(s.value))
    return out


def dictproj_pack_layer_bitmap_host(col_ptr, atom_idx, vals, k: int, d_out: int) -> dict:
    """C_l with the bitmap support index (Eq. (12), a = 0, h = 1)."""
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    atom_idx = np.ascontiguousarray(atom_idx, dtype=np.int32)
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    total = dictproj_layer_packed_entries(col_ptr, k, d_out)
    words = -(-k // 32)
    out = {
        "col_ptr": np.zeros(d_out + 1, np.uint32), "nnz": np.zeros(d_out, np.uint32),
        "codes": np.zeros(total // 2, np.uint8), "scales": np.zeros(total // 16, np.uint8),
        "bitmap": np.zeros(d_out * words, np.uint32),
    }
    s = C.c_float()
    _check(lib().dictproj_pack_layer_bitmap_host(
        _ptr(col_ptr, C.c_int32), _ptr(atom_idx, C.c_int32), _ptr(vals, C.c_float), k, d_out,
        _ptr(out["col_ptr"], C.c_uint32), _ptr(out["nnz"], C.c_uint32), _ptr(out["codes"], C.c_uint8),
        _ptr(out["scales"], C.c_uint8), _ptr(out["bitmap"], C.c_uint32), C.byref(s)))
    out.update(k=k, d_out=d_out, words=words, s=np.float32(s.value))
    return out


def dictproj_pack_layer_blocks_host(col_ptr, atom_idx, vals, k: int, d_out: int) -> dict:
    """C_l with block-structured support: whole aligned 16-atom blocks per column."""
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    atom_idx = np.ascontiguousarray(atom_idx, dtype=np.int32)
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    nblk = int(col_ptr[-1]) // 16
    out = {"blk_ptr": np.zeros(d_out + 1, np.uint32), "blk_idx": np.zeros(max(nblk, 1), np.uint16),
           "codes": np.zeros(max(nblk, 1) * 8, np.uint8), "scales": np.zeros(max(nblk, 1), np.uint8)}
    s = C.c_float()
    _check(lib().dictproj_pack_layer_blocks_host(
        _ptr(col_ptr, C.c_int32), _ptr(atom_idx, C.c_int32), _ptr(vals, C.c_float), k, d_out,
        _ptr(out["blk_ptr"], C.c_uint32), _ptr(out["blk_idx"], C.c_uint16), _ptr(out["codes"], C.c_uint8),
        _ptr(out["scales"], C.c_uint8), C.byref(s)))
    out["blk_idx"] = out["blk_idx"][:nblk]
    out["codes"] = out["codes"][:nblk * 8]
    out["scales"] = out["scales"][:nblk]
    out.update(k=k, d_out=d_out, s=np.float32(s.value))
    return out


def dictproj_pack_layer_fmt_host(col_ptr, atom_idx, vals, k: int, d_out: int, fmt: str) -> dict:
    """C_l with FP16 / FP8 / INT8 values (Table 4) and the u8 index."""
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    atom_idx = np.ascontiguousarray(atom_idx, dtype=np.int32)
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    total = dictproj_layer_packed_entries(col_ptr, k, d_out)
    nseg = -(-k // 256)
    f = CFMT[fmt]
    vb = lib().dictproj_cfmt_value_bytes(f)
    out = {
        "col_ptr": np.zeros(d_out + 1, np.uint32), "nnz": np.zeros(d_out, np.uint32),
        "values": np.zeros(total, np.uint16 if vb == 2 else np.uint8),
        "idx": np.zeros(total, np.uint8), "seg_start": np.zeros(d_out * nseg, np.uint16),
    }
    s = C.c_float()
    _check(lib().dictproj_pack_layer_fmt_host(
        _ptr(col_ptr, C.c_int32), _ptr(atom_idx, C.c_int32), _ptr(vals, C.c_float), k, d_out, f,
        _ptr(out["col_ptr"], C.c_uint32), _ptr(out["nnz"], C.c_uint32), out["values"].ctypes.data_as(C.c_void_p),
        _ptr(out["idx"], C.c_uint8), _ptr(out["seg_start"], C.c_uint16), C.byref(s)))
    out.update(k=k, d_out=d_out, nseg=nseg, fmt=fmt, s=np.float32(s.value))
    return out


# ---------------------------------------------------------------- budget and packed files
def dictproj_rank_for_budget(rho_fac: float, n: int, d_in: int, d_out: int, align: int = 1) -> int:
    """Eq. (3): dictionary rank for a factorisation reduction rho_fac, rounded down to `align`."""
    k = C.c_int()
    _check(lib().dictproj_rank_for_budget(float(rho_fac), n, d_in, d_out, align, C.byref(k)))
    return k.value


def dictproj_budget(n: int, d_in: int, d_out: int, k: int, p: float) -> dict:
    """Eq. (2): N0, Np, rho, G."""
    v = [C.c_double() for _ in range(4)]
    _check(lib().dictproj_budget(n, d_in, d_out, k, float(p), *[C.byref(x) for x in v]))
    return dict(zip(("N0", "Np", "rho", "G"), [x.value for x in v]))


def dictproj_group_file_write(path: str, packed: dict):
    codes = np.ascontiguousarray(packed["codes"], np.uint8)
    scales = np.ascontiguousarray(packed["scales"], np.uint8)
    _check(lib().dictproj_group_file_write(os.fsencode(path), _ptr(codes, C.c_uint8), _ptr(scales, C.c_uint8),
                                           float(packed["s"]), packed["d_in"], packed["k"]))


def dictproj_group_file_read(path: str) -> dict:
    d_in, k = C.c_int(), C.c_int()
    _check(lib().dictproj_group_file_info(os.fsencode(path), C.byref(d_in), C.byref(k)))
    out = {"codes": np.zeros(d_in.value * k.value // 2, np.uint8),
           "scales": np.zeros(d_in.value * k.value // 16, np.uint8)}
    s = C.c_float()
    _check(lib().dictproj_group_file_read(os.fsencode(path), _ptr(out["codes"], C.c_uint8),
                                          _ptr(out["scales"], C.c_uint8), C.byref(s), d_in.value, k.value))
    out.update(d_in=d_in.value, k=k.value, s=np.float32(s.value))
    return out


def dictproj_layer_file_write(path: str, packed: dict):
    a = {n: np.ascontiguousarray(packed[n]) for n in ("col_ptr", "codes", "scales", "idx", "seg_start")}
    _check(lib().dictproj_layer_file_write(os.fsencode(path), _ptr(a["col_ptr"], C.c_uint32),
                                           _ptr(a["codes"], C.c_uint8), _ptr(a["scales"], C.c_uint8),
                                           _ptr(a["idx"], C.c_uint8), _ptr(a["seg_start"], C.c_uint16),
                                           float(packed["s"]), packed["k"], packed["d_out"]))


def dictproj_layer_file_read(path: str) -> dict:
    k, d_out, total = C.c_int(), C.c_int(), C.c_size_t()
    _check(lib().dictproj_layer_file_info(os.fsencode(path), C.byref(k), C.byref(d_out), C.byref(total)))
    K, O, T = k.value, d_out.value, total.value
    nseg = -(-K // 256)
    out = {"col_ptr": np.zeros(O + 1, np.uint32), "codes": np.zeros(T // 2, np.uint8),
           "scales": np.zeros(T // 16, np.uint8), "idx": np.zeros(T, np.uint8),
           "seg_start": np.zeros(O * nseg, np.uint16)}
    s = C.c_float()
    _check(lib().dictproj_layer_file_read(os.fsencode(path), _ptr(out["col_ptr"], C.c_uint32),
                                          _ptr(out["codes"], C.c_uint8), _ptr(out["scales"], C.c_uint8),
                                          _ptr(out["idx"], C.c_uint8), _ptr(out["seg_start"], C.c_uint16),
                                          C.byref(s), K, O, T))
    out.update(k=K, d_out=O, nseg=nseg, s=np.float32(s.value))
    return out


# ---------------------------------------------------------------- device objects
class Group:
    """Owns a dictproj_group handle (packed D_g + Z scratch on the device)."""

    def __init__(self, handle: int, d_in: int, k: int, max_tokens: int):
        self.handle, self.d_in, self.k, self.max_tokens = handle, d_in, k, max_tokens

    def free(self):
        if self.handle:
            lib().dictproj_free_group(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


class Layer:
    """Owns a dictproj_layer handle (packed C_l on the device)."""

    def __init__(self, handle: int, k: int, d_out: int):
        self.handle, self.k, self.d_out = handle, k, d_out

    def free(self):
        if self.handle:
            lib().dictproj_free_layer(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def dictproj_group_upload(packed: dict, max_tokens: int) -> Group:
    h = C.c_void_p()
    codes = np.ascontiguousarray(packed["codes"], np.uint8)
    scales = np.ascontiguousarray(packed["scales"], np.uint8)
    _check(lib().dictproj_group_upload(_ptr(codes, C.c_uint8), _ptr(scales, C.c_uint8),
                                       float(packed["s"]), packed["d_in"], packed["k"], max_tokens,
                                       C.byref(h)))
    return Group(h.value, packed["d_in"], packed["k"], max_tokens)


def dictproj_pack_group(D: np.ndarray, max_tokens: int) -> Group:
    D = np.ascontiguousarray(D, dtype=np.float32)
    h = C.c_void_p()
    _check(lib().dictproj_pack_group(_ptr(D, C.c_float), D.shape[0], D.shape[1], max_tokens, C.byref(h)))
    return Group(h.value, D.shape[0], D.shape[1], max_tokens)


def dictproj_layer_upload(packed: dict) -> Layer:
    h = C.c_void_p()
    a = {n: np.ascontiguousarray(packed[n]) for n in ("col_ptr", "codes", "scales", "idx", "seg_start")}
    _check(lib().dictproj_layer_upload(_ptr(a["col_ptr"], C.c_uint32), _ptr(a["codes"], C.c_uint8),
                                       _ptr(a["scales"], C.c_uint8), _ptr(a["idx"], C.c_uint8),
                                       _ptr(a["seg_start"], C.c_uint16), float(packed["s"]),
                                       packed["k"], packed["d_out"], C.byref(h)))
    return Layer(h.value, packed["k"], packed["d_out"])


def dictproj_pack_layer(col_ptr, atom_idx, vals, k: int, d_out: int) -> Layer:
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    atom_idx = np.ascontiguousarray(atom_idx, dtype=np.int32)
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    h = C.c_void_p()
    _check(lib().dictproj_pack_layer(_ptr(col_ptr, C.c_int32), _ptr(atom_idx, C.c_int32),
                                     _ptr(vals, C.c_float), k, d_out, C.byref(h)))
    return Layer(h.value, k, d_out)


def dictproj_layer_upload_fmt(packed: dict) -> Layer:
    """Upload a layer packed by dictproj_pack_layer_fmt_host (FP16 / FP8 / INT8 values)."""
    h = C.c_void_p()
    a = {n: np.ascontiguousarray(packed[n]) for n in ("col_ptr", "values", "idx", "seg_start")}
    _check(lib().dictproj_layer_upload_fmt(_ptr(a["col_ptr"], C.c_uint32), a["values"].ctypes.data_as(C.c_void_p),
                                           _ptr(a["idx"], C.c_uint8), _ptr(a["seg_start"], C.c_uint16),
                                           float(packed["s"]), packed["k"], packed["d_out"], CFMT[packed["fmt"]],
                                           C.byref(h)))
    return Layer(h.value, packed["k"], packed["d_out"])


def dictproj_pack_layer_fmt(col_ptr, atom_idx, vals, k: int, d_out: int, fmt: str) -> Layer:
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    atom_idx = np.ascontiguousarray(atom_idx, dtype=np.int32)
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    h = C.c_void_p()
    _check(lib().dictproj_pack_layer_fmt(_ptr(col_ptr, C.c_int32), _ptr(atom_idx, C.c_int32),
                                         _ptr(vals, C.c_float), k, d_out, CFMT[fmt], C.byref(h)))
    return Layer(h.value, k, d_out)


def dictproj_layer_format(layer: Layer) -> str:
    f = C.c_int()
    _check(lib().dictproj_layer_format(layer.handle, C.byref(f)))
    return {v: k for k, v in CFMT.items()}[f.value]


def dictproj_layer_export_fmt(layer: Layer) -> dict:
    k, d_out = layer.k, layer.d_out
    t, n = C.c_size_t(), C.c_size_t()
    _check(lib().dictproj_layer_info(layer.handle, None, None, C.byref(t), C.byref(n)))
    fmt = dictproj_layer_format(layer)
    vb = lib().dictproj_cfmt_value_bytes(CFMT[fmt])
    nseg = -(-k // 256)
    out = {"col_ptr": np.zeros(d_out + 1, np.uint32), "values": np.zeros(t.value, np.uint16 if vb == 2 else np.uint8),
           "idx": np.zeros(t.value, np.uint8), "seg_start": np.zeros(d_out * nseg, np.uint16)}
    s = C.c_float()
    _check(lib().dictproj_layer_export_fmt(layer.handle, _ptr(out["col_ptr"], C.c_uint32),
                                           out["values"].ctypes.data_as(C.c_void_p), _ptr(out["idx"], C.c_uint8),
                                           _ptr(out["seg_start"], C.c_uint16), C.byref(s)))
    out.update(k=k, d_out=d_out, nseg=nseg, fmt=fmt, s=np.float32(s.value))
    return out


def dictproj_layer_upload_bitmap(packed: dict) -> Layer:
    """Upload a layer packed by dictproj_pack_layer_bitmap_host."""
    h = C.c_void_p()
    a = {n: np.ascontiguousarray(packed[n]) for n in ("col_ptr", "codes", "scales", "bitmap")}
    _check(lib().dictproj_layer_upload_bitmap(_ptr(a["col_ptr"], C.c_uint32), _ptr(a["codes"], C.c_uint8),
                                              _ptr(a["scales"], C.c_uint8), _ptr(a["bitmap"], C.c_uint32),
                                              float(packed["s"]), packed["k"], packed["d_out"], C.byref(h)))
    return Layer(h.value, packed["k"], packed["d_out"])


def dictproj_pack_layer_bitmap(col_ptr, atom_idx, vals, k: int, d_out: int) -> Layer:
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    atom_idx = np.ascontiguousarray(atom_idx, dtype=np.int32)
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    h = C.c_void_p()
    _check(lib().dictproj_pack_layer_bitmap(_ptr(col_ptr, C.c_int32), _ptr(atom_idx, C.c_int32),
                                            _ptr(vals, C.c_float), k, d_out, C.byref(h)))
    return Layer(h.value, k, d_out)


def dictproj_layer_upload_blocks(packed: dict) -> Layer:
    """Upload a layer packed by dictproj_pack_layer_blocks_host."""
    h = C.c_void_p()
    a = {n: np.ascontiguousarray(packed[n]) for n in ("blk_ptr", "blk_idx", "codes", "scales")}
    blk_idx = a["blk_idx"] if a["blk_idx"].size else np.zeros(1, np.uint16)
    codes = a["codes"] if a["codes"].size else np.zeros(8, np.uint8)
    scales = a["scales"] if a["scales"].size else np.zeros(1, np.uint8)
    _check(lib().dictproj_layer_upload_blocks(_ptr(a["blk_ptr"], C.c_uint32), _ptr(blk_idx, C.c_uint16),
                                              _ptr(codes, C.c_uint8), _ptr(scales, C.c_uint8), float(packed["s"]),
                                              packed["k"], packed["d_out"], C.byref(h)))
    return Layer(h.value, packed["k"], packed["d_out"])


def dictproj_pack_layer_blocks(col_ptr, atom_idx, vals, k: int, d_out: int) -> Layer:
    col_ptr = np.ascontiguousarray(col_ptr, dtype=np.int32)
    atom_idx = np.ascontiguousarray(atom_idx, dtype=np.int32)
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    h = C.c_void_p()
    _check(lib().dictproj_pack_layer_blocks(_ptr(col_ptr, C.c_int32), _ptr(atom_idx, C.c_int32),
                                            _ptr(vals, C.c_float), k, d_out, C.byref(h)))
    return Layer(h.value, k, d_out)


def dictproj_layer_index_format(layer: Layer) -> str:
    f = C.c_int()
    _check(lib().dictproj_layer_index_format(layer.handle, C.byref(f)))
    return {v: k for k, v in IFMT.items()}[f.value]


def dictproj_layer_export_bitmap(layer: Layer) -> dict:
    k, d_out = layer.k, layer.d_out
    t = C.c_size_t()
    _check(lib().dictproj_layer_info(layer.handle, None, None, C.byref(t), None))
    words = -(-k // 32)
    out = {"col_ptr": np.zeros(d_out + 1, np.uint32), "codes": np.zeros(t.value // 2, np.uint8),
           "scales": np.zeros(t.value // 16, np.uint8), "bitmap": np.zeros(d_out * words, np.uint32)}
    s = C.c_float()
    _check(lib().dictproj_layer_export_bitmap(layer.handle, _ptr(out["col_ptr"], C.c_uint32),
                                              _ptr(out["codes"], C.c_uint8), _ptr(out["scales"], C.c_uint8),
                                              _ptr(out["bitmap"], C.c_uint32), C.byref(s)))
    out.update(k=k, d_out=d_out, words=words, s=np.float32(s.value))
    return out


def dictproj_layer_export_blocks(layer: Layer) -> dict:
    k, d_out = layer.k, layer.d_out
    t = C.c_size_t()
    _check(lib().dictproj_layer_info(layer.handle, None, None, C.byref(t), None))
    nblk = t.value // 16
    out = {"blk_ptr": np.zeros(d_out + 1, np.uint32), "blk_idx": np.zeros(max(nblk, 1), np.uint16),
           "codes": np.zeros(max(nblk, 1) * 8, np.uint8), "scales": np.zeros(max(nblk, 1), np.uint8)}
    s = C.c_float()
    _check(lib().dictproj_layer_export_blocks(layer.handle, _ptr(out["blk_ptr"], C.c_uint32),
                                              _ptr(out["blk_idx"], C.c_uint16), _ptr(out["codes"], C.c_uint8),
                                              _ptr(out["scales"], C.c_uint8), C.byref(s)))
    out["blk_idx"] = out["blk_idx"][:nblk]
    out["codes"] = out["codes"][:nblk * 8]
    out["scales"] = out["scales"][:nblk]
    out.update(k=k, d_out=d_out, s=np.float32(s.value))
    return out


def dictproj_pack(D, max_tokens: int, layers) -> tuple:
    """layers: list of (col_ptr, atom_idx, vals, d_out). Returns (Group, [Layer])."""
    D = np.ascontiguousarray(D, dtype=np.float32)
    d_in, k = D.shape
    n = len(layers)
    keep = [(np.ascontiguousarray(c, np.int32), np.ascontiguousarray(a, np.int32),
             np.ascontiguousarray(v, np.float32)) for c, a, v, _ in layers]
    cp = (_i32p * n)(*[_ptr(c, C.c_int32) for c, _, _ in keep])
    ai = (_i32p * n)(*[_ptr(a, C.c_int32) for _, a, _ in keep])
    vv = (_f32p * n)(*[_ptr(v, C.c_float) for _, _, v in keep])
    do = (C.c_int * n)(*[int(d) for *_, d in layers])
    gh = C.c_void_p()
    lh = (C.c_void_p * n)()
    _check(lib().dictproj_pack(_ptr(D, C.c_float), d_in, k, max_tokens, n, cp, ai, vv, do,
                               C.byref(gh), lh))
    return Group(gh.value, d_in, k, max_tokens), [Layer(lh[i], k, layers[i][3]) for i in range(n)]


def dictproj_group_export(g: Group) -> dict:
    nc, ns = dictproj_group_packed_sizes(g.d_in, g.k)
    codes, scales, s = np.zeros(nc, np.uint8), np.zeros(ns, np.uint8), C.c_float()
    _check(lib().dictproj_group_export(g.handle, _ptr(codes, C.c_uint8), _ptr(scales, C.c_uint8),
                                       C.byref(s)))
    return {"d_in": g.d_in, "k": g.k, "codes": codes, "scales": scales, "s": np.float32(s.value)}


def dictproj_layer_info(l: Layer) -> dict:
    k, d_out, t, nz = C.c_int(), C.c_int(), C.c_size_t(), C.c_size_t()
    _check(lib().dictproj_layer_info(l.handle, C.byref(k), C.byref(d_out), C.byref(t), C.byref(nz)))
    return {"k": k.value, "d_out": d_out.value, "total": t.value, "nnz_total": nz.value}


def dictproj_group_info(g: Group) -> dict:
    d_in, k, mt = C.c_int(), C.c_int(), C.c_int()
    _check(lib().dictproj_group_info(g.handle, C.byref(d_in), C.byref(k), C.byref(mt)))
    return {"d_in": d_in.value, "k": k.value, "max_tokens": mt.value}


def dictproj_layer_export(l: Layer) -> dict:
    info = dictproj_layer_info(l)
    T, d_out, k = info["total"], l.d_out, l.k
    nseg = -(-k // 256)
    out = {"col_ptr": np.zeros(d_out + 1, np.uint32), "codes": np.zeros(T // 2, np.uint8),
           "scales": np.zeros(T // 16, np.uint8), "idx": np.zeros(T, np.uint8),
           "seg_start": np.zeros(d_out * nseg, np.uint16)}
    s = C.c_float()
    _check(lib().dictproj_layer_export(l.handle, _ptr(out["col_ptr"], C.c_uint32), _ptr(out["codes"], C.c_uint8),
                                       _ptr(out["scales"], C.c_uint8), _ptr(out["idx"], C.c_uint8),
                                       _ptr(out["seg_start"], C.c_uint16), C.byref(s)))
    out.update(k=k, d_out=d_out, nseg=nseg, s=np.float32(s.value))
    return out


# ---------------------------------------------------------------- forward
def dictproj_forward(X_ptr: int, M: int, layer: Layer, group: Group, Y_ptr: int, stream: int = 0):
    _check(lib().dictproj_forward(C.c_void_p(X_ptr), M, layer.handle, group.handle, C.c_void_p(Y_ptr),
                                  C.c_void_p(stream)))


def dictproj_set_decode_kernels(which: int) -> None:
    """Process-wide choice of decode kernels: DECODE_AUTO, DECODE_FUSED or DECODE_SPLIT."""
    _check(lib().dictproj_set_decode_kernels(which))


def dictproj_get_decode_kernels() -> int:
    return int(lib().dictproj_get_decode_kernels())


def dictproj_forward_path(X_ptr: int, M: int, layer: Layer, group: Group, Y_ptr: int, stream: int = 0,
                          path: int = PATH_AUTO):
    _check(lib().dictproj_forward_path(C.c_void_p(X_ptr), M, layer.handle, group.handle,
                                       C.c_void_p(Y_ptr), C.c_void_p(stream), path))


def dictproj_forward_status(X_ptr, M, layer_handle, group_handle, Y_ptr, stream=0, path=PATH_AUTO) -> int:
    """Raw status of a forward call (no exception), for boundary tests."""
    return lib().dictproj_forward_path(C.c_void_p(X_ptr), M, layer_handle, group_handle,
                                       C.c_void_p(Y_ptr), C.c_void_p(stream), path)


def dictproj_forward_batch(X_ptrs, M: int, layers, groups, Y_ptrs, stream: int = 0):
    """Independent projections in one call (lists of equal length <= 4)."""
    n = len(layers)
    arr = lambda vals: (C.c_void_p * n)(*[C.c_void_p(v) for v in vals])
    _check(lib().dictproj_forward_batch(n, arr(X_ptrs), M, arr([l.handle for l in layers]),
                                        arr([g.handle for g in groups]), arr(Y_ptrs), C.c_void_p(stream)))


def dictproj_forward_batch_stages(X_ptrs, M: int, layers, groups, Y_ptrs, stream: int = 0, stages: int = 3):
    """dictproj_forward_batch launching only the stage kernels in the mask
    (1 dictionary, 2 coefficient, 3 both) of the two-kernel decode path."""
    n = len(layers)
    arr = lambda vals: (C.c_void_p * n)(*[C.c_void_p(v) for v in vals])
    _check(lib().dictproj_forward_batch_stages(n, arr(X_ptrs), M, arr([l.handle for l in layers]),
                                               arr([g.handle for g in groups]), arr(Y_ptrs), C.c_void_p(stream),
                                               stages))


def dictproj_decode_batch_plan(shapes, M: int, n_sm: int):
    """Grid of a batched two-kernel decode call, host only. shapes: list of
    (d_in, k, d_out, stored entries). Returns a list of dicts with dict_ctas,
    dict_slices and coeff_ctas per projection."""
    n = len(shapes)
    ints = lambda j: (C.c_int * n)(*[int(sh[j]) for sh in shapes])
    ent = (C.c_longlong * n)(*[int(sh[3]) for sh in shapes])
    dc, ds, cc = (C.c_int * n)(), (C.c_int * n)(), (C.c_int * n)()
    _check(lib().dictproj_decode_batch_plan(n, ints(0), ints(1), ints(2), ent, M, n_sm, dc, ds, cc))
    return [{"dict_ctas": dc[i], "dict_slices": ds[i], "coeff_ctas": cc[i]} for i in range(n)]


def dictproj_group_save(group: "Group", path: str):
    _check(lib().dictproj_group_save(group.handle, os.fsencode(path)))


def dictproj_group_load(path: str, max_tokens: int) -> "Group":
    h = C.c_void_p()
    _check(lib().dictproj_group_load(os.fsencode(path), max_tokens, C.byref(h)))
    d_in, k, mt = C.c_int(), C.c_int(), C.c_int()
    _check(lib().dictproj_group_info(h.value, C.byref(d_in), C.byref(k), C.byref(mt)))
    return Group(h.value, d_in.value, k.value, mt.value)


def dictproj_layer_save(layer: "Layer", path: str):
    _check(lib().dictproj_layer_save(layer.handle, os.fsencode(path)))


def dictproj_layer_load(path: str) -> "Layer":
    h = C.c_void_p()
    _check(lib().dictproj_layer_load(os.fsencode(path), C.byref(h)))
    k, d_out = C.c_int(), C.c_int()
    _check(lib().dictproj_layer_info(h.value, C.byref(k), C.byref(d_out), None, None))
    return Layer(h.value, k.value, d_out.value)


def dictproj_dictionary_stage(X_ptr: int, M: int, group: Group, Z_ptr: int, stream: int = 0):
    _check(lib().dictproj_dictionary_stage(C.c_void_p(X_ptr), M, group.handle, C.c_void_p(Z_ptr),
                                           C.c_void_p(stream)))


def dictproj_dictionary_stage_prefill(X_ptr: int, M: int, group: Group, Z_ptr: int, stream: int = 0):
    """Z (device fp16 [M][k]) = s_D X D_g on the tensor cores."""
    _check(lib().dictproj_dictionary_stage_prefill(C.c_void_p(X_ptr), M, group.handle, C.c_void_p(Z_ptr),
                                                   C.c_void_p(stream)))


def dictproj_group_reserve_prefill(group: Group, max_d_out: int):
    """Reserve the group's prefill coefficient scratch for layers with up to max_d_out columns."""
    _check(lib().dictproj_group_reserve_prefill(group.handle, max_d_out))


def dictproj_coefficient_stage(Z_ptr: int, M: int, layer: Layer, Y_ptr: int, stream: int = 0):
    _check(lib().dictproj_coefficient_stage(C.c_void_p(Z_ptr), M, layer.handle, C.c_void_p(Y_ptr),
                                            C.c_void_p(stream)))


def dictproj_forward_noalloc(group: DeviceGroup, layer: DeviceLayer, X_ptr: int, M: int, Y_ptr: int,
                             stream: int = 0):
    _check(lib().dictproj_forward_noalloc(C.byref(group), C.byref(layer), C.c_void_p(X_ptr), M,
                                          C.c_void_p(Y_ptr), C.c_void_p(stream)))


def dictproj_forward_noalloc_status(group: DeviceGroup, layer: DeviceLayer, X_ptr: int, M: int, Y_ptr: int,
                                    stream: int = 0) -> int:
    """Raw status of a no-allocation forward (no exception)."""
    return lib().dictproj_forward_noalloc(C.byref(group), C.byref(layer), C.c_void_p(X_ptr), M,
                                          C.c_void_p(Y_ptr), C.c_void_p(stream))


def dictproj_check(stream: int = 0):
    _check(lib().dictproj_check(C.c_void_p(stream)))


def dictproj_check_status(stream: int = 0) -> int:
    """dictproj_check without raising: the status code."""
    return lib().dictproj_check(C.c_void_p(stream))


def dictproj_selftest_wait_timeout(cycles: int, stream: int = 0):
    _check(lib().dictproj_selftest_wait_timeout(int(cycles), C.c_void_p(stream)))


def dictproj_launch_count(X_ptrs, M: int, layers, groups) -> int:
    """Kernels one forward call (a batch of len(layers) projections) launches."""
    n = len(layers)
    arr = C.c_void_p * n
    cnt = C.c_int()
    _check(lib().dictproj_launch_count(n, arr(*[C.c_void_p(int(x)) for x in X_ptrs]), M,
                                       arr(*[l.handle for l in layers]), arr(*[g.handle for g in groups]),
                                       C.byref(cnt)))
    return cnt.value


def dictproj_diag_gather_times(buf_ptr: int, max_ctas: int):
    """Arm (device buffer of 2 * max_ctas u64) or disarm (buf_ptr 0) the gather
    kernel's per-CTA start / end timestamps."""
    _check(lib().dictproj_diag_gather_times(C.c_void_p(buf_ptr or None), max_ctas))


def dictproj_diag_phase_times(max_ctas: int = 1024) -> np.ndarray:
    """Phase marks (ns) of the last fused decode launch, shape (ctas, 16)."""
    out = np.zeros(max_ctas * 16, np.uint64)
    n = C.c_int()
    _check(lib().dictproj_diag_phase_times(out.ctypes.data_as(C.POINTER(C.c_ulonglong)), max_ctas, C.byref(n)))
    return out[:n.value * 16].reshape(n.value, 16)
