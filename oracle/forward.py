"""fp64 forward of the dictionary-compressed projection (TEST INFRASTRUCTURE).

Follows Eq. (1) of the technical review ("Prerequisites: projections, rank and
calibration"): rows of X are tokens, W_l is d_in x d_out,

    W_l ~= D_g C_l,   Z_l = X_l D_g,   Y_l ~= Z_l C_l.

Both factors are decoded from their packed NVFP4 bytes by table lookup over all
16 E2M1 codes and the E4M3 scale codes; every product and sum is fp64.  The
GPU path computes the same quantity; its only differences are fp16 X / Y,
fp32 accumulation and, at prefill, an fp16 Z.
"""
from __future__ import annotations

import numpy as np

from .nvfp4 import E2M1_TABLE, E4M3_TABLE
from .pack import SEG, coeff_entry_atoms, unpack_nibbles


def decode_dictionary(pd: dict) -> np.ndarray:
    """D-hat as fp64, shape (d_in, k)."""
    d_in, k = pd["d_in"], pd["k"]
    codes = unpack_nibbles(pd["codes"]).reshape(k, d_in)
    sc = np.asarray(pd["scales"]).reshape(k, d_in // 16)
    vals = E2M1_TABLE[codes] * np.repeat(E4M3_TABLE[sc], 16, axis=1) * float(pd["s"])
    return np.ascontiguousarray(vals.T)


def decode_coeff_entries(pc: dict):
    """(atoms int64, values fp64) of every stored entry, padding included."""
    codes = unpack_nibbles(pc["codes"])
    sc = np.repeat(np.asarray(pc["scales"]), 16)
    vals = E2M1_TABLE[codes] * E4M3_TABLE[sc] * float(pc["s"])
    return coeff_entry_atoms(pc), vals


def decode_coeff_bitmap_entries(pb: dict):
    """(atoms int64, values fp64) of the stored entries of a bitmap-indexed C_l;
    padding entries (no bit) get atom -1 and value 0."""
    from .pack import bitmap_entry_atoms
    codes = unpack_nibbles(pb["codes"])
    sc = np.repeat(np.asarray(pb["scales"]), 16)
    vals = E2M1_TABLE[codes] * E4M3_TABLE[sc] * float(pb["s"])
    atoms = bitmap_entry_atoms(pb)
    return atoms, np.where(atoms >= 0, vals, 0.0)


def forward_factored_bitmap(X: np.ndarray, pd: dict, pb: dict) -> np.ndarray:
    """(X D) C in fp64 with C in the bitmap index format: Y[:, o] = sum over the
    column's set bits j, in order, of Z[:, j] times the j-th stored value."""
    Z = np.asarray(X).astype(np.float64) @ decode_dictionary(pd)
    atoms, vals = decode_coeff_bitmap_entries(pb)
    ptr = pb["col_ptr"].astype(np.int64)
    Y = np.zeros((Z.shape[0], pb["d_out"]), dtype=np.float64)
    for o in range(pb["d_out"]):
        a = atoms[ptr[o]:ptr[o + 1]]
        v = vals[ptr[o]:ptr[o + 1]]
        keep = a >= 0
        Y[:, o] = Z[:, a[keep]] @ v[keep]
    return Y


def decode_coeff_fmt_entries(pf: dict):
    """(atoms, values fp64) of every stored entry of a C_l packed by
    pack_coeff_fmt (any of Table 4's coefficient formats)."""
    from . import valuefmt as VF
    fmt = pf.get("fmt", "nvfp4")
    if fmt == "nvfp4":
        return decode_coeff_entries(pf)
    if fmt == "fp16":
        vals = VF.fp16_decode(pf["values"])
    elif fmt == "fp8":
        vals = VF.fp8_decode(pf["values"], pf["s"])
    else:
        vals = VF.int8_decode(pf["values"].view(np.int8), pf["s"])
    return coeff_entry_atoms(pf), vals


def forward_factored_fmt(X: np.ndarray, pd: dict, pf: dict) -> np.ndarray:
    """(X D) C in fp64 with NVFP4 D and C in any of Table 4's formats."""
    Z = np.asarray(X).astype(np.float64) @ decode_dictionary(pd)
    atoms, vals = decode_coeff_fmt_entries(pf)
    ptr = pf["col_ptr"].astype(np.int64)
    Y = np.zeros((Z.shape[0], pf["d_out"]), dtype=np.float64)
    contrib = Z[:, atoms] * vals[None, :]
    nonempty = np.flatnonzero(np.diff(ptr) > 0)
    if nonempty.size:
        Y[:, nonempty] = np.add.reduceat(contrib, ptr[nonempty], axis=1)
    return Y


def decode_coeff_block_entries(pk: dict):
    """(atoms, values fp64) of every stored entry of a block-structured C_l:
    entry 16 b + i is atom 16 * blk_idx[b] + i."""
    codes = unpack_nibbles(pk["codes"])
    sc = np.repeat(np.asarray(pk["scales"]), 16)
    vals = E2M1_TABLE[codes] * E4M3_TABLE[sc] * float(pk["s"])
    atoms = (pk["blk_idx"].astype(np.int64)[:, None] * 16 + np.arange(16)).reshape(-1)
    return atoms, vals


def forward_factored_blocks(X: np.ndarray, pd: dict, pk: dict) -> np.ndarray:
    """(X D) C in fp64 with a block-structured C_l."""
    Z = np.asarray(X).astype(np.float64) @ decode_dictionary(pd)
    atoms, vals = decode_coeff_block_entries(pk)
    ptr = pk["blk_ptr"].astype(np.int64) * 16
    Y = np.zeros((Z.shape[0], pk["d_out"]), dtype=np.float64)
    contrib = Z[:, atoms] * vals[None, :]
    nonempty = np.flatnonzero(np.diff(ptr) > 0)
    if nonempty.size:
        Y[:, nonempty] = np.add.reduceat(contrib, ptr[nonempty], axis=1)
    return Y


def decode_coeff_dense(pc: dict) -> np.ndarray:
    """C-hat as a dense fp64 (k, d_out) matrix, zeros off the support."""
    k, d_out = pc["k"], pc["d_out"]
    atoms, vals = decode_coeff_entries(pc)
    ptr = pc["col_ptr"].astype(np.int64)
    cols = np.repeat(np.arange(d_out), np.diff(ptr))
    C = np.zeros((k, d_out), dtype=np.float64)
    np.add.at(C, (atoms, cols), vals)  # padding entries add exact zeros
    return C


def expand_weight(Dhat: np.ndarray, Chat: np.ndarray) -> np.ndarray:
    """W = D C (fp64), the weight the factorisation stands for."""
    return np.asarray(Dhat, np.float64) @ np.asarray(Chat, np.float64)


def forward_dense(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Y = X W with X converted exactly from fp16 to fp64."""
    return np.asarray(X).astype(np.float64) @ W


def sparse_columns_product(Z: np.ndarray, pc: dict) -> np.ndarray:
    """Y[:, o] = sum over the stored entries q of column o of Z[:, atom_q] * c_q.

    Written directly from the column-compressed definition (no sparse-library
    call): gather the Z columns of every entry, scale, and sum per column."""
    atoms, vals = decode_coeff_entries(pc)
    ptr = pc["col_ptr"].astype(np.int64)
    Z = np.asarray(Z, np.float64)
    M = Z.shape[0]
    d_out = pc["d_out"]
    Y = np.zeros((M, d_out), dtype=np.float64)
    contrib = Z[:, atoms] * vals[None, :]
    nonempty = np.flatnonzero(np.diff(ptr) > 0)
    if nonempty.size:
        Y[:, nonempty] = np.add.reduceat(contrib, ptr[nonempty], axis=1)
    return Y


def forward_factored(X: np.ndarray, pd: dict, pc: dict) -> np.ndarray:
    """(X D) C in fp64: the two-stage order of Eq. (1)."""
    Z = np.asarray(X).astype(np.float64) @ decode_dictionary(pd)
    return sparse_columns_product(Z, pc)


def decode_projection(pd: dict, pc: dict) -> dict:
    """Both factors decoded once: D-hat (d_in, k) and C's entries (atoms, values)."""
    atoms, vals = decode_coeff_entries(pc)
    return {"Dhat": decode_dictionary(pd), "atoms": atoms, "vals": vals,
            "ptr": pc["col_ptr"].astype(np.int64), "d_out": pc["d_out"]}


def forward_factored_decoded(X: np.ndarray, dec: dict) -> np.ndarray:
    """(X D) C in fp64 on factors already decoded by decode_projection."""
    Z = np.asarray(X).astype(np.float64) @ dec["Dhat"]
    ptr = dec["ptr"]
    Y = np.zeros((Z.shape[0], dec["d_out"]), dtype=np.float64)
    contrib = Z[:, dec["atoms"]] * dec["vals"][None, :]
    nonempty = np.flatnonzero(np.diff(ptr) > 0)
    if nonempty.size:
        Y[:, nonempty] = np.add.reduceat(contrib, ptr[nonempty], axis=1)
    return Y


def forward_reference(X: np.ndarray, pd: dict, pc: dict) -> np.ndarray:
    """X (D C) in fp64: decode both factors, expand W densely, multiply."""
    W = expand_weight(decode_dictionary(pd), decode_coeff_dense(pc))
    return forward_dense(X, W)


def forward_brute(X, Dhat, Chat) -> np.ndarray:
    """Triple loop Y[m,o] = sum_j (sum_i X[m,i] D[i,j]) C[j,o]; tiny inputs only."""
    X = np.asarray(X).astype(np.float64)
    M, d_in = X.shape
    k, d_out = np.asarray(Chat).shape
    Y = np.zeros((M, d_out))
    for m in range(M):
        z = [0.0] * k
        for j in range(k):
            acc = 0.0
            for i in range(d_in):
                acc += float(X[m, i]) * float(Dhat[i, j])
            z[j] = acc
        for o in range(d_out):
            acc = 0.0
            for j in range(k):
                c = float(Chat[j, o])
                if c != 0.0:
                    acc += z[j] * c
            Y[m, o] = acc
    return Y


def sampled_outputs(X: np.ndarray, pd: dict, pc: dict, rows, cols) -> np.ndarray:
    """Y[rows, cols] one by one (for full-size parity on sampled outputs)."""
    Dhat = decode_dictionary(pd)
    atoms, vals = decode_coeff_entries(pc)
    ptr = pc["col_ptr"].astype(np.int64)
    X64 = np.asarray(X).astype(np.float64)
    out = np.zeros(len(rows))
    for n, (m, o) in enumerate(zip(rows, cols)):
        a = atoms[ptr[o]:ptr[o + 1]]
        v = vals[ptr[o]:ptr[o + 1]]
        z = X64[m] @ Dhat[:, a]
        out[n] = float(z @ v)
    return out


def sampled_outputs_rows(X: np.ndarray, pd: dict, pc: dict, rows, cols) -> np.ndarray:
    """Y[rows, cols] in the two-stage order of Eq. (1), restricted to what the
    samples need: Z = X[r] D-hat for each distinct sampled token row r (fp64),
    then for each sample the column's stored entries, sum of Z[r, atom] * value."""
    rows = np.asarray(rows, np.int64)
    cols = np.asarray(cols, np.int64)
    Dhat = decode_dictionary(pd)
    atoms, vals = decode_coeff_entries(pc)
    ptr = pc["col_ptr"].astype(np.int64)
    urows, inv = np.unique(rows, return_inverse=True)
    Z = np.asarray(X)[urows].astype(np.float64) @ Dhat
    out = np.zeros(rows.size)
    for n in range(rows.size):
        o = cols[n]
        a = atoms[ptr[o]:ptr[o + 1]]
        v = vals[ptr[o]:ptr[o + 1]]
        out[n] = float(Z[inv[n], a] @ v)
    return out


def within_tolerance(y_test: np.ndarray, y_ref: np.ndarray, rel_fro: float = 5e-3,
                     elem: float = 1e-2):
    """The parity bar: relative Frobenius error <= 5e-3 and every element
    |err| <= 1e-2 * (1 + |y|).  Returns (ok, rel_fro_err, worst_elem_ratio)."""
    y_test = np.asarray(y_test, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    if y_test.shape != y_ref.shape:
        return False, float("inf"), float("inf")
    if not np.all(np.isfinite(y_test)):
        return False, float("inf"), float("inf")
    err = y_test - y_ref
    den = np.linalg.norm(y_ref)
    rf = float(np.linalg.norm(err) / den) if den > 0 else float(np.linalg.norm(err))
    ratio = np.abs(err) / (elem * (1.0 + np.abs(y_ref)))
    worst = float(ratio.max()) if ratio.size else 0.0
    return (rf <= rel_fro and worst <= 1.0), rf, worst


__all__ = [
    "SEG", "decode_dictionary", "decode_coeff_entries", "decode_coeff_dense", "expand_weight",
    "forward_dense", "sparse_columns_product", "forward_factored", "forward_reference",
    "forward_brute", "sampled_outputs", "sampled_outputs_rows", "within_tolerance", "decode_projection",
    "forward_factored_decoded", "decode_coeff_bitmap_entries", "forward_factored_bitmap",
    "decode_coeff_fmt_entries", "forward_factored_fmt", "decode_coeff_block_entries", "forward_factored_blocks",
]
