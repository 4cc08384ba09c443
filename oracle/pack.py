"""Packed byte layouts of D_g and C_l (TEST INFRASTRUCTURE; the bit-exact contract).

The pages say only "NVFP4, 8-bit scale per block of sixteen values" (technical
review, "From retained values to measured decoding") and that the export holds
"dictionary, per-layer codes, scales and support" (review Algorithm 2, export
step).  Everything else below is a plain reading, written out here once so the
CUDA library's packer can be compared with it byte for byte.

Dictionary D_g (d_in x k, Eq. (1)):
  * quantisation blocks: 16 consecutive d_in entries of one atom (the
    reduction dimension);
  * codes  uint8[k][d_in/2]: element i of atom j at byte j*d_in/2 + i/2, even i
    in the low nibble (atom-major, i.e. K-major for Z = X D);
  * scales uint8[k][d_in/16], E4M3;  s_D fp32.  Requires d_in % 16 == 0.

Coefficients C_l (k x d_out, column-compressed per output channel):
  * column o stores its nnz_o retained atoms in ascending order, then is padded
    with zero entries (code 0, index 0) up to P_o = 16*ceil(nnz_o/16);
  * col_ptr uint32[d_out+1]: padded entry offsets;  nnz uint32[d_out];
  * quantisation blocks: 16 consecutive *stored* entries of a column (the
    structural zeros are not quantised; padding entries are zeros of the block);
    s_C from the amax of the stored values;
  * codes  uint8[total/2]: entry e (global padded index) at byte e/2, even e in
    the low nibble;  scales uint8[total/16];
  * idx    uint8[total]: atom mod 256 (the 8-bit index of Eq. (12)'s a = 8
    case, relative to 256-atom segments);
  * seg_start uint16[d_out][nseg], nseg = ceil(k/256): entry offset, relative
    to the column start, of the first entry whose atom is >= 256*s.  The atom of
    entry q is 256*s(q) + idx with s(q) = max{s : seg_start[s] <= q}; padding
    entries therefore sit in the last segment (atom 256*(nseg-1) < k).

Bitmap-indexed C_l (pack_coeff_bitmap): the same values, codes, scales and
padding; the index is one bit per logical position instead (Eq. (12), a = 0,
h = 1): bitmap uint32[d_out][ceil(k/32)], bit j % 32 of word j // 32 of row o set
iff atom j is retained in column o.
"""
from __future__ import annotations

import numpy as np

from .nvfp4 import E2M1_BLOCK, quantize_blocks, tensor_scale

PAD = 16
SEG = 256


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte, even position in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    if c.size % 2:
        raise ValueError("odd number of codes")
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out


def pack_dictionary(D: np.ndarray) -> dict:
    """Quantise and lay out D_g (d_in x k fp32)."""
    D = np.asarray(D, dtype=np.float32)
    d_in, k = D.shape
    if d_in % E2M1_BLOCK:
        raise ValueError("d_in must be a multiple of 16")
    s = tensor_scale(D)
    atoms = np.ascontiguousarray(D.T)  # [k][d_in]
    codes, sc = quantize_blocks(atoms.reshape(-1, E2M1_BLOCK), s)
    return {
        "d_in": d_in,
        "k": k,
        "codes": pack_nibbles(codes),  # k * d_in / 2
        "scales": sc.astype(np.uint8),  # k * d_in / 16
        "s": np.float32(s),
    }


def pack_coeff(col_ptr: np.ndarray, atom_idx: np.ndarray, vals: np.ndarray, k: int,
               d_out: int) -> dict:
    """Quantise and lay out C_l given in unpadded CSC form (atoms ascending)."""
    col_ptr = np.asarray(col_ptr, dtype=np.int64)
    atom_idx = np.asarray(atom_idx, dtype=np.int64)
    vals = np.asarray(vals, dtype=np.float32)
    if col_ptr.shape != (d_out + 1,) or col_ptr[0] != 0:
        raise ValueError("bad col_ptr")
    nnz = np.diff(col_ptr)
    if np.any(nnz < 0) or np.any(nnz > k):
        raise ValueError("bad column length")
    for o in range(d_out):
        a = atom_idx[col_ptr[o]:col_ptr[o + 1]]
        if a.size and (a[0] < 0 or a[-1] >= k or np.any(np.diff(a) <= 0)):
            raise ValueError("atoms must be ascending, unique and < k")
    nseg = -(-k // SEG)
    padded = -(-nnz // PAD) * PAD
    pptr = np.zeros(d_out + 1, dtype=np.int64)
    pptr[1:] = np.cumsum(padded)
    total = int(pptr[-1])

    pvals = np.zeros(total, dtype=np.float32)
    patoms = np.zeros(total, dtype=np.int64)
    seg_start = np.zeros((d_out, nseg), dtype=np.int64)
    for o in range(d_out):
        a = atom_idx[col_ptr[o]:col_ptr[o + 1]]
        n = a.size
        pvals[pptr[o]:pptr[o] + n] = vals[col_ptr[o]:col_ptr[o + 1]]
        patoms[pptr[o]:pptr[o] + n] = a
        for s in range(nseg):
            seg_start[o, s] = int(np.searchsorted(a, SEG * s, side="left"))
    s_c = tensor_scale(vals)
    codes, sc = quantize_blocks(pvals.reshape(-1, E2M1_BLOCK), s_c)
    idx = (patoms % SEG).astype(np.uint8)
    return {
        "k": k,
        "d_out": d_out,
        "nseg": nseg,
        "col_ptr": pptr.astype(np.uint32),
        "nnz": nnz.astype(np.uint32),
        "codes": pack_nibbles(codes),  # total / 2
        "scales": sc.astype(np.uint8),  # total / 16
        "idx": idx,  # total
        "seg_start": seg_start.astype(np.uint16).reshape(-1),  # d_out * nseg
        "s": np.float32(s_c),
    }


def pack_coeff_fmt(col_ptr: np.ndarray, atom_idx: np.ndarray, vals: np.ndarray, k: int, d_out: int,
                   fmt: str) -> dict:
    """C_l with its values in one of Table 4's coefficient formats (fp16, fp8,
    int8; see valuefmt) and the same index, padding and column pointers as
    pack_coeff. The values array holds one code per stored entry (padding
    entries: code 0): uint8 for fp8 / int8 (int8 as two's complement), uint16
    bit patterns for fp16; s is the per-tensor fp32 scale (1 for fp16)."""
    from . import valuefmt as VF
    if fmt == "nvfp4":
        return pack_coeff(col_ptr, atom_idx, vals, k, d_out)
    if fmt not in VF.FORMATS:
        raise ValueError(f"unknown coefficient format {fmt}")
    pc = pack_coeff(col_ptr, atom_idx, vals, k, d_out)
    col_ptr = np.asarray(col_ptr, dtype=np.int64)
    vals = np.asarray(vals, dtype=np.float32)
    pptr = pc["col_ptr"].astype(np.int64)
    total = int(pptr[-1])
    pvals = np.zeros(total, dtype=np.float32)
    for o in range(d_out):
        n = int(col_ptr[o + 1] - col_ptr[o])
        pvals[pptr[o]:pptr[o] + n] = vals[col_ptr[o]:col_ptr[o + 1]]
    if fmt == "fp16":
        s, codes = np.float32(1.0), VF.fp16_encode(pvals)
    elif fmt == "fp8":
        s = VF.fp8_scale(vals)
        codes = VF.fp8_encode(pvals, s)
    else:
        s = VF.int8_scale(vals)
        codes = VF.int8_encode(pvals, s).view(np.uint8)
    out = {n: pc[n] for n in ("k", "d_out", "nseg", "col_ptr", "nnz", "idx", "seg_start")}
    out.update(fmt=fmt, values=codes, s=np.float32(s))
    return out


BLOCK = 16


def pack_coeff_blocks(col_ptr: np.ndarray, atom_idx: np.ndarray, vals: np.ndarray, k: int, d_out: int) -> dict:
    """C_l with block-structured support (the review's "Let the accelerator
    constrain the support"; the paper names block-structured sparsity as future
    work): every column's support is a union of whole aligned blocks of 16
    consecutive atoms. A kept block is exactly one NVFP4 block (its 16 values,
    one E4M3 scale), so the values, codes and scales equal those of pack_coeff on
    the same support, and the index is one uint16 block number per 16 values:
      blk_ptr uint32[d_out+1]  kept blocks before each column;
      blk_idx uint16[nblk]     block number (atom // 16), ascending per column;
      codes   uint8[nblk*8], scales uint8[nblk], s fp32 (per tensor)."""
    col_ptr = np.asarray(col_ptr, dtype=np.int64)
    atom_idx = np.asarray(atom_idx, dtype=np.int64)
    if k % BLOCK:
        raise ValueError("k must be a multiple of 16")
    for o in range(d_out):
        a = atom_idx[col_ptr[o]:col_ptr[o + 1]]
        if a.size % BLOCK or np.any(a.reshape(-1, BLOCK) != (a[::BLOCK, None] // BLOCK) * BLOCK + np.arange(BLOCK)):
            raise ValueError(f"column {o}: support is not a union of aligned 16-atom blocks")
    pc = pack_coeff(col_ptr, atom_idx, vals, k, d_out)
    nblk = np.diff(col_ptr) // BLOCK
    blk_ptr = np.zeros(d_out + 1, dtype=np.int64)
    blk_ptr[1:] = np.cumsum(nblk)
    return {
        "k": k,
        "d_out": d_out,
        "blk_ptr": blk_ptr.astype(np.uint32),
        "blk_idx": (atom_idx[::BLOCK] // BLOCK).astype(np.uint16),
        "codes": pc["codes"],
        "scales": pc["scales"],
        "s": pc["s"],
    }


def pack_coeff_bitmap(col_ptr: np.ndarray, atom_idx: np.ndarray, vals: np.ndarray, k: int,
                      d_out: int) -> dict:
    """C_l with a bitmap support index: the review's Eq. (12) case a = 0, h = 1
    ("From retained values to measured decoding": one bit per logical position,
    no per-value index bits).

    The stored values, their padding, blocks, codes, scales and s_C are exactly
    those of pack_coeff (the index format does not change what is quantised).
    In place of idx and seg_start each column o has a bitmap of k bits,
    uint32[d_out][ceil(k/32)]: bit (j mod 32) of word j // 32 is set iff atom j
    is retained in column o. Its set bits, in ascending order, are the column's
    stored entries in storage order; padding entries have no bit."""
    pc = pack_coeff(col_ptr, atom_idx, vals, k, d_out)
    col_ptr = np.asarray(col_ptr, dtype=np.int64)
    atom_idx = np.asarray(atom_idx, dtype=np.int64)
    words = -(-k // 32)
    mask = np.zeros((d_out, words * 32), dtype=bool)  # mask[o, j]: atom j retained in column o
    mask[np.repeat(np.arange(d_out), np.diff(col_ptr)), atom_idx] = True
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)  # bit b of a word has weight 2^b
    bitmap = (mask.reshape(d_out, words, 32).astype(np.uint64) * weights).sum(axis=2).astype(np.uint32)
    return {
        "k": k,
        "d_out": d_out,
        "words": words,
        "col_ptr": pc["col_ptr"],
        "nnz": pc["nnz"],
        "codes": pc["codes"],
        "scales": pc["scales"],
        "bitmap": bitmap.reshape(-1),  # d_out * ceil(k/32)
        "s": pc["s"],
    }


def bitmap_entry_atoms(pb: dict) -> np.ndarray:
    """Atom of every stored entry of a bitmap-indexed C_l (padding entries: -1):
    the j-th stored entry of a column is the column's j-th set bit."""
    d_out, words = pb["d_out"], pb["words"]
    ptr = pb["col_ptr"].astype(np.int64)
    bm = pb["bitmap"].reshape(d_out, words)
    bits = (bm[:, :, None].astype(np.uint64) >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    mask = bits.reshape(d_out, words * 32).astype(bool)  # mask[o, j]: bit j of row o
    atoms = np.full(int(ptr[-1]), -1, dtype=np.int64)
    for o in range(d_out):
        set_bits = np.flatnonzero(mask[o])
        atoms[ptr[o]:ptr[o] + set_bits.size] = set_bits
    return atoms


def coeff_entry_atoms(pc: dict) -> np.ndarray:
    """Atom of every stored entry (padding included), from idx and seg_start."""
    d_out, nseg = pc["d_out"], pc["nseg"]
    ptr = pc["col_ptr"].astype(np.int64)
    seg_start = pc["seg_start"].astype(np.int64).reshape(d_out, nseg)
    atoms = np.zeros(int(ptr[-1]), dtype=np.int64)
    for o in range(d_out):
        P = int(ptr[o + 1] - ptr[o])
        q = np.arange(P)
        # s(q) = max{s : seg_start[s] <= q}
        s_of_q = np.searchsorted(seg_start[o], q, side="right") - 1
        atoms[ptr[o]:ptr[o + 1]] = SEG * s_of_q + pc["idx"][ptr[o]:ptr[o + 1]]
    return atoms
