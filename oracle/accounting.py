"""Budget, byte and multiply-add accounting (TEST INFRASTRUCTURE).

Each function restates one passage of the technical review "DictLLM: Shared
Dictionaries for Post-Training Compression":

  eq2_budget        Eq. (2): N0 = n d_in d_out, Np = d_in k + n (1-p) k d_out.
  eq3_rank          Eq. (3): k = floor((1-rho_fac) n d_in d_out / (d_in + n d_out)).
  retained_fraction Np / N0 with the unrounded Eq. (3) rank ("The budget" section:
                    0.8 (1 - 2p/3) ~= 0.6965 for p = 0.194, two square layers).
  mac_fraction      "From retained values to measured decoding": ideal sparse
                    factored decode does n k [d_in + (1-p) d_out] multiply-adds per
                    token against n d_in d_out dense.
  nvfp4_bits        4 value bits + 8 scale bits / 16 = 4.5 bits per value.
  eq12_breakeven    Eq. (12): a sparse array saves bytes iff p > (a + h) / (b + a).
  call_bytes        algorithmic bytes of one forward call in the packed layouts
                    (D and C values, indices, scales; X and Y), padding excluded.
"""
from __future__ import annotations

import math


def eq2_budget(n: int, d_in: int, d_out: int, k: float, p: float):
    N0 = n * d_in * d_out
    Np = d_in * k + n * (1.0 - p) * k * d_out
    return {"N0": N0, "Np": Np, "rho": 1.0 - Np / N0, "G": N0 / Np}


def eq3_rank(rho_fac: float, n: int, d_in: int, d_out: int) -> int:
    return int(math.floor((1.0 - rho_fac) * n * d_in * d_out / (d_in + n * d_out)))


def eq3_rank_real(rho_fac: float, n: int, d_in: int, d_out: int) -> float:
    return (1.0 - rho_fac) * n * d_in * d_out / (d_in + n * d_out)


def retained_fraction(rho_fac: float, n: int, d_in: int, d_out: int, p: float) -> float:
    k = eq3_rank_real(rho_fac, n, d_in, d_out)
    b = eq2_budget(n, d_in, d_out, k, p)
    return b["Np"] / b["N0"]


def dictionary_share(rho_fac: float, n: int, d_in: int, d_out: int) -> float:
    """Fraction of the original group count that the dictionary alone costs."""
    k = eq3_rank_real(rho_fac, n, d_in, d_out)
    return d_in * k / (n * d_in * d_out)


def mac_fraction(n: int, k: float, d_in: int, d_out: int, p: float) -> float:
    return n * k * (d_in + (1.0 - p) * d_out) / (n * d_in * d_out)


def nvfp4_bits(value_bits: int = 4, scale_bits: int = 8, block: int = 16) -> float:
    return value_bits + scale_bits / block


def eq12_breakeven(a: float, b: float, h: float) -> float:
    return (a + h) / (b + a)


def eq12_saves(p: float, a: float, b: float, h: float) -> bool:
    q = 1.0 - p
    return q * (b + a) + h < b


def call_bytes(M: int, d_in: int, d_out: int, k: int, nnz_per_col, x_bytes: int = 2,
               y_bytes: int = 2) -> dict:
    """Algorithmic bytes of one forward call (unpadded).

    D: d_in k / 2 code bytes + d_in k / 16 scale bytes + 4 (fp32 s_D).
    C: per column ceil(nnz/2) code bytes + ceil(nnz/16) scale bytes + nnz index
       bytes + 2 ceil(k/256) segment-start bytes + 4 column-pointer bytes; + 4.
    X, Y: M (d_in + d_out) fp16."""
    if isinstance(nnz_per_col, int):
        cols = [nnz_per_col] * d_out
    else:
        cols = list(nnz_per_col)
    nseg = max(1, -(-k // 256))
    dbytes = d_in * k // 2 + d_in * k // 16 + 4
    cbytes = 4 + sum(-(-n // 2) + -(-n // 16) + n + 2 * nseg + 4 for n in cols)
    xy = M * (d_in * x_bytes + d_out * y_bytes)
    return {"D": dbytes, "C": cbytes, "XY": xy, "total": dbytes + cbytes + xy}


def call_flops(M: int, d_in: int, k: int, nnz_total: int) -> dict:
    """2 M d_in k for the dictionary stage, 2 M nnz for the coefficient stage."""
    return {"dict": 2 * M * d_in * k, "coeff": 2 * M * nnz_total,
            "total": 2 * M * (d_in * k + nnz_total)}
