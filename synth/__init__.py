"""Seeded synthetic workloads for the dictionary-compressed projection.

This module only draws random numbers. It holds none of the method's arithmetic
(no quantisation, no packing, no products): it produces the *inputs* that both
the fp64 oracle and the CUDA path consume.

Shapes follow the LLaMA-7B projection shapes of the DictLLM paper
(arXiv 2611.08082; Table A14 measures decode on LLaMA-7B at batch one):
attention q/k/v/o 4096x4096, gate/up 4096x11008, down 11008x4096.

Every tensor comes from its own generator,
``numpy.random.default_rng(SeedSequence([cfg, group, ptype, layer, tensor_id]))``,
so a tensor does not depend on the order in which tensors are generated.

Recipe (stated once, used everywhere):
  * D_g  (d_in x k, fp32):  N(0, 1/d_in).
  * C_l nonzeros (fp32):     N(0, 1/k).  At the tiny shape (d_in=256, k=128) these
    are exactly N(0, 1/256) and N(0, 1/128).
  * C_l support: every output column keeps exactly nnz = k - floor((1-rho)*k)
    atoms (the per-column removal count floor(p*k) of the technical review's
    pruning algorithm, with p = 1 - rho), drawn uniformly without replacement and
    sorted ascending.  ``nnz_per_column`` below is that count.
  * X (M x d_in, fp16): N(0, 1) drawn in fp32 then rounded to fp16; the prefill
    workload scales round(0.01*d_in) channels (uniform without replacement, per
    layer) by 20 before rounding.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# tensor ids inside a SeedSequence key
T_D, T_SUPPORT, T_CVALS, T_X, T_OUTLIER, T_DENSITY = 0, 1, 2, 3, 4, 5

PROJ_TYPES = ("q", "k", "v", "o", "gate", "up", "down")
# LLaMA-7B projection shapes (d_in, d_out) and the dictionary width k used for
# each projection type in these workloads.
LLAMA7B_SHAPES = {
    "q": (4096, 4096, 2048),
    "k": (4096, 4096, 2048),
    "v": (4096, 4096, 2048),
    "o": (4096, 4096, 2048),
    "gate": (4096, 11008, 3072),
    "up": (4096, 11008, 3072),
    "down": (11008, 4096, 3072),
}
# which projections read the same activation inside one transformer layer
INPUT_SITE = {"q": 0, "k": 0, "v": 0, "o": 1, "gate": 2, "up": 2, "down": 3}


def nnz_per_column(k: int, rho: float) -> int:
    """Retained atoms per output column at density rho: k - floor((1-rho)*k)."""
    return k - int(math.floor((1.0 - rho) * k))


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(x) for x in key]))


def gen_dictionary(cfg: int, group: int, ptype: int, d_in: int, k: int) -> np.ndarray:
    """D_g as fp32, shape (d_in, k), row-major; entries N(0, 1/d_in)."""
    g = _rng(cfg, group, ptype, 0, T_D)
    d = g.standard_normal((d_in, k), dtype=np.float32)
    d *= np.float32(1.0 / math.sqrt(d_in))
    return d


def gen_support(cfg: int, group: int, ptype: int, layer: int, k: int, d_out: int,
                nnz: int) -> np.ndarray:
    """Sorted atom indices, shape (d_out, nnz), int32.

    Uniform without replacement per column via a partial Fisher-Yates shuffle
    run for all columns at once (nnz vectorised swap steps)."""
    if nnz < 0 or nnz > k:
        raise ValueError("nnz out of range")
    g = _rng(cfg, group, ptype, layer, T_SUPPORT)
    dt = np.int16 if k <= 32767 else np.int32
    perm = np.tile(np.arange(k, dtype=dt), (d_out, 1))
    rows = np.arange(d_out)
    for i in range(nnz):
        j = i + g.integers(0, k - i, size=d_out)
        a = perm[rows, i].copy()
        perm[rows, i] = perm[rows, j]
        perm[rows, j] = a
    sup = np.sort(perm[:, :nnz].astype(np.int32), axis=1)
    return sup


@dataclass
class SparseCoeff:
    """C_l in column-compressed form (unpadded), fp32 values."""
    k: int
    d_out: int
    col_ptr: np.ndarray  # int32 (d_out+1,)
    atom_idx: np.ndarray  # int32 (nnz_total,), ascending within a column
    vals: np.ndarray  # float32 (nnz_total,)

    @property
    def nnz_total(self) -> int:
        return int(self.col_ptr[-1])


def gen_coeff(cfg: int, group: int, ptype: int, layer: int, k: int, d_out: int,
              rho: float) -> SparseCoeff:
    """C_l (k x d_out) with exactly nnz_per_column(k, rho) nonzeros per column."""
    nnz = nnz_per_column(k, rho)
    sup = gen_support(cfg, group, ptype, layer, k, d_out, nnz)
    g = _rng(cfg, group, ptype, layer, T_CVALS)
    vals = g.standard_normal(d_out * nnz, dtype=np.float32)
    vals *= np.float32(1.0 / math.sqrt(k))
    col_ptr = (np.arange(d_out + 1, dtype=np.int64) * nnz).astype(np.int32)
    return SparseCoeff(k=k, d_out=d_out, col_ptr=col_ptr,
                       atom_idx=sup.reshape(-1).copy(), vals=vals)


def gen_coeff_blocks(cfg: int, group: int, ptype: int, layer: int, k: int, d_out: int, rho: float,
                     block: int = 16) -> SparseCoeff:
    """C_l (k x d_out) whose support is block-structured: every column keeps
    nb = k/block - floor((1-rho) k/block) whole aligned blocks of `block`
    consecutive atoms, drawn uniformly without replacement; the retained values
    are N(0, 1/k)."""
    if k % block:
        raise ValueError("k must be a multiple of the block size")
    kb = k // block
    nb = kb - int(math.floor((1.0 - rho) * kb))
    blocks = gen_support(cfg, group, ptype, layer, kb, d_out, nb)  # sorted block numbers per column
    atoms = (blocks[:, :, None] * block + np.arange(block, dtype=np.int32)[None, None, :]).reshape(d_out, -1)
    g = _rng(cfg, group, ptype, layer, T_CVALS)
    vals = g.standard_normal(d_out * nb * block, dtype=np.float32)
    vals *= np.float32(1.0 / math.sqrt(k))
    col_ptr = (np.arange(d_out + 1, dtype=np.int64) * nb * block).astype(np.int32)
    return SparseCoeff(k=k, d_out=d_out, col_ptr=col_ptr, atom_idx=atoms.reshape(-1).astype(np.int32).copy(),
                       vals=vals)


def gen_activations(cfg: int, layer: int, site: int, M: int, d_in: int,
                    outlier_frac: float = 0.0, outlier_gain: float = 20.0) -> np.ndarray:
    """X as fp16, shape (M, d_in), row-major."""
    g = _rng(cfg, 0, site, layer, T_X)
    x = g.standard_normal((M, d_in), dtype=np.float32)
    if outlier_frac > 0.0:
        n_out = int(round(outlier_frac * d_in))
        go = _rng(cfg, 0, site, layer, T_OUTLIER)
        ch = go.choice(d_in, size=n_out, replace=False)
        x[:, ch] *= np.float32(outlier_gain)
    return x.astype(np.float16)


def draw_density(cfg: int, group: int, ptype: int, layer: int, lo: float, hi: float) -> float:
    """Per-projection density drawn uniformly in [lo, hi)."""
    g = _rng(cfg, group, ptype, layer, T_DENSITY)
    return float(lo + (hi - lo) * g.random())


# ----------------------------------------------------------------------------
# Workload descriptions
# ----------------------------------------------------------------------------
@dataclass
class Projection:
    """One projection call: layer `layer` of group `group`, type `ptype`."""
    cfg: int
    name: str
    group: int
    layer: int  # global layer index
    ptype: int
    d_in: int
    d_out: int
    k: int
    rho: float
    site: int


@dataclass
class Workload:
    cfg: int
    name: str
    projections: list = field(default_factory=list)
    tokens: tuple = (1,)
    outlier_frac: float = 0.0

    def groups(self):
        """Distinct (group, ptype) dictionaries with their shapes, in first-use order."""
        seen = {}
        for p in self.projections:
            key = (p.group, p.ptype)
            if key not in seen:
                seen[key] = (p.d_in, p.k)
        return seen


def tiny() -> Workload:
    """One group of 2 layers, d_in=d_out=256, k=128, density 0.5, M in {1,4}."""
    w = Workload(cfg=0, name="tiny", tokens=(1, 4))
    for layer in range(2):
        w.projections.append(Projection(0, "tiny", 0, layer, 0, 256, 256, 128, 0.5, 0))
    return w


def attention_group() -> Workload:
    """q,k,v,o, each its own dictionary shared by 2 layers; density 0.3; M=1."""
    w = Workload(cfg=1, name="llama7b-attn-group", tokens=(1,))
    for layer in range(2):
        for t, nm in enumerate(("q", "k", "v", "o")):
            d_in, d_out, k = LLAMA7B_SHAPES[nm]
            w.projections.append(Projection(1, nm, 0, layer, t, d_in, d_out, k, 0.3,
                                            INPUT_SITE[nm]))
    return w


def mlp_groups() -> Workload:
    """gate/up (4096->11008) and down (11008->4096), k=3072, density 0.25, M in {1,8}."""
    w = Workload(cfg=2, name="llama7b-mlp-groups", tokens=(1, 8))
    for layer in range(2):
        for nm in ("gate", "up", "down"):
            d_in, d_out, k = LLAMA7B_SHAPES[nm]
            w.projections.append(Projection(2, nm, 0, layer, PROJ_TYPES.index(nm), d_in,
                                            d_out, k, 0.25, INPUT_SITE[nm]))
    return w


def full_step(n_layers: int = 32, cfg: int = 3, rho_fixed: float | None = None,
              tokens=(1,), outlier_frac: float = 0.0, name: str = "llama7b-linear-stack") -> Workload:
    """All 7 projection types of n_layers layers in groups of 2, model order
    (q,k,v,o,gate,up,down per layer); density U[0.2,0.4] per projection unless fixed."""
    w = Workload(cfg=cfg, name=name, tokens=tokens, outlier_frac=outlier_frac)
    for layer in range(n_layers):
        group = layer // 2
        for t, nm in enumerate(PROJ_TYPES):
            d_in, d_out, k = LLAMA7B_SHAPES[nm]
            rho = rho_fixed if rho_fixed is not None else draw_density(cfg, group, t, layer, 0.2, 0.4)
            w.projections.append(Projection(cfg, nm, group, layer, t, d_in, d_out, k, rho,
                                            INPUT_SITE[nm]))
    return w


def prefill(n_layers: int = 32) -> Workload:
    """Shapes of the full stack, density 0.3, M in {128, 512, 2048}, 1% outlier channels x20."""
    return full_step(n_layers=n_layers, cfg=4, rho_fixed=0.3, tokens=(128, 512, 2048),
                     outlier_frac=0.01, name="llama7b-prefill")


WORKLOADS = {0: tiny, 1: attention_group, 2: mlp_groups, 3: full_step, 4: prefill}


def projection_inputs(p: Projection):
    """(D fp32, C SparseCoeff) for a projection."""
    D = gen_dictionary(p.cfg, p.group, p.ptype, p.d_in, p.k)
    C = gen_coeff(p.cfg, p.group, p.ptype, p.layer, p.k, p.d_out, p.rho)
    return D, C
