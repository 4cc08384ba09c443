"""Test inputs whose NVFP4 quantisation is exact (no method arithmetic here:
a generator of integer factors and their exact product).

With every NVFP4 block holding an entry of magnitude 2688 = 6 x 448 (the tensor
amax), the tensor scale is 1 and every block scale the E4M3 maximum 448, and
values 448 x {0, .5, 1, 1.5, 2, 3, 4, 6} quantise without error. The quantised
forward must then equal the exact product of the original factors."""
import numpy as np

GRID = np.array([224, 448, 672, 896, 1344, 1792, 2688], np.int64)


def exact_block(rng, n, keep=16):
    v = rng.choice(GRID, size=n) * rng.choice([-1, 1], size=n)
    for b in range(0, n, keep):  # each block of `keep` entries holds +-2688
        v[b + rng.integers(0, min(keep, n - b))] = 2688 * rng.choice([-1, 1])
    return v


def exact_case(seed=0, d_in=64, k=512, M=3, blocks=False):
    rng = np.random.default_rng(seed)
    D = np.zeros((d_in, k), np.int64)
    for a in range(k):  # atom-major blocks of 16 d_in entries
        D[:, a] = exact_block(rng, d_in)
        D[rng.random(d_in) < 0.3, a] = 0
        for b in range(0, d_in, 16):
            if not np.any(np.abs(D[b:b + 16, a]) == 2688):
                D[b, a] = 2688
    cols = []
    if blocks:  # unions of aligned 16-atom blocks, every block one NVFP4 block
        for o in range(12):
            bl = np.sort(rng.choice(k // 16, size=int(rng.integers(0, 6)), replace=False))
            cols.append(np.concatenate([np.arange(16 * b, 16 * b + 16) for b in bl]).astype(np.int64)
                        if bl.size else np.zeros(0, np.int64))
    else:  # sizes that are and are not multiples of 16, atoms in both 256-atom segments
        for nnz in (0, 16, 20, 32, 47, 64, 1, 16, 100, 33, 256, 5):
            cols.append(np.sort(rng.choice(k, size=nnz, replace=False)).astype(np.int64))
    col_ptr = np.zeros(len(cols) + 1, np.int64)
    col_ptr[1:] = np.cumsum([c.size for c in cols])
    atoms = np.concatenate(cols) if col_ptr[-1] else np.zeros(0, np.int64)
    vals = np.concatenate([exact_block(rng, c.size) if c.size else np.zeros(0, np.int64) for c in cols])
    Cd = np.zeros((k, len(cols)), np.int64)
    for o, c in enumerate(cols):
        Cd[c, o] = vals[col_ptr[o]:col_ptr[o + 1]]
    X = rng.integers(-3, 4, size=(M, d_in)).astype(np.float16)
    exact = X.astype(np.int64) @ D @ Cd  # integers below 2^53: exact in fp64 as well
    return X, D.astype(np.float32), col_ptr, atoms, vals.astype(np.float32), k, len(cols), exact
