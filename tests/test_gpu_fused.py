"""The fused decode kernel (one kernel per call, weights staged through shared
memory by TMA, one grid-wide exchange of partial Z) against the fp64 oracle.

This module selects it for every decode call (dictproj_set_decode_kernels with
DECODE_FUSED; the library's default sends NVFP4 projections to the faster
two-kernel path). These cases cover its edges: a reduction
length that leaves a partial 512-element piece (zero-filled out of bounds), a
single 16-atom tile, 32 segments of 256 atoms, fewer output columns than SMs
(CTAs without columns), empty / full / one-atom columns, columns that straddle
segment boundaries, batches of up to four different shapes with aliased inputs,
M = 8 with two k = 3072 projections (their Z tables do not fit shared memory
together, so they are loaded one after the other), CUDA-graph replay and long
chains of calls (the launch epochs of the exchange advance every call)."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dictionary_compressed_linear_b200 as dp  # noqa: E402
from gpu_helpers import (assert_parity, device_projection, oracle_forward,  # noqa: E402
                         oracle_projection, run_forward)


@pytest.fixture(autouse=True, scope="module")
def _fused_kernel():
    dp.dictproj_set_decode_kernels(dp.DECODE_FUSED)
    yield
    dp.dictproj_set_decode_kernels(dp.DECODE_AUTO)


def _case(seed, d_in, k, d_out, rho):
    return synth.gen_dictionary(40, seed, 0, d_in, k), synth.gen_coeff(40, seed, 0, 0, k, d_out, rho)


@pytest.mark.parametrize("d_in,k,d_out,rho", [
    (512, 256, 300, 0.3),      # one piece per atom row
    (544, 512, 200, 0.3),      # second piece 32 of 512 elements wide
    (4128, 2064, 4100, 0.3),   # ragged everything
    (11008, 3072, 4096, 0.3),  # down projection
    (1024, 16, 64, 1.0),       # a single tile
    (512, 8192, 64, 0.05),     # 32 segments
    (2048, 512, 96, 0.5),      # fewer columns than SMs
    (4096, 3072, 11008, 0.4),  # gate/up at the densest stack density
])
@pytest.mark.parametrize("M", [1, 2, 5, 8])
def test_fused_shapes(d_in, k, d_out, rho, M):
    D, C = _case(1, d_in, k, d_out, rho)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(40, M, 0, M, d_in)
    if (k + 256) * 8 * 4 > 227 * 1024 and M > 4:
        # Z of k atoms for 8 token slots exceeds shared memory: refused before any launch
        Xd = torch.from_numpy(X).cuda()
        Y = torch.full((M, d_out), 3.0, dtype=torch.float16, device="cuda")
        st = torch.cuda.current_stream().cuda_stream
        assert dp.dictproj_forward_status(Xd.data_ptr(), M, l.handle, g.handle, Y.data_ptr(), st) == -9
        torch.cuda.synchronize()
        assert torch.all(Y == 3.0)
        return
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc), f"fused d_in={d_in} k={k} d_out={d_out} M={M}")


def _custom_layer(k, d_out, cols, seed=0):
    rng = np.random.default_rng(seed)
    ptr = np.zeros(d_out + 1, np.int32)
    ptr[1:] = np.cumsum([c.size for c in cols])
    atoms = np.concatenate(cols).astype(np.int32)
    vals = (rng.standard_normal(atoms.size) / np.sqrt(k)).astype(np.float32)
    return synth.SparseCoeff(k=k, d_out=d_out, col_ptr=ptr, atom_idx=atoms, vals=vals)


@pytest.mark.parametrize("M", [1, 4, 8])
def test_fused_degenerate_columns(M):
    rng = np.random.default_rng(5)
    k, d_in = 1008, 512
    kinds = [0, k, 1, 15, 16, 17, 255, 256, 257, 3]
    cols = [np.sort(rng.choice(k, size=kinds[o % len(kinds)], replace=False)) for o in range(333)]
    cols[7] = np.array([0, 600, 1007])
    cols[8] = np.arange(240, 272)
    cols[9] = np.arange(0, 1008, 63)
    C = _custom_layer(k, 333, cols)
    D = synth.gen_dictionary(41, 0, 0, d_in, k)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(41, 0, 0, M, d_in)
    y = run_forward(g, l, X)
    assert_parity(y, oracle_forward(X, pd, pc, dense=True), f"fused degenerate M={M}")
    assert np.all(y[:, 0] == 0.0)


@pytest.mark.parametrize("M", [1, 3, 8])
def test_fused_batches(M):
    shapes = [(4096, 2048, 4096, 0.2), (4096, 2048, 4096, 0.4), (11008, 3072, 4096, 0.3), (544, 512, 200, 0.3)]
    projs = []
    for i, (d_in, k, d_out, rho) in enumerate(shapes):
        D, C = _case(10 + i, d_in, k, d_out, rho)
        g, l = device_projection(D, C, max_tokens=8)
        projs.append((g, l, oracle_projection(D, C), d_in, d_out))
    Xn = [synth.gen_activations(42, i, 0, M, p[3]) for i, p in enumerate(projs)]
    Xn[1] = Xn[0]
    Xs = [torch.from_numpy(x).cuda() for x in Xn]
    Xs[1] = Xs[0]  # two projections read the same activation
    Ys = [torch.full((M, p[4]), float("nan"), dtype=torch.float16, device="cuda") for p in projs]
    st = torch.cuda.current_stream().cuda_stream
    for n in (2, 3, 4):
        dp.dictproj_forward_batch([x.data_ptr() for x in Xs[:n]], M, [p[1] for p in projs[:n]],
                                  [p[0] for p in projs[:n]], [y.data_ptr() for y in Ys[:n]], st)
        torch.cuda.synchronize()
        for i in range(n):
            pd, pc = projs[i][2]
            assert_parity(Ys[i].float().cpu().numpy().astype(np.float64), oracle_forward(Xn[i], pd, pc),
                          f"batch of {n}, entry {i}, M={M}")


def test_fused_mlp_pair_at_m8_loads_z_tables_in_turn():
    projs = []
    for i in range(2):
        D, C = _case(20 + i, 4096, 3072, 11008, 0.3)
        projs.append((*device_projection(D, C, max_tokens=8), oracle_projection(D, C)))
    X_np = synth.gen_activations(43, 0, 0, 8, 4096)
    X = torch.from_numpy(X_np).cuda()
    Ys = [torch.full((8, 11008), float("nan"), dtype=torch.float16, device="cuda") for _ in projs]
    st = torch.cuda.current_stream().cuda_stream
    dp.dictproj_forward_batch([X.data_ptr()] * 2, 8, [p[1] for p in projs], [p[0] for p in projs],
                              [y.data_ptr() for y in Ys], st)
    torch.cuda.synchronize()
    for (g, l, (pd, pc)), y in zip(projs, Ys):
        assert_parity(y.float().cpu().numpy().astype(np.float64), oracle_forward(X_np, pd, pc), "gate/up M=8")


def test_fused_long_chain_in_a_graph_is_exact_and_repeatable():
    # 40 calls on one group and two layers, captured once and replayed 5 times: the
    # exchange's epochs advance 200 times and every replay must give the same bits.
    # Odd calls read the previous call's output, even calls a fresh activation.
    D = synth.gen_dictionary(44, 0, 0, 1024, 512)
    Cs = [synth.gen_coeff(44, 0, 0, j, 512, 1024, 0.3) for j in range(2)]
    g = dp.dictproj_pack_group(D, 8)
    ls = [dp.dictproj_pack_layer(C.col_ptr, C.atom_idx, C.vals, 512, 1024) for C in Cs]
    pd, _ = oracle_projection(D, Cs[0])
    pcs = [oracle_projection(D, C)[1] for C in Cs]
    fresh = [torch.from_numpy(synth.gen_activations(44, i, 0, 2, 1024)).cuda() for i in range(0, 40, 2)]
    outs = [torch.empty((2, 1024), dtype=torch.float16, device="cuda") for _ in range(40)]
    ins = [fresh[i // 2] if i % 2 == 0 else outs[i - 1] for i in range(40)]
    s = torch.cuda.Stream()

    def chain():
        for i in range(40):
            dp.dictproj_forward(ins[i].data_ptr(), 2, ls[i % 2], g, outs[i].data_ptr(), s.cuda_stream)

    with torch.cuda.stream(s):
        chain()
    s.synchronize()
    ref = [o.clone() for o in outs]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        chain()
    for _ in range(5):
        with torch.cuda.stream(s):
            for o in outs:
                o.fill_(float("nan"))
            graph.replay()
        s.synchronize()
        for a, b in zip(outs, ref):
            assert torch.equal(a, b)
    del graph
    for i in range(40):  # each call against the oracle on the call's own input
        x = (fresh[i // 2] if i % 2 == 0 else ref[i - 1]).cpu().numpy()
        assert_parity(ref[i].float().cpu().numpy().astype(np.float64), oracle_forward(x, pd, pcs[i % 2]), f"call {i}")
    assert dp.dictproj_check_status(s.cuda_stream) == 0


def test_decode_kernel_choice_sets_the_launch_count():
    D, C = _case(9, 1024, 512, 300, 0.3)
    g, l = device_projection(D, C, max_tokens=8)
    X = torch.zeros((1, 1024), dtype=torch.float16, device="cuda")
    assert dp.dictproj_launch_count([X.data_ptr()], 1, [l], [g]) == 1  # this module: fused
    dp.dictproj_set_decode_kernels(dp.DECODE_SPLIT)
    try:
        assert dp.dictproj_launch_count([X.data_ptr()], 1, [l], [g]) == 2
        dp.dictproj_set_decode_kernels(dp.DECODE_AUTO)
        assert dp.dictproj_launch_count([X.data_ptr()], 1, [l], [g]) == 2  # NVFP4: the two-kernel path
    finally:
        dp.dictproj_set_decode_kernels(dp.DECODE_FUSED)
