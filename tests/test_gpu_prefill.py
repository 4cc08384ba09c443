"""Prefill path (tcgen05 tensor-core GEMMs) against the fp64 oracle.

The dictionary stage Z = s_D X D_g is checked on its own (Z is fp16 with s_D
applied before rounding), then the whole forward Y = X D_g C_l at the shapes of
the prefill workload (LLaMA-7B projections, 1 % of input channels scaled x20),
with ragged token counts, atom counts and reduction lengths that leave partial
128 x 256 tiles and partial 64-element stages. The largest case compares
sampled outputs that the oracle computes one by one.
"""
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
from oracle import forward as F  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _build():
    from dictionary_compressed_linear_b200 import build
    build.build()


def _case(seed, d_in, k, d_out, rho):
    D = synth.gen_dictionary(4, seed, 0, d_in, k)
    C = synth.gen_coeff(4, seed, 0, 0, k, d_out, rho)
    return D, C


@pytest.mark.parametrize("d_in,k,M", [(256, 128, 16), (512, 272, 129), (4096, 2048, 128),
                                      (4128, 2064, 200), (11008, 3072, 256)])
def test_dictionary_stage_prefill(d_in, k, M):
    D = synth.gen_dictionary(4, 1, 0, d_in, k)
    g = dp.dictproj_pack_group(D, max(M, 8))
    pd = dp.dictproj_pack_group_host(D)
    X = synth.gen_activations(4, 0, 0, M, d_in, outlier_frac=0.01)
    Xd = torch.from_numpy(X).cuda()
    Z = torch.full((M, k), float("nan"), dtype=torch.float16, device="cuda")
    dp.dictproj_dictionary_stage_prefill(Xd.data_ptr(), M, g, Z.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    z_ref = X.astype(np.float64) @ F.decode_dictionary(pd)
    assert_parity(Z.float().cpu().numpy().astype(np.float64), z_ref, f"Z d_in={d_in} k={k} M={M}")


@pytest.mark.parametrize("d_in,k,d_out,rho,M", [
    (256, 128, 256, 0.5, 16),       # tiny shapes, one partial tile
    (4096, 2048, 4096, 0.3, 128),   # attention projection
    (4096, 2048, 4096, 0.3, 512),
    (4128, 2064, 4100, 0.3, 200),   # ragged d_in, k, d_out (d_out % 8 != 0) and M
    (11008, 3072, 4096, 0.3, 128),  # down projection
])
def test_prefill_forward(d_in, k, d_out, rho, M):
    D, C = _case(2, d_in, k, d_out, rho)
    g, l = device_projection(D, C, max_tokens=M)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(4, 0, 2, M, d_in, outlier_frac=0.01)
    y = run_forward(g, l, X)
    assert_parity(y, oracle_forward(X, pd, pc), f"prefill d_in={d_in} k={k} d_out={d_out} M={M}")


def test_prefill_gate_m2048_sampled():
    # gate/up shape at the largest prefill size; 4000 outputs checked one by one
    d_in, k, d_out, M = 4096, 3072, 11008, 2048
    D, C = _case(3, d_in, k, d_out, 0.3)
    g, l = device_projection(D, C, max_tokens=M)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(4, 1, 2, M, d_in, outlier_frac=0.01)
    y = run_forward(g, l, X)
    rng = np.random.default_rng(7)
    rows = np.concatenate([rng.integers(0, M, 3900), [0, M - 1] * 50])
    cols = np.concatenate([rng.integers(0, d_out, 3900), [0, d_out - 1] * 50])
    ref = F.sampled_outputs(X, pd, pc, rows, cols)
    assert_parity(y[rows, cols], ref, "gate M=2048 sampled")
    assert np.all(np.isfinite(y))


def test_prefill_deterministic_and_matches_oracle_twice():
    D, C = _case(5, 1024, 512, 768, 0.3)
    g, l = device_projection(D, C, max_tokens=300)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(4, 2, 0, 300, 1024, outlier_frac=0.01)
    y1 = run_forward(g, l, X)
    y2 = run_forward(g, l, X)
    assert np.array_equal(y1, y2)
    assert_parity(y1, oracle_forward(X, pd, pc), "prefill 300 tokens")


def test_prefill_requires_reserved_scratch():
    D, C = _case(6, 256, 128, 512, 0.5)
    g = dp.dictproj_pack_group(D, 64)
    l = dp.dictproj_pack_layer(C.col_ptr, C.atom_idx, C.vals, C.k, C.d_out)
    X = torch.zeros((32, 256), dtype=torch.float16, device="cuda")
    Y = torch.full((32, 512), 3.0, dtype=torch.float16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert dp.dictproj_forward_status(X.data_ptr(), 32, l.handle, g.handle, Y.data_ptr(), st) == -5
    assert "dictproj_group_reserve_prefill" in dp.dictproj_last_error()
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)
    dp.dictproj_group_reserve_prefill(g, 256)   # too small still
    assert dp.dictproj_forward_status(X.data_ptr(), 32, l.handle, g.handle, Y.data_ptr(), st) == -5
    dp.dictproj_group_reserve_prefill(g, 512)
    assert dp.dictproj_forward_status(X.data_ptr(), 32, l.handle, g.handle, Y.data_ptr(), st) == 0
    torch.cuda.synchronize()
    assert torch.all(Y == 0.0)


def test_prefill_in_cuda_graph():
    D, C = _case(7, 512, 256, 512, 0.3)
    g, l = device_projection(D, C, max_tokens=256)
    pd, pc = oracle_projection(D, C)
    X_np = synth.gen_activations(4, 3, 0, 256, 512, outlier_frac=0.01)
    X = torch.from_numpy(X_np).cuda()
    Y = torch.empty((256, 512), dtype=torch.float16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dp.dictproj_forward(X.data_ptr(), 256, l, g, Y.data_ptr(), s.cuda_stream)  # warm-up outside capture
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        dp.dictproj_forward(X.data_ptr(), 256, l, g, Y.data_ptr(), s.cuda_stream)
    Y.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert_parity(Y.float().cpu().numpy().astype(np.float64), oracle_forward(X_np, pd, pc), "graph replay")
    del graph


@pytest.mark.parametrize("M", [128, 512, 2048])
@pytest.mark.parametrize("name", ["q", "gate", "down"])
def test_benchmarked_prefill_configurations(name, M):
    """Exactly the inputs and launch configuration bench.py times for the prefill
    leg (same seeds, same M, so the same token-tile width per shape), checked on
    4000 sampled outputs: 16 token rows (first and last included) x 250 columns."""
    import bench
    D, C, X = bench.prefill_inputs(name, M)
    pg = dp.dictproj_pack_group_host(D)
    pc = dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, C.k, C.d_out)
    g = dp.dictproj_group_upload(pg, M)
    dp.dictproj_group_reserve_prefill(g, C.d_out)
    l = dp.dictproj_layer_upload(pc)
    y = run_forward(g, l, X)
    assert np.all(np.isfinite(y))
    pd_o, pc_o = oracle_projection(D, C)
    rng = np.random.default_rng(1000 + M)
    trows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 14, replace=False)]))
    rows = np.repeat(trows, 250)
    cols = np.concatenate([np.concatenate([[0, C.d_out - 1], rng.choice(C.d_out, 248, replace=False)])
                           for _ in trows])
    ref = F.sampled_outputs_rows(X, pd_o, pc_o, rows, cols)
    assert_parity(y[rows, cols], ref, f"bench prefill {name} M={M}")
