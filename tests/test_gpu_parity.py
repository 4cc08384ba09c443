"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Bar (fp16 in/out, fp32 accumulation): relative Frobenius error <= 5e-3 and every
element |err| <= 1e-2 * (1 + |y|). Packed bytes are compared bit for bit.
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


@pytest.fixture(scope="module", autouse=True)
def _build():
    from dictionary_compressed_linear_b200 import build
    build.build()


def _case(cfg, group, ptype, layer, d_in, k, d_out, rho):
    D = synth.gen_dictionary(cfg, group, ptype, d_in, k)
    C = synth.gen_coeff(cfg, group, ptype, layer, k, d_out, rho)
    return D, C


# ------------------------------------------------------------------ tiny workload
@pytest.mark.parametrize("M", [1, 4])
def test_tiny_workload_all_layers(M):
    w = synth.tiny()
    for p in w.projections:
        D, C = synth.projection_inputs(p)
        g, l = device_projection(D, C, max_tokens=8)
        pd, pc = oracle_projection(D, C)
        X = synth.gen_activations(0, p.layer, p.site, M, p.d_in)
        y = run_forward(g, l, X)
        assert_parity(y, oracle_forward(X, pd, pc, dense=True), f"tiny layer {p.layer} M={M}")


# ------------------------------------------------------------------ LLaMA shapes, decode
@pytest.mark.parametrize("name", ["q", "o"])
def test_attention_projection_m1(name):
    w = synth.attention_group()
    p = [q for q in w.projections if q.name == name and q.layer == 1][0]
    D, C = synth.projection_inputs(p)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(1, p.layer, p.site, 1, p.d_in)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc), f"attn {name}")


@pytest.mark.parametrize("name,M", [("gate", 1), ("down", 1), ("up", 8), ("down", 8)])
def test_mlp_projection(name, M):
    w = synth.mlp_groups()
    p = [q for q in w.projections if q.name == name and q.layer == 0][0]
    D, C = synth.projection_inputs(p)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(2, p.layer, p.site, M, p.d_in)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc), f"mlp {name} M={M}")


# ------------------------------------------------------------------ ragged token counts
@pytest.fixture(scope="module")
def mid():
    D, C = _case(10, 0, 0, 0, 512, 256, 300, 0.3)
    g, l = device_projection(D, C, max_tokens=160)
    pd, pc = oracle_projection(D, C)
    return g, l, pd, pc


@pytest.mark.parametrize("M", [1, 2, 3, 5, 6, 7, 8])
def test_decode_ragged_m(mid, M):
    g, l, pd, pc = mid
    X = synth.gen_activations(10, M, 0, M, 512)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc, dense=True), f"M={M}")


@pytest.mark.parametrize("M", [1, 8, 9, 40, 128, 160])
def test_prefill_path(mid, M):
    g, l, pd, pc = mid
    X = synth.gen_activations(10, M, 1, M, 512, outlier_frac=0.01)
    y = run_forward(g, l, X, path=dp.PATH_PREFILL)
    assert_parity(y, oracle_forward(X, pd, pc, dense=True), f"prefill M={M}")


# ------------------------------------------------------------------ degenerate layers
def _custom_layer(k, d_out, cols, seed=0):
    rng = np.random.default_rng(seed)
    ptr = np.zeros(d_out + 1, np.int32)
    ptr[1:] = np.cumsum([c.size for c in cols])
    atoms = np.concatenate(cols).astype(np.int32) if cols else np.zeros(0, np.int32)
    vals = (rng.standard_normal(atoms.size) / np.sqrt(k)).astype(np.float32)
    return synth.SparseCoeff(k=k, d_out=d_out, col_ptr=ptr, atom_idx=atoms, vals=vals)


@pytest.mark.parametrize("M", [1, 3, 8, 20])
def test_degenerate_columns(M):
    rng = np.random.default_rng(3)
    k, d_in = 1008, 64
    kinds = [0, k, 1, 15, 16, 17, 255, 256, 257, 3]
    cols = []
    for o in range(45):  # d_out not a multiple of the 32-column CTA tile
        n = kinds[o % len(kinds)]
        cols.append(np.sort(rng.choice(k, size=n, replace=False)))
    cols[7] = np.array([0, 600, 1007])  # empty segments in between
    cols[8] = np.arange(240, 272)  # one block straddling a segment boundary
    C = _custom_layer(k, 45, cols)
    D = synth.gen_dictionary(11, 0, 0, d_in, k)
    g, l = device_projection(D, C, max_tokens=32)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(11, 0, 0, M, d_in)
    y = run_forward(g, l, X)
    yr = oracle_forward(X, pd, pc, dense=True)
    assert_parity(y, yr, f"degenerate M={M}")
    assert np.all(y[:, 0] == 0.0)  # an empty column gives exact zeros


def test_smallest_shapes():
    D, C = _case(12, 0, 0, 0, 32, 16, 1, 1.0)
    g, l = device_projection(D, C, max_tokens=1)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(12, 0, 0, 1, 32)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc, dense=True), "smallest")


def test_all_zero_input_gives_zero():
    D, C = _case(13, 0, 0, 0, 256, 128, 64, 0.5)
    g, l = device_projection(D, C, max_tokens=4)
    y = run_forward(g, l, np.zeros((4, 256), np.float16))
    assert np.all(y == 0.0)


# ------------------------------------------------------------------ bit-exact packed bytes
def test_device_bytes_match_oracle_layout():
    D, C = _case(14, 0, 0, 0, 4096, 2048, 700, 0.3)
    g, l = device_projection(D, C, max_tokens=1)
    pd, pc = oracle_projection(D, C)
    eg = dp.dictproj_group_export(g)
    assert np.array_equal(eg["codes"], pd["codes"]) and np.array_equal(eg["scales"], pd["scales"])
    assert eg["s"] == pd["s"]
    el = dp.dictproj_layer_export(l)
    for n in ("col_ptr", "codes", "scales", "idx", "seg_start"):
        assert np.array_equal(el[n], pc[n]), n
    assert el["s"] == pc["s"]


# ------------------------------------------------------------------ determinism and graphs
def test_deterministic_bits(mid):
    g, l, pd, pc = mid
    X = synth.gen_activations(10, 99, 0, 8, 512)
    a = run_forward(g, l, X)
    b = run_forward(g, l, X)
    assert np.array_equal(a, b)


def test_cuda_graph_capture_and_side_stream(mid):
    g, l, pd, pc = mid
    X = torch.from_numpy(synth.gen_activations(10, 98, 0, 4, 512)).cuda()
    Y = torch.zeros((4, 300), dtype=torch.float16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dp.dictproj_forward(X.data_ptr(), 4, l, g, Y.data_ptr(), s.cuda_stream)  # warm-up
    s.synchronize()
    ref = Y.clone()
    Y.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        dp.dictproj_forward(X.data_ptr(), 4, l, g, Y.data_ptr(), s.cuda_stream)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, ref)
    yr = oracle_forward(X.cpu().numpy(), pd, pc, dense=True)
    assert_parity(Y.float().cpu().numpy().astype(np.float64), yr, "graph")


def test_chain_of_calls_sharing_a_group():
    # two layers of one group, the second reading the first's output: the
    # dependency wait must order Z scratch reuse and X reads
    D = synth.gen_dictionary(15, 0, 0, 256, 128)
    C1 = synth.gen_coeff(15, 0, 0, 0, 128, 256, 0.5)
    C2 = synth.gen_coeff(15, 0, 0, 1, 128, 256, 0.5)
    g = dp.dictproj_pack_group(D, 8)
    l1 = dp.dictproj_pack_layer(C1.col_ptr, C1.atom_idx, C1.vals, 128, 256)
    l2 = dp.dictproj_pack_layer(C2.col_ptr, C2.atom_idx, C2.vals, 128, 256)
    pd, pc1 = oracle_projection(D, C1)
    _, pc2 = oracle_projection(D, C2)
    X = torch.from_numpy(synth.gen_activations(15, 0, 0, 2, 256)).cuda()
    Y1 = torch.empty((2, 256), dtype=torch.float16, device="cuda")
    Y2 = torch.empty((2, 256), dtype=torch.float16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    for _ in range(3):
        dp.dictproj_forward(X.data_ptr(), 2, l1, g, Y1.data_ptr(), st)
        dp.dictproj_forward(Y1.data_ptr(), 2, l2, g, Y2.data_ptr(), st)
    torch.cuda.synchronize()
    y1 = Y1.float().cpu().numpy().astype(np.float64)
    assert_parity(y1, oracle_forward(X.cpu().numpy(), pd, pc1, dense=True), "chain 1")
    y2 = Y2.float().cpu().numpy().astype(np.float64)
    assert_parity(y2, oracle_forward(Y1.cpu().numpy(), pd, pc2, dense=True), "chain 2")


def test_full_and_stage_mask_calls_interleaved_on_one_group():
    # full calls, single calls and stage-mask calls share the group's Z scratch;
    # interleaved on one stream they stay ordered, in eager launches and in graph
    # replays, with no bounded wait giving up
    D = synth.gen_dictionary(20, 0, 0, 2048, 1024)
    C = synth.gen_coeff(20, 0, 0, 0, 1024, 1500, 0.3)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    Xn = [synth.gen_activations(20, i, 0, 2, 2048) for i in range(3)]
    Xs = [torch.from_numpy(x).cuda() for x in Xn]
    Y = torch.empty((2, 1500), dtype=torch.float16, device="cuda")
    outs = [torch.empty_like(Y) for _ in range(3)]
    s = torch.cuda.Stream()

    def seq():
        for i, x in enumerate(Xs):
            dp.dictproj_forward(x.data_ptr(), 2, l, g, outs[i].data_ptr(), s.cuda_stream)
            dp.dictproj_forward_batch_stages([x.data_ptr()], 2, [l], [g], [Y.data_ptr()], s.cuda_stream, 1)
            dp.dictproj_forward_batch_stages([x.data_ptr()], 2, [l], [g], [Y.data_ptr()], s.cuda_stream, 2)
            dp.dictproj_forward_batch([x.data_ptr()], 2, [l], [g], [Y.data_ptr()], s.cuda_stream)
    with torch.cuda.stream(s):
        seq()
    dp.dictproj_check(s.cuda_stream)
    first = [o.clone() for o in outs]
    for x, o in zip(Xn, outs):
        assert_parity(o.float().cpu().numpy().astype(np.float64), oracle_forward(x, pd, pc), "interleaved calls")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        seq()
    for o in outs:
        o.fill_(float("nan"))
    with torch.cuda.stream(s):
        for _ in range(20):
            graph.replay()
    dp.dictproj_check(s.cuda_stream)
    for a, b in zip(first, outs):
        assert torch.equal(a, b)


# ------------------------------------------------------------------ batched forward
@pytest.mark.parametrize("M", [1, 3, 8, 12])
def test_batch_matches_single_calls_bitwise(M):
    shapes = [(512, 256, 300, 0.3), (512, 256, 200, 0.25), (1024, 512, 96, 0.4)]
    projs = []
    for i, (d_in, k, d_out, rho) in enumerate(shapes):
        D = synth.gen_dictionary(16, i, 0, d_in, k)
        C = synth.gen_coeff(16, i, 0, 0, k, d_out, rho)
        g, l = device_projection(D, C, max_tokens=16)
        projs.append((g, l, d_in, d_out))
    Xs = [torch.from_numpy(synth.gen_activations(16, i, 0, M, d)).cuda() for i, (_, _, d, _) in enumerate(projs)]
    Xs[1] = Xs[0]  # q/k/v style: two projections read the same activation
    Ys = [torch.empty((M, do), dtype=torch.float16, device="cuda") for (_, _, _, do) in projs]
    Yr = [torch.empty((M, do), dtype=torch.float16, device="cuda") for (_, _, _, do) in projs]
    st = torch.cuda.current_stream().cuda_stream
    dp.dictproj_forward_batch([x.data_ptr() for x in Xs], M, [p[1] for p in projs], [p[0] for p in projs],
                              [y.data_ptr() for y in Ys], st)
    for (g, l, _, _), x, y in zip(projs, Xs, Yr):
        dp.dictproj_forward(x.data_ptr(), M, l, g, y.data_ptr(), st)
    torch.cuda.synchronize()
    for a, b in zip(Ys, Yr):
        assert torch.equal(a, b)


@pytest.mark.parametrize("M", [1, 8])
def test_mixed_shape_batch_with_byte_proportional_grid(M):
    # LLaMA-7B shapes of different sizes in one call: the dictionary grid shares a
    # J that differs from some lone plans and the gather CTAs follow stored
    # entries; each output still meets the oracle bar, and the stage-mask calls
    # (dictionary kernel, then coefficient kernel) reproduce the full call bit for bit
    shapes = [(4096, 2048, 4096, 0.3), (11008, 3072, 4096, 0.25), (4096, 3072, 11008, 0.25)]
    projs, refs = [], []
    for i, (d_in, k, d_out, rho) in enumerate(shapes):
        D, C = _case(19, i, i, 0, d_in, k, d_out, rho)
        g, l = device_projection(D, C, max_tokens=8)
        projs.append((g, l, d_in, d_out))
        refs.append(oracle_projection(D, C))
    Xn = [synth.gen_activations(19, i, 0, M, d) for i, (_, _, d, _) in enumerate(projs)]
    Xs = [torch.from_numpy(x).cuda() for x in Xn]
    Ys = [torch.full((M, do), float("nan"), dtype=torch.float16, device="cuda") for (_, _, _, do) in projs]
    args = ([x.data_ptr() for x in Xs], M, [p[1] for p in projs], [p[0] for p in projs])
    st = torch.cuda.current_stream().cuda_stream
    dp.dictproj_forward_batch(*args, [y.data_ptr() for y in Ys], st)
    torch.cuda.synchronize()
    for y, x, (pd, pc), i in zip(Ys, Xn, refs, range(3)):
        assert_parity(y.float().cpu().numpy().astype(np.float64), oracle_forward(x, pd, pc), f"mixed batch {i} M={M}")
    Y2 = [torch.full_like(y, float("nan")) for y in Ys]
    dp.dictproj_forward_batch_stages(*args, [y.data_ptr() for y in Y2], st, 1)
    torch.cuda.synchronize()
    assert all(torch.isnan(y.float()).all() for y in Y2)  # the dictionary kernel alone writes no output
    dp.dictproj_forward_batch_stages(*args, [y.data_ptr() for y in Y2], st, 2)
    torch.cuda.synchronize()
    for a, b in zip(Ys, Y2):
        assert torch.equal(a, b)
    for bad in (0, 4):
        with pytest.raises(dp.DictprojError) as e:
            dp.dictproj_forward_batch_stages(*args, [y.data_ptr() for y in Y2], st, bad)
        assert e.value.status == -5
    plan = dp.dictproj_decode_batch_plan(
        [(d_in, k, d_out, int(np.asarray(pc["col_ptr"])[-1])) for (d_in, k, d_out, _), (_, pc) in zip(shapes, refs)],
        M, torch.cuda.get_device_properties(0).multi_processor_count)
    assert all(p["dict_ctas"] >= 1 and p["coeff_ctas"] >= 1 for p in plan)


def test_batched_projections_finish_together():
    # a q/k/v-like batch (4096 -> 32768 columns, so that the work spans tens of
    # microseconds against the global timer's ticks) with C densities 0.2 / 0.3 /
    # 0.4: the gather kernel hands its CTAs out so that the projection that would
    # finish last gets the next one (a warp takes whole columns; a column costs two
    # 256-entry windows plus its windows). Measured from the start of their column
    # work (device timestamps of the gather kernel's CTAs, median of 5 launches),
    # the three projections finish within 10% of each other, and within 10% of
    # the spread that cost predicts
    rhos = (0.2, 0.3, 0.4)
    projs = []
    for i, rho in enumerate(rhos):
        D, C = _case(24, i, i, 0, 4096, 2048, 32768, rho)
        projs.append(device_projection(D, C, max_tokens=8))
    X = torch.from_numpy(synth.gen_activations(24, 0, 0, 1, 4096)).cuda()
    Ys = [torch.empty((1, 32768), dtype=torch.float16, device="cuda") for _ in rhos]
    st = torch.cuda.current_stream().cuda_stream
    call = lambda: dp.dictproj_forward_batch([X.data_ptr()] * 3, 1, [p[1] for p in projs], [p[0] for p in projs],
                                             [y.data_ptr() for y in Ys], st)
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    totals = [dp.dictproj_layer_info(l)["total"] for _, l in projs]
    plan = dp.dictproj_decode_batch_plan([(4096, 2048, 32768, t) for t in totals], 1, n_sm)
    ctas = [p["coeff_ctas"] for p in plan]
    model = [-(-(-(-32768 // n)) // 32) * (2 + (t / 32768 + 128) / 256) for n, t in zip(ctas, totals)]
    buf = torch.zeros(2 * sum(ctas), dtype=torch.int64, device="cuda")
    call()
    torch.cuda.synchronize()
    ratios, last = [], []
    dp.dictproj_diag_gather_times(buf.data_ptr(), sum(ctas))
    try:
        for _ in range(5):
            buf.zero_()
            call()
            torch.cuda.synchronize()
            t = buf.view(-1, 2).cpu().numpy().astype(np.float64)
            assert np.all(t[:, 1] >= t[:, 0]) and np.all(t[:, 0] > 0)
            start, b, ends = t[:, 0].min(), 0, []
            for n in ctas:
                ends.append(t[b:b + n, 1].max() - start)
                b += n
            ratios.append(max(ends) / min(ends))
            last.append(ends)
    finally:
        dp.dictproj_diag_gather_times(0, 0)
    r = float(np.median(ratios))
    assert r <= 1.10 and r <= max(model) / min(model) * 1.10, (ratios, model, ctas, last)


def test_batch_rejects_repeated_group():
    D = synth.gen_dictionary(17, 0, 0, 64, 32)
    C = synth.gen_coeff(17, 0, 0, 0, 32, 16, 0.5)
    g, l = device_projection(D, C, max_tokens=2)
    X = torch.zeros((1, 64), dtype=torch.float16, device="cuda")
    Y = torch.zeros((1, 16), dtype=torch.float16, device="cuda")
    with pytest.raises(dp.DictprojError) as e:
        dp.dictproj_forward_batch([X.data_ptr()] * 2, 1, [l, l], [g, g], [Y.data_ptr()] * 2, 0)
    assert e.value.status == -4


# ------------------------------------------------------------------ long columns
@pytest.mark.parametrize("M", [1, 3])
def test_columns_longer_than_1024_entries(M):
    # k = 3072 at density 0.4 stores 1229 entries per column (1232 padded): the
    # gather kernel holds such a column in five 256-entry windows, the last one
    # past entry 1024
    D, C = _case(18, 0, 0, 0, 512, 3072, 96, 0.4)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    assert int(np.diff(pc["col_ptr"]).max()) > 1024
    X = synth.gen_activations(18, 0, 0, M, 512)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc), f"long columns M={M}")


# ------------------------------------------------------------------ layers the gather kernel does not hold
@pytest.mark.parametrize("M", [1, 3, 8])
def test_columns_longer_than_1280_entries(M):
    # k = 3072 at density 0.9 stores 2765 entries per column (2768 padded),
    # beyond the gather kernel's 1280; dictproj_forward routes the layer to the
    # direct coefficient kernel
    D, C = _case(19, 0, 0, 0, 256, 3072, 64, 0.9)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    assert int(np.diff(pc["col_ptr"]).max()) > 1280
    X = synth.gen_activations(19, 0, 0, M, 256)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc), f"columns > 1280 entries M={M}")


@pytest.mark.parametrize("M", [1, 3, 4])
def test_more_than_32_segments(M):
    # k = 8448 has 33 segments of 256 atoms (the gather holds at most 32): the
    # layer runs on the direct coefficient kernel
    D, C = _case(20, 0, 0, 0, 256, 8448, 64, 0.05)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    assert pc["nseg"] == 33
    X = synth.gen_activations(20, 0, 0, M, 256)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc), f"33 segments M={M}")


def test_k_beyond_shared_memory_is_rejected_before_launch():
    # (k + 256) * 8 floats of Z exceed the per-block shared memory at M = 8 for
    # k = 8192: UNSUPPORTED, nothing launched; k = 7008 is the largest that fits
    D, C = _case(21, 0, 0, 0, 64, 8192, 32, 0.02)
    g, l = device_projection(D, C, max_tokens=8)
    X = torch.zeros((8, 64), dtype=torch.float16, device="cuda")
    Y = torch.full((8, 32), 3.0, dtype=torch.float16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert dp.dictproj_forward_status(X.data_ptr(), 8, l.handle, g.handle, Y.data_ptr(), st) == -9
    assert "shared memory" in dp.dictproj_last_error()
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)
    assert dp.dictproj_forward_status(X.data_ptr(), 4, l.handle, g.handle, Y.data_ptr(), st) == 0
    torch.cuda.synchronize()
    assert torch.all(Y[:4] == 0.0)


@pytest.mark.parametrize("M", [1, 8])
def test_largest_k_that_fits_at_m8(M):
    D, C = _case(22, 0, 0, 0, 64, 7008, 48, 0.05)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(22, 0, 0, M, 64)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc), f"k=7008 M={M}")


# ------------------------------------------------------------------ partial 128-element units of d_in
@pytest.mark.parametrize("d_in", [160, 4128])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_decode_d_in_not_a_multiple_of_128(d_in, M):
    D, C = _case(23, 0, 0, 0, d_in, 512, 200, 0.3)
    g, l = device_projection(D, C, max_tokens=8)
    pd, pc = oracle_projection(D, C)
    X = synth.gen_activations(23, 0, 0, M, d_in)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc, dense=True), f"d_in={d_in} M={M}")


# ------------------------------------------------------------------ bounded waits
def test_bounded_wait_times_out_and_the_device_stays_usable(mid):
    g, l, pd, pc = mid
    st = torch.cuda.current_stream().cuda_stream
    assert dp.dictproj_check_status(st) == 0
    dp.dictproj_selftest_wait_timeout(1 << 20, st)  # ~0.5 ms at 2 GHz; nothing can complete the wait
    assert dp.dictproj_check_status(st) == -8
    assert "gave up" in dp.dictproj_last_error()
    assert dp.dictproj_check_status(st) == 0  # the word was cleared
    X = synth.gen_activations(10, 77, 0, 2, 512)
    assert_parity(run_forward(g, l, X), oracle_forward(X, pd, pc, dense=True), "after a timeout")
    assert dp.dictproj_check_status(st) == 0
