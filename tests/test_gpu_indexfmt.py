"""Bitmap (Eq. (12), a = 0, h = 1) and block-structured C_l through the C ABI,
against the fp64 oracle's own packings: device bytes identical to the oracle's
layouts, decode (M <= 8, the two-kernel path with each format's coefficient
kernel) and prefill (each format's densify kernel, the shared tcgen05 GEMM)
within tolerance, batches mixing index formats, CUDA-graph replay, and the
calls that do not take these layers refused before any launch."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dictionary_compressed_linear_b200 as dp  # noqa: E402
from gpu_helpers import assert_parity, run_forward  # noqa: E402
from oracle import forward as F  # noqa: E402
from oracle.pack import pack_coeff_bitmap, pack_coeff_blocks, pack_dictionary  # noqa: E402


def _custom(k, d_out, cols, seed=0):
    rng = np.random.default_rng(seed)
    ptr = np.zeros(d_out + 1, np.int32)
    ptr[1:] = np.cumsum([c.size for c in cols])
    atoms = np.concatenate(cols).astype(np.int32) if cols else np.zeros(0, np.int32)
    vals = (rng.standard_normal(atoms.size) / np.sqrt(k)).astype(np.float32)
    return synth.SparseCoeff(k=k, d_out=d_out, col_ptr=ptr, atom_idx=atoms, vals=vals)


def _bitmap_proj(seed, d_in, k, d_out, rho, max_tokens=8, C=None):
    D = synth.gen_dictionary(70, seed, 0, d_in, k)
    C = C if C is not None else synth.gen_coeff(70, seed, 0, 0, k, d_out, rho)
    g = dp.dictproj_pack_group(D, max_tokens)
    l = dp.dictproj_pack_layer_bitmap(C.col_ptr, C.atom_idx, C.vals, k, C.d_out)
    if max_tokens > 8:
        dp.dictproj_group_reserve_prefill(g, C.d_out)
    return g, l, pack_dictionary(D), pack_coeff_bitmap(C.col_ptr, C.atom_idx, C.vals, k, C.d_out)


def _blocks_proj(seed, d_in, k, d_out, rho, max_tokens=8, C=None):
    D = synth.gen_dictionary(71, seed, 0, d_in, k)
    C = C if C is not None else synth.gen_coeff_blocks(71, seed, 0, 0, k, d_out, rho)
    g = dp.dictproj_pack_group(D, max_tokens)
    l = dp.dictproj_pack_layer_blocks(C.col_ptr, C.atom_idx, C.vals, k, C.d_out)
    if max_tokens > 8:
        dp.dictproj_group_reserve_prefill(g, C.d_out)
    return g, l, pack_dictionary(D), pack_coeff_blocks(C.col_ptr, C.atom_idx, C.vals, k, C.d_out)


def test_device_bytes_match_the_oracle():
    g, l, _, pb = _bitmap_proj(1, 512, 2080, 300, 0.3)
    assert dp.dictproj_layer_index_format(l) == "bitmap"
    e = dp.dictproj_layer_export_bitmap(l)
    for n in ("col_ptr", "codes", "scales", "bitmap"):
        assert np.array_equal(e[n], np.asarray(pb[n]).reshape(-1)), n
    assert e["s"] == pb["s"]
    g, l, _, pk = _blocks_proj(2, 512, 2048, 300, 0.3)
    assert dp.dictproj_layer_index_format(l) == "blocks"
    e = dp.dictproj_layer_export_blocks(l)
    for n in ("blk_ptr", "blk_idx", "codes", "scales"):
        assert np.array_equal(e[n], np.asarray(pk[n]).reshape(-1)), n
    assert e["s"] == pk["s"]
    for exp in (dp.dictproj_layer_export, dp.dictproj_layer_export_bitmap):
        with pytest.raises(dp.DictprojError) as err:
            exp(l)
        assert err.value.status == -9


@pytest.mark.parametrize("d_in,k,d_out,rho,M", [
    (4096, 2048, 4096, 0.3, 1), (4096, 3072, 11008, 0.25, 1), (11008, 3072, 4096, 0.25, 1),
    (4096, 2048, 4096, 0.3, 3), (4096, 3072, 2048, 0.4, 8), (544, 48, 70, 0.5, 2),
    (1024, 8192, 64, 0.05, 1), (512, 256, 20, 1.0, 5)])
def test_bitmap_decode_parity(d_in, k, d_out, rho, M):
    g, l, pd, pb = _bitmap_proj(3, d_in, k, d_out, rho)
    X = synth.gen_activations(70, M, 0, M, d_in)
    assert_parity(run_forward(g, l, X), F.forward_factored_bitmap(X, pd, pb), f"bitmap decode M={M}")


@pytest.mark.parametrize("d_in,k,d_out,rho,M", [
    (4096, 2048, 4096, 0.3, 1), (4096, 3072, 11008, 0.25, 1), (11008, 3072, 4096, 0.25, 1),
    (4096, 2048, 4096, 0.3, 4), (4096, 3072, 2048, 0.4, 8), (544, 48, 70, 0.5, 2),
    (1024, 8192, 64, 0.05, 1), (512, 256, 20, 1.0, 5)])
def test_blocks_decode_parity(d_in, k, d_out, rho, M):
    g, l, pd, pk = _blocks_proj(4, d_in, k, d_out, rho)
    X = synth.gen_activations(71, M, 0, M, d_in)
    assert_parity(run_forward(g, l, X), F.forward_factored_blocks(X, pd, pk), f"blocks decode M={M}")


@pytest.mark.parametrize("M", [1, 8])
def test_degenerate_columns(M):
    k, d_in = 96, 256
    cols = [np.array([], np.int32), np.arange(k, dtype=np.int32), np.array([95], np.int32),
            np.array([0, 31, 32, 63, 64], np.int32), np.array([], np.int32)]
    C = _custom(k, len(cols), cols)
    g, l, pd, pb = _bitmap_proj(5, d_in, k, 0, 0.0, C=C)
    X = synth.gen_activations(72, M, 0, M, d_in)
    y = run_forward(g, l, X)
    assert_parity(y, F.forward_factored_bitmap(X, pd, pb), f"bitmap degenerate M={M}")
    assert np.all(y[:, 0] == 0) and np.all(y[:, 4] == 0)
    bcols = [np.array([], np.int32), np.arange(k, dtype=np.int32), np.arange(80, 96, dtype=np.int32),
             np.concatenate([np.arange(0, 16), np.arange(48, 64)]).astype(np.int32), np.array([], np.int32)]
    C = _custom(k, len(bcols), bcols)
    g, l, pd, pk = _blocks_proj(6, d_in, k, 0, 0.0, C=C)
    y = run_forward(g, l, X)
    assert_parity(y, F.forward_factored_blocks(X, pd, pk), f"blocks degenerate M={M}")
    assert np.all(y[:, 0] == 0) and np.all(y[:, 4] == 0)


@pytest.mark.parametrize("M", [16, 200])
def test_prefill_parity(M):
    g, l, pd, pb = _bitmap_proj(7, 1024, 512, 768, 0.3, max_tokens=256)
    X = synth.gen_activations(73, M, 0, M, 1024, outlier_frac=0.01)
    assert_parity(run_forward(g, l, X), F.forward_factored_bitmap(X, pd, pb), f"bitmap prefill M={M}")
    g, l, pd, pk = _blocks_proj(8, 1024, 512, 768, 0.3, max_tokens=256)
    assert_parity(run_forward(g, l, X), F.forward_factored_blocks(X, pd, pk), f"blocks prefill M={M}")


def test_batch_mixing_index_formats_and_graph_replay():
    from oracle.pack import pack_coeff
    D = [synth.gen_dictionary(74, i, 0, 2048, 1024) for i in range(3)]
    C = [synth.gen_coeff(74, 0, 0, 0, 1024, 900, 0.3), synth.gen_coeff(74, 1, 0, 0, 1024, 900, 0.3),
         synth.gen_coeff_blocks(74, 2, 0, 0, 1024, 900, 0.3)]
    gs = [dp.dictproj_pack_group(d, 8) for d in D]
    ls = [dp.dictproj_pack_layer(C[0].col_ptr, C[0].atom_idx, C[0].vals, 1024, 900),
          dp.dictproj_pack_layer_bitmap(C[1].col_ptr, C[1].atom_idx, C[1].vals, 1024, 900),
          dp.dictproj_pack_layer_blocks(C[2].col_ptr, C[2].atom_idx, C[2].vals, 1024, 900)]
    refs = [lambda X, i=0: F.forward_factored(X, pack_dictionary(D[0]), pack_coeff(C[0].col_ptr, C[0].atom_idx, C[0].vals, 1024, 900)),
            lambda X: F.forward_factored_bitmap(X, pack_dictionary(D[1]), pack_coeff_bitmap(C[1].col_ptr, C[1].atom_idx, C[1].vals, 1024, 900)),
            lambda X: F.forward_factored_blocks(X, pack_dictionary(D[2]), pack_coeff_blocks(C[2].col_ptr, C[2].atom_idx, C[2].vals, 1024, 900))]
    X_np = synth.gen_activations(75, 0, 0, 2, 2048)
    X = torch.from_numpy(X_np).cuda()
    Ys = [torch.full((2, 900), float("nan"), dtype=torch.float16, device="cuda") for _ in range(3)]
    s = torch.cuda.Stream()
    call = lambda: dp.dictproj_forward_batch([X.data_ptr()] * 3, 2, ls, gs, [y.data_ptr() for y in Ys], s.cuda_stream)
    with torch.cuda.stream(s):
        call()
    s.synchronize()
    first = [y.clone() for y in Ys]
    for y, ref in zip(Ys, refs):
        assert_parity(y.float().cpu().numpy().astype(np.float64), ref(X_np), "mixed index formats")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        call()
    for y in Ys:
        y.fill_(float("nan"))
    with torch.cuda.stream(s):
        for _ in range(3):
            graph.replay()
    s.synchronize()
    for a, b in zip(first, Ys):
        assert torch.equal(a, b)  # replays are bit-identical to the eager call


def test_calls_that_do_not_take_index_layers_refuse():
    g, l, _, _ = _bitmap_proj(9, 512, 512, 64, 0.3)
    X = torch.zeros((1, 512), dtype=torch.float16, device="cuda")
    Y = torch.full((1, 64), 3.0, dtype=torch.float16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    dp.dictproj_set_decode_kernels(dp.DECODE_FUSED)
    try:
        assert dp.dictproj_forward_status(X.data_ptr(), 1, l.handle, g.handle, Y.data_ptr(), st) == -9
    finally:
        dp.dictproj_set_decode_kernels(dp.DECODE_AUTO)
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)
    with pytest.raises(dp.DictprojError) as err:
        dp.dictproj_layer_save(l, "/tmp/never-written-bitmap.dpj")
    assert err.value.status == -9
