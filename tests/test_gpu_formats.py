"""FP16 / FP8 / INT8 coefficient values (the paper's Table 4 formats, NVFP4
dictionary) through the C ABI, against the fp64 oracle's own packing.

The fused decode kernel and the prefill path decode every format; the device
bytes match the oracle's layout bit for bit; calls that no path serves for these
formats are refused before any launch."""
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
from oracle.pack import pack_coeff_fmt, pack_dictionary  # noqa: E402

FORMATS = ["fp16", "fp8", "int8"]


def _proj(seed, d_in, k, d_out, rho, fmt, max_tokens=8):
    D = synth.gen_dictionary(60, seed, 0, d_in, k)
    C = synth.gen_coeff(60, seed, 0, 0, k, d_out, rho)
    g = dp.dictproj_pack_group(D, max_tokens)
    l = dp.dictproj_pack_layer_fmt(C.col_ptr, C.atom_idx, C.vals, k, d_out, fmt)
    if max_tokens > 8:
        dp.dictproj_group_reserve_prefill(g, d_out)
    return g, l, pack_dictionary(D), pack_coeff_fmt(C.col_ptr, C.atom_idx, C.vals, k, d_out, fmt)


@pytest.mark.parametrize("fmt", FORMATS)
def test_device_bytes_match_the_oracle(fmt):
    g, l, pd, pf = _proj(1, 512, 2048, 700, 0.3, fmt)
    assert dp.dictproj_layer_format(l) == fmt
    e = dp.dictproj_layer_export_fmt(l)
    for n in ("col_ptr", "values", "idx", "seg_start"):
        assert np.array_equal(e[n], pf[n]), n
    assert e["s"] == pf["s"]
    with pytest.raises(dp.DictprojError) as err:
        dp.dictproj_layer_export(l)
    assert err.value.status == -9


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("d_in,k,d_out,rho,M", [(4096, 2048, 4096, 0.3, 1), (4096, 2048, 4096, 0.3, 3),
                                                (11008, 3072, 4096, 0.25, 1), (4096, 3072, 11008, 0.25, 8),
                                                (544, 512, 200, 0.5, 5)])
def test_decode_parity(fmt, d_in, k, d_out, rho, M):
    g, l, pd, pf = _proj(2, d_in, k, d_out, rho, fmt)
    X = synth.gen_activations(60, M, 0, M, d_in)
    assert_parity(run_forward(g, l, X), F.forward_factored_fmt(X, pd, pf), f"{fmt} decode M={M}")


def test_batch_of_mixed_formats():
    projs = [_proj(10 + i, 4096, 2048, 4096, 0.3, f) for i, f in enumerate(["nvfp4", "fp8", "int8", "fp16"])]
    X_np = synth.gen_activations(61, 0, 0, 2, 4096)
    X = torch.from_numpy(X_np).cuda()
    Ys = [torch.full((2, 4096), float("nan"), dtype=torch.float16, device="cuda") for _ in projs]
    dp.dictproj_forward_batch([X.data_ptr()] * 4, 2, [p[1] for p in projs], [p[0] for p in projs],
                              [y.data_ptr() for y in Ys], torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    for (g, l, pd, pf), y in zip(projs, Ys):
        assert_parity(y.float().cpu().numpy().astype(np.float64), F.forward_factored_fmt(X_np, pd, pf),
                      "mixed-format batch")


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("M", [16, 200])
def test_prefill_parity(fmt, M):
    g, l, pd, pf = _proj(3, 1024, 512, 768, 0.3, fmt, max_tokens=256)
    X = synth.gen_activations(62, M, 0, M, 1024, outlier_frac=0.01)
    assert_parity(run_forward(g, l, X), F.forward_factored_fmt(X, pd, pf), f"{fmt} prefill M={M}")


def test_paths_that_do_not_decode_the_format_refuse_before_launch():
    # k = 8448 (33 segments of 256 atoms) is beyond the fused kernel's range: the
    # two-kernel decode path reads NVFP4 only, so the call is refused and Y is untouched
    g, l, pd, pf = _proj(4, 256, 8448, 64, 0.05, "fp8")
    X = torch.zeros((1, 256), dtype=torch.float16, device="cuda")
    Y = torch.full((1, 64), 3.0, dtype=torch.float16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert dp.dictproj_forward_status(X.data_ptr(), 1, l.handle, g.handle, Y.data_ptr(), st) == -9
    assert "fused kernel" in dp.dictproj_last_error()
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)
    with pytest.raises(dp.DictprojError) as err:
        dp.dictproj_layer_save(l, "/tmp/never-written.dpj")
    assert err.value.status == -9
