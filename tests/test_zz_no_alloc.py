"""dictproj_forward_noalloc: the decode-path forward for callers that cannot
allocate device memory at call time (runtimes that reserve all device memory
up front in their own arena; work enqueued while a stream is being captured
into a CUDA graph). It keeps the Z scratch in a file-scope device array instead
of allocating, and must match the fp64 oracle (and dictproj_forward) on two
calls in a row.

The test itself allocates its inputs and outputs with torch; only the entry
point under test must not allocate. Collected last on purpose."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dictionary_compressed_linear_b200 as dp  # noqa: E402
from oracle.forward import forward_factored, within_tolerance  # noqa: E402
from oracle.pack import pack_coeff, pack_dictionary  # noqa: E402


def _device_views(pg, pc):
    """Caller-owned device copies of the packed bytes, and the C structs viewing them."""
    keep = {n: torch.from_numpy(np.ascontiguousarray(pg[n])).cuda() for n in ("codes", "scales")}
    for n in ("col_ptr", "codes", "scales", "idx", "seg_start"):
        a = np.ascontiguousarray(pc[n])
        if a.dtype == np.uint32:
            a = a.view(np.int32)
        elif a.dtype == np.uint16:
            a = a.view(np.int16)
        keep["c_" + n] = torch.from_numpy(a).cuda()
    g = dp.DeviceGroup(keep["codes"].data_ptr(), keep["scales"].data_ptr(), float(pg["s"]), pg["d_in"], pg["k"])
    l = dp.DeviceLayer(keep["c_col_ptr"].data_ptr(), keep["c_codes"].data_ptr(), keep["c_scales"].data_ptr(),
                       keep["c_idx"].data_ptr(), keep["c_seg_start"].data_ptr(), float(pc["s"]), pc["k"],
                       pc["d_out"])
    return g, l, keep


@pytest.mark.parametrize("d_in,k,d_out,rho,M", [
    (4096, 2048, 4096, 0.3, 1), (4096, 2048, 4096, 0.3, 8),  # attention projection
    (11008, 3072, 4096, 0.25, 3),                             # down projection
    (256, 128, 256, 0.5, 4),                                  # tiny shape
    (256, 3072, 64, 0.9, 1),                                  # columns of 2768 padded entries
    (256, 8448, 64, 0.05, 2),                                 # 33 segments of 256 atoms
])
def test_noalloc_matches_oracle_and_forward_twice(d_in, k, d_out, rho, M):
    D = synth.gen_dictionary(30, 0, 0, d_in, k)
    C = synth.gen_coeff(30, 0, 0, 0, k, d_out, rho)
    pg = dp.dictproj_pack_group_host(D)
    pc = dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    X_np = synth.gen_activations(30, 0, 0, M, d_in)
    X = torch.from_numpy(X_np).cuda()
    st = torch.cuda.current_stream().cuda_stream
    ref = forward_factored(X_np, pack_dictionary(D), pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out))
    g, l, keep = _device_views(pg, pc)
    outs = []
    for _ in range(2):  # two calls in a row share the static scratch
        Y = torch.full((M, d_out), float("nan"), dtype=torch.float16, device="cuda")
        dp.dictproj_forward_noalloc(g, l, X.data_ptr(), M, Y.data_ptr(), st)
        torch.cuda.synchronize()
        outs.append(Y.float().cpu().numpy().astype(np.float64))
    for y in outs:
        ok, rf, worst = within_tolerance(y, ref)
        assert ok, (rf, worst)
    assert np.array_equal(outs[0], outs[1])
    # and the allocating entry point agrees with it
    g_ref = dp.dictproj_group_upload(pg, 8)
    l_ref = dp.dictproj_layer_upload(pc)
    Y_ref = torch.empty((M, d_out), dtype=torch.float16, device="cuda")
    dp.dictproj_forward(X.data_ptr(), M, l_ref, g_ref, Y_ref.data_ptr(), st)
    torch.cuda.synchronize()
    ok, rf, worst = within_tolerance(outs[0], Y_ref.float().cpu().numpy().astype(np.float64))
    assert ok, (rf, worst)


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    # (k + 256) * 8 > 49152 for k = 6144 at M = 8; at M = 1 the same k fits
    d_in, k, d_out = 64, 6144, 16
    D = synth.gen_dictionary(31, 0, 0, d_in, k)
    C = synth.gen_coeff(31, 0, 0, 0, k, d_out, 0.01)
    pg = dp.dictproj_pack_group_host(D)
    pc = dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, k, d_out)
    g, l, keep = _device_views(pg, pc)
    X_np = synth.gen_activations(31, 0, 0, 8, d_in)
    X = torch.from_numpy(X_np).cuda()
    Y = torch.full((8, d_out), 3.0, dtype=torch.float16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert dp.dictproj_forward_noalloc_status(g, l, X.data_ptr(), 8, Y.data_ptr(), st) == -5
    assert "static scratch" in dp.dictproj_last_error()
    torch.cuda.synchronize()
    assert torch.all(Y == 3.0)
    assert dp.dictproj_forward_noalloc_status(g, l, X.data_ptr(), 1, Y.data_ptr(), st) == 0
    torch.cuda.synchronize()
    ref = forward_factored(X_np[:1], pack_dictionary(D), pack_coeff(C.col_ptr, C.atom_idx, C.vals, k, d_out))
    ok, rf, worst = within_tolerance(Y[:1].float().cpu().numpy().astype(np.float64), ref)
    assert ok, (rf, worst)
    assert torch.all(Y[1:] == 3.0)
