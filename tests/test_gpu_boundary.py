"""Boundary behaviour of the C ABI on a GPU: every invalid call returns its
documented status before any launch (the output buffer is left untouched),
and host-injected faults leave nothing allocated."""
import os
import subprocess
import sys

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import dictionary_compressed_linear_b200 as dp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def proj():
    D = synth.gen_dictionary(20, 0, 0, 256, 128)
    C = synth.gen_coeff(20, 0, 0, 0, 128, 64, 0.5)
    g = dp.dictproj_pack_group(D, 4)
    l = dp.dictproj_pack_layer(C.col_ptr, C.atom_idx, C.vals, 128, 64)
    D2 = synth.gen_dictionary(20, 1, 0, 256, 64)
    g2 = dp.dictproj_pack_group(D2, 4)
    return g, l, g2


def _status(X, M, l, g, Y, path=dp.PATH_AUTO):
    return dp.dictproj_forward_status(X, M, l.handle if l else None, g.handle if g else None, Y,
                                      torch.cuda.current_stream().cuda_stream, path)


def test_invalid_calls_return_codes_and_do_not_launch(proj):
    g, l, g2 = proj
    X = torch.zeros((8, 256 + 8), dtype=torch.float16, device="cuda")
    Y = torch.full((8, 64 + 8), 7.0, dtype=torch.float16, device="cuda")
    x, y = X.data_ptr(), Y.data_ptr()
    assert _status(0, 1, l, g, y) == -1
    assert _status(x, 1, None, g, y) == -1
    assert _status(x, 0, l, g, y) == -5
    assert _status(x, 5, l, g, y) == -5  # above max_tokens = 4
    assert _status(x, 1, l, g2, y) == -4  # k mismatch
    assert _status(x + 2, 1, l, g, y) == -3
    assert _status(x, 1, l, g, y + 8) == -3
    assert _status(x, 1, l, g, y, path=7) == -5
    torch.cuda.synchronize()
    assert torch.all(Y == 7.0)  # nothing was written
    assert _status(x, 1, l, g, y) == 0


def test_decode_path_refuses_large_m():
    D = synth.gen_dictionary(21, 0, 0, 64, 32)
    C = synth.gen_coeff(21, 0, 0, 0, 32, 16, 0.5)
    g = dp.dictproj_pack_group(D, 16)
    l = dp.dictproj_pack_layer(C.col_ptr, C.atom_idx, C.vals, 32, 16)
    X = torch.zeros((16, 64), dtype=torch.float16, device="cuda")
    Y = torch.zeros((16, 16), dtype=torch.float16, device="cuda")
    assert dp.dictproj_forward_status(X.data_ptr(), 9, l.handle, g.handle, Y.data_ptr(), 0,
                                      dp.PATH_DECODE) == -9


def test_shape_errors_at_creation():
    with pytest.raises(dp.DictprojError) as e:
        dp.dictproj_pack_group(np.ones((48, 16), np.float32), 1)  # d_in % 32 != 0
    assert e.value.status == -2
    with pytest.raises(dp.DictprojError) as e:
        dp.dictproj_pack_group(np.ones((64, 24), np.float32), 1)  # k % 16 != 0
    assert e.value.status == -2
    with pytest.raises(dp.DictprojError) as e:
        dp.dictproj_pack_group(np.ones((64, 32), np.float32), 0)
    assert e.value.status == -5
    with pytest.raises(dp.DictprojError) as e:
        dp.dictproj_pack_layer(np.array([0, 1]), np.array([40]), np.ones(1, np.float32), 32, 1)
    assert e.value.status == -5


def test_upload_rejects_corrupt_layout():
    C = synth.gen_coeff(22, 0, 0, 0, 512, 8, 0.3)
    pc = dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, 512, 8)
    bad = dict(pc, col_ptr=pc["col_ptr"].copy())
    bad["col_ptr"][3] += 8  # not a multiple of 16
    with pytest.raises(dp.DictprojError) as e:
        dp.dictproj_layer_upload(bad)
    assert e.value.status == -5
    bad = dict(pc, seg_start=pc["seg_start"].copy())
    bad["seg_start"][1] = 60000
    with pytest.raises(dp.DictprojError) as e:
        dp.dictproj_layer_upload(bad)
    assert e.value.status == -5


@pytest.mark.parametrize("kind,status", [("alloc", -7), ("copy", -6)])
def test_injected_host_faults(kind, status):
    code = (
        "import numpy as np, torch, dictionary_compressed_linear_b200 as dp\n"
        "torch.cuda.init()\n"
        "free0 = torch.cuda.mem_get_info()[0]\n"
        "for _ in range(20):\n"
        "    try:\n"
        "        dp.dictproj_pack_group(np.ones((4096, 2048), np.float32), 8)\n"
        "        raise SystemExit('no error')\n"
        "    except dp.DictprojError as e:\n"
        f"        assert e.status == {status}, e\n"
        "free1 = torch.cuda.mem_get_info()[0]\n"
        "assert free0 - free1 < 64 << 20, (free0, free1)\n"
        "print('ok')\n")
    env = dict(os.environ, DICTPROJ_FAULT=kind, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


def test_pack_convenience_all_or_nothing():
    D = synth.gen_dictionary(23, 0, 0, 64, 32)
    good = synth.gen_coeff(23, 0, 0, 0, 32, 8, 0.5)
    g, ls = dp.dictproj_pack(D, 2, [(good.col_ptr, good.atom_idx, good.vals, 8)] * 2)
    assert len(ls) == 2 and g.handle and all(l.handle for l in ls)
    with pytest.raises(dp.DictprojError):
        dp.dictproj_pack(D, 2, [(good.col_ptr, good.atom_idx, good.vals, 8),
                                (np.array([0, 1]), np.array([99]), np.ones(1, np.float32), 1)])


def test_save_and_load_handles_through_files(tmp_path):
    D, C = synth.gen_dictionary(0, 0, 0, 512, 256), synth.gen_coeff(0, 0, 0, 0, 256, 384, 0.3)
    g = dp.dictproj_pack_group(D, 8)
    l = dp.dictproj_pack_layer(C.col_ptr, C.atom_idx, C.vals, 256, 384)
    dp.dictproj_group_save(g, str(tmp_path / "g.dpj"))
    dp.dictproj_layer_save(l, str(tmp_path / "l.dpj"))
    g2 = dp.dictproj_group_load(str(tmp_path / "g.dpj"), 8)
    l2 = dp.dictproj_layer_load(str(tmp_path / "l.dpj"))
    X = torch.from_numpy(synth.gen_activations(0, 0, 0, 3, 512)).cuda()
    st = torch.cuda.current_stream().cuda_stream
    Y1 = torch.empty((3, 384), dtype=torch.float16, device="cuda")
    Y2 = torch.full((3, 384), float("nan"), dtype=torch.float16, device="cuda")
    dp.dictproj_forward(X.data_ptr(), 3, l, g, Y1.data_ptr(), st)
    dp.dictproj_forward(X.data_ptr(), 3, l2, g2, Y2.data_ptr(), st)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
