"""Shared helpers for the GPU tests: build projections through the C ABI and
compute the oracle's answer for the same packed factors."""
import numpy as np
import torch

import dictionary_compressed_linear_b200 as dp
from oracle import forward as F
from oracle.pack import pack_coeff, pack_dictionary


def device_projection(D, C, max_tokens):
    """(group, layer) on the GPU via the library's packer."""
    g = dp.dictproj_pack_group(D, max_tokens)
    l = dp.dictproj_pack_layer(C.col_ptr, C.atom_idx, C.vals, C.k, C.d_out)
    dp.dictproj_group_reserve_prefill(g, C.d_out)
    return g, l


def oracle_projection(D, C):
    return pack_dictionary(D), pack_coeff(C.col_ptr, C.atom_idx, C.vals, C.k, C.d_out)


def run_forward(g, l, X_np, path=dp.PATH_AUTO, stream=None):
    X = torch.from_numpy(np.ascontiguousarray(X_np)).cuda()
    M = X.shape[0]
    Y = torch.full((M, l.d_out), float("nan"), dtype=torch.float16, device="cuda")
    s = stream or torch.cuda.current_stream()
    dp.dictproj_forward_path(X.data_ptr(), M, l, g, Y.data_ptr(), s.cuda_stream, path)
    s.synchronize()
    return Y.float().cpu().numpy().astype(np.float64)


def oracle_forward(X_np, pd, pc, dense=False):
    if dense:
        return F.forward_reference(X_np, pd, pc)
    return F.forward_factored(X_np, pd, pc)


def assert_parity(y_gpu, y_ref, what=""):
    ok, rf, worst = F.within_tolerance(y_gpu, y_ref)
    assert ok, f"{what}: rel-Frobenius {rf:.3e} (bar 5e-3), worst |err|/(1e-2(1+|y|)) {worst:.3f} (bar 1)"
    return rf, worst
