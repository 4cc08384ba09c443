"""Full-size parity in the launch configuration the benchmark times.

The first two layers of the LLaMA-7B-shaped stack (one group of each of the 7
projection types: 4096 x 4096 with k = 2048, 4096 -> 11008 and 11008 -> 4096
with k = 3072, densities drawn in [0.2, 0.4]) run exactly as bench.py runs a
decode step: q/k/v and gate/up batched into one call each, the step captured in
a CUDA graph and replayed. Every output of every projection is compared with the oracle's
fp64 factored forward, computed from the oracle's own packing of the same
seeded factors."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU container
    pytest.skip("needs a CUDA device", allow_module_level=True)

import bench  # noqa: E402
import dictionary_compressed_linear_b200 as dp  # noqa: E402
from oracle import forward as F  # noqa: E402
from oracle.pack import pack_coeff, pack_dictionary  # noqa: E402


def test_first_group_of_the_stack_in_the_bench_launch_configuration():
    wl = synth.full_step(n_layers=2)
    stack = bench.Stack(wl, 1, torch, dp, lambda msg: None)
    s = torch.cuda.Stream()
    graph = bench.capture(torch, s, lambda: stack.forward_all(dp, s.cuda_stream, batched=True))
    stack.y.fill_(float("nan"))
    with torch.cuda.stream(s):
        graph.replay()
    s.synchronize()
    y = stack.y.float().cpu().numpy().astype(np.float64)
    del graph
    packed = {}
    for i, p in enumerate(wl.projections):
        D, C = synth.projection_inputs(p)
        if (p.group, p.ptype) not in packed:
            packed[(p.group, p.ptype)] = pack_dictionary(D)
        pd = packed[(p.group, p.ptype)]
        pc = pack_coeff(C.col_ptr, C.atom_idx, C.vals, p.k, p.d_out)
        X = synth.gen_activations(wl.cfg, p.layer, p.site, 1, p.d_in, wl.outlier_frac)
        ref = F.forward_factored(X, pd, pc)[0]
        got = y[stack.y_off[i]:stack.y_off[i] + p.d_out]
        ok, rf, worst = F.within_tolerance(got, ref)
        assert ok, f"{p.name} layer {p.layer}: rel-Frobenius {rf:.3e}, worst {worst:.3f}"
