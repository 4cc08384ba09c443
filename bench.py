#!/usr/bin/env python
"""Benchmark of the dictionary-compressed projection forward on B200.

Default workload: one decode step (M = 1 token) through the full LLaMA-7B-shaped
linear stack: 32 layers in 16 groups of 2, all 7 projection types (q, k, v, o,
gate, up, down), 112 NVFP4 dictionaries and 224 sparse NVFP4 coefficient
matrices with densities drawn uniformly in [0.2, 0.4], synthetic seeded data.
A step is the 224 dictproj_forward calls in model order, captured in one CUDA
graph. Packed weights total ~2.6 GB, far larger than L2, so every step streams
from HBM without an explicit flush.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). With N > 1 (torchrun, one process per GPU) every
rank runs an independent replica of the step (the path has no collective);
value = tokens of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "linear-layer decode tokens/s (LLaMA-7B shapes, M=1); HBM GB/s as % of peak"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------- accounting
def nnz_cols(p):
    return synth.nnz_per_column(p.k, p.rho)


def d_bytes(p):
    return p.d_in * p.k // 2 + p.d_in * p.k // 16 + 4


def c_bytes(p):
    n = nnz_cols(p)
    nseg = max(1, -(-p.k // 256))
    return 4 + p.d_out * (-(-n // 2) + -(-n // 16) + n + 2 * nseg + 4)


def stage_bytes(p, M):
    mp = 1 if M <= 1 else 2 if M <= 2 else 4 if M <= 4 else 8
    dict_stage = d_bytes(p) + 2 * M * p.d_in + 4 * p.k * mp
    coeff_stage = c_bytes(p) + 4 * p.k * mp + 2 * M * p.d_out
    return dict_stage, coeff_stage


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense fp16 tensor-core peak in TFLOP/s: the measured bf16 burst figure (fp16
    and bf16 dense MMA have the same rate), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops; fp16 dense rate is the same)"
    return 1590.0, "fallback 1590 TFLOP/s"


def kernel_source_hash(files=("decode.cu", "common.cuh"), region=None):
    """sha256 prefix of the kernel sources; `region` = (start marker, end marker)
    restricts the first file to the text between them (one kernel of a file)."""
    h = hashlib.sha256()
    for i, fn in enumerate(files):
        with open(os.path.join(ROOT, "dictionary_compressed_linear_b200", "csrc", fn), "rb") as f:
            data = f.read()
        if region and i == 0:
            a = data.find(region[0].encode())
            b = data.find(region[1].encode(), a + 1)
            if a < 0 or b < 0:
                return None
            data = data[a:b]
        h.update(data)
    return h.hexdigest()[:16]


def profiled(kernel_name, key="bytes_per_launch"):
    """A figure from the committed ncu summary (profiles/traffic.json), if the
    kernel's source is unchanged since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel_name)
    if not e:
        return None
    files = tuple(e.get("source_files", ["decode.cu", "common.cuh"]))
    region = tuple(e["source_region"]) if e.get("source_region") else None
    if e.get("source_hash") != kernel_source_hash(files, region):
        return None
    return e.get(key)


def profiled_traffic(kernel_name, algorithmic_bytes):
    """DRAM bytes of one launch: the measured DRAM / algorithmic byte ratio of the
    ncu capture, scaled to this launch's algorithmic bytes (traffic grows in
    proportion to the packed bytes a launch streams)."""
    r = profiled(kernel_name, "traffic_ratio")
    return None if r is None else int(round(r * algorithmic_bytes))


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(value, dist, device):
    """The largest `value` over all ranks (every rank gets it); `value` when there
    is no process group. Rank timings are combined this way: the job takes as
    long as its slowest replica."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank, world, ms):
    """Whole-job tokens/s of `world` independent replicas that took `ms` (the
    max over ranks) for `tokens_per_rank` tokens each."""
    return world * tokens_per_rank / (ms / 1e3)


# ----------------------------------------------------------------------------- per-shape decode rows
SHAPE_ROWS = (("q", 1, 0.3), ("k", 1, 0.3), ("v", 1, 0.3), ("o", 1, 0.3),
              ("gate", 2, 0.25), ("up", 2, 0.25), ("down", 2, 0.25))


def call_bytes(d_in, d_out, k, rho, M):
    """Algorithmic bytes of one projection call: packed D, packed C (u8 index,
    unpadded), X and Y."""
    n = synth.nnz_per_column(k, rho)
    nseg = max(1, -(-k // 256))
    return (d_in * k // 2 + d_in * k // 16 + 4 + 4 + d_out * (-(-n // 2) + -(-n // 16) + n + 2 * nseg + 4)
            + 2 * M * (d_in + d_out))


def per_shape_bench(torch, dp, stream, peak, tokens=(1, 8), reps=5):
    """Each LLaMA-7B projection shape alone (densities of the attention and MLP
    workloads: 0.3 and 0.25), one dictproj_forward per call, chained in a CUDA
    graph over R device copies of the packed weights whose total exceeds 4x the L2
    size, so that every call streams its weights from HBM."""
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    sh = stream.cuda_stream
    rows = {}
    for name, cfg, rho in SHAPE_ROWS:
        d_in, d_out, k = synth.LLAMA7B_SHAPES[name]
        pt = synth.PROJ_TYPES.index(name)
        D = synth.gen_dictionary(cfg, 0, pt, d_in, k)
        C = synth.gen_coeff(cfg, 0, pt, 0, k, d_out, rho)
        pg = dp.dictproj_pack_group_host(D)
        pc = dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, k, d_out)
        R = -(-4 * l2 // call_bytes(d_in, d_out, k, rho, 1)) + 1
        gs = [dp.dictproj_group_upload(pg, 8) for _ in range(R)]
        ls = [dp.dictproj_layer_upload(pc) for _ in range(R)]
        row = {"d_in": d_in, "d_out": d_out, "k": k, "density": rho, "weight_copies": R}
        for M in tokens:
            X = torch.from_numpy(synth.gen_activations(cfg, 0, synth.INPUT_SITE[name], M, d_in)).cuda()
            Y = torch.empty((M, d_out), dtype=torch.float16, device="cuda")

            def chain():
                for i in range(R):
                    dp.dictproj_forward(X.data_ptr(), M, ls[i], gs[i], Y.data_ptr(), sh)
            g = capture(torch, stream, chain)
            time_replays(torch, stream, g, 3)
            ms = time_replays(torch, stream, g, reps) / (reps * R)
            del g
            b = call_bytes(d_in, d_out, k, rho, M)
            gbs = b / (ms / 1e3) / 1e9
            row[f"M={M}"] = {"us_per_call": round(ms * 1e3, 3), "bytes_per_call": b, "GB/s": round(gbs, 1),
                             "frac": round(gbs / peak, 4),
                             "launches_per_call": dp.dictproj_launch_count([X.data_ptr()], M, [ls[0]], [gs[0]])}
        rows[name] = row
        del gs, ls
    return {"workload": "each projection shape alone: configs 1-2 (attention q/k/v/o 4096->4096 k=2048 density 0.3; "
                        "gate/up 4096->11008 and down 11008->4096, k=3072, density 0.25), M=1 and M=8, "
                        "one call per projection chained in a CUDA graph over R weight copies > 4x L2",
            "peak_GB/s": peak, "rows": rows}


# ----------------------------------------------------------------------------- prefill leg
PREFILL_SHAPES = ("q", "gate", "down")
PREFILL_TOKENS = (128, 512, 2048)


def prefill_inputs(name, M):
    """The prefill workload's inputs for one projection type at M tokens: D (fp32
    d_in x k), C (density 0.3) and X (fp16 M x d_in, 1% of channels x20)."""
    d_in, d_out, k = synth.LLAMA7B_SHAPES[name]
    pt = synth.PROJ_TYPES.index(name)
    D = synth.gen_dictionary(4, 0, pt, d_in, k)
    C = synth.gen_coeff(4, 0, pt, 0, k, d_out, 0.3)
    X = synth.gen_activations(4, 0, synth.INPUT_SITE[name], M, d_in, 0.01)
    return D, C, X


def prefill_bench(torch, dp, stream, tokens=PREFILL_TOKENS, reps=20):
    """Prefill (M tokens) of one projection of each LLaMA-7B shape class: the
    dictionary stage alone (tcgen05, the tensor-bound step) and the whole forward,
    timed with CUDA events over graphs of `reps` calls alternating two weight sets
    (C density 0.3, 1% of input channels x20, as in the prefill workload).
    TFLOP/s count the method's own work: 2 M d_in k for the dictionary stage and
    2 M (d_in k + nnz) for the forward (the dense-equivalent 2 M (d_in k + k d_out)
    that the densified coefficient GEMM executes is given beside it)."""
    sh = stream.cuda_stream
    peak, peak_src = measured_tensor_peak()
    out = {"workload": "prefill, M in {128, 512, 2048}: q (4096->4096, k=2048), gate (4096->11008, k=3072), "
                       "down (11008->4096, k=3072); C density 0.3; X fp16 N(0,1), 1% channels x20",
           "peak_tflops": peak, "peak_source": peak_src, "shapes": {}}
    for name in PREFILL_SHAPES:
        d_in, d_out, k = synth.LLAMA7B_SHAPES[name]
        D, C, _ = prefill_inputs(name, 1)
        nnz = int(C.col_ptr[-1])
        pg = dp.dictproj_pack_group_host(D)
        pc = dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, k, d_out)
        Mmax = max(tokens)
        gs = [dp.dictproj_group_upload(pg, Mmax) for _ in range(2)]
        for g in gs:
            dp.dictproj_group_reserve_prefill(g, d_out)
        ls = [dp.dictproj_layer_upload(pc) for _ in range(2)]
        res = {}
        for M in tokens:
            X = torch.from_numpy(prefill_inputs(name, M)[2]).cuda()
            Z = torch.empty((M, k), dtype=torch.float16, device="cuda")
            Y = torch.empty((M, d_out), dtype=torch.float16, device="cuda")
            r = {}
            for what in ("dictionary_stage", "forward"):
                def chain():
                    for i in range(reps):
                        if what == "dictionary_stage":
                            dp.dictproj_dictionary_stage_prefill(X.data_ptr(), M, gs[i % 2], Z.data_ptr(), sh)
                        else:
                            dp.dictproj_forward(X.data_ptr(), M, ls[i % 2], gs[i % 2], Y.data_ptr(), sh)
                g = capture(torch, stream, chain)
                time_replays(torch, stream, g, 3)
                ms = time_replays(torch, stream, g, 5) / (5 * reps)
                del g
                flops = 2.0 * M * d_in * k + (2.0 * M * nnz if what == "forward" else 0.0)
                tf = flops / (ms / 1e3) / 1e12
                r[what] = {"us": round(ms * 1e3, 2), "TFLOP/s": round(tf, 1), "frac": round(tf / peak, 4),
                           "flops": flops}
                if what == "forward":
                    dense = 2.0 * M * (d_in * k + k * d_out)
                    r[what]["dense_equivalent_TFLOP/s"] = round(dense / (ms / 1e3) / 1e12, 1)
            if M == 2048:
                r["dictionary_stage"]["tensor_pipe_util_ncu"] = profiled(f"k_dict_prefill:{name}", "tensor_util")
            res[f"M={M}"] = r
        out["shapes"][name] = res
        del gs, ls
    return out


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- workload
def _pack_group_worker(spec):
    cfg, group, ptype, d_in, k = spec
    import dictionary_compressed_linear_b200 as dp
    D = synth.gen_dictionary(cfg, group, ptype, d_in, k)
    return spec, dp.dictproj_pack_group_host(D)


def _pack_layer_worker(spec):
    i, cfg, group, ptype, layer, k, d_out, rho = spec
    import dictionary_compressed_linear_b200 as dp
    C = synth.gen_coeff(cfg, group, ptype, layer, k, d_out, rho)
    return i, dp.dictproj_pack_layer_host(C.col_ptr, C.atom_idx, C.vals, k, d_out)


class Stack:
    """The packed weights of the linear stack on one GPU, plus activation buffers.

    Generation and host packing run in a spawn-started process pool; the main
    process only uploads the packed bytes."""

    def __init__(self, workload, M, torch, dp, log):
        import multiprocessing as mp
        self.w, self.M = workload, M
        t0 = time.time()
        gspecs = {}
        for p in workload.projections:
            gspecs.setdefault((p.group, p.ptype), (p.cfg, p.group, p.ptype, p.d_in, p.k))
        lspecs = [(i, p.cfg, p.group, p.ptype, p.layer, p.k, p.d_out, p.rho)
                  for i, p in enumerate(workload.projections)]
        self.groups, self.layers = {}, [None] * len(lspecs)
        nproc = max(1, min(len(os.sched_getaffinity(0)), 16))
        with mp.get_context("spawn").Pool(nproc) as pool:
            for spec, packed in pool.imap_unordered(_pack_group_worker, list(gspecs.values())):
                self.groups[(spec[1], spec[2])] = dp.dictproj_group_upload(packed, max(M, 8))
            for i, packed in pool.imap_unordered(_pack_layer_worker, lspecs):
                self.layers[i] = dp.dictproj_layer_upload(packed)
        log(f"packed {len(self.groups)} dictionaries and {len(self.layers)} coefficient matrices "
            f"in {time.time() - t0:.1f}s ({nproc} processes)")
        # one contiguous activation buffer per direction; every slice 256-byte aligned
        sites = {}
        off = 0
        for p in workload.projections:
            key = (p.layer, p.site)
            if key not in sites:
                sites[key] = (off, p.d_in)
                off += -(-M * p.d_in // 128) * 128
        self.x_off = sites
        self.x_elems = off
        self.y_off = []
        off = 0
        for p in workload.projections:
            self.y_off.append(off)
            off += -(-M * p.d_out // 128) * 128
        self.y_elems = off
        xh = np.zeros(self.x_elems, np.float16)
        for (layer, site), (o, d_in) in sites.items():
            x = synth.gen_activations(workload.cfg, layer, site, M, d_in, workload.outlier_frac)
            xh[o:o + M * d_in] = x.reshape(-1)
        self.x_host = torch.from_numpy(xh).pin_memory()
        self.x = self.x_host.cuda()
        self.y = torch.zeros(self.y_elems, dtype=torch.float16, device="cuda")
        self.y_host = torch.zeros(self.y_elems, dtype=torch.float16).pin_memory()

    def call_groups(self, batched):
        """Projections issued together: the ones of one layer reading the same input
        (q/k/v, gate/up) when batched, else one call per projection."""
        calls, cur = [], []
        for i, p in enumerate(self.w.projections):
            if cur and (not batched or (p.layer, p.site) != cur[-1][1]):
                calls.append([j for j, _ in cur])
                cur = []
            cur.append((i, (p.layer, p.site)))
        if cur:
            calls.append([j for j, _ in cur])
        return calls

    def calls(self, batched):
        """(X pointers, layers, groups, Y pointers) of every call of the step, in order."""
        xp, yp = self.x.data_ptr(), self.y.data_ptr()
        out = []
        for call in self.call_groups(batched):
            xs, ls, gs, ys = [], [], [], []
            for i in call:
                p = self.w.projections[i]
                xs.append(xp + 2 * self.x_off[(p.layer, p.site)][0])
                ls.append(self.layers[i])
                gs.append(self.groups[(p.group, p.ptype)])
                ys.append(yp + 2 * self.y_off[i])
            out.append((xs, ls, gs, ys))
        return out

    def launches_per_step(self, dp, batched=True):
        """Kernels one step launches, as the library reports for each of its calls."""
        return sum(dp.dictproj_launch_count(xs, self.M, ls, gs) for xs, ls, gs, _ in self.calls(batched))

    def forward_all(self, dp, stream_handle, batched=True):
        for xs, ls, gs, ys in self.calls(batched):
            if len(ls) == 1:
                dp.dictproj_forward(xs[0], self.M, ls[0], gs[0], ys[0], stream_handle)
            else:
                dp.dictproj_forward_batch(xs, self.M, ls, gs, ys, stream_handle)


def capture(torch, stream, fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()  # warm-up outside capture
    stream.synchronize()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def stage_rooflines(torch, dp, stack, stream, M, peak, batched=True, reps=20):
    """Average launch time and HBM roofline of each stage kernel of the two-kernel
    decode path in the step's own launch configuration: the step's calls (the same
    batches, grids and Z scratch, through dictproj_forward_batch_stages) captured
    twice, once launching only the dictionary kernels and once only the coefficient
    kernels (which then read the Z the last full step left: the same work)."""
    sh = stream.cuda_stream
    projs = stack.w.projections
    calls = stack.calls(batched)

    def stage_only(mask):
        def fn():
            for xs, ls, gs, ys in calls:
                dp.dictproj_forward_batch_stages(xs, M, ls, gs, ys, sh, mask)
        return fn

    out = {}
    for name, mask, byte_idx in (("k_dict_decode", 1, 0), ("k_coeff_gather", 2, 1)):
        g = capture(torch, stream, stage_only(mask))
        time_replays(torch, stream, g, 3)
        ms = time_replays(torch, stream, g, reps) / reps
        del g
        nbytes = sum(stage_bytes(p, M)[byte_idx] for p in projs)
        per_launch_ms = ms / len(calls)
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"ms_per_step": round(ms, 4), "launches": len(calls), "projections": len(projs),
                     "avg_launch_us": round(per_launch_ms * 1e3, 3),
                     "algorithmic_bytes_per_launch": int(nbytes / len(calls)), "GB/s": round(gbs, 1),
                     "frac": round(gbs / peak, 4)}
    return out


def time_replays(torch, stream, graph, n, pre=None, post=None):
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(n):
            if pre:
                pre()
            graph.replay()
            if post:
                post()
        b.record(stream)
    b.synchronize()
    return a.elapsed_time(b)


# ----------------------------------------------------------------------------- oracle legs
def oracle_layer_sample(workload, layer_index=0):
    """Decoded fp64 factors and inputs of the 7 projections of one layer."""
    from oracle import forward as F
    from oracle.pack import pack_coeff, pack_dictionary
    sample = []
    for p in workload.projections:
        if p.layer != layer_index:
            continue
        D, C = synth.projection_inputs(p)
        dec = F.decode_projection(pack_dictionary(D), pack_coeff(C.col_ptr, C.atom_idx, C.vals, p.k, p.d_out))
        X = synth.gen_activations(workload.cfg, p.layer, p.site, 1, p.d_in, workload.outlier_frac)
        sample.append((p, dec, X))
    return sample


def cpu_baseline(workload, n_layers, budget_s=12.0):
    """Oracle (fp64 factored forward on pre-decoded factors) on one layer's 7
    projections, repeated for about `budget_s` seconds, scaled to the stack."""
    from oracle import forward as F
    t0 = time.time()
    sample = oracle_layer_sample(workload)
    decode_s = time.time() - t0
    reps, spent = 0, 0.0
    while spent < budget_s or reps == 0:
        t = time.perf_counter()
        for p, dec, X in sample:
            F.forward_factored_decoded(X, dec)
        spent += time.perf_counter() - t
        reps += 1
        if reps >= 200:
            break
    layer_s = spent / reps
    return {"value": 1.0 / (n_layers * layer_s), "unit": "tokens/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"layer 0 (7 projections, M=1) of the {n_layers}-layer stack, fp64 factored "
                      f"forward on pre-decoded factors, {reps} repetitions ({spent:.1f}s), "
                      f"scaled x{n_layers}; one-off decode+pack of the sample took {decode_s:.1f}s"}


def step_config(wl, n_layers, M, world, batched=True):
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": f"{wl.name}: {n_layers} layers in {n_layers // 2} groups x 7 projection "
                        "types (LLaMA-7B shapes), NVFP4 D/C, C density U[0.2,0.4], M=1",
            "tokens_per_step": M, "projections_per_step": len(wl.projections),
            "weights": "nvfp4 (E2M1 + E4M3/16 + fp32)", "activations": "fp16", "accumulate": "fp32",
            "l2": "inputs larger than L2 (packed weights ~2.6 GB, no flush needed)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def run_reference(args, budget_s=200.0):
    """--impl reference: the oracle timed on the host cores (rank 0 only).

    A step is the whole stack's forward: the fp64 factored forward of all
    n_layers x 7 projections in model order, each layer reusing the 7 decoded
    factors of layer 0 (same shapes; decoding all 224 would take minutes). If
    warm-up + timed steps of the whole stack would not fit `budget_s`, a step is
    instead the first S projections of that sequence and a step then counts as
    S / (n_layers x 7) tokens, so that value and ms_per_step describe exactly
    what was timed."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    from oracle import forward as F
    wl = synth.full_step(n_layers=args.layers)
    t_setup = time.perf_counter()
    sample = oracle_layer_sample(wl)
    setup_s = time.perf_counter() - t_setup
    n_proj = args.layers * len(sample)
    # probe: one pass over the 7 projections gives the time per projection
    t = time.perf_counter()
    for p, dec, X in sample:
        F.forward_factored_decoded(X, dec)
    per_proj = (time.perf_counter() - t) / len(sample)
    steps_total = args.warmup + args.steps
    S = n_proj
    if steps_total * n_proj * per_proj > budget_s:
        S = max(1, int(budget_s / (steps_total * per_proj)))
    seq = [sample[i % len(sample)] for i in range(S)]

    def one_step():
        for p, dec, X in seq:
            F.forward_factored_decoded(X, dec)

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    timed_s = time.perf_counter() - t0
    ms_per_step = 1e3 * timed_s / args.steps
    tokens_per_step = S / n_proj
    value = tokens_per_step * args.steps / timed_s
    what = (f"each step = the fp64 oracle's factored forward of all {n_proj} projections of the stack "
            f"in model order" if S == n_proj else
            f"each step = the first {S} of the stack's {n_proj} projections in model order "
            f"({tokens_per_step:.4f} token per step), sized to fit {budget_s:.0f}s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": step_config(wl, args.layers, 1, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)),
                         "kind": "oracle",
                         "sample": f"{what}; every layer reuses layer 0's 7 decoded factors (pre-decoded in "
                                   f"{setup_s:.0f}s); {args.steps} timed steps in {timed_s:.1f}s"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- main arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--stage-reps", type=int, default=50)
    ap.add_argument("--ref-budget", type=float, default=200.0,
                    help="--impl reference: seconds that warm-up plus timed steps may take")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill (M = 128, 512, 2048) leg")
    ap.add_argument("--no-shapes", action="store_true", help="skip the per-projection-shape rows (M = 1, 8)")
    ap.add_argument("--decode-kernels", choices=("auto", "fused", "split"), default="auto",
                    help="decode kernels for M <= 8 calls (dictproj_set_decode_kernels); default: the library's choice")
    ap.add_argument("--no-batch", action="store_true",
                    help="one dictproj_forward per projection instead of batching q/k/v and gate/up")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args, args.ref_budget)

    import torch
    import dictionary_compressed_linear_b200 as dp

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def log(msg):
        if rank == 0:
            print(f"[bench] {msg}", file=sys.stderr, flush=True)

    from dictionary_compressed_linear_b200 import build
    if rank == 0:
        build.build()
    if dist:
        dist.barrier()

    dp.dictproj_set_decode_kernels({"auto": dp.DECODE_AUTO, "fused": dp.DECODE_FUSED,
                                    "split": dp.DECODE_SPLIT}[args.decode_kernels])
    wl = synth.full_step(n_layers=args.layers)
    M = 1
    stack = Stack(wl, M, torch, dp, log)
    stream = torch.cuda.Stream()
    sh = stream.cuda_stream
    graph = capture(torch, stream, lambda: stack.forward_all(dp, sh, batched=not args.no_batch))
    calls_per_step = len(stack.call_groups(not args.no_batch))
    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            graph.replay()
    stream.synchronize()

    # ---------------- timed region
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ms = time_replays(torch, stream, graph, args.steps)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(ms, dist, "cuda")
    ms_per_step = ms / args.steps
    value = replica_throughput(M * args.steps, world, ms)
    # the same step with one call per projection, for comparison
    ms_unbatched = None
    if not args.no_batch:
        g_u = capture(torch, stream, lambda: stack.forward_all(dp, sh, batched=False))
        time_replays(torch, stream, g_u, 5)
        ms_unbatched = time_replays(torch, stream, g_u, max(10, args.steps // 4)) / max(10, args.steps // 4)
        del g_u

    # ---------------- roofline of the dominant kernel
    launches_per_step = stack.launches_per_step(dp, batched=not args.no_batch)
    step_bytes = sum(d_bytes(p) + c_bytes(p) + 2 * M * (p.d_in + p.d_out) for p in wl.projections)
    peak, peak_kind = measured_peaks()
    peak_source = "measured (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6650 GB/s"
    if launches_per_step == calls_per_step:  # every call is one fused launch: the step itself times it
        avg_launch_ms = ms_per_step / launches_per_step
        bytes_per_launch = step_bytes / launches_per_step
        kernel, stages = "k_decode_fused", None
        timing = ("the timed step itself: CUDA events on the launching stream around the replays of the step's "
                  "graph; every launch is k_decode_fused, one per call")
    else:  # two-kernel path: each stage's kernel timed in a graph of that stage's launches of the step alone
        stages = stage_rooflines(torch, dp, stack, stream, M, peak, batched=not args.no_batch)
        dom = max(stages, key=lambda n: stages[n]["ms_per_step"])
        avg_launch_ms = stages[dom]["avg_launch_us"] / 1e3
        bytes_per_launch = stages[dom]["algorithmic_bytes_per_launch"]
        kernel = dom
        timing = ("CUDA events on the launching stream around replays of a graph of the step's own calls "
                  "(same batches, grids and Z scratch) that launches only this kernel "
                  "(dictproj_forward_batch_stages); the dominant kernel is the one with the larger share of the step")
    achieved = bytes_per_launch / (avg_launch_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": profiled_traffic(kernel, bytes_per_launch),
                "kernel": kernel, "peak_source": peak_source,
                "avg_launch_us": round(avg_launch_ms * 1e3, 3), "algorithmic_bytes_per_launch": int(bytes_per_launch),
                "launches_per_step": launches_per_step, "timing": timing}
    if stages:
        roofline["stages"] = stages

    # ---------------- step-level accounting
    d_once = sum(d_bytes(p) for p in {(q.group, q.ptype): q for q in wl.projections}.values())
    step_bytes_once = d_once + sum(c_bytes(p) + 2 * M * (p.d_in + p.d_out) for p in wl.projections)
    step_gbs = step_bytes / (ms_per_step / 1e3) / 1e9

    # ---------------- end to end through the C ABI with host buffers
    h2d = stack.x_host.numel() * 2
    d2h = stack.y_host.numel() * 2
    e2e_steps = max(3, min(args.steps, 500))

    def pre():
        stack.x.copy_(stack.x_host, non_blocking=True)

    def post():
        stack.y_host.copy_(stack.y, non_blocking=True)

    time_replays(torch, stream, graph, 3, pre, post)
    ms_e2e = time_replays(torch, stream, graph, e2e_steps, pre, post)
    e2e_value = replica_throughput(M * e2e_steps, world, max_over_ranks(ms_e2e, dist, "cuda"))

    del graph
    del stack
    torch.cuda.empty_cache()
    shapes = None
    if not args.no_shapes:
        shapes = per_shape_bench(torch, dp, stream, peak)
    prefill = None
    if not args.no_prefill:
        prefill = prefill_bench(torch, dp, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.layers)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": step_config(wl, args.layers, M, world),
        "calls_per_step": calls_per_step,
        "batching": "q/k/v and gate/up share a call (dictproj_forward_batch)" if not args.no_batch
                    else "one dictproj_forward per projection",
        "decode_kernels": {"auto": "library default (two-kernel path for NVFP4 layers)",
                           "fused": "fused single kernel", "split": "two-kernel path"}[args.decode_kernels],
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 2), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "shapes": shapes,
        "clocks": clocks,
        "step": {"algorithmic_bytes": step_bytes, "GB/s": round(step_gbs, 1),
                 "ms_per_step_one_call_per_projection": round(ms_unbatched, 5) if ms_unbatched else None,
                 "frac_of_peak": round(step_gbs / peak, 4),
                 "algorithmic_bytes_dictionary_once_per_group": step_bytes_once,
                 "GB/s_dictionary_once_per_group": round(step_bytes_once / (ms_per_step / 1e3) / 1e9, 1)},
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
