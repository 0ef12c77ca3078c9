"""Benchmark of the paired-4:8 NVFP4 MoE hot path on B200.

A step is one pass of the whole hot path over one batch: route + permute,
dispatch-quantise, gate_up grouped sparse GEMM, SwiGLU + requantise, down
grouped sparse GEMM, router-weighted combine (weight packing is offline and
not timed).  The default workload is the Kimi-K2.5-shaped MoE layer (384
experts, top-8, hidden 7168, intermediate 2048 -> gate_up N = 4096) swept over
T = 1, 4, 16, ..., 16384 tokens with uniform and Zipf(1.1) routing; the headline
numbers are those of T = 4096 with Zipf routing, and every point of the sweep
is in `sweep`.  Synthetic data of the pages' distributions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

Prints one JSON line (rank 0).  `value` is the effective TFLOP/s of the
step's grouped GEMMs (2 * M * K per routed row, the pages' App. D.2
definition) over all ranks; `weight_gbs` the packed expert weights the step
reads.  Device time: the step is captured once as a CUDA graph and replayed;
CUDA events around each replay on the launching stream, L2 flushed (256 MiB
write) before every step outside the events; max over ranks.  Event nodes
inside a second graph give the per-kernel breakdown of the same replays.
`e2e`: the same metric through moesq_moe_layer_host with the step's inputs
and output in pinned host memory (copies inside the timed region).
`--gpus N` with N > 1 starts N ranks (torch.distributed.run, one per GPU).
`--impl reference` times the CPU oracle on a bounded token sample instead.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import socket
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synthetic as S  # noqa: E402
from grouped_gemm_moesq_b200.metrics import packed_weight_bytes  # noqa: E402

METRIC = "paired-4:8 NVFP4 grouped GEMM TFLOP/s + weight GB/s vs roofline, per token count"

KIMI = (384, 8, 7168, 2048)        # experts, top-k, hidden, intermediate
LAYER_T = (1, 4, 16, 64, 256, 1024, 4096, 16384)

# name -> (E, k, H, I, T, routing, kind).  kind: "layer" (the whole path,
# SwiGLU + requantisation fused into the gate_up GEMM), "layer_unfused" (the
# same with SwiGLU + requantisation as a kernel of its own),
# "gemm" (route + quantise + gate_up GEMM), "gemm_down" (route + quantise +
# down GEMM), "quant_gemm" (fixed grouping, routed once outside the step:
# activation quantisation + gate_up GEMM, as the paper's kernel benchmark),
# "quant_gemm_down" (the same with the down shape).
WORKLOADS = {
    "30b_layer_t256": (128, 8, 2048, 768, 256, "uniform", "layer"),
    "tiny_layer_t64": (8, 2, 512, 256, 64, "uniform", "layer"),
    "kimi_gateup_t1": KIMI + (1, "uniform", "gemm"),
    "kimi_gateup_t16": KIMI + (16, "uniform", "gemm"),
    "kimi_gateup_t64": KIMI + (64, "uniform", "gemm"),
    "kimi_gateup_t256": KIMI + (256, "uniform", "gemm"),
    "kimi_down_t8192_zipf": KIMI + (8192, "zipf", "gemm_down"),
    "30b_gateup_t256": (128, 8, 2048, 768, 256, "uniform", "gemm"),
    # compute-bound probes: 32 experts of the Kimi shapes, 4096 rows each
    "cb_gateup_e32_n4096": (32, 8, 7168, 2048, 16384, "fixed4096", "quant_gemm"),
    "cb_down_e32_n4096": (32, 8, 7168, 2048, 16384, "fixed4096", "quant_gemm_down"),
}
for _t in LAYER_T:
    WORKLOADS["kimi_layer_t%d" % _t] = KIMI + (_t, "uniform", "layer")
    WORKLOADS["kimi_layer_t%d_zipf" % _t] = KIMI + (_t, "zipf", "layer")
WORKLOADS["kimi_layer_t4096_zipf_unfused"] = KIMI + (4096, "zipf", "layer_unfused")
WORKLOADS["30b_layer_t256_unfused"] = (128, 8, 2048, 768, 256, "uniform", "layer_unfused")
WORKLOADS["30b_layer_t4096"] = (128, 8, 2048, 768, 4096, "uniform", "layer")
# The paper's Table 11 setting (App. D, B200): Kimi gate_up over all 384
# experts, expert g receiving N * {1, 3/4, 1/2, 1/4}[g % 4] rows, timed as
# activation quantisation + grouped GEMM (bf16 in, bf16 out); the step is
# those two calls.  Value: the paper's latency in us and its effective
# TFLOP/s (2 M K sum(n) / t).
TAB11 = {8: (760.0, 148.0), 16: (793.0, 284.0), 32: (843.0, 535.0), 64: (925.0, 975.0),
         128: (912.0, 1978.0), 256: (1370.0, 2633.0)}
for _n in TAB11:
    WORKLOADS["tab11_n%d" % _n] = KIMI + (30 * _n, "tab11", "quant_gemm")

# Sweeps: one JSON line whose headline is one point and whose `sweep` holds
# every point (all share the packed weights).
SWEEPS = {
    "kimi_layer": {"points": ["kimi_layer_t%d%s" % (t, r) for t in LAYER_T for r in ("", "_zipf")],
                   "headline": "kimi_layer_t4096_zipf"},
    "tab11": {"points": ["tab11_n%d" % n for n in TAB11], "headline": "tab11_n64"},
}
DEFAULT_WORKLOAD = "kimi_layer"

# The paper's kernel sweep (App. D.2, Table 8): (M, K) of each layer, the
# maximum per-expert token counts N and the expert-group counts G; expert g
# receives N * {1, 3/4, 1/2, 1/4}[g % 4] rows.  Sparse kernel and dense
# NVFP4 control, each with its fastest configuration, on the same
# activations; speedup = t_dense / t_sparse.
TAB8 = {
    "kimi_gate_up": (4096, 7168, (32, 64, 128, 256, 512, 1024), (24, 48, 96, 192, 384)),
    "kimi_down": (7168, 2048, (32, 64, 128, 256, 512, 1024), (24, 48, 96, 192, 384)),
    "30b_gate_up": (1536, 2048, (16, 32, 64, 128, 256, 512, 1024), (8, 16, 32, 64, 128)),
    "30b_down": (2048, 768, (16, 32, 64, 128, 256, 512, 1024), (8, 16, 32, 64, 128)),
}

SPEC_HBM_GBS = 8000.0       # B200 HBM3e specification (8 TB/s), beside the measured copy rate
PAPER_SPARSE_FP4_TFLOPS = 18000.0   # the pages' sparse FP4 tensor peak, dense-equivalent
FP4_OVER_BF16 = 4.0    # nominal dense tensor-core ratio, fp4 : bf16 (9 : 2.25 PFLOP/s)
SPARSE_FACTOR = 2.0    # a structured-sparse MMA runs the dense-equivalent contraction at twice the rate


def load_peaks():
    """HBM copy GB/s and dense bf16 TFLOP/s (burst) measured on this GPU type,
    else an earlier measurement of the same pool."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d.get("hbm_gbs", 6650.0), "bf16_tflops": d.get("bf16_tflops", 1590.0),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def strip_c_comments(text):
    """C/C++ source without comments and whitespace (string literals in
    these sources hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", "", text)


def gemm_source_sha():
    """Hash of the code (comments and whitespace removed) of the sources the
    grouped GEMM kernel is built from; a DRAM traffic record taken with ncu
    is only used while it matches."""
    h = hashlib.sha256()
    for f in ("gemm.cuh", "common.cuh"):
        h.update(strip_c_comments(open(os.path.join(ROOT, "grouped_gemm_moesq_b200", "csrc", f)).read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload, gemm):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the ncu summaries under profiles/, or None."""
    sha = gemm_source_sha()
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for ln in open(path):
            if ln.startswith("traffic-record: "):
                rec = json.loads(ln[len("traffic-record: "):])
                if rec.get("workload") == workload and rec.get("gemm") == gemm and rec.get("source_sha") == sha:
                    return rec["dram_bytes_per_launch"]
    return None


def gemm_roofline(gbytes, gfl, gemm_ms, peaks, traffic, gname):
    """Roofline of one grouped GEMM launch: the bound is whichever ideal time
    is longer, algorithmic bytes at the HBM copy rate or dense-equivalent
    flops at the sparse NVFP4 tensor rate; both fractions are reported."""
    hbm_peak = peaks["hbm_gbs"]
    tc_peak = peaks["bf16_tflops"] * FP4_OVER_BF16 * SPARSE_FACTOR
    hbm_ach = gbytes / (gemm_ms * 1e-3) / 1e9
    tc_ach = gfl / (gemm_ms * 1e-3) / 1e12
    if gbytes / (hbm_peak * 1e9) >= gfl / (tc_peak * 1e12):
        roofline = {"bound": "hbm", "achieved": hbm_ach, "peak": hbm_peak, "unit": "GB/s",
                    "frac": hbm_ach / hbm_peak}
    else:
        roofline = {"bound": "tensor", "achieved": tc_ach, "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": tc_ach / tc_peak}
    roofline.update({"traffic": traffic, "algorithmic_bytes": gbytes, "dense_equiv_flops": gfl,
                     "kernel": "grouped_sparse_gemm (%s)" % gname, "kernel_ms": gemm_ms,
                     "hbm_frac": hbm_ach / hbm_peak, "tensor_frac": tc_ach / tc_peak,
                     "hbm_frac_of_spec": hbm_ach / SPEC_HBM_GBS,
                     "tensor_frac_of_paper_peak": tc_ach / PAPER_SPARSE_FP4_TFLOPS,
                     "peak_source": "%s (tensor peak = dense bf16 burst x %g fp4/bf16 x %g sparse)"
                     % (peaks["source"], FP4_OVER_BF16, SPARSE_FACTOR)})
    return roofline


def host_cpu():
    """Host threads available to this process and the CPU model."""
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    try:
        nproc = len(os.sched_getaffinity(0))
    except AttributeError:
        nproc = os.cpu_count()
    return nproc, model


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of one GPU's clocks and throttle reasons while
    sampling is on; start/stop may be called repeatedly (one window per
    timed region) and `summary` covers all windows."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None
        self.rows = []
        self.ok = True

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            self.ok = False

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)
        os.unlink(self.path)
        self.proc = None

    def summary(self):
        rows = self.rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [v for v in sm if v > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ work accounting
def main_gemm_shape(kind, H, I):
    """(M, K) of the workload's main grouped GEMM."""
    return (H, I) if kind in ("gemm_down", "quant_gemm_down") else (2 * I, H)


def step_work(E, k, H, I, T, counts_gu, kind):
    """(flops, weight bytes, per-GEMM algorithmic bytes, per-GEMM dense-equivalent
    flops) of one step."""
    R = int(np.asarray(counts_gu).sum()) if kind.startswith("quant_gemm") else T * k
    touched = int((np.asarray(counts_gu) > 0).sum())
    if kind in ("gemm_down", "quant_gemm_down"):
        M, K = H, I
        flops = 2.0 * M * K * R
        wbytes = touched * packed_weight_bytes(M, K)
        return flops, wbytes, {"down": wbytes + R * (K // 2 + K // 32) + R * M * 2}, {"down": flops}
    gu_w = touched * packed_weight_bytes(2 * I, H)
    # output: the bf16 gate_up rows, or (fused layer) the requantised h rows
    gu_out = R * (I // 2 + I // 32) if kind == "layer" else R * 2 * I * 2
    gu_bytes = gu_w + R * (H // 2 + H // 32) + gu_out
    gu_fl = 2.0 * 2 * I * H * R
    if kind in ("gemm", "quant_gemm"):
        return gu_fl, gu_w, {"gate_up": gu_bytes}, {"gate_up": gu_fl}
    dn_w = touched * packed_weight_bytes(H, I)
    dn_bytes = dn_w + R * (I // 2 + I // 32) + R * H * 2
    dn_fl = 2.0 * H * I * R
    return gu_fl + dn_fl, gu_w + dn_w, {"gate_up": gu_bytes, "down": dn_bytes}, {"gate_up": gu_fl, "down": dn_fl}


def launches_per_step(kind, T):
    """Kernels of this library one step launches: routing is top-k plus one
    finishing kernel for T <= 512 tokens, else top-k, count, scan, scatter;
    then quantise and the GEMM, and for the layer SwiGLU, down GEMM, combine."""
    route = 0 if kind.startswith("quant_gemm") else (2 if T <= 512 else 4)
    return route + 2 + {"layer": 2, "layer_unfused": 3}.get(kind, 0)


def rank_seed(seed, rank):
    """Seed of one rank's token batch: every rank draws its own batch
    (independent replicas, weak scaling)."""
    return seed + 7919 * rank


def max_over_ranks(values, device="cpu"):
    """Element-wise maximum of a list of floats over all ranks of the default
    process group (identity without one).  Every rank must call it."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(flops_per_rank, world, ms):
    """Whole-job TFLOP/s: all ranks' work over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def fixed_count_logits(T, want, k=8):
    """0/1 router logits [T, E] whose top-k gives expert g exactly want[g]
    rows (sum(want) = T * k): every token takes the k experts with the most
    rows still to fill (ties to the lower id)."""
    left = np.array(want, np.int64)
    E = left.size
    assert left.sum() == T * k
    lg = np.zeros((T, E), np.float32)
    for t in range(T):
        pick = np.lexsort((np.arange(E), -left))[:k]
        assert (left[pick] > 0).all()
        lg[t, pick] = 1.0
        left[pick] -= 1
    return lg


def tab11_logits(T, E, k=8):
    """The Table 11 pattern: expert g gets N * {4, 3, 2, 1}[g % 4] / 4 rows,
    N = T / 30."""
    n = T // 30
    return fixed_count_logits(T, [n * (4 - g % 4) // 4 for g in range(E)], k)


def logits_for(routing, seed, T, E):
    if routing == "tab11":
        return tab11_logits(T, E)
    if routing.startswith("fixed"):
        n = int(routing[len("fixed"):])
        return fixed_count_logits(T, [n] * E)
    return S.zipf_logits_np(seed, T, E) if routing == "zipf" else S.uniform_logits_np(seed, T, E)


def parse_gemm_config(text):
    """'128:296:1,64:296:1' -> {"main": (128, 296, 1), "down": (64, 296, 1)}
    (the down configuration defaults to the main one)."""
    parts = [tuple(int(v) for v in p.split(":")) for p in text.split(",")]
    if not 1 <= len(parts) <= 2 or any(len(p) != 3 for p in parts):
        raise argparse.ArgumentTypeError("expected TILE_N:NUM_CTAS:SM_MODE[,TILE_N:NUM_CTAS:SM_MODE]")
    return {"main": parts[0], "down": parts[-1]}


def workload_points(name):
    """(points, headline) of a workload name: a sweep or a single workload."""
    if name in SWEEPS:
        return list(SWEEPS[name]["points"]), SWEEPS[name]["headline"]
    return [name], name


# ------------------------------------------------------------------ CUDA arm
def run_cuda(args, rank, world, local_rank):
    """Times every point of the workload on this rank's GPU.  Returns
    {"points": {name: point}, "headline": name, "clocks": {...}}."""
    import torch
    import grouped_gemm_moesq_b200 as m
    from grouped_gemm_moesq_b200 import build as cuda_build
    from cuda.bindings import runtime as cudart

    if rank == 0 or not os.path.exists(cuda_build.LIB):
        cuda_build.build()
    m.load()
    torch.cuda.set_device(local_rank)
    dev = "cuda"
    seed = 1234
    stream = torch.cuda.current_stream()
    points, headline = workload_points(args.workload)
    clocks = ClockSampler(local_rank)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    # packed weights, drawn on the GPU (same bits as the host generator) and
    # packed 8 experts at a time; shared by every point with the same shapes
    wcache = {}

    def weights(linear, E, M, K, layout=0):
        key = (linear, E, M, K, layout)
        if key not in wcache:
            pw = m.PackedWeights(E, M, K, layout=layout)
            for e0 in range(0, E, 8):
                n = min(8, E - e0)
                w = torch.stack([S.expert_weights_bf16_torch(seed, linear, e, M, K, dev) for e in range(e0, e0 + n)])
                m.moesq_pack_weights(w, e0, n, pw)
                del w
            torch.cuda.synchronize()
            wcache[key] = pw
        return wcache[key]

    def cu_event():
        err, e = cudart.cudaEventCreate()
        assert err == cudart.cudaError_t.cudaSuccess
        return e

    # this GPU's measured ceiling for the MMA the GEMM issues (no memory traffic)
    fp4_peak = {"sparse_n256_1cta": m.moesq_mma_peak(1, 256, 1), "sparse_n128_2cta": m.moesq_mma_peak(1, 128, 2),
                "dense_n256_1cta": m.moesq_mma_peak(0, 256, 1),
                "sparse_n128_2cta_with_scale_copies": m.moesq_mma_peak(1, 128, 2, with_copies=True)}

    results = {}
    for name in points:
        E, k, H, I, T, routing, kind = WORKLOADS[name]
        down_main = kind in ("gemm_down", "quant_gemm_down")
        if down_main:
            w_main, w_dn = weights(1, E, H, I), None
        else:
            # the fused layer reads its gate_up stack in the SwiGLU kernel row order
            w_main = weights(0, E, 2 * I, H, m.LAYOUT_SWIGLU if kind == "layer" else m.LAYOUT_PLAIN)
            w_dn = weights(1, E, H, I) if kind.startswith("layer") else None

        # this rank's batch (independent replicas: weak scaling, no data-path collective)
        K_in = I if down_main else H
        x = S.activations_bf16_torch(rank_seed(seed, rank), T, K_in, dev)
        lg_np = logits_for(routing, rank_seed(seed, rank), T, E)
        lg = torch.from_numpy(lg_np).to(dev)
        rb = m.RoutingBuffers(T, E, k)
        ga = torch.empty(E, dtype=torch.float32, device=dev)
        gh = torch.empty(E, dtype=torch.float32, device=dev)
        if kind.startswith("layer"):
            ws = torch.empty(m.moesq_layer_workspace_bytes(T, k, E, H, I), dtype=torch.uint8, device=dev)
            m.moesq_calibrate_layer(x, lg, T, k, w_main, w_dn, ga, gh, ws)
            del ws
        else:
            m.moesq_act_global_scale(x, ga[:1])
            ga.fill_(float(ga[:1].item()))
        a_codes, a_scales = m.act_buffers(rb.rows_cap, K_in)
        # the fused layer never materialises the bf16 gate_up output
        y_main = None if kind == "layer" else torch.empty(rb.rows_cap, w_main.M, dtype=torch.bfloat16, device=dev)
        if kind.startswith("layer"):
            h_codes, h_scales = m.act_buffers(rb.rows_cap, I)
            y_dn = torch.empty(rb.rows_cap, H, dtype=torch.bfloat16, device=dev)
            out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)

        # GEMM configurations, frozen by moesq_gemm_autotune after the warm-up
        # and before the graphs are captured (or given by --gemm-config)
        tuned = {"main": (0, 0, 0), "down": (0, 0, 0)}

        def c_route_quant():
            m.moesq_route_permute(lg, rb)
            m.moesq_quantize_act(x, T, K_in, rb, ga, rb.rows_cap, a_codes, a_scales)

        def c_gemm_main():
            tn, nc, cps = tuned["main"]
            if kind == "layer":     # gate_up GEMM + SwiGLU + requantisation in one kernel
                m.moesq_grouped_sparse_gemm_swiglu(w_main, a_codes, a_scales, rb.rows_cap, rb.counts, rb.row_offsets,
                                                   ga, gh, h_codes, h_scales, tile_n=tn, num_ctas=nc, sm_mode=cps)
            else:
                m.moesq_grouped_sparse_gemm(w_main, a_codes, a_scales, rb.rows_cap, rb.counts, rb.row_offsets, ga,
                                            y_main, tile_n=tn, num_ctas=nc, sm_mode=cps)

        if kind.startswith("quant_gemm"):     # fixed grouping: routed once, outside the step
            m.moesq_route_permute(lg, rb)
            comps = [("quant", lambda: m.moesq_quantize_act(x, T, K_in, rb, ga, rb.rows_cap, a_codes, a_scales)),
                     ("gemm_main", c_gemm_main)]
        else:
            comps = [("route_quant", c_route_quant), ("gemm_main", c_gemm_main)]
        if kind == "layer_unfused":
            comps += [("swiglu_quant", lambda: m.moesq_swiglu_quant(y_main, I, rb, gh, h_codes, h_scales))]
        if kind.startswith("layer"):
            comps += [("gemm_down", lambda: m.moesq_grouped_sparse_gemm(
                          w_dn, h_codes, h_scales, rb.rows_cap, rb.counts, rb.row_offsets, gh, y_dn,
                          tile_n=tuned["down"][0], num_ctas=tuned["down"][1], sm_mode=tuned["down"][2])),
                      ("combine", lambda: m.moesq_combine(y_dn, H, rb, out))]

        def step_eager():
            for _, f in comps:
                f()

        for _ in range(args.warmup):
            flush.zero_()
            step_eager()
        torch.cuda.synchronize()
        st, word = m.moesq_get_device_error()
        if st != 0:
            raise RuntimeError("%s: device error word %#x during warm-up" % (name, word))
        if args.gemm_config:
            tuned["main"] = args.gemm_config["main"]
            if kind.startswith("layer"):
                tuned["down"] = args.gemm_config["down"]
        elif kind == "layer":
            tuned["main"] = m.moesq_gemm_swiglu_autotune(w_main, a_codes, a_scales, rb.rows_cap, rb.counts,
                                                         rb.row_offsets, ga, gh, h_codes, h_scales, reps=3)[0]
        else:
            tuned["main"] = m.moesq_gemm_autotune(w_main, a_codes, a_scales, rb.rows_cap, rb.counts,
                                                  rb.row_offsets, ga, y_main, reps=3)[0]
        if kind.startswith("layer") and not args.gemm_config:
            tuned["down"] = m.moesq_gemm_autotune(w_dn, h_codes, h_scales, rb.rows_cap, rb.counts,
                                                  rb.row_offsets, gh, y_dn, reps=3)[0]
        step_eager()                          # outputs of the tuned configuration
        torch.cuda.synchronize()
        counts = rb.counts.cpu().numpy()

        # One CUDA graph per step (the pages time CUDA-graph replays, App. D.2),
        # and a second one with external event-record nodes between the
        # components: the same replays give the per-kernel breakdown on the
        # launching stream.
        cev = [cu_event() for _ in range(len(comps) + 1)]
        g_step = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step):
            step_eager()
        g_prof = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_prof):
            cs = torch.cuda.current_stream().cuda_stream
            for j, (_, f) in enumerate(comps):
                cudart.cudaEventRecordWithFlags(cev[j], cs, cudart.cudaEventRecordExternal)
                f()
            cudart.cudaEventRecordWithFlags(cev[-1], cs, cudart.cudaEventRecordExternal)
        flush.zero_()
        g_step.replay()
        g_prof.replay()
        torch.cuda.synchronize()

        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        clocks.start()
        time.sleep(0.2)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            g_step.replay()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clocks.stop()
        part_ms = {pname: [] for pname, _ in comps}
        for i in range(args.steps):             # per-kernel breakdown, same flush discipline
            flush.zero_()
            g_prof.replay()
            torch.cuda.synchronize()
            for j, (pname, _) in enumerate(comps):
                err, dt = cudart.cudaEventElapsedTime(cev[j], cev[j + 1])
                assert err == cudart.cudaError_t.cudaSuccess, err
                part_ms[pname].append(dt)
        st, word = m.moesq_get_device_error()
        if st != 0:
            raise RuntimeError("%s: device error word %#x in the timed region" % (name, word))
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        parts = {pname: statistics.mean(v) for pname, v in part_ms.items()}
        del g_step, g_prof
        for e in cev:
            cudart.cudaEventDestroy(e)

        # e2e through the public host-buffer entry point (layer workloads):
        # pinned host input and logits in, output back, inside the timed region
        e2e = None
        if kind.startswith("layer"):
            wsh = torch.empty(m.moesq_layer_host_workspace_bytes(T, k, E, H, I), dtype=torch.uint8, device=dev)
            xh = x.view(torch.int16).cpu().pin_memory()
            lh = torch.from_numpy(lg_np).pin_memory()
            oh = torch.empty(T, H, dtype=torch.int16).pin_memory()
            for _ in range(args.warmup):
                m.moesq_moe_layer_host(xh, lh, T, k, w_main, w_dn, ga, gh, oh, wsh)
            e2e_ms = []
            for _ in range(args.steps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                m.moesq_moe_layer_host(xh, lh, T, k, w_main, w_dn, ga, gh, oh, wsh)
                b.record(stream)
                b.synchronize()
                e2e_ms.append(a.elapsed_time(b))
            e2e = {"ms_per_step": statistics.mean(e2e_ms),
                   "h2d_bytes_per_step": T * H * 2 + T * E * 4, "d2h_bytes_per_step": T * H * 2}
            del wsh, xh, lh, oh

        flops, wbytes, gemm_bytes, gemm_fl = step_work(E, k, H, I, T, counts, kind)
        t_max, e2e_max = max_over_ranks([ms, e2e["ms_per_step"] if e2e else 0.0], device=dev)
        if e2e:
            e2e["ms_per_step"] = e2e_max
        results[name] = dict(kind=kind, E=E, k=k, H=H, I=I, T=T, routing=routing, ms=t_max, parts=parts,
                             flops=flops, wbytes=wbytes, gemm_bytes=gemm_bytes, gemm_fl=gemm_fl, e2e=e2e,
                             tuned=dict(tuned), launches=launches_per_step(kind, T), counts=counts)
        del x, lg, rb, a_codes, a_scales, y_main
        if kind.startswith("layer"):
            del h_codes, h_scales, y_dn, out
        torch.cuda.empty_cache()
    return {"points": results, "headline": headline, "clocks": clocks.summary(), "fp4_peak": fp4_peak}


# ------------------------------------------------------------------ sparse vs dense sweep (Table 8)
def tab8_counts(N, G):
    return np.array([N * (4 - g % 4) // 4 for g in range(G)], np.int64)


def run_tab8(args):
    """Times the sparse kernel and the dense NVFP4 control over Table 8's
    G x N grid on one GPU; prints one JSON line with every configuration."""
    import ctypes
    import torch
    import grouped_gemm_moesq_b200 as m
    from grouped_gemm_moesq_b200 import binding as B
    from grouped_gemm_moesq_b200 import build as cuda_build
    cuda_build.build()
    m.load()
    dev = "cuda"
    seed = 1234
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sms = torch.cuda.get_device_properties(0).multi_processor_count

    def time_graph(fn, reps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        ts = []
        for _ in range(args.warmup):
            flush.zero_()
            g.replay()
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        del g
        return statistics.median(ts)

    clocks = ClockSampler(0)
    clocks.start()
    layers = {}
    entries = []
    tot_fl, tot_sp = 0.0, 0.0
    for layer, (M, K, Ns, Gs) in TAB8.items():
        Emax = max(Gs)
        linear = 1 if layer.endswith("down") else 0
        pw = m.PackedWeights(Emax, M, K)
        dw = m.DenseWeights(Emax, M, K)
        for e0 in range(0, Emax, 8):
            n = min(8, Emax - e0)
            w = torch.stack([S.expert_weights_bf16_torch(seed, linear, e, M, K, dev) for e in range(e0, e0 + n)])
            m.moesq_pack_weights(w, e0, n, pw)
            m.moesq_pack_dense_nvfp4(w, e0, n, dw)
            del w
        torch.cuda.synchronize()
        speedups = []
        for G in Gs:
            ws = B.moesq_weights(G, M, K, pw.values.data_ptr(), pw.mask.data_ptr(), pw.scales.data_ptr(),
                                 pw.global_scale.data_ptr(), pw.ktiles.data_ptr())
            wd = B.moesq_dense_weights(G, M, K, dw.codes.data_ptr(), dw.scales.data_ptr(),
                                       dw.global_scale.data_ptr(), dw.dtiles.data_ptr())
            for N in Ns:
                counts = tab8_counts(N, G)
                ro = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)]).astype(np.int32)
                rc = int(ro[-1])
                x = S.activations_bf16_torch(seed + G, rc, K, dev)
                ga = torch.empty(1, dtype=torch.float32, device=dev)
                m.moesq_act_global_scale(x, ga)
                gam = ga.expand(G).contiguous()
                codes, scales = m.act_buffers(rc, K)
                m.moesq_quantize_act(x, rc, K, None, ga, rc, codes, scales)
                s16 = m.scales16_buffer(rc, K)
                m.moesq_expand_scales16(scales, rc, K, s16)
                cnt = torch.from_numpy(counts.astype(np.int32)).to(dev)
                rof = torch.from_numpy(ro).to(dev)
                y = torch.empty(rc, M, dtype=torch.bfloat16, device=dev)
                del x
                cand_s = [(64, 2 * sms, 1), (128, 2 * sms, 1), (64, sms, 1), (128, sms, 1)] + \
                         ([(128, 2 * sms, 2)] if M % 256 == 0 else [])
                cand_d = [(64, 2 * sms), (128, 2 * sms), (64, sms), (128, sms)]

                def sparse(c):
                    cfg = B.moesq_gemm_config(*c)
                    B._check(B.load().moesq_grouped_sparse_gemm(
                        ctypes.byref(ws), B._ptr(codes), B._ptr(scales), rc, B._ptr(cnt), B._ptr(rof), B._ptr(gam),
                        B._ptr(y), ctypes.byref(cfg), B._stream()), "sparse")

                def dense(c):
                    cfg = B.moesq_gemm_config(c[0], c[1], 1)
                    B._check(B.load().moesq_grouped_dense_gemm(
                        ctypes.byref(wd), B._ptr(codes), B._ptr(s16), rc, B._ptr(cnt), B._ptr(rof), B._ptr(gam),
                        B._ptr(y), ctypes.byref(cfg), B._stream()), "dense")

                ts = {c: time_graph(lambda c=c: sparse(c), 3) for c in cand_s}
                td = {c: time_graph(lambda c=c: dense(c), 3) for c in cand_d}
                bs, bd = min(ts, key=ts.get), min(td, key=td.get)
                t_s = time_graph(lambda: sparse(bs), args.steps)
                t_d = time_graph(lambda: dense(bd), args.steps)
                fl = 2.0 * M * K * counts.sum()
                tot_fl += fl
                tot_sp += t_s
                speedups.append(t_d / t_s)
                entries.append({"layer": layer, "M": M, "K": K, "G": G, "N": N, "sparse_ms": t_s, "dense_ms": t_d,
                                "speedup": t_d / t_s, "sparse_tflops": fl / (t_s * 1e-3) / 1e12,
                                "dense_tflops": fl / (t_d * 1e-3) / 1e12,
                                "sparse_config": {"tile_n": bs[0], "num_ctas": bs[1], "sm_mode": bs[2]},
                                "dense_config": {"tile_n": bd[0], "num_ctas": bd[1]}})
                del codes, scales, s16, y, cnt, rof
            st, word = m.moesq_get_device_error()
            if st != 0:
                raise RuntimeError("%s: device error word %#x" % (layer, word))
        layers[layer] = {"geomean_speedup": float(np.exp(np.mean(np.log(speedups)))),
                         "min_speedup": float(min(speedups)), "max_speedup": float(max(speedups)),
                         "configs": len(speedups)}
        del pw, dw
        torch.cuda.empty_cache()
    clocks.stop()
    line = {"metric": METRIC, "value": tot_fl / (tot_sp * 1e-3) / 1e12,
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_sp, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x ue4m3 products, f32 accumulate, bf16 out)",
            "data": "synthetic (seeded; Table 8 shapes, per-expert counts N x {1, 3/4, 1/2, 1/4})",
            "config": {"workload": "tab8_sweep", "timing": "CUDA-graph replay of one GEMM launch, median, L2 "
                       "flushed (256 MiB write) before every replay; each kernel with its fastest configuration",
                       "value": "sparse effective TFLOP/s summed over the sweep (total flops / total time)"},
            "layers": layers, "clocks": clocks.summary(), "sweep_tab8": entries,
            "gpu_launches": 2 * len(entries) * args.steps}
    print(json.dumps(line))


# ------------------------------------------------------------------ oracle (CPU) arm
_ORACLE_PREP = {}


def _host_weights(seed, linear, e, M, K):
    """One expert's seeded bf16 weight bits: drawn by the generator's torch
    path on a GPU when one is present (seconds less per Kimi expert), else on
    the host; the bits are the same."""
    try:
        import torch
        if torch.cuda.is_available():
            w = S.expert_weights_bf16_torch(seed, linear, int(e), M, K, "cuda")
            return w.view(torch.int16).cpu().numpy().view(np.uint16)
    except ImportError:
        pass
    return S.expert_weights_bf16_np(seed, linear, int(e), M, K)


def oracle_prepare(workload, n_tokens, seed=1234):
    """Inputs, routing, packed weights (the touched experts only) and the
    activation global scales of the first n_tokens tokens of the workload's
    batch; made once per run, outside every timed region.  For the layer the
    global scales are the oracle's own calibration on that sample."""
    key = (workload, n_tokens, seed)
    if key in _ORACLE_PREP:
        return _ORACLE_PREP[key]
    import oracle as O
    E, k, H, I, T, routing, kind = WORKLOADS[workload]
    n = min(n_tokens, T)
    down_main = kind in ("gemm_down", "quant_gemm_down")
    K_in = I if down_main else H
    x = S.activations_bf16_np(seed, T, K_in, rows=n)
    lg = logits_for(routing, seed, T, E)[:n]
    used = np.nonzero(O.route(lg, k).counts)[0]

    def packed(linear, M, K):
        w = np.stack([_host_weights(seed, linear, e, M, K) for e in used])
        pk = O.pack_weights(w)
        full = O.Packed(np.zeros((E, M, K // 4), np.uint8), np.zeros((E, M, K // 16), np.uint8),
                        np.zeros((E, M, K // 32), np.uint8), np.ones(E, np.float32))
        full.values[used], full.mask[used], full.scales[used], full.gamma[used] = \
            pk.values, pk.mask, pk.scales, pk.gamma
        return full

    prep = {"n": n, "x": x, "lg": lg, "k": k, "kind": kind,
            "ga": np.full(E, O.act_global_scale(x), np.float32)}
    if down_main:
        prep["pk"] = packed(1, H, I)
        prep["flops"] = 2.0 * H * I * n * k
    else:
        prep["pk"] = packed(0, 2 * I, H)
        prep["flops"] = 2.0 * 2 * I * H * n * k
        if kind.startswith("layer"):
            prep["pk_dn"] = packed(1, H, I)
            prep["flops"] = 2.0 * 3 * I * H * n * k
            prep["ga"], prep["gh"] = O.calibrate_layer(x, lg, k, prep["pk"], prep["pk_dn"])
    _ORACLE_PREP[key] = prep
    return prep


def run_oracle_sample(workload, n_tokens, seed=1234):
    """Times one pass of the oracle over the prepared token sample (routing,
    quantisation and the GEMM(s), or the whole layer).  Returns (seconds,
    dense-equivalent flops)."""
    import oracle as O
    p = oracle_prepare(workload, n_tokens, seed)
    t0 = time.perf_counter()
    if p["kind"].startswith("layer"):
        O.moe_layer(p["x"], p["lg"], p["k"], p["pk"], p["pk_dn"], p["ga"], p["gh"])
    else:
        rt = O.route(p["lg"], p["k"])
        a_c, a_s = O.permute_quantize(p["x"], rt, p["ga"])
        O.grouped_gemm(p["pk"], a_c, a_s, rt.offsets, p["ga"])
    return time.perf_counter() - t0, p["flops"]


def oracle_baseline(workload, min_seconds=5.0):
    """The oracle's rate on the token sample, repeated until min_seconds of
    CPU work (the preparation is not timed).  Returns (TFLOP/s, seconds,
    passes, tokens)."""
    n = oracle_sample_tokens(workload)
    secs, fl, passes = 0.0, 0.0, 0
    while secs < min_seconds or passes == 0:
        s_, f_ = run_oracle_sample(workload, n)
        secs, fl, passes = secs + s_, fl + f_, passes + 1
    return fl / secs / 1e12, secs, passes, n


def oracle_sample_tokens(workload):
    """Tokens of the oracle sample: about 2.5e9 multiply-adds per pass, and
    few enough touched experts (about 150 M weights to draw and pack) that
    the preparation stays under a minute or so."""
    E, k, H, I, T, routing, kind = WORKLOADS[workload]
    per_expert = 3 * I * H if kind.startswith("layer") else H * I if kind in ("gemm_down", "quant_gemm_down") else 2 * I * H
    by_macs = int(2.5e9 // (k * per_expert))
    by_prep = int(150e6 // (k * per_expert))
    return max(1, min(T, by_macs, by_prep))


def cpu_baseline_record(value, n, T, passes, secs, what):
    nproc, model = host_cpu()
    return {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": "first %d of %d tokens of %s, %d passes (%.1f s), one host thread" % (n, T, what, passes, secs),
            "host_threads_available": nproc, "cpu_model": model}


# ------------------------------------------------------------------ main
def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def launch_ranks(n):
    """Re-runs this script as n ranks under torch.distributed.run on this
    node (one process per GPU, rendezvous on 127.0.0.1), bounded by timeout;
    returns the launcher's exit code."""
    cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", str(n), "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def point_entry(name, r, peaks):
    """One sweep entry: the point's step time, throughput and GEMM fractions."""
    ent = {"workload": name, "tokens": r["T"], "routing": r["routing"], "ms_per_step": r["ms"],
           "tflops": r["flops"] / (r["ms"] * 1e-3) / 1e12,
           "weight_gbs": r["wbytes"] / (r["ms"] * 1e-3) / 1e9, "breakdown_ms": r["parts"],
           "expert_rows": {"min": int(r["counts"].min()), "max": int(r["counts"].max()),
                           "touched": int((r["counts"] > 0).sum())},
           "gemm_config": {g: {"tile_n": tn, "num_ctas": nc, "sm_mode": cps}
                           for g, (tn, nc, cps) in r["tuned"].items() if tn}}
    gemms = {}
    for gname, part in (("gate_up", "gemm_main"), ("down", "gemm_down" if r["kind"].startswith("layer") else "gemm_main")):
        if gname in r["gemm_bytes"] and part in r["parts"]:
            rf = gemm_roofline(r["gemm_bytes"][gname], r["gemm_fl"][gname], r["parts"][part], peaks, None, gname)
            gemms[gname] = {"ms": r["parts"][part], "hbm_frac": rf["hbm_frac"], "tensor_frac": rf["tensor_frac"],
                            "bound": rf["bound"], "frac": rf["frac"]}
    ent["gemms"] = gemms
    if r["e2e"]:
        ent["e2e_ms"] = r["e2e"]["ms_per_step"]
        ent["e2e_tflops"] = r["flops"] / (r["e2e"]["ms_per_step"] * 1e-3) / 1e12
    return ent


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=None)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(set(WORKLOADS) | set(SWEEPS) | {"tab8_sweep"}))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gemm-config", default=None, type=parse_gemm_config,
                    help="TILE_N:NUM_CTAS:SM_MODE of the main GEMM[,of the down GEMM]: fixed configurations "
                         "instead of the autotuner (profiling runs reproduce the timed launches)")
    args = ap.parse_args()

    if "WORLD_SIZE" not in os.environ and args.gpus is not None and args.gpus > 1:
        sys.exit(launch_ranks(args.gpus))
    if args.workload == "tab8_sweep":
        run_tab8(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus is not None and args.gpus != world:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    points, headline = workload_points(args.workload)
    E, k, H, I, T, routing, kind = WORKLOADS[headline]
    config = {"workload": args.workload, "headline": headline, "experts": E, "top_k": k, "hidden": H,
              "intermediate": I, "tokens_per_gpu": T, "routing": routing, "step": kind}

    if args.impl == "reference":
        if rank != 0:
            return
        n = oracle_sample_tokens(headline)
        oracle_prepare(headline, n)             # inputs and packed weights, not timed
        for _ in range(args.warmup):
            run_oracle_sample(headline, n)
        secs, fl = [], 0.0
        for _ in range(args.steps):
            s, fl = run_oracle_sample(headline, n)
            secs.append(s)
        v = fl / statistics.mean(secs) / 1e12
        rconfig = dict(config, timing="host wall clock (time.perf_counter) around each oracle pass over the "
                                      "token sample; one host thread",
                       l2="n/a (CPU oracle; inputs resident in host memory)")
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": rconfig,
                "cpu_baseline": cpu_baseline_record(v, n, T, args.steps, sum(secs), headline),
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))

    res = run_cuda(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    peaks = load_peaks()
    r = res["points"][res["headline"]]
    ms = r["ms"]
    value = job_throughput(r["flops"], world, ms)
    weight_gbs = world * r["wbytes"] / (ms * 1e-3) / 1e9
    gname = "down" if r["kind"] in ("gemm_down", "quant_gemm_down") else "gate_up"
    gemm_ms = r["parts"]["gemm_main"]
    gbytes, gfl = r["gemm_bytes"][gname], r["gemm_fl"][gname]
    roofline = gemm_roofline(gbytes, gfl, gemm_ms, peaks, profiled_traffic(res["headline"], gname), gname)
    if res.get("fp4_peak"):
        mp = max(v for k_, v in res["fp4_peak"].items() if k_.startswith("sparse") and "copies" not in k_)
        roofline["tensor_frac_of_measured_fp4"] = roofline["dense_equiv_flops"] / (gemm_ms * 1e-3) / 1e12 / mp
        roofline["measured_fp4_sparse_peak"] = mp
        roofline["peak_source"] += ("; measured sparse FP4 MMA peak %.0f TFLOP/s (moesq_mma_peak, back-to-back "
                                    "tcgen05.mma.sp kind::mxf4nvf4 on every SM)" % mp)
    tab11_n = r["T"] // 30 if res["headline"].startswith("tab11_") else None
    vs_baseline = value / TAB11[tab11_n][1] if tab11_n else None
    config.update({"gemm_config_source": "fixed (--gemm-config)" if args.gemm_config else "moesq autotune",
                   "l2": "flushed (256 MiB write) before every step, outside the timed events",
                   "timing": "CUDA-graph replay of the step, CUDA events on the launching stream"})
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": vs_baseline, "dtype": "nvfp4 (e2m1 x ue4m3 products, f32 accumulate, bf16 out)",
            "data": "synthetic (seeded; pages' shapes and distributions)", "config": config,
            "weight_gbs": weight_gbs, "breakdown_ms": r["parts"], "roofline": roofline,
            "gemm_config": {g: {"tile_n": tn, "num_ctas": nc, "sm_mode": cps}
                            for g, (tn, nc, cps) in r["tuned"].items() if tn},
            "clocks": res["clocks"], "gpu_launches": r["launches"] * args.steps,
            "fp4_mma_peak_tflops": res.get("fp4_peak"),
            "expert_rows": {"min": int(r["counts"].min()), "max": int(r["counts"].max()),
                            "touched": int((r["counts"] > 0).sum())}}
    if r["e2e"]:
        e = r["e2e"]
        line["e2e"] = {"value": job_throughput(r["flops"], world, e["ms_per_step"]), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": e["h2d_bytes_per_step"], "d2h_bytes_per_step": e["d2h_bytes_per_step"],
                       "ms_per_step": e["ms_per_step"]}
    if len(res["points"]) > 1:
        line["sweep"] = [point_entry(nm, res["points"][nm], peaks) for nm in points]
    if world == 1 and not args.no_cpu_baseline:
        v, secs, passes, n = oracle_baseline(res["headline"])
        line["cpu_baseline"] = cpu_baseline_record(v, n, r["T"], passes, secs, res["headline"])
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
