"""Benchmark of the paired-4:8 NVFP4 MoE hot path on B200.

A step is one pass of the whole hot path over one batch: route + permute,
dispatch-quantise, gate_up grouped sparse GEMM, SwiGLU + requantise, down
grouped sparse GEMM, router-weighted combine (weight packing is offline and
not timed).  The default workload is the 30B-class MoE layer (128 experts,
top-8, hidden 2048, intermediate 768 -> gate_up N = 1536, T = 256 tokens,
uniform router logits), synthetic data of the pages' distributions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

Prints one JSON line (rank 0).  `value` is the effective TFLOP/s of the
step's two grouped GEMMs (2 * M * K per routed row, the pages' App. D.2
definition) over all ranks; `weight_gbs` the packed expert weights the step
reads.  Device time: the step is captured once as a CUDA graph and replayed;
CUDA events around each replay on the launching stream, L2 flushed (256 MiB
write) before every step outside the events; max over ranks.  Event nodes
inside the graph give the per-kernel breakdown of the same replays.  `e2e`: the same metric through moesq_moe_layer_host with the step's
inputs and output in pinned host memory (copies inside the timed region).
`--impl reference` times the CPU oracle on a bounded token sample instead.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
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

# name -> (E, k, H, I, T, routing, kind); kind "layer" or "gemm" (route + quantise + gate_up GEMM)
WORKLOADS = {
    "30b_layer_t256": (128, 8, 2048, 768, 256, "uniform", "layer"),
    "tiny_layer_t64": (8, 2, 512, 256, 64, "uniform", "layer"),
    "kimi_layer_t1": (384, 8, 7168, 2048, 1, "uniform", "layer"),
    "kimi_layer_t16": (384, 8, 7168, 2048, 16, "uniform", "layer"),
    "kimi_layer_t64": (384, 8, 7168, 2048, 64, "uniform", "layer"),
    "kimi_layer_t256": (384, 8, 7168, 2048, 256, "uniform", "layer"),
    "kimi_layer_t4096_zipf": (384, 8, 7168, 2048, 4096, "zipf", "layer"),
    "kimi_gateup_t1": (384, 8, 7168, 2048, 1, "uniform", "gemm"),
    "kimi_gateup_t16": (384, 8, 7168, 2048, 16, "uniform", "gemm"),
    "kimi_gateup_t64": (384, 8, 7168, 2048, 64, "uniform", "gemm"),
    "kimi_gateup_t256": (384, 8, 7168, 2048, 256, "uniform", "gemm"),
    "kimi_down_t8192_zipf": (384, 8, 7168, 2048, 8192, "zipf", "gemm_down"),
    "30b_gateup_t256": (128, 8, 2048, 768, 256, "uniform", "gemm"),
}
# The paper's Table 11 setting (App. D, B200): Kimi gate_up over all 384
# experts, expert g receiving N * {1, 3/4, 1/2, 1/4}[g % 4] rows, timed as
# activation quantisation + grouped GEMM (bf16 in, bf16 out); the step is
# those two calls.  Value: the paper's latency in us and its effective
# TFLOP/s (2 M K sum(n) / t).
TAB11 = {8: (760.0, 148.0), 16: (793.0, 284.0), 32: (843.0, 535.0), 64: (925.0, 975.0),
         128: (912.0, 1978.0), 256: (1370.0, 2633.0)}
for _n in TAB11:
    WORKLOADS["tab11_n%d" % _n] = (384, 8, 7168, 2048, 30 * _n, "tab11", "quant_gemm")
DEFAULT_WORKLOAD = "30b_layer_t256"


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
                     "peak_source": "%s (tensor peak = dense bf16 burst x %g fp4/bf16 x %g sparse)"
                     % (peaks["source"], FP4_OVER_BF16, SPARSE_FACTOR)})
    return roofline


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

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

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
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
def step_work(E, k, H, I, T, counts_gu, kind):
    """(flops, weight bytes, per-GEMM algorithmic bytes, per-GEMM dense-equivalent
    flops) of one step."""
    R = T * k
    touched = int((np.asarray(counts_gu) > 0).sum())
    if kind == "gemm_down":
        M, K = H, I
        flops = 2.0 * M * K * R
        wbytes = touched * packed_weight_bytes(M, K)
        return flops, wbytes, {"down": wbytes + R * (K // 2 + K // 32) + R * M * 2}, {"down": flops}
    gu_w = touched * packed_weight_bytes(2 * I, H)
    gu_bytes = gu_w + R * (H // 2 + H // 32) + R * 2 * I * 2
    gu_fl = 2.0 * 2 * I * H * R
    if kind in ("gemm", "quant_gemm"):
        return gu_fl, gu_w, {"gate_up": gu_bytes}, {"gate_up": gu_fl}
    dn_w = touched * packed_weight_bytes(H, I)
    dn_bytes = dn_w + R * (I // 2 + I // 32) + R * H * 2
    dn_fl = 2.0 * H * I * R
    return gu_fl + dn_fl, gu_w + dn_w, {"gate_up": gu_bytes, "down": dn_bytes}, {"gate_up": gu_fl, "down": dn_fl}


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


def tab11_logits(T, E, k=8):
    """0/1 router logits whose top-k gives expert g exactly
    N * {4, 3, 2, 1}[g % 4] / 4 rows (N = T / 30): every token takes the k
    experts with the most rows still to fill (ties to the lower id)."""
    n = T // 30
    left = np.array([n * (4 - g % 4) // 4 for g in range(E)], np.int64)
    assert left.sum() == T * k
    lg = np.zeros((T, E), np.float32)
    for t in range(T):
        pick = np.lexsort((np.arange(E), -left))[:k]
        assert (left[pick] > 0).all()
        lg[t, pick] = 1.0
        left[pick] -= 1
    return lg


def logits_for(routing, seed, T, E):
    if routing == "tab11":
        return tab11_logits(T, E)
    return S.zipf_logits_np(seed, T, E) if routing == "zipf" else S.uniform_logits_np(seed, T, E)


# ------------------------------------------------------------------ CUDA arm
def run_cuda(args, rank, world, local_rank):
    import torch
    import grouped_gemm_moesq_b200 as m
    from grouped_gemm_moesq_b200 import build as cuda_build

    if rank == 0 or not os.path.exists(cuda_build.LIB):
        cuda_build.build()
    m.load()
    torch.cuda.set_device(local_rank)
    dev = "cuda"
    E, k, H, I, T, routing, kind = WORKLOADS[args.workload]
    seed = 1234
    stream = torch.cuda.current_stream()

    # weights: drawn on the GPU (same bits as the host generator) and packed, 8 experts at a time
    def make_weights(linear, M, K):
        pw = m.PackedWeights(E, M, K)
        for e0 in range(0, E, 8):
            n = min(8, E - e0)
            w = torch.stack([S.expert_weights_bf16_torch(seed, linear, e, M, K, dev) for e in range(e0, e0 + n)])
            m.moesq_pack_weights(w, e0, n, pw)
            del w
        return pw

    if kind == "gemm_down":
        w_main = make_weights(1, H, I)
        w_dn = None
    else:
        w_main = make_weights(0, 2 * I, H)
        w_dn = make_weights(1, H, I) if kind == "layer" else None
    torch.cuda.synchronize()

    # per-rank batch (independent replicas: weak scaling, no data-path collective)
    K_in = I if kind == "gemm_down" else H
    x_np = S.activations_bf16_np(rank_seed(seed, rank), T, K_in)
    lg_np = logits_for(routing, rank_seed(seed, rank), T, E)
    x = torch.from_numpy(x_np.view(np.int16).copy()).to(dev).view(torch.bfloat16)
    lg = torch.from_numpy(lg_np).to(dev)

    rb = m.RoutingBuffers(T, E, k)
    ga = torch.empty(E, dtype=torch.float32, device=dev)
    gh = torch.empty(E, dtype=torch.float32, device=dev)
    if kind == "layer":
        ws = torch.empty(m.moesq_layer_workspace_bytes(T, k, E, H, I), dtype=torch.uint8, device=dev)
        m.moesq_calibrate_layer(x, lg, T, k, w_main, w_dn, ga, gh, ws)
    else:
        m.moesq_act_global_scale(x, ga[:1])
        ga.fill_(float(ga[:1].item()))
    a_codes, a_scales = m.act_buffers(rb.rows_cap, K_in)
    M_main = w_main.M
    y_main = torch.empty(rb.rows_cap, M_main, dtype=torch.bfloat16, device=dev)
    if kind == "layer":
        h_codes, h_scales = m.act_buffers(rb.rows_cap, I)
        y_dn = torch.empty(rb.rows_cap, H, dtype=torch.bfloat16, device=dev)
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)

    # the hot path as its ABI calls, one callable per component
    def c_route_quant():
        m.moesq_route_permute(lg, rb)
        m.moesq_quantize_act(x, T, K_in, rb, ga, rb.rows_cap, a_codes, a_scales)

    # GEMM configurations, frozen by moesq_gemm_autotune after the warm-up
    # and before the graphs are captured
    tuned = {"main": (0, 0), "down": (0, 0)}

    def c_gemm_main():
        tn, nc = tuned["main"]
        m.moesq_grouped_sparse_gemm(w_main, a_codes, a_scales, rb.rows_cap, rb.counts, rb.row_offsets, ga, y_main,
                                    tile_n=tn, num_ctas=nc)

    if kind == "quant_gemm":                  # fixed grouping: routed once, outside the step
        m.moesq_route_permute(lg, rb)
        comps = [("quant", lambda: m.moesq_quantize_act(x, T, K_in, rb, ga, rb.rows_cap, a_codes, a_scales)),
                 ("gemm_main", c_gemm_main)]
    else:
        comps = [("route_quant", c_route_quant), ("gemm_main", c_gemm_main)]
    if kind == "layer":
        comps += [("swiglu_quant", lambda: m.moesq_swiglu_quant(y_main, I, rb, gh, h_codes, h_scales)),
                  ("gemm_down", lambda: m.moesq_grouped_sparse_gemm(w_dn, h_codes, h_scales, rb.rows_cap, rb.counts,
                                                                    rb.row_offsets, gh, y_dn, tile_n=tuned["down"][0],
                                                                    num_ctas=tuned["down"][1])),
                  ("combine", lambda: m.moesq_combine(y_dn, H, rb, out))]

    def step_eager():
        for _, f in comps:
            f()

    # routing: top-k plus one finishing kernel for T <= 512 tokens, else top-k, count, scan and scatter
    launches_per_step = (0 if kind == "quant_gemm" else 2 if T <= 512 else 4) + 2 + (3 if kind == "layer" else 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        step_eager()
    torch.cuda.synchronize()
    st, word = m.moesq_get_device_error()
    if st != 0:
        raise RuntimeError("device error word %#x during warm-up" % word)
    tuned["main"] = m.moesq_gemm_autotune(w_main, a_codes, a_scales, rb.rows_cap, rb.counts, rb.row_offsets, ga,
                                          y_main, reps=3)[0]
    if kind == "layer":
        tuned["down"] = m.moesq_gemm_autotune(w_dn, h_codes, h_scales, rb.rows_cap, rb.counts, rb.row_offsets, gh,
                                              y_dn, reps=3)[0]
    step_eager()                              # outputs of the tuned configuration
    torch.cuda.synchronize()
    counts = rb.counts.cpu().numpy()

    # One CUDA graph per step (the pages time CUDA-graph replays, App. D.2),
    # with external event-record nodes between the components: the same
    # replays give the per-kernel breakdown on the launching stream.
    from cuda.bindings import runtime as cudart

    def cu_event():
        err, e = cudart.cudaEventCreate()
        assert err == cudart.cudaError_t.cudaSuccess
        return e

    cev = [cu_event() for _ in range(len(comps) + 1)]
    g_step = torch.cuda.CUDAGraph()          # the timed step: kernels only
    with torch.cuda.graph(g_step):
        step_eager()
    g_prof = torch.cuda.CUDAGraph()          # the same kernels with event nodes between them
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

    def ev():
        return torch.cuda.Event(enable_timing=True)

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    t_wall0 = time.perf_counter()
    evs = [(ev(), ev()) for _ in range(args.steps)]
    part_ms = {name: [] for name, _ in comps}
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        g_step.replay()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall0
    for i in range(args.steps):                 # per-kernel breakdown, same flush discipline
        flush.zero_()
        g_prof.replay()
        torch.cuda.synchronize()
        for j, (name, _) in enumerate(comps):
            err, dt = cudart.cudaEventElapsedTime(cev[j], cev[j + 1])
            assert err == cudart.cudaError_t.cudaSuccess, err
            part_ms[name].append(dt)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    st, word = m.moesq_get_device_error()
    if st != 0:
        raise RuntimeError("device error word %#x in the timed region" % word)

    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    parts = {name: statistics.mean(v) for name, v in part_ms.items()}
    del g_step, g_prof
    for e in cev:
        cudart.cudaEventDestroy(e)

    # e2e through the public host-buffer entry point (layer workloads)
    e2e = None
    if kind == "layer":
        wsh = torch.empty(m.moesq_layer_host_workspace_bytes(T, k, E, H, I), dtype=torch.uint8, device=dev)
        xh = torch.from_numpy(x_np.view(np.int16).copy()).pin_memory()
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

    flops, wbytes, gemm_bytes, gemm_fl = step_work(E, k, H, I, T, counts, kind)
    t_max, e2e_max = max_over_ranks([ms, e2e["ms_per_step"] if e2e else 0.0], device=dev)
    if e2e:
        e2e["ms_per_step"] = e2e_max
    return dict(kind=kind, E=E, k=k, H=H, I=I, T=T, routing=routing, ms=t_max, parts=parts, flops=flops,
                wbytes=wbytes, gemm_bytes=gemm_bytes, gemm_fl=gemm_fl, e2e=e2e, tuned=tuned, clocks=clk, launches=launches_per_step * args.steps,
                wall_s=t_wall, counts=counts)


# ------------------------------------------------------------------ oracle (CPU) arm
_ORACLE_PREP = {}


def oracle_prepare(workload, n_tokens, seed=1234):
    """Inputs, routing and packed weights (the touched experts only) of the
    first n_tokens tokens of the workload's batch; made once per run, outside
    every timed region."""
    key = (workload, n_tokens, seed)
    if key in _ORACLE_PREP:
        return _ORACLE_PREP[key]
    import oracle as O
    E, k, H, I, T, routing, kind = WORKLOADS[workload]
    n = min(n_tokens, T)
    K_in = I if kind == "gemm_down" else H
    x = S.activations_bf16_np(seed, T, K_in, rows=n)
    lg = logits_for(routing, seed, T, E)[:n]
    used = np.nonzero(O.route(lg, k).counts)[0]

    def packed(linear, M, K):
        w = np.stack([S.expert_weights_bf16_np(seed, linear, int(e), M, K) for e in used])
        pk = O.pack_weights(w)
        full = O.Packed(np.zeros((E, M, K // 4), np.uint8), np.zeros((E, M, K // 16), np.uint8),
                        np.zeros((E, M, K // 32), np.uint8), np.ones(E, np.float32))
        full.values[used], full.mask[used], full.scales[used], full.gamma[used] = \
            pk.values, pk.mask, pk.scales, pk.gamma
        return full

    prep = {"n": n, "x": x, "lg": lg, "k": k, "kind": kind,
            "ga": np.full(E, O.act_global_scale(x), np.float32), "gh": np.full(E, 64.0, np.float32)}
    if kind == "gemm_down":
        prep["pk"] = packed(1, H, I)
        prep["flops"] = 2.0 * H * I * n * k
    else:
        prep["pk"] = packed(0, 2 * I, H)
        prep["flops"] = 2.0 * 2 * I * H * n * k
        if kind == "layer":
            prep["pk_dn"] = packed(1, H, I)
            prep["flops"] = 2.0 * 3 * I * H * n * k
    _ORACLE_PREP[key] = prep
    return prep


def run_oracle_sample(workload, n_tokens, seed=1234):
    """Times one pass of the oracle over the prepared token sample (routing,
    quantisation and the GEMMs, or the whole layer).  Returns (seconds, flops)."""
    import oracle as O
    p = oracle_prepare(workload, n_tokens, seed)
    t0 = time.perf_counter()
    if p["kind"] == "layer":
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
    per_token_macs = k * (3 * I * H if kind == "layer" else 2 * I * H if kind in ("gemm", "quant_gemm") else H * I)
    weights_per_expert = 3 * I * H if kind == "layer" else 2 * I * H if kind in ("gemm", "quant_gemm") else H * I
    by_macs = int(2.5e9 // per_token_macs)
    by_prep = int(150e6 // (k * weights_per_expert))
    return max(1, min(T, by_macs, by_prep))


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    E, k, H, I, T, routing, kind = WORKLOADS[args.workload]
    config = {"workload": args.workload, "experts": E, "top_k": k, "hidden": H, "intermediate": I,
              "tokens_per_gpu": T, "routing": routing, "step": kind,
              "l2": "flushed (256 MiB write) before every step, outside the timed events",
              "timing": "CUDA-graph replay of the step, CUDA events on the launching stream"}

    if args.impl == "reference":
        if rank != 0:
            return
        n = oracle_sample_tokens(args.workload)
        oracle_prepare(args.workload, n)        # inputs and packed weights, not timed
        for _ in range(args.warmup):
            run_oracle_sample(args.workload, n)
        secs, fl = [], 0.0
        for _ in range(args.steps):
            s, fl = run_oracle_sample(args.workload, n)
            secs.append(s)
        v = fl / statistics.mean(secs) / 1e12
        cores = 1
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                 "sample": "first %d of %d tokens of the workload per step" % (n, T)},
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))

    r = run_cuda(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    peaks = load_peaks()
    ms = r["ms"]
    value = job_throughput(r["flops"], world, ms)
    weight_gbs = world * r["wbytes"] / (ms * 1e-3) / 1e9
    gname = "down" if r["kind"] == "gemm_down" else "gate_up"
    gemm_ms = r["parts"]["gemm_main"]
    gbytes, gfl = r["gemm_bytes"][gname], r["gemm_fl"][gname]
    roofline = gemm_roofline(gbytes, gfl, gemm_ms, peaks, profiled_traffic(args.workload, gname), gname)
    tab11_n = T // 30 if args.workload.startswith("tab11_") else None
    vs_baseline = value / TAB11[tab11_n][1] if tab11_n else None
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": vs_baseline, "dtype": "nvfp4 (e2m1 x ue4m3 products, f32 accumulate, bf16 out)",
            "data": "synthetic (seeded; pages' shapes and distributions)", "config": config,
            "weight_gbs": weight_gbs, "breakdown_ms": r["parts"], "roofline": roofline,
            "gemm_config": {name: {"tile_n": tn, "num_ctas": nc} for name, (tn, nc) in r["tuned"].items()
                            if tn},
            "clocks": r["clocks"], "gpu_launches": r["launches"],
            "expert_rows": {"min": int(r["counts"].min()), "max": int(r["counts"].max()),
                            "touched": int((r["counts"] > 0).sum())}}
    if r["e2e"]:
        e = r["e2e"]
        line["e2e"] = {"value": job_throughput(r["flops"], world, e["ms_per_step"]), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": e["h2d_bytes_per_step"], "d2h_bytes_per_step": e["d2h_bytes_per_step"],
                       "ms_per_step": e["ms_per_step"]}
    if world == 1 and not args.no_cpu_baseline:
        v, secs, passes, n = oracle_baseline(args.workload)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                                "sample": "first %d of %d tokens of the workload, %d passes (%.1f s)"
                                % (n, T, passes, secs)}
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
