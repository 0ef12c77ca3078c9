"""Multi-rank host logic of bench.py on CPU: two gloo ranks, as torchrun
would launch them on two GPUs.  Each rank draws its own token batch (weak
scaling, no data-path collective); the only collective is the max of the
timings over ranks, and the job throughput counts every rank's work over the
slowest rank's time."""
import json
import os
import socket

import numpy as np
import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    import bench
    import synthetic as S
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [1.0 + rank, 5.0 - rank, 0.25 * rank]          # rank 1 is slower in the first entry only
        got = bench.max_over_ranks(ms)
        x = S.activations_bf16_np(bench.rank_seed(1234, rank), 4, 64)
        lg = bench.logits_for("zipf", bench.rank_seed(1234, rank), 4, 16)
        dist.barrier()
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"max": got, "x": x.astype(np.int64).tolist(), "lg": lg.tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_own_batches(tmp_path):
    mp = pytest.importorskip("torch.multiprocessing")
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(world)]
    for i in range(world):
        assert r[i]["max"] == [2.0, 5.0, 0.25]
    assert r[0]["x"] != r[1]["x"]                            # independent token batches
    assert r[0]["lg"] != r[1]["lg"]


def test_single_process_max_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 0.5]) == [3.0, 0.5]


def test_job_throughput_counts_all_ranks_over_slowest():
    import bench
    # 4 ranks, 1e12 dense-equivalent flops each, slowest rank 2 ms
    assert bench.job_throughput(1e12, 4, 2.0) == pytest.approx(2000.0)
    assert bench.rank_seed(7, 0) == 7 and bench.rank_seed(7, 3) != bench.rank_seed(7, 2)


def test_tab11_pattern_routes_to_the_paper_counts():
    """The Table 11 workloads' router logits: top-8 through the oracle's
    router gives expert g exactly N * {1, 3/4, 1/2, 1/4}[g % 4] rows."""
    import bench
    import oracle as O
    for n in (8, 16):
        T = 30 * n
        rt = O.route(bench.tab11_logits(T, 384), 8)
        want = np.array([n * (4 - g % 4) // 4 for g in range(384)])
        assert (rt.counts == want).all()


def test_gemm_roofline_picks_the_longer_ideal_time():
    """Decode-like launch (bytes dominate) is HBM-bound, a launch with many
    rows per expert is tensor-bound; fractions are achieved / peak."""
    import bench
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "source": "measured"}
    r = bench.gemm_roofline(3.0e9, 1.0e11, 0.5, peaks, None, "gate_up")        # 0.5 ms
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(3.0e9 / 0.5e-3 / 1e9 / 6000.0)
    tc_peak = 1500.0 * bench.FP4_OVER_BF16 * bench.SPARSE_FACTOR
    r = bench.gemm_roofline(1.0e9, 2.0e15, 1.0, peaks, 123, "down")             # 1 ms
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["traffic"] == 123
    assert r["frac"] == pytest.approx(2.0e15 / 1e-3 / 1e12 / tc_peak)
    assert r["hbm_frac"] == pytest.approx(1.0e9 / 1e-3 / 1e9 / 6000.0)


def test_traffic_record_needs_the_current_gemm_source():
    """profiles/ records are only used while their source hash matches."""
    import bench
    sha = bench.gemm_source_sha()
    t = bench.profiled_traffic("30b_layer_t256", "gate_up")
    assert t is None or isinstance(t, int)
    assert bench.profiled_traffic("no_such_workload", "gate_up") is None
    assert len(sha) == 16


def test_bench_line_has_the_contract_keys(monkeypatch, capsys):
    """bench.main() composes one JSON line with every key of the contract,
    the headline point's numbers and one sweep entry per point (a stand-in
    for the CUDA run supplies the measured parts)."""
    import json
    import sys
    import bench
    points, headline = bench.workload_points(bench.DEFAULT_WORKLOAD)
    assert headline in points and len(points) == 16

    def fake_point(name):
        E, k, H, I, T, routing, kind = bench.WORKLOADS[name]
        counts = np.full(E, max(1, T * k // E))
        flops, wbytes, gbytes, gfl = bench.step_work(E, k, H, I, T, counts, kind)
        return dict(kind=kind, E=E, k=k, H=H, I=I, T=T, routing=routing, ms=0.5,
                    parts={"route_quant": 0.05, "gemm_main": 0.2, "swiglu_quant": 0.02, "gemm_down": 0.2,
                           "combine": 0.03},
                    flops=flops, wbytes=wbytes, gemm_bytes=gbytes, gemm_fl=gfl,
                    e2e={"ms_per_step": 0.9, "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 2},
                    tuned={"main": (128, 296, 1), "down": (128, 296, 1)}, launches=bench.launches_per_step(kind, T),
                    counts=counts)

    def fake_run(args, rank, world, local_rank):
        return {"points": {nm: fake_point(nm) for nm in points}, "headline": headline,
                "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}}

    monkeypatch.setattr(bench, "run_cuda", fake_run)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "20", "--warmup", "3", "--no-cpu-baseline"])
    bench.main()
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "clocks", "gpu_launches"):
        assert key in line, key
    assert line["config"]["workload"] == bench.DEFAULT_WORKLOAD and line["config"]["headline"] == headline
    assert line["config"]["experts"] == 384 and line["config"]["tokens_per_gpu"] == 4096
    assert 0 < line["roofline"]["frac"]
    # routing (4 kernels at T = 4096), quantise, fused gate_up + SwiGLU, down GEMM, combine
    assert line["e2e"]["value"] > 0 and line["gpu_launches"] == 20 * (4 + 1 + 1 + 1 + 1)
    assert bench.launches_per_step("layer_unfused", 4096) == 4 + 5
    flops = fake_point(headline)["flops"]
    assert line["value"] == pytest.approx(flops / 0.5e-3 / 1e12)
    assert [e["workload"] for e in line["sweep"]] == points
    assert {e["tokens"] for e in line["sweep"]} == set(bench.LAYER_T)
    assert all(set(e["gemms"]) == {"gate_up", "down"} for e in line["sweep"])


def test_gpus_flag_must_match_the_launcher(monkeypatch):
    """Under a launcher, --gpus must equal WORLD_SIZE."""
    import sys
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4"])
    with pytest.raises(SystemExit):
        bench.main()


def test_fixed_count_logits_give_the_asked_counts():
    import bench
    import oracle as O
    want = [4, 0, 2, 6, 4]
    rt = O.route(bench.fixed_count_logits(8, want, k=2), 2)
    assert list(rt.counts) == want


def test_tab8_pattern_and_shapes():
    """Table 8's per-expert counts N * {1, 3/4, 1/2, 1/4} and its four layers."""
    import bench
    assert bench.tab8_counts(32, 8).tolist() == [32, 24, 16, 8, 32, 24, 16, 8]
    assert set(bench.TAB8) == {"kimi_gate_up", "kimi_down", "30b_gate_up", "30b_down"}
    assert bench.TAB8["kimi_down"][:2] == (7168, 2048) and bench.TAB8["30b_down"][:2] == (2048, 768)
    assert len(bench.TAB8["kimi_gate_up"][2]) * len(bench.TAB8["kimi_gate_up"][3]) == 30


def test_gemm_config_flag():
    """--gemm-config fixes the main (and down) GEMM configuration."""
    import argparse
    import bench
    assert bench.parse_gemm_config("128:296:1") == {"main": (128, 296, 1), "down": (128, 296, 1)}
    assert bench.parse_gemm_config("128:296:1,64:148:2") == {"main": (128, 296, 1), "down": (64, 148, 2)}
    for bad in ("128", "128:296", "1:2:3,4:5:6,7:8:9"):
        with pytest.raises(argparse.ArgumentTypeError):
            bench.parse_gemm_config(bad)


def test_step_work_algorithmic_bytes():
    """The per-GEMM algorithmic bytes the roofline divides by: packed weights
    of the touched experts (11 M K / 32 each), the
    NVFP4 activation rows in (K/2 codes + K/32 scales per row) and the
    output: bf16 rows, or for the fused layer the requantised h rows."""
    import bench
    from grouped_gemm_moesq_b200.metrics import packed_weight_bytes
    E, k, H, I, T = 8, 2, 512, 256, 64
    counts = np.array([10, 0, 30, 5, 0, 40, 20, 23])
    R = T * k
    assert packed_weight_bytes(2 * I, H) == 11 * 2 * I * H // 32
    fl, wb, gb, gf = bench.step_work(E, k, H, I, T, counts, "layer")
    touched = 6
    gu_w, dn_w = touched * packed_weight_bytes(2 * I, H), touched * packed_weight_bytes(H, I)
    assert wb == gu_w + dn_w
    assert gb["gate_up"] == gu_w + R * (H // 2 + H // 32) + R * (I // 2 + I // 32)      # fused: h out
    assert gb["down"] == dn_w + R * (I // 2 + I // 32) + R * H * 2
    assert gf["gate_up"] == 2.0 * 2 * I * H * R and gf["down"] == 2.0 * H * I * R and fl == gf["gate_up"] + gf["down"]
    _, _, gb_u, _ = bench.step_work(E, k, H, I, T, counts, "layer_unfused")
    assert gb_u["gate_up"] == gu_w + R * (H // 2 + H // 32) + R * 2 * I * 2             # unfused: bf16 y_gu out
    _, _, gb_q, gf_q = bench.step_work(E, k, H, I, T, counts, "quant_gemm")
    Rq = int(counts.sum())                                                               # fixed grouping: routed rows
    assert gb_q == {"gate_up": gu_w + Rq * (H // 2 + H // 32) + Rq * 2 * I * 2}
    assert gf_q == {"gate_up": 2.0 * 2 * I * H * Rq}
