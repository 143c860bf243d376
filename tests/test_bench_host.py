"""Host-side logic of bench.py on the CPU: the max-over-ranks reduction and whole-job
throughput with two gloo ranks (the replica layout of multi-GPU runs), the per-stage
algorithmic work, and the reference arm's JSON line on the tiny fp32 workload."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from fine_grained_mixture_route_b200 import workloads as W  # noqa: E402


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    bench.init_dist(world, "gloo")
    try:
        step_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
        ms = bench.reduce_max(step_ms, "cpu")
        bench.barrier()
        q.put((rank, ms, bench.aggregate_throughput(1000, world, ms)))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, tput in res:
        assert ms == 15.0
        assert abs(tput - 2 * 1000 / 0.015) < 1e-6


def test_stage_work_sums_to_layer_flops():
    for name, cfg in W.CONFIGS.items():
        w = bench.stage_work(cfg, cfg.n_experts)
        assert abs(sum(f for f, _ in w.values()) - cfg.flops()) < 1e-6 * cfg.flops(), name
        assert all(b > 0 for _, b in w.values())
    dec = W.CONFIGS["decode"]
    # weight bytes of the whole layer when every expert is touched: 256 routed + 1 shared
    per_expert = (3 * 7168 * 2048 + 2 * 2048 + 7168) * 2
    assert abs(bench.layer_bytes(dec, 256) - (257 * per_expert + 256 * 7168 * 2 + 2 * 256 * 7168 * 2)) < 1
    # e4m3 routed experts: same FLOPs; routed weights at 1 byte plus one fp32 scale per row
    for name, cfg in W.CONFIGS.items():
        if cfg.dtype == torch.bfloat16:
            w8 = bench.stage_work(cfg, cfg.n_experts, e4m3=True)
            assert abs(sum(f for f, _ in w8.values()) - cfg.flops()) < 1e-6 * cfg.flops(), name
            assert w8["gemm1_swiglu"][1] < bench.stage_work(cfg, cfg.n_experts)["gemm1_swiglu"][1]
    routed8 = 3 * 7168 * 2048 + (2 * 2048 + 7168) * 4 + (2 * 2048 + 7168) * 2
    assert abs(bench.layer_bytes(dec, 256, e4m3=True)
               - (256 * routed8 + per_expert + 256 * 7168 * 2 + 2 * 256 * 7168 * 2)) < 1
    # block-scaled weights: one scale byte per 32 weights at this shape (whole 1 KB tiles), same FLOPs
    assert bench.mx_scale_bytes_per_expert(dec) == (2 * 2048 * 7168 // 32, 7168 * 2048 // 32)
    routed_mx = 3 * 7168 * 2048 + 3 * 7168 * 2048 // 32 + (2 * 2048 + 7168) * 2
    assert abs(bench.layer_bytes(dec, 256, e4m3=True, mx=True)
               - (256 * routed_mx + per_expert + 256 * 7168 * 2 + 2 * 256 * 7168 * 2)) < 1
    wm, w8 = bench.stage_work(dec, 256, e4m3=True, mx=True), bench.stage_work(dec, 256, e4m3=True)
    assert [f for f, _ in wm.values()] == [f for f, _ in w8.values()]
    S = 256 * 8
    # gemm1: weight scales per run instead of per row; x scales per run instead of per row; h as
    # codes + run scales instead of bf16
    assert wm["gemm1_swiglu"][1] - w8["gemm1_swiglu"][1] == \
        256 * (2 * 2048 * 7168 // 32 - 2 * 2048 * 4) + S * (7168 // 32 - 4) + S * (2048 + 2048 // 32 - 2 * 2048)
    # gemm2: no hidden-row quantisation (bf16 h read, codes and row scales written), run scales of h and W2
    assert wm["gemm2"][1] - w8["gemm2"][1] == \
        256 * (7168 * 2048 // 32 - 7168 * 4) - (S * 2048 * 2 + S * 2048 + S * 4) + S * (2048 // 32 - 4)
    assert wm["gather"][1] - w8["gather"][1] == S * (7168 // 32 - 4)
    # ragged shapes pay whole tiles: inter 80 and d 208 -> one 128-row group, two 128-input chunks
    rag = W.scaled(W.CONFIGS["small"], d=208, inter=80)
    assert bench.mx_scale_bytes_per_expert(rag) == (1 * 2 * 1024, 1 * 1 * 1024)


def test_backward_work_is_twice_the_forward():
    """Backward FLOPs: twice the expert and shared FLOPs of the forward (data and weight gradients)
    plus three router-sized products (recomputed logits, dz . C, dz^T x) against the forward's one."""
    for name, cfg in W.CONFIGS.items():
        if cfg.dtype != torch.bfloat16:
            continue
        fw = sum(f for f, _ in bench.stage_work(cfg, cfg.n_experts).values())
        bw = sum(f for f, _ in bench.bwd_stage_work(cfg, cfg.n_experts).values())
        router = 2.0 * cfg.T * cfg.d * cfg.n_experts
        assert abs(bw - (2 * fw + router)) < 1e-9 * bw, name
        assert all(b > 0 for _, b in bench.bwd_stage_work(cfg, cfg.n_experts).values())


def test_reference_arm_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["metric"] == bench.METRIC


def test_warmup_must_be_three():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
    with pytest.raises(SystemExit):                     # e4m3 routed experts need a bf16 layer
        bench.main(["--workload", "tiny", "--routed-fmt", "e4m3"])
    with pytest.raises(SystemExit):
        bench.main(["--workload", "tiny", "--routed-fmt", "mxfp8"])


def test_cpu_baseline_sample_grows_to_the_target():
    import oracle.moe_oracle as O
    cfg = W.CONFIGS["tiny"]
    L = W.make_layer(cfg, "cpu", 0)
    idx = O.route(L["x"].double().numpy(), L["centroids"].double().numpy(), cfg.top_k)["idx"]
    # a first sample under min_s grows (here up to max_tokens); one at or above it is reported as is
    grown = bench.cpu_baseline(cfg, L, idx, n_tokens=4, target_s=1e9, min_s=1e9, max_tokens=40)
    assert "first 40 tokens" in grown["sample"] and grown["value"] > 0 and grown["kind"] == "oracle"
    kept = bench.cpu_baseline(cfg, L, idx, n_tokens=4, min_s=0.0)
    assert "first 4 tokens" in kept["sample"]
    capped = bench.cpu_baseline(cfg, L, idx, n_tokens=4, target_s=1e9, min_s=1e9, max_tokens=10**6)
    assert f"first {cfg.T} tokens" in capped["sample"]                 # never more than the batch


def test_routing_stats():
    import math
    u = bench.routing_stats([5] * 8)
    assert u["experts_touched"] == 8 and u["max_over_mean"] == 1.0
    assert abs(u["hit_entropy"] - math.log(8)) < 1e-12 and u["hit_entropy"] == pytest.approx(u["hit_entropy_max"])
    one = bench.routing_stats([0, 0, 12, 0])
    assert one["experts_touched"] == 1 and one["hit_entropy"] == 0.0 and one["max_over_mean"] == 4.0
    two = bench.routing_stats([3, 1, 0, 0])
    assert two["hit_entropy"] == pytest.approx(-(0.75 * math.log(0.75) + 0.25 * math.log(0.25)))
