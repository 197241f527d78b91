"""Host-side pieces of bench.py that need no GPU: the max-over-ranks timing
reduction and whole-job aggregation of the multi-GPU (replica) path, run as
two gloo ranks on CPU, and the reference arm (the CPU oracle) end to end."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 180.0][rank]           # the slower rank sets the job time
        ms = bench._max_over_ranks(local_ms, True, torch.device("cpu"))
        bench._barrier(True)
        rate = bench.whole_job_rate(1000.0, ms, world)
        q.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 2000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, rate in got:
        assert ms == 180.0
        assert rate == pytest.approx(2 * 1000.0 / 0.180)


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0", "--cpu-rows", "8"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_flop_accounting_matches_the_published_workload_figures():
    """pairs and FLOPs per step (fwd 4 pairs d, bwd 10 pairs d) against the
    figures derived for each workload: 32K dense, 256K dense, 256K Top-K,
    1M Top-K offload."""
    import bench
    from paged_kv_chunk_query_b200 import synth
    W = synth.WORKLOADS
    cases = [("qwen32k", False, 536_887_296, 26.94),
             ("qwen256k", False, 34_359_869_440, 1724.0),
             ("qwen256k_topk", True, 1_626_472_448, 81.6),
             ("qwen1m_topk_offload", True, 6_559_367_168, 329.1)]
    for name, sparse, pairs_per_head, tflop in cases:
        w = W[name]
        pairs = bench.step_pairs(w, sparse)
        assert pairs == pairs_per_head * w.num_q_heads, name
        total = 14.0 * pairs * w.head_dim / 1e12
        assert abs(total - tflop) <= 0.06 * max(1.0, tflop / 100), (name, total)
    # a recent-only window covering the whole past is dense
    w = W["qwen256k"]
    assert bench.step_pairs(synth.Workload("x", 28, 4, 128, 64, 4096, 64, seed=1,
                                           window=4096), False) == bench.step_pairs(w, False)


def test_clock_scaled_peak_and_step_fractions():
    """The burst tensor peak scales with the SM clock the run held; without a
    clock record there is no scaled peak (and no scaled fraction)."""
    import bench
    assert bench.clock_scaled_peak(1654.6, 1965.0, 1965.0) == 1654.6
    assert abs(bench.clock_scaled_peak(1654.6, 1710.0, 1965.0) - 1654.6 * 1710.0 / 1965.0) < 1e-9
    assert bench.clock_scaled_peak(1654.6, None, 1965.0) is None
    assert bench.clock_scaled_peak(1654.6, 1710.0, None) is None
    peaks = {"bf16": 1654.6, "bf16_sustained": 1359.8, "sm_max_mhz": 1965.0}
    f = bench.step_fractions(784.1, peaks, 1710.0)
    assert abs(f["of_sustained"] - 784.1 / 1359.8) < 1e-12
    assert abs(f["of_burst"] - 784.1 / 1654.6) < 1e-12
    assert abs(f["of_clock_normalised"] - 784.1 / (1654.6 * 1710.0 / 1965.0)) < 1e-12
    assert bench.step_fractions(784.1, peaks, None)["of_clock_normalised"] is None
