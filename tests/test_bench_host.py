"""Host logic of bench.py without a GPU: the max-over-ranks timing and the
barrier over two gloo ranks, the reference arm's JSON line (rank 0 only),
and the bounded oracle samples of the CPU baseline (bf16 and INT8)."""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

from block_sparse_attention_34_b200.configs import WORKLOADS
from block_sparse_attention_34_b200.synth import make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    got_ws, got_rank, _ = bench.dist_env()
    bench.init_dist(got_ws, "gloo")
    # each rank's own time; every rank must see the slowest one
    m = bench.max_over_ranks(1.5 * (got_rank + 1), got_ws, torch.device("cpu"))
    bench.barrier(got_ws)
    q.put((got_rank, m))
    torch.distributed.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 3.0), (1, 3.0)]


def run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env,
                          capture_output=True, text=True, timeout=300)


def test_reference_arm_json_line():
    r = run_bench(["--impl", "reference", "--workload", "tiny_4x8x8", "--steps", "2",
                   "--warmup", "1", "--ref-blocks", "2"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in d
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1


def test_reference_arm_other_ranks_do_nothing():
    r = run_bench(["--impl", "reference", "--workload", "tiny_4x8x8", "--steps", "1",
                   "--warmup", "1"], {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_cpu_baseline_samples():
    sys.path.insert(0, ROOT)
    import bench
    from oracle import paro_ref as ref

    w = WORKLOADS["small_8x16x16"]
    q, k, v, perms = make_inputs(w, heads=1)
    _, _, s = ref.pooled_scores(q.double().numpy(), k.double().numpy(), (w.F, w.H, w.W),
                                perms[:1], w.block)
    idx = ref.select_topk(s, ref.k_for_density(w.NB, w.density))
    for int8 in (False, True):
        tf, dt, sample = bench.cpu_baseline(w, q, k, v, perms, idx, budget_s=1e9, max_blocks=3,
                                            int8=int8)
        assert tf > 0 and dt > 0
        assert sample.startswith("head 0, query blocks 0..2 of ")
    # the sample never reaches the ragged last query block
    _, _, sample = bench.cpu_baseline(w, q, k, v, perms, idx, budget_s=1e9)
    assert f"0..{w.NB - 2} of {w.NB}" in sample


def test_int8_peak_uses_nominal_ratio():
    sys.path.insert(0, ROOT)
    import bench

    peaks = {"bf16_tflops_sustained": 1000.0, "bf16_tflops": 1500.0}
    # the burst figure is the default denominator (kernels timed in short steps)
    assert bench.tensor_peak(peaks, "bf16") == 1500.0
    assert bench.tensor_peak(peaks, "int8") == 3000.0
    assert bench.tensor_peak(peaks, "int8", "bf16_tflops_sustained") == 2000.0


def test_percentiles_pick_order_statistics():
    sys.path.insert(0, ROOT)
    import bench

    xs = [5.0, 1.0, 3.0, 2.0, 4.0, 9.0, 7.0, 8.0, 6.0, 10.0, 0.0]
    p = bench.percentiles(xs)
    assert p == {"p10": 1.0, "p50": 5.0, "p90": 9.0}
    assert bench.percentiles([2.5]) == {"p10": 2.5, "p50": 2.5, "p90": 2.5}


def test_sweep_options_parse_and_refuse_without_cuda():
    """--sweep with --pasa-only / --selection-only parses, and with no CUDA
    device the run stops with a message instead of falling back to the CPU."""
    sys.path.insert(0, ROOT)
    import pytest
    import bench

    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present: the sweep would run")
    for extra in (["--pasa-only"], ["--selection-only"], []):
        with pytest.raises(SystemExit) as e:
            bench.main(["--sweep", *extra])
        assert "CUDA" in str(e.value)


def test_pasa_cpu_baseline_runs_the_oracle():
    sys.path.insert(0, ROOT)
    import bench

    w = WORKLOADS["small_8x16x16"]
    q, k, v, perms = make_inputs(w, heads=1)
    tf, dt, sample = bench.pasa_cpu_baseline(w, q, k, v, perms)
    assert tf > 0 and dt > 0
    assert f"all {w.NB} query blocks" in sample


def test_sics_cpu_baseline_runs_the_oracle():
    sys.path.insert(0, ROOT)
    import bench

    w = WORKLOADS["small_8x16x16"]
    q, k, _, _ = make_inputs(w, heads=1)
    gbs, dt, sample = bench.sics_cpu_baseline(w, q, k)
    assert gbs > 0 and dt > 0 and "head 0" in sample


def test_default_line_cpu_baseline_takes_the_oracles_lists():
    """The default line's CPU baseline, as bench.py builds it: the oracle's
    own kept lists of head 0 (never the GPU's), then the bounded sample, on
    the default 720p workload (one query block) and the INT8 long clip."""
    sys.path.insert(0, ROOT)
    import bench

    for name, int8 in (("720p_21x45x80", False), ("longclip_33x45x80_int8", True)):
        w = WORKLOADS[name]
        q, k, v, perms = make_inputs(w, heads=1)
        idx = bench.oracle_idx_head0(w, q, k, perms, w.density)
        from oracle import paro_ref as ref
        assert idx.shape == (w.B, 1, w.NB, ref.k_for_density(w.NB, w.density))
        assert (idx[..., 0] <= np.arange(w.NB)).all()  # ascending lists that hold the diagonal
        assert all(i in idx[0, 0, i] for i in range(w.NB))
        tf, dt, sample = bench.cpu_baseline(w, q, k, v, perms, idx, budget_s=1e9, max_blocks=1,
                                            int8=int8)
        assert tf > 0 and "query blocks 0..0" in sample
