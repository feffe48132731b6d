"""Host-side logic of bench.py without a GPU: the max over ranks through a real
two-rank gloo process group, the whole-job aggregation, and the reference arm's
rank handling (rank 0 prints one JSON line, other ranks exit without work)."""
import datetime
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench as b
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    # each rank's "device time"; the job's time is the slowest rank's
    v = b.max_over_ranks(dist, [2.5, 7.25][rank], torch.device("cpu"))
    dist.barrier()
    q.put((rank, v))
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 7.25, 1: 7.25}


def test_max_over_ranks_without_process_group():
    assert bench.max_over_ranks(None, 3.5, None) == 3.5


def test_whole_job_value_is_weak_scaling_aggregate():
    # 2 ranks each moving 1 GB in at most 10 ms: 200 GB/s for the job
    assert bench.whole_job_gbps(2, 1e9, 10.0) == pytest.approx(200.0)
    assert bench.whole_job_gbps(1, 1e9, 10.0) == pytest.approx(100.0)


def test_reference_arm_only_rank0_prints(monkeypatch, capsys):
    monkeypatch.setattr(bench, "oracle_sample_run",
                        lambda spec, seconds=10.0, outs_per_rep=None: (0.25, 4, "fake sample"))
    args = bench.parse_args(["--impl", "reference", "--steps", "2", "--warmup", "1", "--gpus", "2"])
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["value"] == 0.25
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 4
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    for k in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in line


def test_prefill_reference_arm_reports_tflops(monkeypatch, capsys):
    monkeypatch.setattr(bench, "oracle_prefill_sample",
                        lambda seconds=10.0, threads=None: (0.0007, 8, "fake prefill sample"))
    args = bench.parse_args(["--impl", "reference", "--workload", "prefill-qwen3-8b",
                             "--steps", "2", "--warmup", "1"])
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["metric"].startswith("prefill GEMM")
    assert line["value"] == pytest.approx(0.0007)
    assert line["e2e"]["unit"] == "TFLOP/s" and line["cpu_baseline"]["unit"] == "TFLOP/s"
    assert line["config"]["workload"] == "prefill-qwen3-8b"


def test_tensor_peak_reads_the_measured_file():
    import json as _json
    try:
        with open(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")) as f:
            mp_ = _json.load(f)
    except OSError:
        mp_ = {}
    for sustained, key, fallback in ((True, "bf16_tflops_sustained", 1400.0), (False, "bf16_tflops", 1590.0)):
        if key in mp_:
            assert bench.measured_tensor_peak(sustained) == (float(mp_[key]), "measured " + key)
        else:
            assert bench.measured_tensor_peak(sustained) == (fallback, "fallback")


def test_prefill_weights_shapes_and_ranges():
    import numpy as np
    q, s, z = bench.prefill_weights(np.random.default_rng(0), 256, 128, 6)
    assert q.shape == (256, 128) and q.dtype == np.uint8 and q.max() < 64
    assert s.shape == z.shape == (2, 128) and s.dtype == z.dtype == np.float16
    assert (s > 0).all() and (z <= 0).all()
