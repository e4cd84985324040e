"""The N > 1 path of bench.py on CPU: two gloo ranks agree on the slowest
rank's step time and on the whole-job rate; the reference arm does no work
on ranks other than 0.  No data-path collective exists: ranks only exchange
the timing."""

import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = 1.0 + rank * 0.5          # rank 1 is the slow one
        m = bench.max_over_ranks(ms, dist, "cpu")
        out[rank] = (m, bench.whole_job_rate(8192, world, m))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_rate():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    m, rate = res[0]
    assert m == pytest.approx(1.5)
    assert rate == pytest.approx(2 * 8192 / 1.5e-3)


def test_reference_arm_is_rank0_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from synthetic import workload

    monkeypatch.setenv("RANK", "1")

    class A:
        gpus, steps, warmup = 2, 3, 3

    assert bench.run_reference(A, workload("qwen3-4b")) == 0


def test_reference_arm_line_keeps_the_contract(monkeypatch, capsys):
    """Rank 0 of the reference arm times the oracle and prints one JSON line
    with the benchmark's keys, "impl": "reference", a cpu_baseline describing
    the run and an e2e with no host-device bytes."""
    import json

    sys.path.insert(0, ROOT)
    import bench
    from synthetic import workload

    monkeypatch.setenv("RANK", "0")

    class A:
        gpus, steps, warmup = 1, 3, 3

    assert bench.run_reference(A, workload("tiny-fp32")) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny-fp32"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["unit"] == d["unit"] and cb["sample"] and cb["blas"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_roofline_peak_follows_the_timed_region():
    """A short region at full clocks is held against the burst GEMM peak; a
    seconds-long region, or one whose clocks fell, against the sustained one."""
    sys.path.insert(0, ROOT)
    import bench

    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    capped = {"sm_mhz": 1410.0, "sm_max_mhz": 1965.0}
    assert bench.choose_peak_kind(0.027, full) == "burst"       # 20 steps of 1.36 ms
    assert bench.choose_peak_kind(0.14, full) == "burst"        # 100 steps
    assert bench.choose_peak_kind(3.3, full) == "sustained"     # 100 steps of 33 ms
    assert bench.choose_peak_kind(0.14, capped) == "sustained"
    assert bench.choose_peak_kind(0.14, {"sm_mhz": None, "sm_max_mhz": None}) == "burst"


def test_forward_launch_count_follows_the_form():
    """The bench's gpu_launches claim: kernels per forward of the default build,
    by the form AUTO (or the caller) takes."""
    import types

    sys.path.insert(0, ROOT)
    import bench
    import weight_gated_mlp_b200 as ittt
    from synthetic import workload

    def count(name, form="auto", clip=0.0, **kw):
        w = workload(name).with_(**kw) if kw else workload(name)
        return bench.forward_launches(ittt, w, types.SimpleNamespace(form=form, clip=clip))

    # gate/up, conv, target, scan, gram + dual output of chunks 0-1, apply
    assert count("qwen3-4b") == 7
    assert count("qwen3-4b", clip=0.3) == 9                 # + norms, row scaling
    assert count("qwen3-4b", T=1024) == 5                   # two chunks: no dual-form head
    assert count("qwen3-4b-128k-c256") == 6                 # AUTO: hybrid (scan, gram, output)
    assert count("qwen3-4b", form="dual") == 6              # gram, output, one-chunk scan
    assert count("qwen3-4b", eta=0.0) == 5                  # W_down0 broadcast, apply
    assert count("tiny-fp32") == 3 + 2 + 1 + 2              # SIMT GEMMs, conv, scan
