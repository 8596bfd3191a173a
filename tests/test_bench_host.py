"""Host-side logic of the benchmark: the multi-rank reduction (gloo, world
size 2, on CPU), the throughput arithmetic, the oracle sample and the
reference arm's contract line."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from packed_attention_b200.workloads import WORKLOADS  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # rank r is slower on the first metric, faster on the second
    vals = bench.max_over_ranks([10.0 + rank, 5.0 - rank], world)
    q.put((rank, vals))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0] == got[1] == [11.0, 5.0]


def test_whole_job_throughput_counts_every_replica():
    w = WORKLOADS[4]
    v1, t1 = bench.whole_job_throughput(w.flops, w.total_tokens, 1, 100, 400.0)
    v2, t2 = bench.whole_job_throughput(w.flops, w.total_tokens, 2, 100, 400.0)
    assert v2 == pytest.approx(2 * v1) and t2 == pytest.approx(2 * t1)
    assert v1 == pytest.approx(w.flops / 4e-3 / 1e12)


def test_oracle_sample_rows_flops_are_per_distinct_row():
    w = WORKLOADS[2]
    rng = np.random.default_rng(0)
    rows, flops = bench.oracle_sample_rows(w, rng, 50)
    assert len(np.unique(rows)) == len(rows)
    lens = np.array(w.seg_lens)
    seg = np.searchsorted(np.cumsum(lens), rows // w.heads, side="right")
    assert flops == 4 * w.head_dim * int(lens[seg].sum())


def test_reference_arm_line_and_non_zero_ranks():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "0", "--steps", "2", "--warmup", "1", "--ref-seconds", "1"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    env1 = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out1 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--config", "0", "--steps", "2", "--warmup", "1"],
                          capture_output=True, text=True, env=env1, timeout=120)
    assert out1.returncode == 0 and out1.stdout.strip() == ""


def test_clock_sampler_waits_for_its_first_row_and_parses(monkeypatch, tmp_path):
    """The sampler blocks until nvidia-smi has written a row (so its start-up
    never overlaps timed work), then reports the median SM clock, the max
    clock and every throttle reason seen. A stand-in for nvidia-smi writes
    two rows after a delay."""
    fake = tmp_path / "fake_smi.py"
    fake.write_text(
        "import sys, time\n"
        "time.sleep(0.3)\n"
        "print('0, 1965, 1965, 330.5, 0x0, Not Active, Not Active, Not Active, Not Active', flush=True)\n"
        "print('0, 1800, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active', flush=True)\n"
        "time.sleep(30)\n")
    real_popen = subprocess.Popen

    def popen(args, **kw):
        assert args[0] == "nvidia-smi" and "-lms" in args
        return real_popen([sys.executable, str(fake)], **kw)

    monkeypatch.setattr(bench.subprocess, "Popen", popen)
    s = bench.ClockSampler(0)
    s.start()
    s.wait_first_row(limit_s=10.0)
    assert os.path.getsize(s.path) > 0
    clocks = s.stop()
    assert clocks["samples"] == 2
    assert clocks["sm_mhz"] == pytest.approx(1882.5)
    assert clocks["sm_max_mhz"] == 1965.0
    assert clocks["reasons"] == ["sw_power_cap"]
    assert clocks["power_w_max"] == pytest.approx(990.1)


def test_clock_sampler_without_nvidia_smi(monkeypatch):
    """No nvidia-smi: the sampler reports nothing and never blocks."""
    def popen(*a, **kw):
        raise OSError("not found")

    monkeypatch.setattr(bench.subprocess, "Popen", popen)
    s = bench.ClockSampler(0)
    s.start()
    s.wait_first_row(limit_s=1.0)
    path = s.path
    assert s.stop() is None
    assert not os.path.exists(path)  # its temporary file is removed too
