"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (127.0.0.1),
each with its own device time, agree on the slowest rank's time and on the
whole-job throughput; the reference arm works on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench.dist_setup()
        ms = bench.max_over_ranks(times[rank], w, "cpu")
        value = bench.job_throughput(1e9, 4, w, ms)
        out[rank] = (w, r, local, ms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_the_whole_job_bytes():
    world, port = 2, _free_port()
    times = [3.0, 5.0]
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, times, out), nprocs=world,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank in (0, 1):
        w, r, local, ms, value = res[rank]
        assert (w, r, local) == (2, rank, rank)
        assert ms == 5.0                                  # the slowest rank
        assert value == pytest.approx(1e9 * 4 * 2 / 5e-3 / 1e9)


def test_single_rank_is_a_no_op():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.job_throughput(2e9, 10, 1, 1000.0) == pytest.approx(20.0)


def _ref_rank(rank, world, out):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import argparse
    import io
    import contextlib
    import bench
    from quantized_recurrent_state_mamba_b200 import workloads as W
    wl = W.tiny()
    args = argparse.Namespace(steps=1, warmup=0, cpu_budget=0.5, cpu_workers=2)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.run_reference(args, wl, "tiny")
    out[rank] = (rc, buf.getvalue())


def test_reference_arm_runs_on_rank_0_only():
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_ref_rank, args=(2, out), nprocs=2, start_method="spawn")
        res = dict(out)
    assert res[0][0] == 0 and res[1][0] == 0
    assert '"impl": "reference"' in res[0][1]
    assert res[1][1] == ""


def test_kernel_source_hash_ignores_comments_only():
    """The ncu summaries stay attached to a kernel through comment edits and
    drop off when its code changes; each kernel family hashes its own
    sources."""
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) { return x + 1; } // one\n/* two\n lines */ int g;"
    b = "int f(int x)  {\n  return x + 1;\n}\n// other words\nint g;"
    c = "int f(int x) { return x + 2; } int g;"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    fams = {bench._kernel_family(w) for w in
            ("decode_130m", "decode_130m_sr", "decode_130m_damp", "scan_370m_all",
             "prefill_370m_mid", "diag_130m")}
    assert fams == {"decode", "damp", "scan", "diag"}
    hashes = {w: bench.kernel_source_hash(w) for w in
              ("decode_130m", "decode_130m_damp", "scan_370m_all", "diag_130m")}
    # the diagnostics pass is the decode kernel in its diagnostics mode
    assert len(set(hashes.values())) == 3
    assert hashes["diag_130m"] == hashes["decode_130m"]
    assert bench.kernel_source_hash("decode_130m_sr") == hashes["decode_130m"]


def test_gpus_n_starts_n_ranks_when_no_launcher_did():
    """bench.py --gpus 2 without a launcher starts two ranks itself
    (torch.distributed.run on 127.0.0.1); with the reference arm rank 0
    prints the one JSON line and reports both ranks."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "0",
                        "--cpu-budget", "0.5", "--cpu-workers", "1"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["cores"] == 1


def test_gpus_n_must_match_the_launcher():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "4", "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "WORLD_SIZE=2" in r.stderr


def test_l2_rotation_counts():
    """A step whose footprint is under 4x the L2 rotates over enough copies
    to reach it; the 130M decode step needs none."""
    sys.path.insert(0, ROOT)
    import bench
    L2 = bench.L2_FALLBACK_BYTES
    big = bench.workload("decode_130m")
    assert bench.footprint_bytes(big, "decode_130m") > 4 * L2
    small = bench.workload("decode_8b_b64_i8a")
    f = bench.footprint_bytes(small, "decode_8b_b64_i8a")
    rows = 64 * 128 * 64
    assert f == rows * (128 + 8) + bench.decode_bytes(small) - 2 * rows * (128 + 8)
    assert f < 4 * L2
