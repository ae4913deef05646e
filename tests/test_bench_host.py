"""Host logic of bench.py, on the CPU: the multi-process plumbing (gloo,
world size 2), the clock-record parser and the profile-backed traffic field.

The benchmark runs one replica per GPU with no collective on the data path;
its only cross-rank steps are barriers and the max-over-ranks of the timed
region, which these tests exercise with the gloo backend.
"""
import hashlib
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench as b
    import torch.distributed as dist
    w, r, _ = b.dist_setup()
    got = b.max_over_ranks(1.5 + r, w)
    b.barrier(w)
    q.put((r, w, got))
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [x[0] for x in res] == [0, 1]
    assert all(x[1] == 2 and x[2] == 2.5 for x in res)


@pytest.mark.slow
def test_reference_arm_under_torchrun_prints_one_line():
    """Two ranks: rank 0 alone times the oracle and prints; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus",
           "2", "--steps", "1", "--warmup", "0"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    # the same workload and config dict as the main arm's line at this world size
    import sws_inputs as W
    assert line["config"] == bench.workload_config(bench.headline_workload(W), 2)
    assert line["ms_per_step"] > 0 and line["extrapolated_ms_per_full_pass"] > line["ms_per_step"]


def test_clock_parser_flags_throttle_reasons():
    c = bench.ClockSampler("00000000:1b:00.0")
    c.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0})()
    c.th = type("T", (), {"join": lambda self, timeout=None: None})()
    c.skip = 0
    c.lines = [
        "00000000:1B:00.0, 1965, 1965, 400.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "00000000:1B:00.0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "00000000:1B:00.0, 1700, 1965, 1001.0, 0x4, Not Active, Not Active, Not Active, Active",
        "00000000:2C:00.0, 900, 1965, 100.0, 0x8, Active, Not Active, Not Active, Not Active",  # another GPU
        "garbage",
    ]
    r = c.stop()
    assert r["samples"] == 3 and r["sm_mhz"] == 1800 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 1001.0


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    csrc = tmp_path / "block_sparse_attention_sws_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_bytes(b"kernel v1")
    digest = hashlib.sha256(b"kernel v1").hexdigest()
    (tmp_path / "profiles" / "p.md").write_text(
        f"# p\n\n- kernel source sha256: `{digest}`\n- dram bytes per launch (read + write): 1234.5\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("p", "k.cu") == 1234.5
    src.write_bytes(b"kernel v2")  # changed since the capture: no traffic figure
    assert bench.profiled_traffic("p", "k.cu") is None
    assert bench.profiled_traffic("missing", "k.cu") is None
