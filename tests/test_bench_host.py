"""Host-side plumbing of bench.py that needs no GPU: the replica launch under torchrun with
world_size 2 (gloo on CPU), the max-over-ranks timing, the reference arm running on rank 0
only, and the clock-sample summary."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_replicas_take_max_over_ranks(tmp_path):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "tests", "dist_worker.py"), str(tmp_path)]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=240)
    assert r.returncode == 0, r.stderr[-2000:]
    res = [json.load(open(tmp_path / f"rank{k}.json")) for k in range(2)]
    for k, x in enumerate(res):
        assert x["rank"] == k and x["world"] == 2 and x["backend"] == "gloo"
        assert x["max"] == 15.0          # 10 + 5 * rank, maximum over both ranks
    assert res[1]["skipped"] is True     # reference arm: rank 1 exits without work


def test_clock_summary_parses_reasons(tmp_path):
    import bench
    path = tmp_path / "clk.csv"
    path.write_text("0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
                    "0, 1900, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
                    "0, 1800, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active\n"
                    "garbage line\n")
    cs = bench.ClockSampler(0)
    cs.proc = object()          # pretend a sampler ran
    cs.path = str(path)
    s = cs.summary()
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]


def test_measured_peaks_present():
    import bench
    peak, kind = bench.measured_peaks()
    assert peak > 1000
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert kind == "measured"


def test_traffic_record_follows_kernel_code_not_comments(tmp_path):
    """The ncu traffic record applies while the kernel's code is the captured code: a comment
    edit keeps the hash, a code edit changes it (checked on a copy of the sources)."""
    import shutil
    import bench
    for rel in bench.KERNEL_SOURCES:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), dst)
    base = bench.kernel_code_hash(str(tmp_path))
    assert base == bench.kernel_code_hash()
    k = tmp_path / bench.KERNEL_SOURCES[0]
    src = k.read_text()
    k.write_text(src.replace("// ", "//  note: ", 3) + "\n/* trailing remark */\n")
    assert bench.kernel_code_hash(str(tmp_path)) == base
    k.write_text(src.replace("kScSlots = 4", "kScSlots = 5", 1))
    assert bench.kernel_code_hash(str(tmp_path)) != base
    # the bench quotes the record only while it was taken on the current kernel code
    rec = json.load(open(os.path.join(ROOT, "profiles", "decode_tc_traffic.json")))
    if rec["code_sha256"] == base:
        assert bench.decode_traffic() is not None
    else:
        assert bench.decode_traffic() is None
