"""Host logic of bench.py on CPU: max-over-ranks timing and whole-job
aggregation across two gloo ranks, the reference arm's rank gating, and the
clock-sample parser."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    r = bench.Ranks("gloo")
    r.barrier()
    ms = 10.0 + 5.0 * rank                      # rank 1 is the slower one
    m = r.max(ms)
    value = bench.aggregate_value(8192, r.world, m / 1e3)
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
        json.dump({"max": m, "value": value, "world": r.world}, f)
    r.barrier()
    r.close()


def test_two_rank_max_and_aggregate(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(2)]
    for d in res:
        assert d["world"] == 2
        assert d["max"] == 15.0                  # every rank sees the slowest rank's time
        assert d["value"] == pytest.approx(2 * 8192 / 0.015)


def test_aggregate_single():
    assert bench.aggregate_value(8192, 1, 0.5e-3) == pytest.approx(16384000.0)


def test_reference_arm_nonzero_rank_exits_without_work(tmp_path):
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_reference_arm_line(tmp_path):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--workload", "wo_1p3b"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"]


def test_clock_parser():
    c = bench.ClockSampler("GPU-x")

    class P:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    class T:
        def join(self, timeout=None):
            pass

    c.proc, c.t = P(), T()
    c.lines = ["0, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Not Active",
               "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
               "0, 1900, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
               "garbage"]
    r = c.stop()
    assert r["sm_mhz"] == 1900 and r["sm_max_mhz"] == 1965 and r["reasons"] == ["sw_power_cap"]
    assert r["samples"] == 3


def test_clock_record_rejection():
    """A timed region is measured again when its clock record shows a hardware
    or thermal slowdown, or a clock far below its maximum with no reason (a
    leftover clock lock); power-cap throttling alone is kept."""
    ok = {"sm_mhz": 1590.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 500}
    assert not bench.clocks_rejected(ok)
    assert not bench.clocks_rejected({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 9})
    for r in bench.BAD_REASONS:
        assert bench.clocks_rejected(dict(ok, reasons=["sw_power_cap", r]))
    assert bench.clocks_rejected({"sm_mhz": 1000.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 50})
    # a low clock with the power cap active is the cap, not a lock
    assert not bench.clocks_rejected(dict(ok, sm_mhz=1000.0))
    # no clock source: nothing to judge
    assert not bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"],
                                      "samples": 0})


def test_traffic_record_follows_its_sources(tmp_path, monkeypatch):
    """DRAM traffic from the committed ncu record is reported only while the
    kernel's sources hash to the digest recorded with it; a changed source (or
    a missing entry) reports nothing."""
    src = tmp_path / "k.cu"
    src.write_text("// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"sources": ["k.cu"], "dram_bytes_per_launch": 12345, "source_sha256": bench.source_digest(["k.cu"])}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"k": rec}))
    assert bench.measured_traffic("k") == 12345
    assert bench.measured_traffic("other") is None
    src.write_text("// kernel v2\n")
    assert bench.measured_traffic("k") is None


def test_profile_commands_use_current_options():
    """Every bench.py command quoted in profiles/*.md (indented command lines,
    with their backslash continuations) parses with bench.py's present options,
    and names only workloads that exist."""
    import glob
    import re
    import shlex
    from ternary_gemm_b200.inputs import WORKLOADS
    found = 0
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        lines = open(path).read().split("\n")
        i = 0
        while i < len(lines):
            line = lines[i]
            if line.startswith("    ") and "bench.py" in line:
                cmd = re.split(r"\s{2,}\(", line.strip())[0]          # a trailing "(aside)" is prose
                while cmd.endswith("\\") and i + 1 < len(lines):
                    i += 1
                    cmd = cmd[:-1] + " " + lines[i].strip()
                words = shlex.split(cmd)
                k = max(j for j, w in enumerate(words) if w.endswith("bench.py"))
                args = [w for w in words[k + 1:] if not re.match(r"^[>|&]|^\d?>", w)]
                a = bench.parse_args(args)
                assert a.workload in WORKLOADS, (path, cmd)
                found += 1
            i += 1
    assert found >= 5


def test_traffic_record_sources_cover_the_kernels_includes():
    """Each DRAM-traffic record digests its kernel file and every library
    header that file includes, directly or not, so any change to the compiled
    kernel withdraws the record."""
    import re
    csrc = os.path.join(ROOT, "ternary_gemm_b200", "csrc")

    def closure(f, seen):
        p = os.path.join(csrc, f)
        if f in seen or not os.path.exists(p):
            return seen
        seen.add(f)
        for inc in re.findall(r'#include\s+"([^"]+)"', open(p).read()):
            closure(inc, seen)
        return seen

    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for key, kernel_file in (("gemm_7b_wdown", "gemm_i8.cu"), ("k1_7b_wdown", "fht_quant_tc.cu")):
        have = {os.path.basename(p) for p in rec[key]["sources"]}
        assert closure(kernel_file, set()) <= have, key
