"""The committed ncu summaries agree with the benchmark that cites them.

Each `profiles/gattn_kernel_<workload>.md` names the command it was captured
with (`-s N -c 1` on the attention kernel: the (N+1)-th call, whose contexts
are the workload's first-call lengths + N), its algorithmic bytes per launch
and its DRAM traffic.  The algorithmic figure must be the bench's own byte
count for that call on the seeded workload, and the bench must take the
traffic only while the summary's source digest matches the kernel sources.
Every ncu command in the summaries keeps the clocks unlocked."""

import glob
import os
import re

import pytest

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = sorted(glob.glob(os.path.join(ROOT, "profiles", "gattn_kernel_*.md")))


def _fields(text):
    vals = {}
    for line in text.splitlines():
        item = line.strip().lstrip("-* ").strip()
        m = re.match(r"(source_sha1|traffic_bytes_per_launch|algorithmic_bytes_per_launch):\s*`?([0-9a-f]+)`?", item)
        if m:
            vals[m.group(1)] = m.group(2)
    return vals


def _commands(text):
    """The ncu commands of the summary, continuation lines joined."""
    lines, cmds = text.splitlines(), []
    for i, line in enumerate(lines):
        if re.search(r"(^|\s)ncu --", line.strip()):
            cmd = line.strip()
            j = i
            while cmd.endswith("\\"):
                j += 1
                cmd = cmd[:-1] + " " + lines[j].strip()
            cmds.append(cmd)
    return cmds


def test_every_summary_names_a_clock_neutral_command():
    files = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))
    assert files
    for path in files:
        cmds = _commands(open(path).read())
        assert cmds, path
        for cmd in cmds:
            assert "--clock-control none" in cmd, (path, cmd)
            assert "python bench.py" in cmd, (path, cmd)


@pytest.mark.parametrize("path", PROFILES, ids=[os.path.basename(p) for p in PROFILES])
def test_attention_summary_matches_the_bench_byte_count(path):
    name = os.path.basename(path)[len("gattn_kernel_"):-len(".md")]
    text = open(path).read()
    vals = _fields(text)
    cmd = _commands(text)[0]
    skip = int(re.search(r"\s-s\s+(\d+)", cmd).group(1))
    assert re.search(r"\s-c\s+1\b", cmd) and "gattn_kernel" in cmd
    if "--workload" in cmd:
        assert re.search(r"--workload\s+%s\b" % re.escape(name), cmd)
    else:
        assert name == "stack36"                 # the bench's default workload
    w = workloads.workload(name)
    L = workloads.context_lengths(w)
    want = bench.kv_bytes(L + skip, w["Hkv"], w["D"], w["S"], w["W"])
    assert int(vals["algorithmic_bytes_per_launch"]) == want
    traffic = int(vals["traffic_bytes_per_launch"])
    assert 1.0 <= traffic / want <= 1.05, traffic / want
    if vals["source_sha1"] == bench.kernel_source_hash():
        assert bench.profiled_traffic(name) == traffic
    else:
        assert bench.profiled_traffic(name) is None
