"""The profile summaries under profiles/ are text that names the commands behind their
figures.  Those commands must run committed files as they stand: every bench.py flag they
pass exists, every ncu command leaves the GPU clocks alone, and every traffic record names a
kernel class and workload that bench.py knows."""
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md")))


def _commands(path):
    """The indented command lines of a summary, continuation lines joined."""
    out, cur = [], ""
    for line in open(path, encoding="utf-8"):
        if not line.startswith("    "):
            if cur:
                out.append(cur)
            cur = ""
            continue
        part = line.strip()
        cur = (cur + " " + part.rstrip("\\").strip()) if cur else part.rstrip("\\").strip()
        if not part.endswith("\\"):
            out.append(cur)
            cur = ""
    if cur:
        out.append(cur)
    return out


def _bench_flags():
    src = open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read()
    return set(re.findall(r'add_argument\("(--[a-z0-9-]+)"', src))


def test_every_summary_names_its_command():
    assert PROFILES
    for p in PROFILES:
        assert any("python bench.py" in c for c in _commands(p)), os.path.basename(p)


@pytest.mark.parametrize("path", PROFILES, ids=[os.path.basename(p) for p in PROFILES])
def test_commands_use_existing_bench_flags(path):
    flags = _bench_flags()
    for cmd in _commands(path):
        for seg in cmd.split("python bench.py")[1:]:
            seg = re.split(r"[>|&]", seg)[0]
            for f in re.findall(r"(--[a-z0-9-]+)", seg):
                assert f in flags, (os.path.basename(path), f)


@pytest.mark.parametrize("path", PROFILES, ids=[os.path.basename(p) for p in PROFILES])
def test_ncu_commands_leave_clocks_alone(path):
    for cmd in _commands(path):
        for seg in re.split(r"&&|;", cmd):
            if seg.strip().startswith("ncu "):
                assert "--clock-control none" in seg, (os.path.basename(path), seg)


def test_traffic_records_name_known_classes_and_workloads():
    import bench
    names = set(bench.CLASS_NAMES.values())
    recs = [ln.split() for ln in open(os.path.join(ROOT, "profiles", "traffic.txt"), encoding="utf-8")
            if ln.strip() and not ln.startswith("#")]
    assert recs
    for f in recs:
        assert len(f) == 4, f
        assert f[0] in names and f[2] == bench.WORKLOAD, f
        assert re.fullmatch(r"[0-9a-f]{16}", f[1]) and float(f[3]) > 0, f
