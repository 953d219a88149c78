"""Every command in profiles/ that runs the bench uses flags the bench still
has, and workloads it knows, so each summary can be reproduced from committed
files."""
import glob
import os
import re

import bench
from workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench_flags():
    src = open(os.path.join(ROOT, "bench.py")).read()
    return set(re.findall(r'add_argument\("(--[a-z0-9-]+)"', src))


def test_profile_commands_use_existing_flags():
    flags = _bench_flags()
    seen = 0
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = open(path).read().replace("\\\n", " ")
        for line in text.splitlines():
            if "python bench.py" not in line:
                continue
            cmd = line[line.index("python bench.py"):].split("#")[0]
            seen += 1
            for f in re.findall(r"(--[a-z0-9-]+)", cmd):
                assert f in flags, f"{os.path.basename(path)}: unknown bench flag {f}"
            m = re.search(r"--workload\s+(\S+)", cmd)
            if m:
                assert m.group(1) in WORKLOADS, f"{os.path.basename(path)}: {m.group(1)}"
    assert seen > 0
    assert bench.METRIC
