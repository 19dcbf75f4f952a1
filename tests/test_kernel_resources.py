"""Every sm_100a kernel of libvi compiles without register spills.

Compiles each csrc/*.cu with the library's own nvcc flags and -Xptxas -v (no
GPU needed) and reads ptxas' report.  The tensor-core kernels run near the
register budget of their launch shapes (the persistent conv at up to 182
registers a thread, the fused attention kernel at 111-125 with 448 threads);
a spill there would move state to local memory on the hot path, so a change
that introduces one fails here, before any GPU run."""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from clip_temporal_modules_b200 import build as vibuild  # noqa: E402

SPILL = re.compile(r"(\d+) bytes spill stores, (\d+) bytes spill loads")
ENTRY = re.compile(r"Compiling entry function '([^']+)'")


def _ptxas_report(src: str, tmp_path) -> str:
    flags = [f for f in vibuild.NVCC_FLAGS if f != "-shared"]
    cmd = [vibuild.nvcc(), *flags, "-I", os.path.join(ROOT, "include"), "-c", "-o",
           str(tmp_path / "k.o"), src]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    return res.stderr


@pytest.mark.parametrize("src", vibuild.sources(), ids=os.path.basename)
def test_no_register_spills(src, tmp_path):
    report = _ptxas_report(src, tmp_path)
    entry, spills = None, []
    for line in report.splitlines():
        m = ENTRY.search(line)
        if m:
            entry = m.group(1)
            continue
        m = SPILL.search(line)
        if m and (int(m.group(1)) or int(m.group(2))):
            spills.append((entry, line.strip()))
    assert not spills, spills
