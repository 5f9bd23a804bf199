"""Launch register counts of the kernels that move registers between
warpgroups with setmaxnreg. Each split was computed for one launch count
(the most __launch_bounds__ allows); ptxas must report exactly that count,
since setmaxnreg.inc can only take registers the launch reserved and a
smaller launch count would leave it waiting. Also: no spills. CPU only (nvcc
cross-compiles; ptxas prints the counts with -v)."""
import os
import re
import subprocess

import pytest

from transformer_attention_gqa_b200 import build as B

# kernel name -> registers per thread at launch (threads x registers = the split's total)
EXPECTED = {"gqa_attn_fwd_kernel": 128, "gqa_attn_bwd_kernel": 128}


@pytest.fixture(scope="module")
def ptxas_report(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("regs") / "lib.so")
    cmd = [B.nvcc_path()] + B.NVCC_FLAGS + ["-Xptxas", "-v", "-o", out, B.SRC]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stderr


def kernel_reports(text):
    """(mangled name, registers, spill store bytes, spill load bytes) per entry function."""
    reps = []
    name = None
    spills = (0, 0)
    for line in text.splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            name = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and name:
            spills = (int(m.group(1)), int(m.group(2)))
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and name:
            reps.append((name, int(m.group(1))) + spills)
            name = None
    return reps


def test_setmaxnreg_kernels_launch_with_the_split_register_count(ptxas_report):
    reps = kernel_reports(ptxas_report)
    seen = {k: 0 for k in EXPECTED}
    for name, regs, st, ld in reps:
        for kern, want in EXPECTED.items():
            if kern in name:
                seen[kern] += 1
                assert regs == want, (name, regs)
                assert st == 0 and ld == 0, (name, st, ld)
    # forward: 3 head dims x (bf16, fp32, masked bf16); backward: 3 head dims
    assert seen == {"gqa_attn_fwd_kernel": 9, "gqa_attn_bwd_kernel": 3}, seen
