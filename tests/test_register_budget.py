"""Register budgets of the coded single-token kernels (CPU: nvcc only).

The int8_hadamard32 kernel at K = 128 holds 128 state values per lane and
runs twelve one-warp CTAs per SM, which leaves 168 registers a thread; the
fp8 kernel runs four CTAs of four warps, 128 registers. Spills or a larger
budget cost those kernels a large share of their speed, so the instantiations
of the configured workloads (slot pools, bf16 inputs, working readout) are
compiled here with ptxas' report and held to both.
"""

import os
import re
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "gated_delta_rule_80_b200", "csrc")
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

# (header, explicit instantiation, register limit)
CASES = [
    ("gdn_group_i8.cuh", "template __global__ void gdn::step_group_i8<0, true, false>(const gdn::StepParams, int64_t);",
     168),
    ("gdn_stream_fp8.cuh",
     "template __global__ void gdn::step_stream_fp8<128, 0, 2, 1>(const gdn::StepParams, int64_t);", 128),
]


@pytest.mark.skipif(not os.path.exists(NVCC), reason="needs nvcc")
@pytest.mark.parametrize("header,inst,limit", CASES)
def test_no_spills_within_budget(header, inst, limit):
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "k.cu")
        with open(src, "w") as f:
            f.write(f'#include "{header}"\n{inst}\n')
        r = subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                            "--expt-relaxed-constexpr", "-I" + CSRC, "-I" + os.path.join(ROOT, "include"),
                            "-Xptxas", "-v", "-c", src, "-o", os.path.join(d, "k.o")],
                           capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    spills = [int(x) for x in re.findall(r"(\d+) bytes spill stores", r.stderr)]
    regs = [int(x) for x in re.findall(r"Used (\d+) registers", r.stderr)]
    assert spills and regs, r.stderr[-2000:]
    assert max(spills) == 0, f"{inst}: {max(spills)} bytes of spill stores"
    assert max(regs) <= limit, f"{inst}: {max(regs)} registers, budget {limit}"
