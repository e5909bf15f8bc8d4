"""Parity of both attention kernels on every bf16, head size 64 case: the
tcgen05 kernel (groups of four block rows over the union of their selected
blocks; the default on dense maps), forced with MRA_ATTN_IMPL=tc, and the
warp-level mma.sync kernel (the default on sparse maps), forced with
MRA_ATTN_IMPL=mma.

The kernel choice is read once per process, so each case runs in a child
process with the variable set; the child compares the CUDA output with the
oracle on the same seeded inputs and reports the error, and checks that the
device status word stayed clear.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import numpy as np, torch
import mra_testlib as tl
from resolution_block_sparse_b200.workloads import WORKLOADS, make_inputs, random_inputs
case = json.loads(sys.argv[2])
if "workload" in case:
    w = WORKLOADS[case["workload"]]
    inputs = make_inputs(w)
    kw = dict(block_per_row=w.block_per_row, approx_mode=w.approx_mode, first_n=w.first_n, diag_n=w.diag_n)
else:
    inputs = random_inputs(case["B"], case["H"], case["N"], 64, dtype=torch.bfloat16, seed=case["seed"],
                           pad_tokens=case.get("pad"), v_scale=1.0)
    kw = dict(block_per_row=case["bpr"], approx_mode=case["mode"], first_n=case["f"], diag_n=case["g"])
gpu = tl.run_gpu(inputs, **kw)
ora = tl.run_oracle(inputs, **kw)
stats = tl.compare(inputs, gpu, ora)
from resolution_block_sparse_b200 import mra_get_device_status
assert mra_get_device_status() == 0, mra_get_device_status()
print("RESULT " + json.dumps(stats))
'''

CASES = [
    {"workload": 4},
    {"workload": 2},
    {"workload": 5},
    {"workload": 3},
    {"B": 1, "H": 2, "N": 1024, "bpr": 4, "mode": 0, "f": 1, "g": 1, "seed": 3, "pad": [100]},
    {"B": 1, "H": 2, "N": 2048, "bpr": 40, "mode": 1, "f": 1, "g": 1, "seed": 4},
    {"B": 2, "H": 3, "N": 288, "bpr": 2, "mode": 0, "f": 1, "g": 1, "seed": 5, "pad": [0, 70]},
    {"B": 1, "H": 1, "N": 8192, "bpr": 2, "mode": 0, "f": 1, "g": 0, "seed": 6},
    {"B": 2, "H": 1, "N": 256, "bpr": 2, "mode": 1, "f": 0, "g": 0, "seed": 7, "pad": [256, 0]},
    {"B": 1, "H": 2, "N": 96, "bpr": 1, "mode": 0, "f": 0, "g": 0, "seed": 8},               # 3 rows: group past the end
    {"B": 2, "H": 2, "N": 512, "bpr": 16, "mode": 0, "f": 0, "g": 0, "seed": 9, "pad": [0, 33]},   # saturated, padded keys
    {"B": 1, "H": 2, "N": 800, "bpr": 3, "mode": 1, "f": 2, "g": 3, "seed": 10, "pad": [100]},
    {"B": 1, "H": 1, "N": 8192, "bpr": 2, "mode": 1, "f": 1, "g": 0, "seed": 11, "pad": [300]},   # split groups, merge
]


@pytest.mark.parametrize("impl", ["tc", "mma"])
@pytest.mark.parametrize("case", CASES, ids=[json.dumps(c, sort_keys=True) for c in CASES])
def test_attention_kernel_parity(case, impl):
    env = dict(os.environ, MRA_ATTN_IMPL=impl)
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, json.dumps(case)], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert "RESULT" in r.stdout
