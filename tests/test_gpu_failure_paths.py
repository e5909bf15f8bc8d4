"""Failure paths, made to happen without faulting or hanging the GPU.

* Device timeout: MRA_TEST_EXPIRE_WAIT=1 makes the first bounded mbarrier wait
  of every CTA of the tcgen05 attention kernel report expiry without waiting.
  The kernel must return (every role stops, its copies and MMAs in flight are
  drained, its tensor memory freed), the device status word must carry
  MRA_DEV_TIMEOUT (mra_status_from_device maps it to MRA_ERR_DEVICE_TIMEOUT),
  and the next call without the hook must be clean and match the oracle.
* Allocation failure: MRA_TEST_FAIL_ALLOC=1 makes the workspace growth fail on
  the host; the call returns MRA_ERR_ALLOC and launches nothing, and a later
  call without the hook succeeds.

Each case runs in a child process (fresh library state); the hooks are read
at every call, so the child sets and clears them between calls.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

TIMEOUT_CHILD = r'''
import os, sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import torch
import mra_testlib as tl
import resolution_block_sparse_b200 as mra
from resolution_block_sparse_b200 import _binding as b
from resolution_block_sparse_b200.workloads import random_inputs
inputs = random_inputs(1, 2, 1024, 64, dtype=torch.bfloat16, seed=31, pad_tokens=[70], v_scale=1.0)
kw = dict(block_per_row=32, approx_mode=0, first_n=0, diag_n=0)   # every block selected: tcgen05 kernel
os.environ["MRA_TEST_EXPIRE_WAIT"] = "1"
gpu = tl.run_gpu(inputs, want_intermediates=False, **kw)
st = gpu["status"]
assert st & b.MRA_DEV_TIMEOUT, st
assert mra.mra_status_from_device(st) == b.MRA_ERR_DEVICE_TIMEOUT
del os.environ["MRA_TEST_EXPIRE_WAIT"]
gpu = tl.run_gpu(inputs, **kw)
stats = tl.compare(inputs, gpu, tl.run_oracle(inputs, **kw))
assert mra.mra_get_device_status() == 0
print("RESULT", stats)
'''

ALLOC_CHILD = r'''
import os, sys
sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
import numpy as np, torch
import mra_testlib as tl
import resolution_block_sparse_b200 as mra
from resolution_block_sparse_b200 import _binding as b
from resolution_block_sparse_b200.workloads import random_inputs
inputs = random_inputs(1, 2, 1024, 64, dtype=torch.bfloat16, seed=32, pad_tokens=[0], v_scale=1.0)
dev = torch.device("cuda:0")
q, k, v = (inputs[x].to(dev) for x in ("q", "k", "v"))
out = torch.full_like(q, float("nan"))
lib = mra.load_library()
os.environ["MRA_TEST_FAIL_ALLOC"] = "1"
st = lib.mra_attention_fwd(b._ptr(q), b._ptr(k), b._ptr(v), None, b._ptr(out), 1, 2, 1024, 64, 4, 1, 1, 1, None)
assert st == b.MRA_ERR_ALLOC, st
assert "allocation" in mra.mra_status_string(st)
torch.cuda.synchronize()
assert torch.isnan(out.float()).all(), "nothing may be written after a failed allocation"
del os.environ["MRA_TEST_FAIL_ALLOC"]
gpu = tl.run_gpu(inputs, block_per_row=4, approx_mode=1, first_n=1, diag_n=1)
tl.compare(inputs, gpu, tl.run_oracle(inputs, block_per_row=4, approx_mode=1, first_n=1, diag_n=1))
print("RESULT ok")
'''


@pytest.mark.parametrize("child,env", [(TIMEOUT_CHILD, {"MRA_ATTN_IMPL": "tc"}), (ALLOC_CHILD, {})],
                         ids=["device_timeout", "alloc_failure"])
def test_failure_path(child, env):
    e = dict(os.environ, **env)
    e.pop("MRA_TEST_EXPIRE_WAIT", None)
    e.pop("MRA_TEST_FAIL_ALLOC", None)
    r = subprocess.run([sys.executable, "-c", child, ROOT], env=e, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert "RESULT" in r.stdout
