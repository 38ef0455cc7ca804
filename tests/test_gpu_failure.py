"""Failure detection without a GPU fault: a copy the fused kernel waits for
never happens (test hook EA_DEBUG_DROP_KV_POS), so its bounded wait runs out.
The kernel must record EA_ERR_TIMEOUT in the status word, leave cleanly
(drain copies and MMAs, free TMEM), and the CUDA context must stay usable.
Runs in a child process because the hook and the wait limit are read once
per process."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, torch
sys.path.insert(0, ROOT)
import workloads
from sparse_attention_head_b200 import _lib
from sparse_attention_head_b200.api import (attn_workspace, ea_get_device_status,
    ea_hybrid_attn_prefill, ea_router_decide, make_params)
w = workloads.get("tiny")
q, k, v = (t.cuda() for t in workloads.make_qkv(w, 0))
mask = workloads.make_fixed_mask(w, 0).cuda()
ws = attn_workspace(make_params(1, 4, 2, 512, 64, 16, 128), "cuda")
ea_hybrid_attn_prefill(q, k, v, mask, 16, 128, workspace=ws)
st = ea_get_device_status(ws)
assert st == _lib.EA_ERR_TIMEOUT, st
assert ea_get_device_status(ws) == 0          # the word was cleared
# the context is still usable: plain torch work and another library call
x = torch.randn(256, 256, device="cuda")
y = (x @ x).sum().item()
assert y == y
w1 = torch.randn(32, 128, device="cuda"); b1 = torch.zeros(32, device="cuda")
w2 = torch.randn(4, 32, device="cuda"); b2 = torch.zeros(4, device="cuda")
m, z = ea_router_decide(k, w1, b1, w2, b2)
torch.cuda.synchronize()
print("TIMEOUT_OK")
'''


def test_dropped_copy_times_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, EA_WAIT_TIMEOUT_MS="300", EA_DEBUG_DROP_KV_POS="3")
    res = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT))], env=env,
                         capture_output=True, text=True, timeout=180)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "TIMEOUT_OK" in res.stdout
