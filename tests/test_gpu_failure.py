"""Failure detection without a GPU fault.  Each test makes a bounded device
wait run out on purpose and checks that the kernel records EA_ERR_TIMEOUT in
the status word, leaves cleanly (drains its copies and MMAs, frees TMEM) and
that the CUDA context stays usable.

The waits are made to run out by the failure-injection hooks, which only the
test build of the library (libea_testhooks.so, compiled with EA_TEST_HOOKS)
carries; libea.so ignores the environment.  Each case runs in a child
process, because the hooks and the wait limit are read once per process:
- a copy the fused kernel waits for never happens (EA_DEBUG_DROP_KV_POS);
- CTA 0 of the routed one-launch path leaves without arriving at one of its
  grid barriers (EA_DEBUG_SKIP_GRID_SYNC), so the other CTAs' bounded
  barrier waits run out."""
import os
import subprocess
import sys

import pytest
import torch

from sparse_attention_head_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# The child loads the test build of the library before any call.
PRELUDE = r'''
import sys, torch
sys.path.insert(0, ROOT)
import workloads
from sparse_attention_head_b200 import _lib
_lib.LIB_PATH = TESTHOOKS
from sparse_attention_head_b200.api import (attn_workspace, ea_get_device_status,
    ea_hybrid_attn_prefill, ea_hybrid_attn_prefill_routed, ea_router_decide, make_params)
w = workloads.get("tiny")
q, k, v = (t.cuda() for t in workloads.make_qkv(w, 0))
mask = workloads.make_fixed_mask(w, 0).cuda()

def context_still_serves_work():
    # plain torch work and a library call no hook touches
    x = torch.randn(256, 256, device="cuda")
    y = (x @ x).sum().item()
    assert y == y
    w1 = torch.randn(32, 128, device="cuda"); b1 = torch.zeros(32, device="cuda")
    w2 = torch.randn(4, 32, device="cuda"); b2 = torch.zeros(4, device="cuda")
    m, z = ea_router_decide(k, w1, b1, w2, b2)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(z).all())
'''

DROPPED_COPY = PRELUDE + r'''
ws = attn_workspace(make_params(1, 4, 2, 512, 64, 16, 128), "cuda")
ea_hybrid_attn_prefill(q, k, v, mask, 16, 128, workspace=ws)
st = ea_get_device_status(ws)
assert st == _lib.EA_ERR_TIMEOUT, st
assert ea_get_device_status(ws) == 0          # the word was cleared
context_still_serves_work()
print("TIMEOUT_OK")
'''

SKIPPED_GRID_ARRIVAL = PRELUDE + r'''
g = torch.Generator().manual_seed(3)
w1 = (torch.randn(32, 128, generator=g) * 0.05).cuda(); b1 = torch.zeros(32, device="cuda")
w2 = (torch.randn(4, 32, generator=g) * 0.2).cuda(); b2 = torch.zeros(4, device="cuda")
ws = torch.zeros(1 << 22, dtype=torch.uint8, device="cuda")
route = torch.full((1, 4), 9, dtype=torch.uint8, device="cuda")
out = torch.full_like(q, 7.0)
ea_hybrid_attn_prefill_routed(q, k, v, w1, b1, w2, b2, 16, 128, route_mask=route, out=out,
                              workspace=ws)
st = ea_get_device_status(ws)
assert st == _lib.EA_ERR_TIMEOUT, st
assert ea_get_device_status(ws) == 0          # status word and barrier cleared
# the launch ended at the barrier: no attention output was written
assert bool((out == 7.0).all())
context_still_serves_work()
print("TIMEOUT_OK")
'''


def _run_child(code: str, env_extra: dict):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    env = dict(os.environ, EA_WAIT_TIMEOUT_MS="300", **env_extra)
    src = code.replace("ROOT", repr(ROOT)).replace("TESTHOOKS", repr(build.TESTHOOKS_LIB))
    res = subprocess.run([sys.executable, "-c", src], env=env, capture_output=True, text=True,
                         timeout=180)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "TIMEOUT_OK" in res.stdout


def test_dropped_copy_times_out_and_context_survives():
    _run_child(DROPPED_COPY, {"EA_DEBUG_DROP_KV_POS": "3"})


@pytest.mark.parametrize("phase", [0, 3])
def test_skipped_grid_arrival_times_out_and_context_survives(phase):
    """Phase 0 is the barrier after pooling, 3 the one after the route mask
    is written (the last before the attention pipeline starts)."""
    _run_child(SKIPPED_GRID_ARRIVAL, {"EA_DEBUG_SKIP_GRID_SYNC": str(phase)})


def test_release_library_ignores_the_hooks():
    """With the hooks' variables set, libea.so still runs the routed launch
    and the fused prefill to completion (status 0)."""
    code = PRELUDE.replace("_lib.LIB_PATH = TESTHOOKS\n", "") + r'''
ws = attn_workspace(make_params(1, 4, 2, 512, 64, 16, 128), "cuda")
ea_hybrid_attn_prefill(q, k, v, mask, 16, 128, workspace=ws)
assert ea_get_device_status(ws) == 0
w1 = torch.randn(32, 128, device="cuda") * 0.05; b1 = torch.zeros(32, device="cuda")
w2 = torch.randn(4, 32, device="cuda") * 0.2; b2 = torch.zeros(4, device="cuda")
wsr = torch.zeros(1 << 22, dtype=torch.uint8, device="cuda")
ea_hybrid_attn_prefill_routed(q, k, v, w1, b1, w2, b2, 16, 128, workspace=wsr)
assert ea_get_device_status(wsr) == 0
print("TIMEOUT_OK")
'''
    _run_child(code, {"EA_DEBUG_DROP_KV_POS": "3", "EA_DEBUG_SKIP_GRID_SYNC": "0"})
