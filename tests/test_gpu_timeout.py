"""The bounded device wait, run out on purpose on a healthy GPU.

Every mbarrier wait in the library gives up after a bounded time, records
MOE_ERR_TIMEOUT in the error word, waits (again bounded) for what its warp
still has in flight and returns, so a copy that never completes cannot hang
the GPU.  This test builds the library with its test hooks and a 2 ms wait
limit, and makes the flat bulk dispatch's first warp announce the bytes of
one load without issuing it: that wait can only run out.  Nothing is left in
flight, so no fault is involved.  Checked: the call returns, the error word
reads MOE_ERR_TIMEOUT, and the next normal dispatch and combine on the same
stream match the oracle bit for bit.

The hooked build runs in a child process (the library is bound once per
process), so the rest of the suite keeps the production build.
"""
import json
import os
import subprocess
import sys

import pytest

from combine_moe_layout_06_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TEST_LIB = os.path.join(ROOT, "combine_moe_layout_06_b200", "_build", "libmoe_layout_testhooks.so")

CHILD = r"""
import json, os, sys, time
import numpy as np
import torch
sys.path.insert(0, os.environ["MOE_ROOT"])
import oracle
from combine_moe_layout_06_b200 import buffers, capi, inputs

T, H, E, k, R = 700, 1024, 16, 4, 4
d = inputs.make_random(T, H, E, k, seed=21)
x, topk, w = d["x"], d["topk_idx"], d["topk_w"]
cfg = capi.config(T, H, E, k, R)
lay = buffers.DeviceLayout(cfg)
topk_dev = torch.from_numpy(topk).cuda()
x_dev = buffers.bf16_from_bits(x)
recv = torch.empty((T * k, H), dtype=torch.bfloat16, device="cuda")
capi.moe_layout(cfg, topk_dev, lay.struct)
torch.cuda.synchronize()
out = {}
os.environ["MOE_TEST_SKIP_LOAD"] = "0"
t0 = time.perf_counter()
capi.moe_dispatch(cfg, lay.struct, x_dev, recv)
torch.cuda.synchronize()
out["hooked_seconds"] = time.perf_counter() - t0
out["hooked_status"] = capi.moe_get_error(lay.struct)
del os.environ["MOE_TEST_SKIP_LOAD"]
recv.view(torch.int16).fill_(0x7F81)
capi.moe_dispatch(cfg, lay.struct, x_dev, recv)
y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
capi.moe_combine(cfg, lay.struct, recv, torch.from_numpy(w).cuda(), y)
torch.cuda.synchronize()
out["next_status"] = capi.moe_get_error(lay.struct)
ref = oracle.layout(topk, E, R)
recv_ref = oracle.dispatch_flat(x, ref["slot"])
out["recv_equal"] = bool(np.array_equal(buffers.bits_of(recv), recv_ref))
out["y_equal"] = bool(np.array_equal(buffers.bits_of(y), oracle.combine(recv_ref, w, ref["slot"])))
print("RESULT " + json.dumps(out))
"""


def test_bounded_wait_runs_out_and_the_next_call_is_exact():
    import torch
    from combine_moe_layout_06_b200 import capi
    assert torch.cuda.is_available()
    build.build(out=TEST_LIB, defines=("MOE_TEST_HOOKS", "MOE_MAX_WAIT_NS=2000000ull"))
    env = dict(os.environ, MOE_LAYOUT_LIB=TEST_LIB, MOE_ROOT=ROOT)
    env.pop("MOE_TEST_SKIP_LOAD", None)
    res = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    line = [ln for ln in res.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    out = json.loads(line[len("RESULT "):])
    assert out["hooked_status"] == capi.MOE_ERR_TIMEOUT
    assert out["hooked_seconds"] < 5.0, "the hooked call returned (two bounded waits of 2 ms)"
    assert out["next_status"] == capi.MOE_OK
    assert out["recv_equal"] and out["y_equal"]
