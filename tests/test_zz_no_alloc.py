"""moe_plan_noalloc: the routing/plan entry point that allocates no device memory.

It is meant for callers that cannot call cudaMalloc when they route a batch (code
under a memory pool that owns the whole device, plugins given only their input and
output buffers, services that forbid allocation after start-up). Its scratch lives in
a fixed static device array inside the library, shared by every call. These tests call
it through the C ABI several times in a row, on shapes of different sizes, with and
without capacity borrowing, and check each result against the CPU oracle's plan of the
same logits and against what the regular moe_plan() writes into its caller-allocated
workspace. A last test runs it in a fresh process under lazy module loading, where its
first call is the one that makes the device reserve the array. The file is collected
last.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GATE_RTOL = 1e-5          # the gate tolerance of the other GPU parity tests
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _noalloc_plan(lib, w, logits, borrow=False):
    shape = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C, borrow=borrow)
    dev = logits.device
    idx = torch.full((w.T, w.k), -1, dtype=torch.int32, device=dev)
    gate = torch.full((w.T, w.k), -1.0, dtype=torch.float32, device=dev)
    rnd = torch.full((w.T, w.k), -1, dtype=torch.int32, device=dev)
    slot = torch.full((w.T, w.k), -1, dtype=torch.int32, device=dev)
    R = ctypes.c_int32(-1)
    load = (ctypes.c_int32 * w.E)()
    stream = torch.cuda.current_stream(dev).cuda_stream
    st = lib.moe_plan_noalloc(ctypes.byref(shape), logits.data_ptr(), idx.data_ptr(), gate.data_ptr(),
                              rnd.data_ptr(), slot.data_ptr(), ctypes.byref(R), load, stream or None)
    assert st == 0, moe.STATUS.get(st, st)
    return dict(topk_idx=idx, gate=gate, round=rnd, slot=slot, R=R.value, load=list(load))


def _regular_plan(w, logits, borrow=False):
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, device=logits.device, borrow=borrow)
    info = layer.plan(logits=logits)
    pt = layer.plan_tensors()
    return dict(topk_idx=pt["topk_idx"].clone(), gate=pt["gate"].clone(), round=pt["round"].clone(),
                slot=pt["slot"].clone(), R=info.R, load=list(info.load)[:w.E])


def _check_against_oracle(w, logits, got, borrow):
    z = logits.cpu().numpy()
    idx = oracle.select_topk(z, w.k)
    p = (oracle.plan_borrow if borrow else oracle.plan)(idx, w.E, w.C)
    assert np.array_equal(got["topk_idx"].cpu().numpy(), idx)
    assert got["R"] == p["R"]
    assert got["load"] == [int(v) for v in p["load"]]
    assert np.array_equal(got["round"].cpu().numpy(), p["round"])
    assert np.array_equal(got["slot"].cpu().numpy(), p["slot"])
    np.testing.assert_allclose(got["gate"].cpu().numpy(), oracle.gates(z, idx), rtol=GATE_RTOL, atol=0.0)


@pytest.mark.parametrize("borrow", [False, True], ids=["own-capacity", "borrowing"])
def test_noalloc_plan_matches_oracle_and_moe_plan_in_a_row(borrow):
    build.build()
    lib = moe.load_library()
    # a larger shape first, then a smaller one, then the larger one again, so that later calls
    # run over whatever earlier ones left in the shared static scratch (with borrowing the
    # smaller shape also has fewer rounds than the one before it)
    for name in ("4k-zipf1", "tiny-zipf1", "4k-zipf1"):
        w = wl.BY_NAME[name]
        logits = wl.generate(w, "cuda", routing_only=True)["logits"]
        got = _noalloc_plan(lib, w, logits, borrow)
        torch.cuda.synchronize()
        _check_against_oracle(w, logits, got, borrow)
        ref = _regular_plan(w, logits, borrow)
        torch.cuda.synchronize()
        assert got["R"] == ref["R"] and got["R"] >= 2
        assert got["load"] == ref["load"]
        assert torch.equal(got["topk_idx"], ref["topk_idx"])
        assert torch.equal(got["round"], ref["round"])
        assert torch.equal(got["slot"], ref["slot"])
        torch.testing.assert_close(got["gate"], ref["gate"], rtol=GATE_RTOL, atol=0.0)


def test_noalloc_plan_rejects_shapes_over_its_scratch():
    lib = moe.load_library()
    # 2^20 tokens x 4 pairs need 32 MiB of row lists: more than the 16 MiB static array.
    shape = moe.make_shape(1 << 20, 64, 8, 4, 64, 1 << 20)
    R = ctypes.c_int32(-1)
    dummy = 1 << 12      # never dereferenced: the size check comes before any launch
    st = lib.moe_plan_noalloc(ctypes.byref(shape), dummy, dummy, dummy, dummy, dummy,
                              ctypes.byref(R), None, None)
    assert st == -8 and R.value == -1


_LAZY_CHILD = r"""
import ctypes, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
import oracle
from dropless_moe_layer_b200 import moe
from dropless_moe_layer_b200 import workloads as wl
lib = moe.load_library()
torch.cuda.set_device(0)
torch.cuda.init()
R = ctypes.c_int32(-1)
# start-up call with an empty batch: under lazy loading this is where the device reserves
# the static scratch array
st = lib.moe_plan_noalloc(ctypes.byref(moe.make_shape(0, 128, 8, 2, 256, 32)), None, None, None,
                          None, None, ctypes.byref(R), None, None)
assert st == 0 and R.value == 0, (st, R.value)
w = wl.BY_NAME["4k-zipf1"]
z = wl.generate(w, "cuda", routing_only=True)["logits"]
out = [torch.empty(w.T, w.k, dtype=t, device="cuda") for t in (torch.int32, torch.float32, torch.int32, torch.int32)]
load = (ctypes.c_int32 * w.E)()
st = lib.moe_plan_noalloc(ctypes.byref(moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C)), z.data_ptr(),
                          *[t.data_ptr() for t in out], ctypes.byref(R), load, None)
assert st == 0, st
p = oracle.plan(oracle.select_topk(z.cpu().numpy(), w.k), w.E, w.C)
assert R.value == p["R"] and list(load) == [int(v) for v in p["load"]]
assert np.array_equal(out[2].cpu().numpy(), p["round"]) and np.array_equal(out[3].cpu().numpy(), p["slot"])
print("lazy-ok", R.value)
"""


def test_noalloc_first_call_under_lazy_module_loading():
    """In a fresh process with CUDA_MODULE_LOADING=LAZY, the start-up call (T = 0) succeeds and
    the next call's plan equals the oracle's."""
    build.build()
    env = dict(os.environ, CUDA_MODULE_LOADING="LAZY")
    res = subprocess.run([sys.executable, "-c", _LAZY_CHILD, ROOT], env=env, capture_output=True, text=True,
                         timeout=300)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-2000:]
    assert "lazy-ok" in res.stdout
