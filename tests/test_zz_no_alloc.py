"""moe_plan_noalloc: the routing/plan entry point that allocates no device memory.

It is meant for callers that cannot call cudaMalloc when they route a batch (code
under a memory pool that owns the whole device, plugins given only their input and
output buffers, services that forbid allocation after start-up). Its scratch lives in
a fixed static device array inside the library. This test calls it through the C ABI
twice in a row, on two different shapes, and checks each result against what the
regular moe_plan() writes into its caller-allocated workspace. It sits in a file of
its own, collected last.
"""
import ctypes

import pytest
import torch

from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GATE_RTOL = 1e-5          # the gate tolerance of the other GPU parity tests


def _noalloc_plan(lib, w, logits):
    shape = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C)
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


def _regular_plan(w, logits):
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, device=logits.device)
    info = layer.plan(logits=logits)
    pt = layer.plan_tensors()
    return dict(topk_idx=pt["topk_idx"].clone(), gate=pt["gate"].clone(), round=pt["round"].clone(),
                slot=pt["slot"].clone(), R=info.R, load=list(info.load)[:w.E])


def test_noalloc_plan_matches_moe_plan_twice_in_a_row():
    build.build()
    lib = moe.load_library()
    # a larger shape first, then a smaller one, so the second call runs over whatever the
    # first left in the shared static scratch
    for name in ("4k-zipf1", "tiny-zipf1"):
        w = wl.BY_NAME[name]
        logits = wl.generate(w, "cuda", routing_only=True)["logits"]
        got = _noalloc_plan(lib, w, logits)
        torch.cuda.synchronize()
        ref = _regular_plan(w, logits)
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
