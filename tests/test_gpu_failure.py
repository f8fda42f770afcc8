"""Failure detection without a GPU fault: a dependency wait of the pipelined launch that can
never be met runs out after its time limit, the launch unwinds, the workspace status word
reports it (MOE_ERR_TIMEOUT), and the context stays usable for the next, correct call.

The wait is made to run out by editing the plan after moe_plan: one round is told its last
128-row block of one expert holds more rows than were dispatched into it, so that block's
gate/up tiles wait for rows that never come. Nothing is written out of bounds (the claimed rows
stay inside the expert's C rows) and no kernel traps or faults."""
import pytest
import torch

from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = -6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


def test_unmeetable_wait_times_out_and_the_context_recovers():
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, schedule="pipeline")
    layer.plan(logits=inp["logits"])
    y_good = layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"]).clone()
    torch.cuda.synchronize()
    assert layer.device_status() == 0

    info = layer.plan(logits=inp["logits"])
    n = layer.plan_tensors()["n"]                      # a view into the workspace
    r = info.R - 1
    row = n[r].cpu()
    e = next(e for e in range(w.E) if 0 < int(row[e]) < w.C and int(row[e]) % 128 != 0)
    n[r, e] = min(w.C, (int(row[e]) // 128 + 1) * 128)  # claim rows nobody dispatches
    torch.cuda.synchronize()
    layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"])
    torch.cuda.synchronize()                           # returns after the 2 s wait limit
    assert layer.device_status() == MOE_ERR_TIMEOUT
    assert int(layer.sync_counters().abs().sum()) == 0  # the last CTA left the counters clean

    layer.plan(logits=inp["logits"])                   # a fresh plan clears the status word
    y = layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(y, y_good)
