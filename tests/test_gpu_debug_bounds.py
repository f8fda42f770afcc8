"""GPU side of the debug bounds checks (MOE_FLAG_DEBUG_BOUNDS).

With the checks on, the layer gives the same bits as the per-round schedule without them. A
bad plan summary injected on the host is refused before any kernel runs. Bad plan entries
injected into the workspace after planning (a slot past the capacity, a row-list token past T,
an expert row count past C) and an overwritten workspace guard are reported by
moe_device_status as MOE_ERR_BOUNDS, with what failed recorded in the workspace header, and the
bad accesses are skipped: every corrupted index is one that a debug check reads before the
access (or, for the GEMM's row gather, a TMA coordinate past the tensor, which reads zeros).
The next plan on the same workspace starts clean."""
import ctypes

import pytest
import torch

from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl

pytestmark = pytest.mark.gpu

HDR_STATUS, HDR_BAD_KIND, HDR_BAD_VALUE = 2, 4, 5
BAD_DISPATCH_ROW, BAD_COMBINE_PAIR, BAD_COMBINE_TOKEN, BAD_GEMM_ROWS, BAD_CANARY = 2, 3, 4, 5, 6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


def _layer(w, inp, debug, borrow=False):
    layer = moe.DroplessMoE(w.T, w.d, w.E, w.k, w.F, w.C, schedule="per_round", borrow=borrow,
                            debug_bounds=debug)
    layer.plan(logits=inp["logits"], x=inp["x"] if w.router == "gemm" else None,
               w_router=inp["w_router"], bias=inp["bias"])
    return layer


def _header(layer):
    return layer._view(layer.layout.header, 8, torch.int32).cpu().tolist()


@pytest.mark.parametrize("name,borrow", [("tiny-zipf1", False), ("4k-zipf1", False), ("4k-zipf1", True)])
def test_checked_run_gives_the_same_bits(name, borrow):
    w = wl.BY_NAME[name]
    inp = wl.generate(w, "cuda")
    ys = []
    for debug in (False, True):
        layer = _layer(w, inp, debug, borrow)
        ys.append(layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"]))
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        if debug:
            assert _header(layer)[HDR_STATUS] == 0 and _header(layer)[HDR_BAD_KIND] == 0
    assert torch.equal(ys[0], ys[1])


def test_host_injected_bad_plan_is_refused_before_any_launch():
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")
    layer = _layer(w, inp, True)
    bad = moe.PlanInfo()
    ctypes.memmove(ctypes.byref(bad), ctypes.byref(layer.info), ctypes.sizeof(bad))
    bad.load[0] += 1
    before = moe.launch_count()
    y = torch.empty(w.T, w.d, dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as err:
        moe.forward(layer.shape, bad, layer.ws, layer.ws_bytes, inp["x"].data_ptr(), inp["w_gate_up"].data_ptr(),
                    inp["w_down"].data_ptr(), y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert err.value.status == -1
    assert moe.launch_count() == before


def _corrupt_and_run(w, inp, corrupt):
    layer = _layer(w, inp, True)
    torch.cuda.synchronize()
    corrupt(layer)
    torch.cuda.synchronize()
    layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"])
    status = layer.device_status()
    hdr = _header(layer)
    # the next plan on the same workspace starts clean, and its forward passes every check
    layer.plan(logits=inp["logits"])
    layer.forward(inp["x"], inp["w_gate_up"], inp["w_down"])
    assert layer.device_status() == 0
    return status, hdr


def test_slot_past_capacity_is_reported():
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")

    def corrupt(layer):
        layer.plan_tensors()["slot"][5, 1] = w.C + 5
    status, hdr = _corrupt_and_run(w, inp, corrupt)
    assert status == -9
    assert hdr[HDR_BAD_KIND] == BAD_COMBINE_PAIR and hdr[HDR_STATUS] & 16


def test_row_token_past_T_is_reported():
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")

    def corrupt(layer):
        L = layer.layout
        row_start = layer._view(L.row_start, 3, torch.int32).cpu().tolist()
        tokens = layer._view(L.row_token, w.T * w.k, torch.int32)
        tokens[row_start[1] + 3] = w.T + 3      # a row of round 1 (combined row by row)
    status, hdr = _corrupt_and_run(w, inp, corrupt)
    assert status == -9
    assert hdr[HDR_BAD_KIND] in (BAD_DISPATCH_ROW, BAD_COMBINE_TOKEN)


def test_expert_rows_past_capacity_are_reported():
    w = wl.BY_NAME["4k-zipf1"]
    inp = wl.generate(w, "cuda")

    def corrupt(layer):
        layer._view(layer.layout.n, w.E, torch.int32)[0] = w.C + 100
    status, hdr = _corrupt_and_run(w, inp, corrupt)
    assert status == -9
    assert hdr[HDR_BAD_KIND] == BAD_GEMM_ROWS and hdr[HDR_BAD_VALUE] == 0


def test_overwritten_guard_is_reported():
    w = wl.BY_NAME["tiny-zipf1"]
    inp = wl.generate(w, "cuda")

    def corrupt(layer):
        L = layer.layout
        end_of_buf = L.buf + (w.E * w.C * w.d * 2 + 255) // 256 * 256   # the guard after buf
        layer.workspace[end_of_buf + 17] ^= 0xFF
    status, hdr = _corrupt_and_run(w, inp, corrupt)
    assert status == -9
    assert hdr[HDR_BAD_KIND] == BAD_CANARY and hdr[HDR_STATUS] & 32
