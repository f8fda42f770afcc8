"""Host side of the debug bounds checks (MOE_FLAG_DEBUG_BOUNDS), run without a GPU: the flag
grows the workspace by one 256-byte guard per region and spaces the regions accordingly, it
refuses the all-pipelined schedule, and a plan summary the planner cannot have produced is
rejected before any CUDA call (the workspace pointer is never dereferenced on the host)."""
import ctypes

import pytest

from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl

REGIONS = ["header", "block_base", "logits", "topk_idx", "gate", "round", "slot", "load", "offsets", "n",
           "row_off", "row_start", "row_token", "row_dst", "buf", "h", "out", "mb_prefix", "sync"]


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load_library()


@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_guards_follow_every_region(lib, name):
    w = wl.BY_NAME[name]
    plain = moe.workspace_layout(moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C, schedule="per_round"))
    dbg = moe.workspace_layout(moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C, debug_bounds=True))
    assert dbg.total_bytes == plain.total_bytes + 256 * len(REGIONS)
    for i, r in enumerate(REGIONS):
        # every region starts 256 bytes later per guard before it, so its size is unchanged
        assert getattr(dbg, r) == getattr(plain, r) + 256 * i, r
    assert dbg.buf2 == dbg.h2 == dbg.out2 == 0       # per-round schedule: no second buffer set


def test_debug_flag_refuses_the_all_pipelined_schedule(lib):
    s = moe.make_shape(256, 128, 8, 2, 256, 32, schedule="pipeline", debug_bounds=True)
    assert moe.workspace_bytes(s) == 0


def _info(w, load, R=None, max_load=None):
    info = moe.PlanInfo()
    for e, v in enumerate(load):
        info.load[e] = v
    info.max_load = max(load) if max_load is None else max_load
    info.R = -(-info.max_load // w.C) if R is None else R
    return info


def _forward(lib, shape, info, ws_bytes):
    fake = 1 << 24        # a 256-byte aligned address the host never dereferences
    return lib.moe_forward(ctypes.byref(shape), ctypes.byref(info), fake, ws_bytes, fake, fake, fake, fake, None)


def test_inconsistent_plan_summary_is_rejected_before_any_launch(lib):
    w = wl.custom(T=64, d=64, E=4, k=2, F=64, C=16)
    shape = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C, debug_bounds=True)
    nbytes = moe.workspace_bytes(shape)
    good = [40, 40, 30, 18]                              # adds up to T k = 128
    launches = moe.launch_count()
    st_good = _forward(lib, shape, _info(w, good), nbytes)
    assert st_good != -1                                 # passes the host checks (no GPU here: fails later)
    for bad in (_info(w, [41, 40, 30, 18]),              # loads do not add up to T k
                _info(w, [40, 40, 30, 18], R=2),         # R is not ceil(max_load / C)
                _info(w, [40, 40, 30, 18], max_load=30),  # max_load is not the loads' maximum
                _info(w, [70, 40, 0, 18])):              # a load above T
        assert _forward(lib, shape, bad, nbytes) == -1
    assert moe.launch_count() == launches
    # without the flag the same summaries are not checked
    plain = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C, schedule="per_round")
    assert _forward(lib, plain, _info(w, [41, 40, 30, 18]), moe.workspace_bytes(plain)) != -1
