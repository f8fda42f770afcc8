"""Host-side checks of the C ABI: the library builds, loads and exports every entry
point that include/moe.h declares, and argument errors are reported as status codes
without touching the GPU (these calls return before any CUDA call)."""
import ctypes

import pytest

from dropless_moe_layer_b200 import build, moe
from dropless_moe_layer_b200 import workloads as wl


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = moe.header_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    for n in ["moe_workspace_bytes", "moe_plan", "moe_forward"]:
        assert n in names


def test_status_strings(lib):
    for code in moe.STATUS:
        assert lib.moe_status_string(code)
    assert lib.moe_status_string(12345) == b"unknown status"


def _bytes_model(w, per_round=False):
    """Workspace size from the layout rules: 256-byte aligned regions; a second set of round
    buffers unless the schedule is per-round only."""
    def a(n):
        return (n + 255) // 256 * 256
    T, E, k, C, d, F = w.T, w.E, w.k, w.C, w.d, w.F
    mr = (T + C - 1) // C
    blocks = (T + 255) // 256
    return (a(320 * 4) + a(T * E * 4) + 4 * a(T * k * 4) + a(E * 4) + a((E + 1) * 4)
            + a(blocks * E * 4) + 2 * a(mr * E * 4) + a((mr + 1) * 4) + 2 * a(T * k * 4)
            + a(E * C * d * 2) + a(E * C * F * 2) + a(E * C * d * 2)
            + a(mr * (E + 1) * 4) + a((448 + 8 * E * ((C + 127) // 128) * 8) * 4)
            + (0 if per_round else a(E * C * d * 2) + a(E * C * F * 2) + a(E * C * d * 2)))


@pytest.mark.parametrize("w", wl.WORKLOADS, ids=lambda w: w.name)
def test_workspace_is_fixed_by_shape(lib, w):
    s = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C)
    n = moe.workspace_bytes(s)
    assert n == _bytes_model(w)
    # the round buffers dominate: E*C*(2d + d_ff) bf16 (dispatch rows, activations, outputs)
    assert n >= w.E * w.C * (2 * w.d + w.F) * 2
    lay = moe.workspace_layout(s)
    assert lay.total_bytes == n
    offs = [lay.header, lay.block_base, lay.logits, lay.topk_idx, lay.gate, lay.round, lay.slot, lay.load,
            lay.offsets, lay.n, lay.row_off, lay.row_start, lay.row_token,
            lay.row_dst, lay.buf, lay.h, lay.out]
    offs += [lay.mb_prefix, lay.sync, lay.buf2, lay.h2, lay.out2]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert lay.max_rounds == (w.T + w.C - 1) // w.C
    s1 = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C, schedule="per_round")
    assert moe.workspace_bytes(s1) == _bytes_model(w, per_round=True)
    lay1 = moe.workspace_layout(s1)
    assert lay1.buf2 == lay1.h2 == lay1.out2 == 0


@pytest.mark.parametrize("kw", [
    dict(E=0), dict(E=257), dict(k=0), dict(k=17, E=32), dict(k=5, E=4), dict(C=0),
    dict(d=96), dict(d=32), dict(d_ff=100), dict(T=-1), dict(d=16448),
])
def test_bad_shapes_are_rejected(lib, kw):
    base = dict(T=64, d=128, E=8, k=2, d_ff=128, C=16)
    base.update(kw)
    s = moe.make_shape(**base)
    assert moe.workspace_bytes(s) == 0
    lay = moe.WorkspaceLayout()
    assert lib.moe_workspace_layout(ctypes.byref(s), ctypes.byref(lay)) == -2


def test_bad_flags_rejected(lib):
    s = moe.make_shape(64, 128, 8, 2, 128, 16)
    for flags in (32, 1 << 31, moe.FLAG_PER_ROUND | moe.FLAG_PIPELINE_ALL,
                  moe.FLAG_BORROW | moe.FLAG_PIPELINE_ALL, moe.FLAG_DEBUG_BOUNDS | moe.FLAG_PIPELINE_ALL):
        s.flags = flags
        assert moe.workspace_bytes(s) == 0
    # borrowing runs per round: no second buffer set, like the per-round schedule
    assert moe.workspace_bytes(moe.make_shape(64, 128, 8, 2, 128, 16, borrow=True)) == \
        moe.workspace_bytes(moe.make_shape(64, 128, 8, 2, 128, 16, schedule="per_round"))
    # the pipelined schedules share one layout; per-round only drops the second buffer set
    assert moe.workspace_bytes(moe.make_shape(64, 128, 8, 2, 128, 16, schedule="pipeline")) == \
        moe.workspace_bytes(moe.make_shape(64, 128, 8, 2, 128, 16))
    assert moe.workspace_bytes(moe.make_shape(64, 128, 8, 2, 128, 16, schedule="per_round")) < \
        moe.workspace_bytes(moe.make_shape(64, 128, 8, 2, 128, 16))


def test_plan_argument_errors_without_gpu(lib):
    s = moe.make_shape(64, 128, 8, 2, 128, 16)
    need = moe.workspace_bytes(s)
    info = moe.PlanInfo()
    P = ctypes.byref
    # null workspace / null info
    assert lib.moe_plan(P(s), 4096, None, None, None, None, need, P(info), None) == -1
    assert lib.moe_plan(P(s), 4096, None, None, None, 1 << 20, need, None, None) == -1
    # neither logits nor (x, w_router)
    assert lib.moe_plan(P(s), None, None, None, None, 1 << 20, need, P(info), None) == -1
    # workspace too small
    assert lib.moe_plan(P(s), 4096, None, None, None, 1 << 20, need - 1, P(info), None) == -3
    # misaligned workspace / logits
    assert lib.moe_plan(P(s), 4096, None, None, None, (1 << 20) + 16, need, P(info), None) == -4
    assert lib.moe_plan(P(s), 4100, None, None, None, 1 << 20, need, P(info), None) == -4


def test_forward_argument_errors_without_gpu(lib):
    s = moe.make_shape(64, 128, 8, 2, 128, 16)
    need = moe.workspace_bytes(s)
    info = moe.PlanInfo()
    info.R = 5                                   # more rounds than ceil(T / C) = 4
    P = ctypes.byref
    ws = 1 << 20
    assert lib.moe_forward(P(s), P(info), ws, need, 4096, 4096, 4096, 4096, None) == -1
    info.R = 1
    assert lib.moe_forward(P(s), None, ws, need, 4096, 4096, 4096, 4096, None) == -1
    assert lib.moe_forward(P(s), P(info), ws, need - 256, 4096, 4096, 4096, 4096, None) == -3
    assert lib.moe_forward(P(s), P(info), ws + 8, need, 4096, 4096, 4096, 4096, None) == -4
    for fn in ("moe_round_dispatch", "moe_round_gate_up", "moe_round_down", "moe_round_combine"):
        f = getattr(lib, fn)
        assert f(P(s), P(info), ws, need - 256, 0, 4096, None) == -3
        assert f(P(s), P(info), ws + 64, need, 0, 4096, None) == -4
    # a plan made with capacity borrowing cannot be run as a plan without it, nor the reverse
    sb = moe.make_shape(64, 128, 8, 2, 128, 16, borrow=True)
    need_b = moe.workspace_bytes(sb)
    info.plan_flags = moe.FLAG_BORROW
    assert lib.moe_forward(P(s), P(info), ws, need, 4096, 4096, 4096, 4096, None) == -1
    assert lib.moe_round_combine(P(s), P(info), ws, need, 0, 4096, None) == -1
    info.plan_flags = 0
    assert lib.moe_forward(P(sb), P(info), ws, need_b, 4096, 4096, 4096, 4096, None) == -1


def _backward_rows2(w, per_round=False):
    """Rows of the second buffer set: E*C/8 rounded up to 64, plus 64 per expert (none with the
    per-round flag)."""
    if per_round:
        return 0
    return (-(-w.E * w.C // 8) + 63) // 64 * 64 + 64 * w.E


def _backward_bytes_model(w, borrow=False, per_round=False):
    """Backward workspace from its layout rules: per-round buffers of E*C rows (with borrowing
    E*C + 64*E: each expert's segment starts at a multiple of 64), [T, k] dgate and unit gates,
    the segment table [max_rounds, E], max_rounds + 1 zero words, and the second set of the
    per-round buffers. No copy of the weights and no transposed copy of the activations."""
    def a(n):
        return (n + 255) // 256 * 256
    T, E, k, C, d, F = w.T, w.E, w.k, w.C, w.d, w.F

    def round_buffers(rows):
        return (3 * a(rows * d * 2) + a(rows * 4) + 2 * a(rows * 2 * F * 2) + a(rows * F * 2)
                + a(rows * (F // 64) * 4))
    rows = E * C + (64 * E if borrow else 0)
    mr = (T + C - 1) // C
    return (round_buffers(rows) + 2 * a(T * k * 4) + a(mr * E * 4) + a((mr + 1) * 4)
            + round_buffers(_backward_rows2(w, per_round)))


@pytest.mark.parametrize("w", wl.WORKLOADS, ids=lambda w: w.name)
def test_backward_workspace_is_fixed_by_shape(lib, w):
    s = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C)
    n = moe.backward_workspace_bytes(s)
    assert n == _backward_bytes_model(w)
    lay = moe.backward_layout(s)
    assert lay.total_bytes == n and lay.rows == w.E * w.C
    offs = [lay.xbuf, lay.dybuf, lay.row_gate, lay.ab, lay.hg, lay.dab, lay.dgate_part, lay.dxbuf, lay.dgate,
            lay.ones, lay.seg_off, lay.zeros]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert lay.rows2 == _backward_rows2(w)
    offs2 = [lay.xbuf2, lay.dybuf2, lay.row_gate2, lay.ab2, lay.hg2, lay.dab2, lay.dgate_part2, lay.dxbuf2]
    assert offs2 == sorted(offs2) and offs2[0] > lay.zeros and all(o % 256 == 0 for o in offs2)
    sb = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C, borrow=True)
    assert moe.backward_workspace_bytes(sb) == _backward_bytes_model(w, borrow=True)
    assert moe.backward_layout(sb).rows == w.E * w.C + 64 * w.E
    sp = moe.make_shape(w.T, w.d, w.E, w.k, w.F, w.C, schedule="per_round")
    assert moe.backward_workspace_bytes(sp) == _backward_bytes_model(w, per_round=True)
    lp = moe.backward_layout(sp)
    assert lp.rows2 == 0 and lp.xbuf2 == 0 and lp.dxbuf2 == 0
    s.flags = 32          # not a flag
    assert moe.backward_workspace_bytes(s) == 0


def test_backward_argument_errors_without_gpu(lib):
    s = moe.make_shape(64, 128, 8, 2, 128, 16)
    need, bneed = moe.workspace_bytes(s), moe.backward_workspace_bytes(s)
    info = moe.PlanInfo()
    info.R = 1
    P = ctypes.byref
    ws, bws, p = 1 << 20, 1 << 24, 4096
    f = lib.moe_backward
    assert f(P(s), None, ws, need, bws, bneed, p, p, p, p, p, p, p, p, None) == -1
    assert f(P(s), P(info), ws, need, None, bneed, p, p, p, p, p, p, p, p, None) == -1
    assert f(P(s), P(info), ws, need, bws, bneed - 256, p, p, p, p, p, p, p, p, None) == -3
    assert f(P(s), P(info), ws, need, bws + 64, bneed, p, p, p, p, p, p, p, p, None) == -4
    assert f(P(s), P(info), ws, need, bws, bneed, p, p, p, p + 4, p, p, p, p, None) == -4
    assert f(P(s), P(info), ws, need, bws, bneed, p, p, p, None, p, p, p, p, None) == -1
    # a plan with capacity borrowing runs on a borrowing shape (its argument checks pass and
    # the call reaches the device check), and only on one
    sb = moe.make_shape(64, 128, 8, 2, 128, 16, borrow=True)
    info.plan_flags = moe.FLAG_BORROW
    assert f(P(sb), P(info), ws, moe.workspace_bytes(sb), bws, moe.backward_workspace_bytes(sb),
             p, p, p, p, p, p, p, p, None) not in (-1, -2, -3, -4)
    assert f(P(s), P(info), ws, need, bws, bneed, p, p, p, p, p, p, p, p, None) == -1


@pytest.mark.parametrize("cmd", [["gcc", "-std=c99", "-x", "c"], ["g++", "-std=c++11", "-x", "c++"]],
                         ids=["c99", "c++11"])
def test_public_header_is_plain_c(cmd):
    """include/moe.h is a C ABI: it compiles on its own, warning-free, as C99 and as C++11."""
    import os
    import shutil
    import subprocess
    if shutil.which(cmd[0]) is None:
        pytest.skip(f"{cmd[0]} not installed")
    header = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")
    out = subprocess.run(cmd + ["-fsyntax-only", "-Wall", "-Wextra", "-Werror", header],
                         capture_output=True, text=True)
    assert out.returncode == 0, out.stderr


def test_profile_kinds_agree_with_the_header():
    import os
    import re
    header = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")
    with open(header) as f:
        n = int(re.search(r"#define MOE_PROFILE_KINDS (\d+)", f.read()).group(1))
    assert moe.PROFILE_KINDS == n == len(moe.PROFILE_NAMES)
    assert set(moe.BACKWARD_GEMM_KINDS) <= set(moe.PROFILE_NAMES)
