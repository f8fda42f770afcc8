"""The benchmark's algorithmic-work accounting (pure host logic): the per-kernel units of one
step add up to the layer's totals however the rounds are split between per-round launches and
the pipelined launch, and nothing counts padding rows."""
import types

import numpy as np
import pytest

import bench
import oracle
from dropless_moe_layer_b200 import workloads as wl


def _plan(name, borrow=False):
    w = wl.BY_NAME[name]
    z = wl.generate(w, "cpu", routing_only=True)["logits"].numpy()
    idx = oracle.select_topk(z, w.k)
    p = (oracle.plan_borrow if borrow else oracle.plan)(idx, w.E, w.C)
    info = types.SimpleNamespace(load=list(p["load"]) + [0] * (256 - w.E), R=p["R"])
    return w, p, info


@pytest.mark.parametrize("name", ["tiny-zipf1", "4k-zipf1"])
def test_work_totals_do_not_depend_on_the_split(name):
    w, p, info = _plan(name)
    pairs = w.T * w.k
    for r0 in range(0, p["R"] + 1):
        work = bench.algorithmic_work(w, info, r0, p["round"], p["n"])
        flops = work["gate_up"][1] + work["down"][1]
        if "pipeline" in work:
            flops += work["pipeline"][1][0]
        assert flops == 6 * pairs * w.d * w.F                      # every pair's GEMM work once
        # combine bytes split exactly between stand-alone launches, the steps that ride on a GEMM
        # launch and the pipelined launch
        rode_comb, rode_disp = bench.ride_plan(w, p["n"], r0)
        assert rode_comb <= set(range(r0)) and rode_disp <= set(range(1, p["R"]))
        comb = work["combine"][1] + bench.combine_bytes(w, p["round"], rode_comb) + (
            bench.combine_bytes(w, p["round"], set(range(r0, p["R"]))) if r0 < p["R"] else 0)
        assert comb == bench.combine_bytes(w, p["round"])
        assert ("pipeline" in work) == (r0 < p["R"])


def test_combine_bytes_closed_form():
    """Each pair's row is read once; each token writes y once per round it has pairs in and
    reads it back on every such round but its first."""
    w, p, info = _plan("tiny-zipf1")
    spans = np.array([len(set(r)) for r in p["round"].tolist()])
    want = w.T * w.k * w.d * 2 + spans.sum() * w.d * 4 + (spans - 1).sum() * w.d * 4
    assert bench.combine_bytes(w, p["round"]) == want


def test_borrowing_plan_rows_feed_the_accounting():
    """With borrowing an expert may hold more than C rows of a round: the accounting takes the
    plan's own n, so the GEMM work still counts every pair once."""
    w, p, info = _plan("4k-zipf1", borrow=True)
    assert p["n"].max() > w.C
    work = bench.algorithmic_work(w, info, p["R"], p["round"], p["n"])
    assert work["gate_up"][1] + work["down"][1] == 6 * w.T * w.k * w.d * w.F


def test_traffic_record_ignores_comments_not_code():
    """The recorded DRAM traffic stays attached to a kernel across edits of its comments and
    layout, and is dropped by an edit of its code."""
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "//kept";\n\n  char c = \'/\';\n'
    assert bench.code_tokens(src) == 'int a = 1;\nconst char* s = "//kept";\nchar c = \'/\';'
    reflowed = 'int   a = 1;   // another note\n  const char* s = "//kept"; // x\nchar c = \'/\';'
    assert bench.code_tokens(reflowed) == bench.code_tokens(src)
    assert bench.code_tokens(src.replace("a = 1", "a = 2")) != bench.code_tokens(src)


def test_backward_flops_split_by_launch_kind():
    """The backward's GEMM launch kinds account for all of its tensor-core work: 16 d d_ff flops
    per routed pair (recompute 4, dh 2, dx 4, dW2 2, dW1 and dW3 4); a round runs its recompute
    and dh either as two launches or as one fused launch, never both."""
    from dropless_moe_layer_b200 import moe
    w = wl.BY_NAME["4k-zipf1"]
    f = bench.BWD_KIND_FLOPS
    assert set(f) == set(moe.BACKWARD_GEMM_KINDS) and set(bench.BWD_FRONT_KINDS) <= set(f)
    assert f["backward_recompute"] + f["backward_dh"] == f["backward_recompute_dh"]
    assert (f["backward_recompute_dh"] + f["backward_dx_wgrad"]) * w.T * w.k * w.d * w.F == bench.backward_flops(w)


def test_ride_plan_follows_the_size_rule():
    """Small copy steps (at most 32 MiB of rows) always ride; a large one rides only when the GEMM
    it would ride on is long enough to hide it at the copy warps' rate."""
    w = wl.BY_NAME["32k-zipf1.2-router-gemm"]
    n = np.zeros((3, w.E), dtype=np.int64)
    n[0, :] = w.C                       # a full round: 262144 rows
    n[1, :4] = w.C                      # 8192 rows (117 MB: not small)
    n[2, 0] = 100                       # a thin round
    comb, disp = bench.ride_plan(w, n, 3)
    assert comb == set()                # round 0's combine outlasts round 1's gate/up; round 1's, round 2's
    assert disp == {1, 2}               # round 1's dispatch hides under round 0's down; round 2's is small
    n2 = np.zeros((2, w.E), dtype=np.int64)
    n2[0, :4] = w.C
    n2[1, :] = w.C
    comb, disp = bench.ride_plan(w, n2, 2)
    assert comb == {0} and disp == set()   # the small round's combine hides under the full round's


def test_backward_roofline_counts():
    """One round, two experts (3 and 1 rows), four tokens each with one pair: the copy part is
    the gather (x bf16 and dy fp32 read, both written back as bf16 rows), the dx rows read by the
    combine and each token's first dx write, plus dz from the logits and dgate; with an
    unbounded tensor peak every GEMM kind is its bytes at the copy peak, and the weight
    gradients are stored once (round 0)."""
    w = wl.custom(name="t", T=4, d=64, E=2, k=1, F=64, C=4)
    info = types.SimpleNamespace(load=[3, 1] + [0] * 254, R=1)
    rnd = np.zeros((4, 1), dtype=np.int64)
    n = np.array([[3, 1]])
    peaks = {"hbm_gbs": 1.0}     # 1 GB/s: seconds = bytes / 1e9
    s, parts = bench.backward_roofline_s(w, info, rnd, peaks, 1e30, n)
    P, A, d, F, T, E, k = 4, 2, 64, 64, 4, 2, 1
    copies = P * d * 6 + P * d * 4 + P * d * 2 + T * d * 4 + T * E * 8 + T * k * 8
    assert parts["copies"] == pytest.approx(copies / 1e9 * 1e3)
    grads = A * 3 * d * F * 4
    assert parts["dx_wgrad"] * 1e6 == pytest.approx(4 * P * 2 * F + A * 2 * F * d * 2 + 3 * P * d * 2 + P * F * 2
                                                     + grads)
    assert s * 1e3 == pytest.approx(sum(parts.values()))
    # a second round holding the same rows again: its gradients are read and written (2x)
    rnd2 = np.array([[0, 1]] * 4)
    info2 = types.SimpleNamespace(load=[6, 2] + [0] * 254, R=2)
    w2 = wl.custom(name="t", T=4, d=64, E=2, k=2, F=64, C=3)
    _, parts2 = bench.backward_roofline_s(w2, info2, rnd2, peaks, 1e30, np.array([[3, 1], [3, 1]]))
    assert parts2["dx_wgrad"] - 2 * parts["dx_wgrad"] == pytest.approx(grads / 1e9 * 1e3)
