"""Python binding of libmoe.so (the C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. PyTorch is used for device memory and streams. There is no CPU path: if
the library is missing or the GPU is not an sm_100 part, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

from .build import LIB_PATH, ROOT

c_i32, c_u32, c_sz, c_vp = ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t, ctypes.c_void_p

MAX_EXPERTS = 256
PROFILE_KINDS = 13
PROFILE_NAMES = ["router_gemm", "topk", "plan", "dispatch", "gate_up", "down", "combine", "pipeline",
                 "backward_recompute", "backward_dh", "backward_dx_wgrad", "backward_copy",
                 "backward_recompute_dh"]
BACKWARD_GEMM_KINDS = ("backward_recompute", "backward_dh", "backward_recompute_dh", "backward_dx_wgrad")
FLAG_RENORM_TOPK = 1
FLAG_PER_ROUND = 2
FLAG_PIPELINE_ALL = 4
FLAG_BORROW = 8
FLAG_DEBUG_BOUNDS = 16
SCHEDULES = {"auto": 0, "per_round": FLAG_PER_ROUND, "pipeline": FLAG_PIPELINE_ALL}

STATUS = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED_SHAPE",
          -3: "MOE_ERR_WORKSPACE_TOO_SMALL", -4: "MOE_ERR_MISALIGNED", -5: "MOE_ERR_CUDA",
          -6: "MOE_ERR_TIMEOUT", -7: "MOE_ERR_NO_DEVICE", -8: "MOE_ERR_NOALLOC_LIMIT", -9: "MOE_ERR_BOUNDS"}


class Shape(ctypes.Structure):
    _fields_ = [("T", c_i32), ("d", c_i32), ("E", c_i32), ("k", c_i32), ("d_ff", c_i32),
                ("C", c_i32), ("flags", c_u32)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("R", c_i32), ("max_load", c_i32), ("load", c_i32 * MAX_EXPERTS),
                ("logits", c_vp), ("topk_idx", c_vp), ("gate", c_vp), ("round", c_vp),
                ("slot", c_vp), ("offsets", c_vp), ("n", c_vp), ("plan_flags", c_u32)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [(name, c_sz) for name in (
        "total_bytes", "header", "logits", "topk_idx", "gate", "round", "slot", "load",
        "offsets", "block_base", "n", "row_off", "row_start", "row_token", "row_dst", "buf", "h", "out",
        "mb_prefix", "sync", "buf2", "h2", "out2")
    ] + [("max_rounds", c_i32), ("plan_blocks", c_i32)]


class BackwardLayout(ctypes.Structure):
    _fields_ = [(name, c_sz) for name in (
        "total_bytes", "xbuf", "dybuf", "row_gate", "ab", "hg", "dab", "dgate_part", "dxbuf", "dgate",
        "ones", "seg_off", "zeros")
    ] + [("rows", c_i32)] + [(name, c_sz) for name in (
        "xbuf2", "dybuf2", "row_gate2", "ab2", "hg2", "dab2", "dgate_part2", "dxbuf2")
    ] + [("rows2", c_i32)]


class MoeError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {STATUS.get(status, status)} ({_status_text(status)})")


_lib: Optional[ctypes.CDLL] = None


def header_symbols() -> list[str]:
    """Names of the entry points declared in include/moe.h."""
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        text = f.read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by dropless_moe_layer_b200.build, or the file named by
    the MOE_LIBRARY_PATH environment variable). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("MOE_LIBRARY_PATH") or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"libmoe.so not found at {path}; build it with "
                           "`python -m dropless_moe_layer_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    sig = {
        "moe_workspace_bytes": (c_sz, [P(Shape)]),
        "moe_workspace_layout": (ctypes.c_int, [P(Shape), P(WorkspaceLayout)]),
        "moe_plan": (ctypes.c_int, [P(Shape), c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, P(PlanInfo), c_vp]),
        "moe_forward": (ctypes.c_int, [P(Shape), P(PlanInfo), c_vp, c_sz, c_vp, c_vp, c_vp, c_vp, c_vp]),
        "moe_round_dispatch": (ctypes.c_int, [P(Shape), P(PlanInfo), c_vp, c_sz, c_i32, c_vp, c_vp]),
        "moe_round_gate_up": (ctypes.c_int, [P(Shape), P(PlanInfo), c_vp, c_sz, c_i32, c_vp, c_vp]),
        "moe_round_down": (ctypes.c_int, [P(Shape), P(PlanInfo), c_vp, c_sz, c_i32, c_vp, c_vp]),
        "moe_round_combine": (ctypes.c_int, [P(Shape), P(PlanInfo), c_vp, c_sz, c_i32, c_vp, c_vp]),
        "moe_device_status": (ctypes.c_int, [P(Shape), c_vp, c_vp]),
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_launch_count": (ctypes.c_uint64, []),
        "moe_profile_enable": (ctypes.c_int, [ctypes.c_int]),
        "moe_profile_read": (ctypes.c_int, [P(c_i32), P(ctypes.c_double)]),
        "moe_plan_noalloc": (ctypes.c_int, [P(Shape), c_vp, c_vp, c_vp, c_vp, c_vp, P(c_i32), P(c_i32), c_vp]),
        "moe_ep_exchange_plan": (ctypes.c_int, [P(Shape), c_i32, c_i32, P(c_i32), c_i32, P(c_i32), P(c_i32),
                                                P(c_i32), P(c_i32), P(c_i32), P(c_i32), P(c_i32)]),
        "moe_ep_workspace_bytes": (c_sz, [P(Shape), c_i32]),
        "moe_ep_plan": (ctypes.c_int, [P(Shape), c_i32, c_i32, P(c_i32), P(PlanInfo), c_vp, c_sz, c_vp, c_sz,
                                       P(c_i32), c_vp]),
        "moe_ep_round_pack": (ctypes.c_int, [P(Shape), c_i32, c_i32, P(c_i32), c_vp, c_sz, c_i32, c_vp, c_vp, c_vp]),
        "moe_ep_round_experts": (ctypes.c_int, [P(Shape), c_i32, c_i32, P(c_i32), c_vp, c_sz, c_i32, c_vp, c_vp,
                                                c_vp, c_vp, c_vp, ctypes.c_int64, c_vp, c_vp]),
        "moe_ep_round_combine": (ctypes.c_int, [P(Shape), c_i32, c_i32, P(c_i32), c_vp, c_sz, c_vp, c_sz, c_i32,
                                                c_vp, c_vp, c_vp]),
        "moe_backward_workspace_bytes": (c_sz, [P(Shape)]),
        "moe_backward_workspace_layout": (ctypes.c_int, [P(Shape), P(BackwardLayout)]),
        "moe_backward": (ctypes.c_int, [P(Shape), P(PlanInfo), c_vp, c_sz, c_vp, c_sz, c_vp, c_vp, c_vp,
                                        c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _status_text(status: int) -> str:
    try:
        return load_library().moe_status_string(status).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(call: str, status: int) -> None:
    if status != 0:
        raise MoeError(call, status)


def make_shape(T: int, d: int, E: int, k: int, d_ff: int, C: int, renorm: bool = False,
               schedule: str = "auto", borrow: bool = False, debug_bounds: bool = False) -> Shape:
    """schedule: "auto" (trailing thin rounds pipelined), "per_round" or "pipeline";
    borrow: capacity borrowing between experts (MOE_FLAG_BORROW); debug_bounds: the library's
    index checks and workspace guards (MOE_FLAG_DEBUG_BOUNDS)."""
    return Shape(T, d, E, k, d_ff, C, (FLAG_RENORM_TOPK if renorm else 0) | SCHEDULES[schedule] |
                 (FLAG_BORROW if borrow else 0) | (FLAG_DEBUG_BOUNDS if debug_bounds else 0))


# ------------------------------------------------------------------------- raw-pointer calls

def workspace_bytes(shape: Shape) -> int:
    return int(load_library().moe_workspace_bytes(ctypes.byref(shape)))


def workspace_layout(shape: Shape) -> WorkspaceLayout:
    lay = WorkspaceLayout()
    _check("moe_workspace_layout", load_library().moe_workspace_layout(ctypes.byref(shape), ctypes.byref(lay)))
    return lay


def plan(shape: Shape, logits: int, x: int, w_router: int, bias: int, ws: int, ws_bytes: int,
         stream: int) -> PlanInfo:
    info = PlanInfo()
    _check("moe_plan", load_library().moe_plan(ctypes.byref(shape), logits or None, x or None,
                                               w_router or None, bias or None, ws, ws_bytes,
                                               ctypes.byref(info), stream or None))
    return info


def forward(shape: Shape, info: PlanInfo, ws: int, ws_bytes: int, x: int, w_gate_up: int,
            w_down: int, y: int, stream: int) -> None:
    _check("moe_forward", load_library().moe_forward(ctypes.byref(shape), ctypes.byref(info), ws, ws_bytes,
                                                     x, w_gate_up, w_down, y, stream or None))


def backward_workspace_bytes(shape: Shape) -> int:
    return int(load_library().moe_backward_workspace_bytes(ctypes.byref(shape)))


def backward_layout(shape: Shape) -> BackwardLayout:
    lay = BackwardLayout()
    _check("moe_backward_workspace_layout",
           load_library().moe_backward_workspace_layout(ctypes.byref(shape), ctypes.byref(lay)))
    return lay


def backward(shape: Shape, info: PlanInfo, ws: int, ws_bytes: int, bws: int, bws_bytes: int, x: int,
             w_gate_up: int, w_down: int, dy: int, dx: int, dw_gate_up: int, dw_down: int, dz: int,
             stream: int) -> None:
    _check("moe_backward", load_library().moe_backward(ctypes.byref(shape), ctypes.byref(info), ws, ws_bytes,
                                                       bws, bws_bytes, x, w_gate_up, w_down, dy, dx,
                                                       dw_gate_up, dw_down, dz, stream or None))


def _round_call(name: str, shape: Shape, info: PlanInfo, ws: int, ws_bytes: int, r: int, ptr: int,
                stream: int) -> None:
    _check(name, getattr(load_library(), name)(ctypes.byref(shape), ctypes.byref(info), ws, ws_bytes,
                                                r, ptr, stream or None))


def round_dispatch(shape, info, ws, ws_bytes, r, x, stream):
    _round_call("moe_round_dispatch", shape, info, ws, ws_bytes, r, x, stream)


def round_gate_up(shape, info, ws, ws_bytes, r, w_gate_up, stream):
    _round_call("moe_round_gate_up", shape, info, ws, ws_bytes, r, w_gate_up, stream)


def round_down(shape, info, ws, ws_bytes, r, w_down, stream):
    _round_call("moe_round_down", shape, info, ws, ws_bytes, r, w_down, stream)


def round_combine(shape, info, ws, ws_bytes, r, y, stream):
    _round_call("moe_round_combine", shape, info, ws, ws_bytes, r, y, stream)


def device_status(shape: Shape, ws: int, stream: int) -> int:
    return int(load_library().moe_device_status(ctypes.byref(shape), ws, stream or None))


def launch_count() -> int:
    return int(load_library().moe_launch_count())


def profile_enable(on: bool) -> None:
    _check("moe_profile_enable", load_library().moe_profile_enable(1 if on else 0))


def profile_read() -> dict:
    counts = (c_i32 * PROFILE_KINDS)()
    ms = (ctypes.c_double * PROFILE_KINDS)()
    _check("moe_profile_read", load_library().moe_profile_read(counts, ms))
    return {PROFILE_NAMES[i]: (int(counts[i]), float(ms[i])) for i in range(PROFILE_KINDS)}


def ep_exchange_plan(shape: Shape, G: int, rank: int, loads) -> dict:
    """Exchange tables of an expert-parallel rank (moe_ep_exchange_plan; host code, no GPU).
    loads: [G, E] integer array of every rank's pair counts per expert. Returns numpy arrays:
    R, base [E], send_counts / send_offsets / recv_counts / recv_offsets [R, G], n_owned [R, E/G]."""
    import numpy as np
    E = shape.E
    lo = np.ascontiguousarray(np.asarray(loads, dtype=np.int32).reshape(G, E))
    P = ctypes.POINTER(c_i32)
    R = c_i32(0)
    base = np.zeros(E, dtype=np.int32)
    lib = load_library()
    _check("moe_ep_exchange_plan", lib.moe_ep_exchange_plan(ctypes.byref(shape), G, rank, lo.ctypes.data_as(P), 0,
                                                            ctypes.byref(R), base.ctypes.data_as(P), None, None,
                                                            None, None, None))
    nr = R.value
    out = {k: np.zeros((nr, G), dtype=np.int32) for k in ("send_counts", "send_offsets", "recv_counts", "recv_offsets")}
    out["n_owned"] = np.zeros((nr, E // G if G > 0 else 0), dtype=np.int32)
    _check("moe_ep_exchange_plan", lib.moe_ep_exchange_plan(
        ctypes.byref(shape), G, rank, lo.ctypes.data_as(P), nr, ctypes.byref(R), base.ctypes.data_as(P),
        *[out[k].ctypes.data_as(P) for k in ("send_counts", "send_offsets", "recv_counts", "recv_offsets", "n_owned")]))
    return dict(out, R=nr, base=base)


# ------------------------------------------------------------------------- torch marshalling

def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _need(t, dtype, shape, name):
    import torch
    if t is None:
        return
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or t.device.type != "cuda":
        raise ValueError(f"{name}: expected contiguous cuda {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


class DroplessMoE:
    """A fixed-memory dropless MoE layer (forward, and backward with recompute) on one B200.

    The workspace (the layer's fixed memory) is allocated once, from the shape alone.
    `plan()` routes one batch; `forward()` runs its rounds; `__call__` does both.
    """

    def __init__(self, T: int, d: int, E: int, k: int, d_ff: int, C: int, renorm: bool = False,
                 device=None, schedule: str = "auto", borrow: bool = False, debug_bounds: bool = False):
        import torch
        self.shape = make_shape(T, d, E, k, d_ff, C, renorm, schedule, borrow, debug_bounds)
        self.ws_bytes = workspace_bytes(self.shape)
        if self.ws_bytes == 0:
            raise ValueError(f"unsupported shape T={T} d={d} E={E} k={k} d_ff={d_ff} C={C}")
        self.device = torch.device(device or "cuda")
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        self.layout = workspace_layout(self.shape)
        self.info: Optional[PlanInfo] = None

    @property
    def ws(self) -> int:
        return int(self.workspace.data_ptr())

    def _stream(self, stream) -> int:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return int(s.cuda_stream)

    def plan(self, logits=None, x=None, w_router=None, bias=None, stream=None) -> PlanInfo:
        import torch
        s = self.shape
        _need(logits, torch.float32, (s.T, s.E), "logits")
        _need(x, torch.bfloat16, (s.T, s.d), "x")
        _need(w_router, torch.bfloat16, (s.E, s.d), "w_router")
        _need(bias, torch.float32, (s.E,), "bias")
        self.info = plan(s, _ptr(logits), _ptr(x), _ptr(w_router), _ptr(bias), self.ws,
                         self.ws_bytes, self._stream(stream))
        return self.info

    def forward(self, x, w_gate_up, w_down, y=None, stream=None):
        import torch
        s = self.shape
        if self.info is None:
            raise RuntimeError("plan() first")
        _need(x, torch.bfloat16, (s.T, s.d), "x")
        _need(w_gate_up, torch.bfloat16, (s.E, 2 * s.d_ff, s.d), "w_gate_up")
        _need(w_down, torch.bfloat16, (s.E, s.d, s.d_ff), "w_down")
        if y is None:
            y = torch.empty(s.T, s.d, dtype=torch.float32, device=self.device)
        _need(y, torch.float32, (s.T, s.d), "y")
        forward(s, self.info, self.ws, self.ws_bytes, _ptr(x), _ptr(w_gate_up), _ptr(w_down),
                _ptr(y), self._stream(stream))
        return y

    def __call__(self, x, w_gate_up, w_down, logits=None, w_router=None, bias=None, y=None,
                 stream=None):
        self.plan(logits=logits, x=x if logits is None else None, w_router=w_router, bias=bias,
                  stream=stream)
        return self.forward(x, w_gate_up, w_down, y=y, stream=stream)

    def backward(self, x, w_gate_up, w_down, dy, stream=None) -> dict:
        """Gradients of the last planned forward given dy [T, d] fp32: dx [T, d], dw_gate_up
        [E, 2 d_ff, d], dw_down [E, d, d_ff], dz [T, E] (all fp32), recomputing each round's
        expert activations on the forward's round schedule. The backward workspace is
        allocated on first use (its size depends on the shape only)."""
        import torch
        s = self.shape
        if self.info is None:
            raise RuntimeError("plan() first")
        _need(x, torch.bfloat16, (s.T, s.d), "x")
        _need(w_gate_up, torch.bfloat16, (s.E, 2 * s.d_ff, s.d), "w_gate_up")
        _need(w_down, torch.bfloat16, (s.E, s.d, s.d_ff), "w_down")
        _need(dy, torch.float32, (s.T, s.d), "dy")
        if getattr(self, "bworkspace", None) is None:
            self.bws_bytes = backward_workspace_bytes(s)
            self.bworkspace = torch.empty(self.bws_bytes, dtype=torch.uint8, device=self.device)
        f32 = dict(dtype=torch.float32, device=self.device)
        g = dict(dx=torch.empty(s.T, s.d, **f32), dw_gate_up=torch.empty(s.E, 2 * s.d_ff, s.d, **f32),
                 dw_down=torch.empty(s.E, s.d, s.d_ff, **f32), dz=torch.empty(s.T, s.E, **f32))
        backward(s, self.info, self.ws, self.ws_bytes, int(self.bworkspace.data_ptr()), self.bws_bytes,
                 _ptr(x), _ptr(w_gate_up), _ptr(w_down), _ptr(dy), _ptr(g["dx"]), _ptr(g["dw_gate_up"]),
                 _ptr(g["dw_down"]), _ptr(g["dz"]), self._stream(stream))
        return g

    # -- views of the plan and of the round buffers (for checking and inspection)
    def _view(self, off: int, count: int, dtype):
        import torch
        itemsize = torch.empty((), dtype=dtype).element_size()
        return self.workspace[off:off + count * itemsize].view(dtype)

    def plan_tensors(self) -> dict:
        import torch
        s, L = self.shape, self.layout
        R = self.info.R if self.info is not None else 0
        return dict(
            topk_idx=self._view(L.topk_idx, s.T * s.k, torch.int32).view(s.T, s.k),
            gate=self._view(L.gate, s.T * s.k, torch.float32).view(s.T, s.k),
            round=self._view(L.round, s.T * s.k, torch.int32).view(s.T, s.k),
            slot=self._view(L.slot, s.T * s.k, torch.int32).view(s.T, s.k),
            load=self._view(L.load, s.E, torch.int32),
            offsets=self._view(L.offsets, s.E + 1, torch.int32),
            n=self._view(L.n, R * s.E, torch.int32).view(R, s.E),
            logits=self._view(L.logits, s.T * s.E, torch.float32).view(s.T, s.E),
        )

    def round_buffer(self):
        """The dispatch buffer as [E, C, d] (expert e's rows at e, 0..). With capacity borrowing
        the round's rows are packed instead: row row_off[r][e] - row_start[r] + slot of the
        flattened [E * C, d] view."""
        import torch
        s, L = self.shape, self.layout
        return self._view(L.buf, s.E * s.C * s.d, torch.bfloat16).view(s.E, s.C, s.d)

    def output_buffer(self):
        import torch
        s, L = self.shape, self.layout
        return self._view(L.out, s.E * s.C * s.d, torch.bfloat16).view(s.E, s.C, s.d)

    def hidden_buffer(self):
        import torch
        s, L = self.shape, self.layout
        return self._view(L.h, s.E * s.C * s.d_ff, torch.bfloat16).view(s.E, s.C, s.d_ff)

    def sync_counters(self):
        """The pipelined launch's dependency counters (all zero between calls)."""
        import torch
        s, L = self.shape, self.layout
        words = 448 + 8 * s.E * ((s.C + 127) // 128) * 8
        return self._view(L.sync, words, torch.int32)

    def round_step(self, step: str, r: int, ptr_tensor, stream=None) -> None:
        fn = dict(dispatch=round_dispatch, gate_up=round_gate_up, down=round_down,
                  combine=round_combine)[step]
        fn(self.shape, self.info, self.ws, self.ws_bytes, r, _ptr(ptr_tensor), self._stream(stream))

    def device_status(self, stream=None) -> int:
        return device_status(self.shape, self.ws, self._stream(stream))
