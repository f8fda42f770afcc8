"""One rank of the expert-parallel layer (include/moe.h, the moe_ep_* calls).

Argument marshalling only: routing, planning, packing, the expert GEMMs and the combine run in
libmoe.so's kernels; PyTorch provides device memory, and the exchange between ranks is the
caller's transport (`forward_distributed` uses torch.distributed: an all-gather of the per-rank
pair counts and, per round, an all-to-all of the packed rows and one back).

"Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, the multi-round dropless MoE
item [section "Scaling MoE", Fig. 6]: the experts are split into groups, one per
expert-parallel rank, and every group runs dispatch -> compute -> collect rounds with a fixed
per-expert capacity. Rank g owns the E/G contiguous experts [g E/G, (g+1) E/G); every rank
holds T tokens and routes them itself.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np

from . import moe


class ExpertParallelRank:
    """Rank `rank` of G. Buffers are allocated once from the shape (fixed memory): send and
    return rows min(T k, E C), received rows E/G * C."""

    def __init__(self, T: int, d: int, E: int, k: int, d_ff: int, C: int, G: int, rank: int, device=None):
        import torch
        if E % G != 0:
            raise ValueError("E must be a multiple of G")
        self.G, self.rank, self.E, self.k, self.C, self.d, self.F = G, rank, E, k, C, d, d_ff
        self.layer = moe.DroplessMoE(T, d, E, k, d_ff, C, device=device, schedule="per_round")
        self.shape = self.layer.shape
        self.device = self.layer.device
        lib = moe.load_library()
        self.ep_bytes = int(lib.moe_ep_workspace_bytes(ctypes.byref(self.shape), G))
        if self.ep_bytes == 0:
            raise ValueError("unsupported expert-parallel shape")
        self.ep_ws = torch.empty(self.ep_bytes, dtype=torch.uint8, device=self.device)
        bf16 = dict(dtype=torch.bfloat16, device=self.device)
        rows_send = min(T * k, E * C)
        self.buf_rows = (E // G) * C
        self.sendbuf = torch.empty(rows_send, d, **bf16)
        self.retbuf = torch.empty(rows_send, d, **bf16)
        self.recvbuf = torch.empty(self.buf_rows, d, **bf16)
        self.h = torch.empty(self.buf_rows, d_ff, **bf16)
        self.out = torch.empty(self.buf_rows, d, **bf16)
        self.loads_all: Optional[np.ndarray] = None
        self.tables: Optional[dict] = None
        self.R = 0

    def _loads_ptr(self):
        return self.loads_all.ctypes.data_as(ctypes.POINTER(moe.c_i32))

    def _stream(self):
        import torch
        return int(torch.cuda.current_stream(self.device).cuda_stream)

    def route(self, logits=None, x=None, w_router=None, bias=None) -> np.ndarray:
        """Top-k routing and the rank's own plan; returns its pair counts per expert [E]."""
        info = self.layer.plan(logits=logits, x=x, w_router=w_router, bias=bias)
        return np.array(info.load[:self.E], dtype=np.int32)

    def plan(self, loads_all) -> int:
        """Every rank's counts [G, E] (all-gathered) -> this rank's plan and exchange tables."""
        self.loads_all = np.ascontiguousarray(np.asarray(loads_all, dtype=np.int32).reshape(self.G, self.E))
        R = moe.c_i32(0)
        lib = moe.load_library()
        moe._check("moe_ep_plan", lib.moe_ep_plan(
            ctypes.byref(self.shape), self.G, self.rank, self._loads_ptr(), ctypes.byref(self.layer.info),
            self.layer.ws, self.layer.ws_bytes, int(self.ep_ws.data_ptr()), self.ep_bytes, ctypes.byref(R),
            self._stream()))
        self.R = R.value
        self.tables = moe.ep_exchange_plan(self.shape, self.G, self.rank, self.loads_all)
        return self.R

    def pack(self, r: int, x):
        """This rank's rows of round r, packed (chunk g for owner g); returns the filled rows."""
        lib = moe.load_library()
        moe._check("moe_ep_round_pack", lib.moe_ep_round_pack(
            ctypes.byref(self.shape), self.G, self.rank, self._loads_ptr(), int(self.ep_ws.data_ptr()),
            self.ep_bytes, r, int(x.data_ptr()), int(self.sendbuf.data_ptr()), self._stream()))
        return self.sendbuf[:int(self.tables["send_counts"][r].sum())]

    def experts(self, r: int, w_gate_up_local, w_down_local):
        """Owner side of round r over recvbuf's received rows; returns the result rows (same order)."""
        lib = moe.load_library()
        moe._check("moe_ep_round_experts", lib.moe_ep_round_experts(
            ctypes.byref(self.shape), self.G, self.rank, self._loads_ptr(), int(self.ep_ws.data_ptr()),
            self.ep_bytes, r, int(self.recvbuf.data_ptr()), int(w_gate_up_local.data_ptr()),
            int(w_down_local.data_ptr()), int(self.h.data_ptr()), int(self.out.data_ptr()), self.buf_rows,
            self.layer.ws, self._stream()))
        return self.out[:int(self.tables["recv_counts"][r].sum())]

    def combine(self, r: int, y) -> None:
        """y (+)= gate * retbuf rows for this rank's pairs of round r."""
        lib = moe.load_library()
        moe._check("moe_ep_round_combine", lib.moe_ep_round_combine(
            ctypes.byref(self.shape), self.G, self.rank, self._loads_ptr(), self.layer.ws, self.layer.ws_bytes,
            int(self.ep_ws.data_ptr()), self.ep_bytes, r, int(self.retbuf.data_ptr()), int(y.data_ptr()),
            self._stream()))

    def forward_distributed(self, x, w_gate_up_local, w_down_local, logits=None, w_router=None, bias=None,
                            group=None):
        """The whole layer on this rank, with torch.distributed (NCCL on GPUs) as the transport."""
        import torch
        import torch.distributed as dist
        counts = torch.as_tensor(self.route(logits=logits, x=x if logits is None else None, w_router=w_router,
                                            bias=bias), device=self.device)
        gathered = [torch.empty_like(counts) for _ in range(self.G)]
        dist.all_gather(gathered, counts, group=group)
        self.plan(torch.stack(gathered).cpu().numpy())
        y = torch.empty(x.shape[0], self.d, dtype=torch.float32, device=self.device)
        for r in range(self.R):
            send = self.pack(r, x)
            sc = [int(v) for v in self.tables["send_counts"][r]]
            rc = [int(v) for v in self.tables["recv_counts"][r]]
            recv = self.recvbuf[:sum(rc)]
            dist.all_to_all_single(recv, send, output_split_sizes=rc, input_split_sizes=sc, group=group)
            out = self.experts(r, w_gate_up_local, w_down_local)
            dist.all_to_all_single(self.retbuf[:sum(sc)], out, output_split_sizes=sc, input_split_sizes=rc,
                                   group=group)
            self.combine(r, y)
        return y
