"""Expert parallelism: one rank's part of a routed-expert MoE layer whose
experts are split over `world` ranks.

Qwen3.8-Flash-Next-RAZOR-96B-A6B-NVFP4 card, serving example: the model is
served with expert parallelism over eight GPUs.  The layer computes exactly
what MoELayer computes; only where an expert's rows are computed moves.  Every
rank holds the router and the shared expert (replicated), the routed experts
[rank * E/world, (rank+1) * E/world), and its own token batch.  A forward is
three phases around two all-to-all exchanges:

  dispatch   routing and permutation of the rank's tokens over all E experts
             (moe_route_permute), the plan (moe_ep_plan: the destination's
             local expert index of every permuted row, rows per rank), and the
             x rows in permuted order (moe_gather_rows) -- that order is
             grouped by destination rank already;
             exchange 1: rows and their expert indices to their ranks;
  compute    the received rows permuted by local expert (moe_permute), the
             grouped SwiGLU experts on them, and their outputs gathered back
             into the received order (moe_gather_rows);
             exchange 2: the outputs back to the ranks they came from, which
             receive them in their own permuted order;
  combine    the weighted combine with the rank's shared expert (moe_combine).

With extra = 1 the same pass scores the experts for RAZOR's Refill-RMS
selection (refill_pass): every token's k + 1 routed rows travel, come back
in FP32, and razor_refill_rms_accumulate adds the rank's statistics at the
tokens' home, where the rows are in the single-GPU layer's permuted order;
layer.refill_allreduce then sums the statistics of all ranks (in rank
order) before razor_select, so every rank keeps the same experts.

The arithmetic of every row is that of the single-GPU layer: the same
kernels, and rows do not interact inside a GEMM tile, so a rank's outputs are
bit-identical to MoELayer's on the same tokens.  The exchanges here are
torch.distributed all_to_all_single calls (NCCL between GPUs, gloo on CPU);
their split sizes need the row counts on the host, one synchronisation per
forward.  A kernel that moves the rows over peer memory inside the GEMMs is
not part of this module.

The steps are taken through an `ops` object (LibraryOps: the C ABI on the
device), so that the orchestration can be exercised on CPU processes with
stand-ins for the kernels.
"""

from __future__ import annotations

from typing import Dict, Optional

import torch

from . import abi


class LibraryOps:
    """The steps of the expert-parallel layer on the device, through the C
    ABI (BF16 / FP16 16-bit weights)."""

    def route_permute(self, x, w_router, bias, k, extra, bufs):
        abi.moe_route_permute(x, w_router, bias, k, extra, topk_idx=bufs["topk_idx"], topk_w=bufs["topk_w"],
                              topk_logit=bufs["topk_logit"], expert_offsets=bufs["offsets"],
                              row_token=bufs["row_token"], slot_row=bufs["slot_row"], ws=bufs["ws_route"])

    def plan(self, offsets, world, rows, row_local_expert, send_counts):
        abi.moe_ep_plan(offsets, world, rows, row_local_expert=row_local_expert, send_counts=send_counts)

    def gather_rows(self, src, index, out):
        if src.dtype == torch.float32:  # FP32 rows moved as pairs of 16-bit halves
            src, out = src.view(torch.bfloat16), out.view(torch.bfloat16)
        abi.moe_gather_rows(src, index, out=out)

    def permute(self, ids, E_local, offsets, row_token, slot_row, ws):
        abi.moe_permute(ids.view(-1, 1), E_local, expert_offsets=offsets, row_token=row_token,
                        slot_row=slot_row.view(-1, 1), ws=ws)

    def experts(self, x_rows, row_token, offsets, w_gate_up, w_down, f, ws):
        R = x_rows.shape[0]
        abi.moe_grouped_swiglu_bf16(x_rows, row_token, offsets, R, w_gate_up, w_down,
                                    out_fp32=f.dtype == torch.float32, f=f, ws=ws)

    def shared(self, x, offsets, w_sh_gate_up, w_sh_down, out, ws):
        T = x.shape[0]
        abi.moe_grouped_swiglu_bf16(x, None, offsets, T, w_sh_gate_up.unsqueeze(0), w_sh_down.unsqueeze(0),
                                    f=out, ws=ws)

    def combine(self, f_home, slot_row, topk_w, shared, y):
        abi.moe_combine(f_home, slot_row, topk_w, shared_out=shared, y=y)

    def refill(self, f_home, slot_row, topk_idx, topk_logit, offsets, sum_sq, count, shared, y, ws):
        abi.razor_refill_rms_accumulate(f_home, slot_row, topk_idx, topk_logit, offsets, sum_sq, count,
                                        shared_out=shared, y_out=y, ws=ws)


class ExpertParallelLayer:
    """One rank of an expert-parallel layer.  weights: the layer's full
    weights (router, bias, shared expert, and either all E experts' w_gate_up
    [E, 2I, H] / w_down [E, H, I] or only this rank's E/world of them with
    E taken from the router).  T_max: the largest token batch of a rank.
    extra = 1: each token also sends its rank-(k+1) row, for refill_pass."""

    def __init__(self, weights: Dict[str, torch.Tensor], k: int, rank: int, world: int, T_max: int,
                 ops=None, device: Optional[torch.device] = None, extra: int = 0):
        self.ops = ops or LibraryOps()
        self.k, self.rank, self.world = k, rank, world
        if extra not in (0, 1):
            raise ValueError("extra must be 0 or 1")
        self.extra = extra
        self.ks = k + extra
        self.E, self.H = weights["w_router"].shape
        if self.E % world:
            raise ValueError(f"E={self.E} is not a multiple of world={world}")
        self.El = self.E // world
        lo = rank * self.El
        gu, wd = weights["w_gate_up"], weights["w_down"]
        if gu.shape[0] == self.E:
            gu, wd = gu[lo:lo + self.El].contiguous(), wd[lo:lo + self.El].contiguous()
        if gu.shape[0] != self.El:
            raise ValueError("expert weights must hold all E experts or this rank's E/world")
        self.w = dict(w_router=weights["w_router"], bias=weights["bias"], w_gate_up=gu, w_down=wd,
                      w_sh_gate_up=weights["w_sh_gate_up"], w_sh_down=weights["w_sh_down"])
        self.dev = device or weights["w_router"].device
        self.adt = weights["w_router"].dtype
        self.I = gu.shape[1] // 2
        self._alloc(T_max)

    def _alloc(self, T_max: int) -> None:
        d, H, k, ks, E, El = self.dev, self.H, self.k, self.ks, self.E, self.El
        rows = T_max * ks
        R_max = self.world * rows  # every rank may send all its rows here
        # the kernels' routing weights are FP32; on CPU (stand-in steps) the
        # activation type
        i32, f32 = torch.int32, (torch.float32 if self.dev.type == "cuda" else self.adt)
        self.T_max = T_max
        b = dict(topk_idx=torch.empty((T_max, ks), dtype=i32, device=d),
                 topk_w=torch.empty((T_max, k), dtype=f32, device=d),
                 topk_logit=torch.empty((T_max, ks), dtype=f32, device=d),
                 offsets=torch.empty((E + 1,), dtype=i32, device=d),
                 row_token=torch.empty((rows,), dtype=i32, device=d),
                 slot_row=torch.empty((T_max, ks), dtype=i32, device=d))
        # the routed outputs: FP32 for the Refill statistics (as in MoELayer)
        fdt = torch.float32 if (self.extra and self.dev.type == "cuda") else self.adt
        if self.dev.type == "cuda":
            b["ws_route"] = abi.workspace(abi.MOE_OP_ROUTE_PERMUTE, T_max, H, E, ks, 0, d)
            self.ws_perm = abi.workspace(abi.MOE_OP_PERMUTE, R_max, H, El, 1, 0, d)
            self.ws_ffn = abi.workspace(abi.MOE_OP_SWIGLU_BF16, R_max, H, El, 1, self.I, d)
            self.ws_sh = abi.workspace(abi.MOE_OP_SWIGLU_BF16, T_max, H, 1, 1, self.I, d)
            self.ws_refill = abi.workspace(abi.MOE_OP_REFILL, T_max, H, E, ks, 0, d) if self.extra else None
        else:
            b["ws_route"] = self.ws_perm = self.ws_ffn = self.ws_sh = self.ws_refill = None
        self.b = b
        self.send_ids = torch.empty((rows,), dtype=i32, device=d)
        self.send_counts = torch.empty((self.world,), dtype=i32, device=d)
        self.send_rows = torch.empty((rows, H), dtype=self.adt, device=d)
        self.recv_ids = torch.empty((R_max,), dtype=i32, device=d)
        self.recv_rows = torch.empty((R_max, H), dtype=self.adt, device=d)
        self.loc_offsets = torch.empty((El + 1,), dtype=i32, device=d)
        self.loc_row = torch.empty((R_max,), dtype=i32, device=d)
        self.loc_slot = torch.empty((R_max,), dtype=i32, device=d)
        self.f_local = torch.empty((R_max, H), dtype=fdt, device=d)
        self.f_ret = torch.empty((R_max, H), dtype=fdt, device=d)
        self.f_home = torch.empty((rows, H), dtype=fdt, device=d)
        self.shared = torch.empty((T_max, H), dtype=self.adt, device=d)
        self.sh_offsets = {}
        self.y = torch.empty((T_max, H), dtype=self.adt, device=d)

    # -- phases ------------------------------------------------------------
    def dispatch(self, x: torch.Tensor):
        """Routing, plan and send rows of this rank's tokens; also its shared
        expert.  Returns (send_rows, send_ids, send_counts) for exchange 1."""
        T = x.shape[0]
        assert T <= self.T_max
        rows = T * self.ks
        b = self.b
        view = {n: (t[:T] if n in ("topk_idx", "topk_w", "topk_logit", "slot_row") else
                    t[:rows] if n == "row_token" else t) for n, t in b.items()}
        self.ops.route_permute(x, self.w["w_router"], self.w["bias"], self.k, self.extra, view)
        self.ops.plan(b["offsets"], self.world, rows, self.send_ids[:rows], self.send_counts)
        self.ops.gather_rows(x, b["row_token"][:rows], self.send_rows[:rows])
        off = self.sh_offsets.get(T)
        if off is None:
            off = torch.tensor([0, T], dtype=torch.int32, device=self.dev)
            self.sh_offsets[T] = off
        self.ops.shared(x, off, self.w["w_sh_gate_up"], self.w["w_sh_down"], self.shared[:T], self.ws_sh)
        self.T = T
        return self.send_rows[:rows], self.send_ids[:rows], self.send_counts

    def compute(self, recv_rows: torch.Tensor, recv_ids: torch.Tensor) -> torch.Tensor:
        """The local experts on the received rows; outputs in received order
        (for exchange 2)."""
        R = recv_rows.shape[0]
        self.ops.permute(recv_ids, self.El, self.loc_offsets, self.loc_row[:R], self.loc_slot[:R], self.ws_perm)
        self.ops.experts(recv_rows, self.loc_row[:R], self.loc_offsets, self.w["w_gate_up"], self.w["w_down"],
                         self.f_local[:R], self.ws_ffn)
        self.ops.gather_rows(self.f_local[:R], self.loc_slot[:R], self.f_ret[:R])
        return self.f_ret[:R]

    def combine(self, f_home: torch.Tensor) -> torch.Tensor:
        """Weighted combine of the rank's own rows (in its permuted order)
        with its shared expert."""
        T = self.T
        y = self.y[:T]
        if self.extra:
            raise RuntimeError("a layer built with extra = 1 scores experts: use refill_pass")
        self.ops.combine(f_home, self.b["slot_row"][:T], self.b["topk_w"][:T], self.shared[:T], y)
        return y

    def refill(self, f_home: torch.Tensor, sum_sq: torch.Tensor, count: torch.Tensor) -> torch.Tensor:
        """Refill-RMS statistics of the rank's tokens added to sum_sq [E] FP64
        and count [E] int64 (its own permuted rows, k + 1 per token), and the
        layer output y of those tokens."""
        if not self.extra:
            raise RuntimeError("refill needs a layer built with extra = 1")
        T = self.T
        y = self.y[:T]
        b = self.b
        self.ops.refill(f_home, b["slot_row"][:T], b["topk_idx"][:T], b["topk_logit"][:T], b["offsets"], sum_sq,
                        count, self.shared[:T], y, self.ws_refill)
        return y


def forward(layer: ExpertParallelLayer, x: torch.Tensor, group=None) -> torch.Tensor:
    """One expert-parallel forward of this rank's tokens x [T, H]; every rank
    of `group` calls it (collectively, in the same order)."""
    return _exchange_and_finish(layer, x, group, lambda f_home: layer.combine(f_home))


def refill_pass(layer: ExpertParallelLayer, x: torch.Tensor, sum_sq: torch.Tensor, count: torch.Tensor,
                group=None) -> torch.Tensor:
    """One expert-parallel Refill-RMS scoring pass of this rank's tokens x
    (layer built with extra = 1): the rank's statistics are added to sum_sq
    and count; combine them over the ranks with layer.refill_allreduce before
    razor_select.  Returns the layer output of x."""
    return _exchange_and_finish(layer, x, group, lambda f_home: layer.refill(f_home, sum_sq, count))


def _exchange_and_finish(layer: ExpertParallelLayer, x: torch.Tensor, group, finish) -> torch.Tensor:
    import torch.distributed as dist

    send_rows, send_ids, send_counts = layer.dispatch(x)
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    sc = [int(v) for v in send_counts.tolist()]
    rc = [int(v) for v in recv_counts.tolist()]
    R = sum(rc)
    recv_rows, recv_ids = layer.recv_rows[:R], layer.recv_ids[:R]
    dist.all_to_all_single(recv_rows, send_rows, rc, sc, group=group)
    dist.all_to_all_single(recv_ids, send_ids, rc, sc, group=group)
    f_ret = layer.compute(recv_rows, recv_ids)
    f_home = layer.f_home[:send_rows.shape[0]]
    dist.all_to_all_single(f_home, f_ret, sc, rc, group=group)
    return finish(f_home)


def forward_emulated(layers, xs, stats=None):
    """The same forward for all ranks of one process (every rank's layer and
    tokens on one device, the exchanges as copies between their buffers), in
    the phase order a real exchange imposes; no kernel waits for another.
    Returns each rank's y.  stats: for layers built with extra = 1, one
    (sum_sq, count) pair per rank, to which each rank's Refill statistics are
    added (refill_pass instead of forward)."""
    W = len(layers)
    sends = [lay.dispatch(x) for lay, x in zip(layers, xs)]
    counts = [[int(v) for v in s[2].tolist()] for s in sends]  # counts[src][dst]
    rets = []
    for d in range(W):
        parts_r, parts_i = [], []
        for s in range(W):
            a = sum(counts[s][:d])
            n = counts[s][d]
            parts_r.append(sends[s][0][a:a + n])
            parts_i.append(sends[s][1][a:a + n])
        R = sum(counts[s][d] for s in range(W))
        rr, ri = layers[d].recv_rows[:R], layers[d].recv_ids[:R]
        torch.cat(parts_r, out=rr)
        torch.cat(parts_i, out=ri)
        rets.append(layers[d].compute(rr, ri))
    ys = []
    for s in range(W):
        home = layers[s].f_home[:sends[s][0].shape[0]]
        parts = []
        for d in range(W):
            a = sum(counts[t][d] for t in range(s))  # rows of ranks before s in d's received order
            parts.append(rets[d][a:a + counts[s][d]])
        torch.cat(parts, out=home)
        ys.append(layers[s].refill(home, *stats[s]) if stats is not None else layers[s].combine(home))
    return ys
