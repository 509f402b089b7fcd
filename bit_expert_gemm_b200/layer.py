"""The routed-expert MoE layer as a sequence of C-ABI calls.

MoELayer owns the device weights of one layer plus every intermediate
buffer and workspace for a maximum token count, so that a forward pass
launches only the library's kernels (no allocation, no host sync).  The
weight format is one of "bf16" (16-bit weights, BF16 or FP16 activations),
"awq_g32" and "nvfp4"; the router and the shared expert are always 16-bit.

forward(x)               x [T, H] on the device -> y [T, H]; with a pre-MoE
                         RMSNorm gain in the weights ("w_norm" [H]) the
                         block's input is the normalised x (one call with
                         the routing: moe_norm_route_permute)
forward_host(xh, yh)     pinned host x -> y in pinned host memory (copies in
                         the stream, for end-to-end measurements)
refill_pass(x, stats)    one Refill-RMS scoring pass (k+1 slots), adds to the
                         statistics and returns y
capture(x, fn)           records one pass (forward, or any callable over the
                         layer's buffers) into a CUDA graph bound to the
                         device buffer x; replaying the graph re-runs the
                         pass on whatever x then holds, without host work
                         between the kernels; graph_kernels then holds the
                         number of kernel launches one replay makes
"""

from __future__ import annotations

from typing import Dict, Optional

import torch

from . import abi


def graph_kernel_nodes(g: "torch.cuda.CUDAGraph") -> int:
    """Kernel nodes of a captured (not yet instantiated) graph: the launches
    that one replay makes."""
    from cuda.bindings import runtime as rt

    graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, nodes, n = rt.cudaGraphGetNodes(graph)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    if n and not nodes:
        err, nodes, n = rt.cudaGraphGetNodes(graph, n)
    kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes[:n]]
    return sum(1 for t in kinds if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)


def prepare_nvfp4_weights(w: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    """Adds NVFP4 copies of the 16-bit expert weights, quantised by the
    library (moe_nvfp4_quantize): gate, up and down of every expert are
    separate tensors with their own global scale.
    w_gu [E, 2I, H/2], sf_gu [E, 2I, H/16], gs_gu [E, 2]; w_d [E, H, I/2],
    sf_d [E, H, I/16], gs_d [E].  The weight scales are also rearranged once
    into the FP4 GEMM's tile order (sfp_gu, sfp_d: moe_nvfp4_prepack_sf), so the
    layer's calls do not redo it every step."""
    gu, wd = w["w_gate_up"], w["w_down"]
    E, I2, H = gu.shape
    I = I2 // 2
    c, sf, gs = abi.moe_nvfp4_quantize(gu.reshape(2 * E, I, H))
    out = dict(w)
    out["w_gu"], out["sf_gu"], out["gs_gu"] = c.reshape(E, I2, H // 2), sf.reshape(E, I2, H // 16), gs.reshape(E, 2)
    c, sf, gs = abi.moe_nvfp4_quantize(wd)
    out["w_d"], out["sf_d"], out["gs_d"] = c, sf, gs
    out["sfp_gu"] = abi.moe_nvfp4_prepack_sf(out["sf_gu"], swiglu=True)
    out["sfp_d"] = abi.moe_nvfp4_prepack_sf(out["sf_d"], swiglu=False)
    return out


class MoELayer:
    def __init__(self, weights: Dict[str, torch.Tensor], k: int, fmt: str = "bf16", T_max: int = 8192,
                 extra: int = 0, device: Optional[torch.device] = None):
        self.w = weights
        self.k = k
        self.fmt = fmt
        self.extra = extra
        self.dev = device or weights["w_router"].device
        self.E, self.H = weights["w_router"].shape
        self.adt = weights["w_router"].dtype
        self.norm = "w_norm" in weights  # pre-MoE RMSNorm, gain 1 + w_norm, eps 1e-6
        self.norm_eps = 1e-6
        self.I_sh = weights["w_sh_down"].shape[1]
        if fmt in ("bf16",):
            self.I = weights["w_gate_up"].shape[1] // 2
        elif fmt == "awq_g32":
            self.I = weights["qw_gu"].shape[2] * 8 // 2
            if "awq_packed" not in weights:
                # the routed weights also tile-packed: the decode kernel fetches each
                # sub-tile, the grouped GEMMs each 128-column unit, with one bulk copy,
                # and both dequantise the pair-ordered codes without byte permutes
                self.w = weights = dict(weights)
                weights["awq_packed"] = abi.moe_awq_prepack_g32(weights["qw_gu"], weights["qz_gu"], weights["sc_gu"],
                                                                weights["qw_d"], weights["qz_d"], weights["sc_d"])
        elif fmt == "nvfp4":
            if "w_gu" not in weights:
                self.w = weights = prepare_nvfp4_weights(weights)
            self.I = weights["w_gu"].shape[1] // 2
        else:
            raise ValueError(fmt)
        self._alloc(T_max)

    def _alloc(self, T_max: int) -> None:
        d, H, E = self.dev, self.H, self.E
        ks = self.k + self.extra
        rows = T_max * ks
        i32 = torch.int32
        self.T_max = T_max
        self.topk_idx = torch.empty((T_max, ks), dtype=i32, device=d)
        self.topk_w = torch.empty((T_max, self.k), dtype=torch.float32, device=d)
        self.topk_logit = torch.empty((T_max, ks), dtype=torch.float32, device=d)
        self.offsets = torch.empty((E + 1,), dtype=i32, device=d)
        self.row_token = torch.empty((rows,), dtype=i32, device=d)
        self.slot_row = torch.empty((T_max, ks), dtype=i32, device=d)
        # routed rows f: FP32 for Refill, else the activation dtype (BF16 for NVFP4)
        f_dt = torch.float32 if self.extra else (self.adt if self.fmt in ("bf16", "awq_g32") else torch.bfloat16)
        self.f = torch.empty((rows, H), dtype=f_dt, device=d)
        self.shared = torch.empty((T_max, H), dtype=self.adt, device=d)
        # optional shared-expert gate (weights key "w_sh_gate", [H]): sigmoid(x . w) per token
        self.sh_gate = torch.empty((T_max,), dtype=torch.float32, device=d) if "w_sh_gate" in self.w else None
        # the normalised block input when the layer carries its pre-MoE RMSNorm
        self.x_norm = torch.empty((T_max, H), dtype=self.adt, device=d) if self.norm else None
        self.y = torch.empty((T_max, H), dtype=self.adt, device=d)
        op = {"bf16": abi.MOE_OP_SWIGLU_BF16, "awq_g32": abi.MOE_OP_SWIGLU_AWQ_G32,
              "nvfp4": abi.MOE_OP_SWIGLU_NVFP4}[self.fmt]
        # route + permute in one call; the T_max workspace covers every T <= T_max
        self.ws_route = abi.workspace(abi.MOE_OP_ROUTE_PERMUTE, T_max, H, E, ks, 0, d)
        self.ws_ffn = abi.workspace(op, T_max, H, E, ks, self.I, d)
        self.ws_sh = abi.workspace(abi.MOE_OP_SWIGLU_BF16, T_max, H, 1, 1, self.I_sh, d)
        # decode-sized batches run a separate shared expert (the library's
        # weight-streaming GEMVs for one dense expert) on a second stream
        self._sh_stream = T_max <= 16
        if self._sh_stream:
            self._side = torch.cuda.Stream(device=d)
        if self.fmt in ("bf16", "awq_g32") and self.I_sh == self.I:
            # routed + shared experts in one call: big enough for every path it
            # takes for T <= T_max (T <= 16, T <= 128, larger)
            op_exp = abi.MOE_OP_EXPERTS_BF16 if self.fmt == "bf16" else abi.MOE_OP_EXPERTS_AWQ_G32
            need = max(abi.moe_workspace_size(op_exp, t, H, E, ks, self.I)
                       for t in {T_max, min(T_max, 128), min(T_max, 16)})
            self.ws_exp = torch.empty(max(256, need), dtype=torch.uint8, device=d)
        else:
            self.ws_exp = None
        self.ws_refill = abi.workspace(abi.MOE_OP_REFILL, T_max, H, E, ks, 0, d)
        self._sh_off = {}

    def _shared_offsets(self, T: int) -> torch.Tensor:
        t = self._sh_off.get(T)
        if t is None:
            t = torch.tensor([0, T], dtype=torch.int32, device=self.dev)
            self._sh_off[T] = t
        return t

    def route(self, x: torch.Tensor) -> torch.Tensor:
        """Routing and permutation of the batch; returns the block's input:
        x, or with a pre-MoE RMSNorm the normalised x (then the shared-expert
        gate, if the layer has one, is computed by the same call)."""
        T = x.shape[0]
        ks = self.k + self.extra
        outs = dict(topk_idx=self.topk_idx[:T], topk_w=self.topk_w[:T], topk_logit=self.topk_logit[:T],
                    expert_offsets=self.offsets, row_token=self.row_token[:T * ks], slot_row=self.slot_row[:T],
                    ws=self.ws_route)
        if self.norm:
            gate = self.sh_gate[:T] if self.sh_gate is not None else None
            abi.moe_norm_route_permute(x, self.w["w_norm"], self.w["w_router"], self.w["bias"], self.k, self.extra,
                                       eps=self.norm_eps, w_shared_gate=self.w.get("w_sh_gate"),
                                       x_norm=self.x_norm[:T], shared_gate=gate, **outs)
            return self.x_norm[:T]
        abi.moe_route_permute(x, self.w["w_router"], self.w["bias"], self.k, self.extra, **outs)
        return x

    def experts(self, x: torch.Tensor) -> torch.Tensor:
        T = x.shape[0]
        rows = T * (self.k + self.extra)
        f = self.f[:rows]
        w = self.w
        if self.fmt == "bf16":
            abi.moe_grouped_swiglu_bf16(x, self.row_token[:rows], self.offsets, rows, w["w_gate_up"], w["w_down"],
                                        out_fp32=f.dtype == torch.float32, f=f, ws=self.ws_ffn)
        elif self.fmt == "awq_g32":
            abi.moe_grouped_swiglu_awq_g32(x, self.row_token[:rows], self.offsets, rows, w["qw_gu"], w["qz_gu"],
                                           w["sc_gu"], w["qw_d"], w["qz_d"], w["sc_d"],
                                           out_fp32=f.dtype == torch.float32, f=f, ws=self.ws_ffn)
        else:
            abi.moe_grouped_swiglu_nvfp4_prepacked(x, self.row_token[:rows], self.offsets, rows, w["w_gu"],
                                                   w["sfp_gu"], w["gs_gu"], w["w_d"], w["sfp_d"], w["gs_d"],
                                                   act_gs_in=w.get("act_gs"), out_fp32=f.dtype == torch.float32,
                                                   f=f, ws=self.ws_ffn)
        return f

    def shared_expert(self, x: torch.Tensor) -> torch.Tensor:
        T = x.shape[0]
        sh = self.shared[:T]
        abi.moe_grouped_swiglu_bf16(x, None, self._shared_offsets(T), T, self.w["w_sh_gate_up"].unsqueeze(0),
                                    self.w["w_sh_down"].unsqueeze(0), out_fp32=False, f=sh, ws=self.ws_sh)
        return sh

    def experts_and_shared(self, x: torch.Tensor):
        """Routed expert rows f and the shared expert's output; one C-ABI call
        (moe_experts_bf16 / moe_experts_awq_g32) for 16-bit and AWQ weights."""
        if self.ws_exp is None:
            if self._sh_stream and x.shape[0] <= 16:
                # decode batch: the shared expert (a few SMs' worth of weight
                # streaming) runs beside the routed experts on a second stream
                cur = torch.cuda.current_stream()
                self._side.wait_stream(cur)
                with torch.cuda.stream(self._side):
                    sh = self.shared_expert(x)
                f = self.experts(x)
                cur.wait_stream(self._side)
                return f, sh
            return self.experts(x), self.shared_expert(x)
        T = x.shape[0]
        rows = T * (self.k + self.extra)
        f = self.f[:rows]
        sh = self.shared[:T]
        w = self.w
        if self.fmt == "bf16":
            abi.moe_experts_bf16(x, self.row_token[:rows], self.offsets, rows, w["w_gate_up"], w["w_down"],
                                 w["w_sh_gate_up"], w["w_sh_down"], out_fp32=f.dtype == torch.float32, f=f,
                                 shared_out=sh, ws=self.ws_exp)
        elif "awq_packed" in w:
            abi.moe_experts_awq_g32_prepacked(x, self.row_token[:rows], self.offsets, rows, w["qw_gu"], w["qz_gu"],
                                              w["sc_gu"], w["qw_d"], w["qz_d"], w["sc_d"], w["awq_packed"],
                                              w["w_sh_gate_up"], w["w_sh_down"], out_fp32=f.dtype == torch.float32,
                                              f=f, shared_out=sh, ws=self.ws_exp)
        else:
            abi.moe_experts_awq_g32(x, self.row_token[:rows], self.offsets, rows, w["qw_gu"], w["qz_gu"], w["sc_gu"],
                                    w["qw_d"], w["qz_d"], w["sc_d"], w["w_sh_gate_up"], w["w_sh_down"],
                                    out_fp32=f.dtype == torch.float32, f=f, shared_out=sh, ws=self.ws_exp)
        return f, sh

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        """y [T, H] = the layer applied to x [T, H]; into `y` if given, else
        into the layer's own output buffer (overwritten by the next pass)."""
        T = x.shape[0]
        assert T <= self.T_max and self.extra == 0
        xin = self.route(x)
        gate = self.block_gate(xin)
        f, sh = self.experts_and_shared(xin)
        y = self.y[:T] if y is None else y
        abi.moe_combine(f, self.slot_row[:T], self.topk_w[:T], shared_out=sh, shared_gate=gate, y=y)
        return y

    def shared_gate(self, x: torch.Tensor) -> Optional[torch.Tensor]:
        """Per-token shared-expert gate (moe_shared_gate), or None without one."""
        if self.sh_gate is None:
            return None
        return abi.moe_shared_gate(x, self.w["w_sh_gate"], gate=self.sh_gate[:x.shape[0]])

    def block_gate(self, xin: torch.Tensor) -> Optional[torch.Tensor]:
        """The shared-expert gate of the block input xin (route's result):
        already computed by the routing call when the layer normalises its
        input, else by moe_shared_gate; None without a gate."""
        if self.sh_gate is None:
            return None
        if self.norm:
            return self.sh_gate[:xin.shape[0]]
        return self.shared_gate(xin)

    def capture(self, x: torch.Tensor, fn=None, warmup: int = 1) -> "torch.cuda.CUDAGraph":
        """CUDA graph of fn(x) (default: forward).  Every launch of the pass
        has fixed pointers (the layer's buffers, x) and host-side arguments,
        so the graph replays it exactly; the pass is run `warmup` times first
        so that one-time host set-up (function attributes, cached offsets)
        happens outside the capture."""
        fn = fn or self.forward
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(warmup):
                fn(x)
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            fn(x)
        self.graph_kernels = graph_kernel_nodes(g)
        g.instantiate()
        return g

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, x_dev: torch.Tensor) -> None:
        """Pinned host x -> device -> forward -> pinned host y, all enqueued on
        the current stream."""
        T = x_host.shape[0]
        x_dev[:T].copy_(x_host, non_blocking=True)
        y = self.forward(x_dev[:T])
        y_host.copy_(y, non_blocking=True)

    def refill_pass(self, x: torch.Tensor, sum_sq: torch.Tensor, count: torch.Tensor) -> torch.Tensor:
        """One Refill-RMS scoring pass over x; statistics are added in place."""
        T = x.shape[0]
        assert self.extra == 1
        xin = self.route(x)
        gate = self.block_gate(xin)
        f, sh = self.experts_and_shared(xin)
        y = self.y[:T]
        # the shared expert cancels in the score; with a gate, y is combined separately
        abi.razor_refill_rms_accumulate(f, self.slot_row[:T], self.topk_idx[:T], self.topk_logit[:T], self.offsets,
                                        sum_sq, count, shared_out=None if gate is not None else sh,
                                        y_out=None if gate is not None else y, ws=self.ws_refill)
        if gate is not None:
            abi.moe_combine(f, self.slot_row[:T], self.topk_w[:T], shared_out=sh, shared_gate=gate, y=y)
        return y


# Tensors of a layer whose leading axis (or, for the flat tile-packed copies,
# whose equal per-expert blocks) belong to one routed expert each.
EXPERT_TENSORS = ("w_router", "bias", "w_gate_up", "w_down", "qw_gu", "qz_gu", "sc_gu", "qw_d", "qz_d", "sc_d",
                  "w_gu", "sf_gu", "gs_gu", "w_d", "sf_d", "gs_d")
EXPERT_PACKED = ("awq_packed", "sfp_gu", "sfp_d")


def slice_layer_weights(w: Dict[str, torch.Tensor], kept: torch.Tensor) -> Dict[str, torch.Tensor]:
    """The pruned layer: every per-expert tensor, router rows and bias
    included, gathered with one kept list (razor_slice, all in the same order);
    the shared expert and any activation scales are unchanged.  kept [keep]
    int32 on the device, normally razor_select's ascending kept set."""
    E = w["w_router"].shape[0]
    out = {}
    for n, t in w.items():
        if n in EXPERT_TENSORS:
            out[n] = abi.razor_slice(t.contiguous(), kept)
        elif n in EXPERT_PACKED:
            out[n] = abi.razor_slice(t.reshape(E, -1), kept).reshape(-1)
        else:
            out[n] = t
    return out


def keep_manifest(kept, E: int, policy: str = "refill_rms", scores=None) -> dict:
    """Keep manifest of one pruned layer: the original expert indices in
    output order (expert j of the pruned layer is original expert
    kept_expert_indices[j]), the budget, and how they were chosen
    ("refill_rms": RMS-aggregated Refill scores; "router_norm": router-row
    L2 norm).  Host-side bookkeeping; kept may be a tensor or a sequence."""
    ids = [int(e) for e in (kept.tolist() if hasattr(kept, "tolist") else kept)]
    if sorted(set(ids)) != ids or (ids and not 0 <= ids[0] <= ids[-1] < E):
        raise ValueError("kept indices must be distinct, ascending and in [0, E)")
    m = {"method": "razor", "policy": policy, "experts_before": E, "experts_kept": len(ids),
         "kept_expert_indices": ids}
    if policy == "refill_rms":
        m["aggregation"] = "rms"
    if scores is not None:
        sc = scores.tolist() if hasattr(scores, "tolist") else list(scores)
        m["kept_scores"] = [float(sc[e]) for e in ids]
    return m


def refill_allreduce(sum_sq: torch.Tensor, count: torch.Tensor, group=None) -> None:
    """Combines the Refill-RMS statistics of all ranks in place: every rank
    ends with the sums and counts of the whole data set, so razor_select
    keeps the same experts everywhere.  The statistics are additive; they are
    gathered and added in rank order (not reduced by the collective), so the
    FP64 sums, and the selection, do not depend on the reduction order.
    sum_sq [E] FP64 and count [E] int64, on the device of the process group's
    backend (CUDA for NCCL, CPU for gloo)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    if world == 1:
        return
    parts_s = [torch.empty_like(sum_sq) for _ in range(world)]
    parts_c = [torch.empty_like(count) for _ in range(world)]
    dist.all_gather(parts_s, sum_sq.contiguous(), group=group)
    dist.all_gather(parts_c, count.contiguous(), group=group)
    total_s, total_c = parts_s[0].clone(), parts_c[0].clone()
    for ps, pc in zip(parts_s[1:], parts_c[1:]):
        total_s += ps
        total_c += pc
    sum_sq.copy_(total_s)
    count.copy_(total_c)


class HostPipeline:
    """Streams token batches from pinned host memory through one layer and
    back, overlapping the upload of batch i+1 and the download of batch i-1
    with the forward of batch i: uploads and downloads run on two copy
    streams, the forward (one CUDA graph per device buffer) on the caller's
    current stream, with two device buffers each for x and y and events
    between them, so a buffer is only refilled once the pass that reads it
    is done.

        pipe = HostPipeline(layer, T)
        for i, (xh, yh) in enumerate(batches):   # pinned host tensors [T, H]
            pipe.step(xh, yh)
        pipe.finish()                            # the current stream waits for the last download

    A host output buffer is complete once finish() (or a later wait on the
    current stream) has returned; a host input buffer may be reused once the
    step after next has been enqueued.

    Decode-sized batches (T <= whole_step_max_T, with graphs) take one CUDA
    graph per (host x, host y) pair instead, holding the upload, the forward
    and the download: a step is then one graph launch on the host, which is
    what bounds a decode step's end-to-end time (the copies are a few KB).
    Those graphs are recorded on the first step with each pair of host
    buffers, so a caller that streams from a fixed set of pinned buffers
    records them all during its warm-up; a host input buffer may then be
    rewritten once the step that reads it has completed on the GPU.
    """

    whole_step_max_T = 256

    def __init__(self, layer: MoELayer, T: int, use_graphs: bool = True):
        assert T <= layer.T_max and layer.extra == 0
        H = layer.w["w_router"].shape[1]
        dev = layer.dev
        self.layer, self.T = layer, T
        self.whole = use_graphs and T <= self.whole_step_max_T
        self._step_graphs = {}
        self.x = [torch.empty((T, H), dtype=layer.adt, device=dev) for _ in range(2)]
        self.y = [torch.empty((T, H), dtype=layer.adt, device=dev) for _ in range(2)]
        self.s_in, self.s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        self.ev_in = [torch.cuda.Event() for _ in range(2)]    # x[b] uploaded
        self.ev_used = [torch.cuda.Event() for _ in range(2)]  # the pass on x[b] is done and y[b] written
        self.ev_out = [torch.cuda.Event() for _ in range(2)]   # y[b] downloaded
        self.graphs = None
        if use_graphs and not self.whole:
            self.graphs = [layer.capture(self.x[b], fn=lambda xx, b=b: layer.forward(xx, y=self.y[b]))
                           for b in range(2)]
        self.i = 0

    def begin(self) -> None:
        """Orders the copy streams after the work already on the current
        stream (for instance a timing event)."""
        cs = torch.cuda.current_stream()
        self.s_in.wait_stream(cs)
        self.s_out.wait_stream(cs)

    def _whole_step(self, x_host: torch.Tensor, y_host: torch.Tensor) -> None:
        """Upload, forward and download of one batch as one graph launch."""
        key = (x_host.data_ptr(), y_host.data_ptr())
        g = self._step_graphs.get(key)
        if g is None:
            x, y, layer = self.x[0], self.y[0], self.layer

            def body():
                x.copy_(x_host, non_blocking=True)
                layer.forward(x, y=y)
                y_host.copy_(y, non_blocking=True)

            g = layer.capture(x, fn=lambda _x: body())
            self._step_graphs[key] = g
        g.replay()
        self.i += 1

    def step(self, x_host: torch.Tensor, y_host: torch.Tensor) -> None:
        if self.whole:
            self._whole_step(x_host, y_host)
            return
        b, cs = self.i & 1, torch.cuda.current_stream()
        if self.i >= 2:
            self.s_in.wait_event(self.ev_used[b])  # the pass two steps back has read x[b]
        with torch.cuda.stream(self.s_in):
            self.x[b].copy_(x_host, non_blocking=True)
            self.ev_in[b].record(self.s_in)
        cs.wait_event(self.ev_in[b])
        if self.i >= 2:
            cs.wait_event(self.ev_out[b])  # y[b] of two steps back has been downloaded
        if self.graphs is not None:
            self.graphs[b].replay()
        else:
            self.layer.forward(self.x[b], y=self.y[b])
        self.ev_used[b].record(cs)
        self.s_out.wait_event(self.ev_used[b])
        with torch.cuda.stream(self.s_out):
            y_host.copy_(self.y[b], non_blocking=True)
            self.ev_out[b].record(self.s_out)
        self.i += 1

    def finish(self) -> None:
        cs = torch.cuda.current_stream()
        cs.wait_stream(self.s_in)
        cs.wait_stream(self.s_out)
