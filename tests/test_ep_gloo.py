"""Expert parallelism on CPU processes (gloo, world size 2 and 4): the
orchestration of ep.py (routing, plan, the two all-to-all exchanges with
their split sizes, the local permutation, the return to the source ranks'
permuted order, the combine) with the steps taken by the oracle instead of
the kernels.  Every rank's output must equal the oracle's whole layer on that
rank's tokens; with extra = 1 (Refill-RMS scoring) every rank's statistics,
after the all-reduce, must equal the oracle's over all ranks' tokens."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

WORLDS = (2, 4)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The steps of ep.ExpertParallelLayer computed by the oracle in float64
    on CPU tensors (the layer's buffers), for testing the orchestration."""

    def route_permute(self, x, w_router, bias, k, extra, bufs):
        from oracle import moe
        r = moe.route(x.numpy(), w_router.numpy(), bias.numpy(), k, extra)
        p = moe.permute(r["idx"], w_router.shape[0])
        self.p = r["p"]
        bufs["topk_idx"].copy_(torch.from_numpy(r["idx"]))
        bufs["topk_w"].copy_(torch.from_numpy(r["w"]))
        bufs["topk_logit"].copy_(torch.from_numpy(np.take_along_axis(r["logits"], r["idx"], axis=1)))
        bufs["offsets"].copy_(torch.from_numpy(p["offsets"]))
        bufs["row_token"].copy_(torch.from_numpy(p["row_token"]))
        bufs["slot_row"].copy_(torch.from_numpy(p["slot_row"]))

    def plan(self, offsets, world, rows, row_local_expert, send_counts):
        off = offsets.numpy().astype(np.int64)
        E = len(off) - 1
        El = E // world
        e = np.searchsorted(off, np.arange(rows), side="right") - 1
        row_local_expert.copy_(torch.from_numpy(e % El))
        send_counts.copy_(torch.from_numpy(off[El::El] - off[:-1:El]))

    def gather_rows(self, src, index, out):
        out.copy_(src[index.long()])

    def permute(self, ids, E_local, offsets, row_token, slot_row, ws):
        from oracle import moe
        p = moe.permute(ids.numpy().astype(np.int64)[:, None], E_local)
        offsets.copy_(torch.from_numpy(p["offsets"]))
        row_token.copy_(torch.from_numpy(p["row_token"]))
        slot_row.copy_(torch.from_numpy(p["slot_row"].ravel()))

    def experts(self, x_rows, row_token, offsets, w_gate_up, w_down, f, ws):
        from oracle import moe
        off = offsets.numpy()
        rt = row_token.numpy().astype(np.int64)
        I = w_gate_up.shape[1] // 2
        for e in range(len(off) - 1):
            a, b = int(off[e]), int(off[e + 1])
            if a < b:
                gu = w_gate_up[e].numpy()
                fe, _ = moe.swiglu_expert(x_rows.numpy()[rt[a:b]], gu[:I], gu[I:], w_down[e].numpy())
                f[a:b] = torch.from_numpy(fe)

    def shared(self, x, offsets, w_sh_gate_up, w_sh_down, out, ws):
        from oracle import moe
        I = w_sh_gate_up.shape[0] // 2
        g = w_sh_gate_up.numpy()
        out.copy_(torch.from_numpy(moe.swiglu_expert(x.numpy(), g[:I], g[I:], w_sh_down.numpy())[0]))

    def combine(self, f_home, slot_row, topk_w, shared, y):
        from oracle import moe
        y.copy_(torch.from_numpy(moe.combine(f_home.numpy(), slot_row.numpy(), topk_w.numpy(), shared.numpy())))

    def refill(self, f_home, slot_row, topk_idx, topk_logit, offsets, sum_sq, count, shared, y, ws):
        from oracle import moe, razor
        k = slot_row.shape[1] - 1
        idx, sr = topk_idx.numpy().astype(np.int64), slot_row.numpy().astype(np.int64)
        d = razor.refill_deltas_closed_form(f_home.numpy(), sr, idx, self.p, k)
        razor.accumulate(sum_sq.numpy(), count.numpy(), d, idx, k)  # in place (shared storage)
        pk = np.take_along_axis(self.p, idx[:, :k], axis=1)
        y.copy_(torch.from_numpy(moe.combine(f_home.numpy(), sr[:, :k], pk / pk.sum(1, keepdims=True),
                                             shared.numpy())))


def _weights(E, H, I, seed):
    g = torch.Generator().manual_seed(seed)
    return dict(w_router=torch.randn((E, H), generator=g, dtype=torch.float64) / H ** 0.5,
                bias=torch.randn((E,), generator=g, dtype=torch.float64) * 1.5,
                w_gate_up=torch.randn((E, 2 * I, H), generator=g, dtype=torch.float64) / H ** 0.5,
                w_down=torch.randn((E, H, I), generator=g, dtype=torch.float64) / I ** 0.5,
                w_sh_gate_up=torch.randn((2 * I, H), generator=g, dtype=torch.float64) / H ** 0.5,
                w_sh_down=torch.randn((H, I), generator=g, dtype=torch.float64) / I ** 0.5)


def _tokens(rank, T, H):
    return torch.randn((T, H), generator=torch.Generator().manual_seed(1000 + rank), dtype=torch.float64)


E, H, I, K = 16, 32, 16, 3


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import datetime

    import torch.distributed as dist

    from bit_expert_gemm_b200 import ep

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = _weights(E, H, I, 7)
        T = 20 + 7 * rank  # ranks hold batches of different sizes
        layer = ep.ExpertParallelLayer(w, K, rank, world, T_max=48, ops=OracleOps(), device=torch.device("cpu"))
        for step in range(2):  # the layer's buffers are reused by a second forward
            x = _tokens(rank + 10 * step, T, H)
            y = ep.forward(layer, x)
            out[f"y{rank}_{step}"] = y.numpy().copy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", WORLDS)
def test_expert_parallel_matches_whole_layer(world):
    from oracle import moe

    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    w = {n: t.numpy() for n, t in _weights(E, H, I, 7).items()}
    for rank in range(world):
        T = 20 + 7 * rank
        for step in range(2):
            x = _tokens(rank + 10 * step, T, H).numpy()
            ref = moe.moe_layer(x, w["w_router"], w["bias"], K,
                                lambda e: (w["w_gate_up"][e, :I], w["w_gate_up"][e, I:], w["w_down"][e]),
                                (w["w_sh_gate_up"][:I], w["w_sh_gate_up"][I:], w["w_sh_down"]))
            assert np.allclose(res[f"y{rank}_{step}"], ref["y"], rtol=1e-12, atol=1e-12), (rank, step)


def _refill_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import datetime

    import torch.distributed as dist

    from bit_expert_gemm_b200 import ep
    from bit_expert_gemm_b200.layer import refill_allreduce

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = _weights(E, H, I, 7)
        T = 20 + 7 * rank
        layer = ep.ExpertParallelLayer(w, K, rank, world, T_max=48, ops=OracleOps(), device=torch.device("cpu"),
                                       extra=1)
        sum_sq = torch.zeros(E, dtype=torch.float64)
        count = torch.zeros(E, dtype=torch.int64)
        for step in range(2):
            x = _tokens(rank + 10 * step, T, H)
            y = ep.refill_pass(layer, x, sum_sq, count)
            out[f"y{rank}_{step}"] = y.numpy().copy()
        refill_allreduce(sum_sq, count)
        out[f"s{rank}"] = sum_sq.numpy().copy()
        out[f"c{rank}"] = count.numpy().copy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", WORLDS)
def test_expert_parallel_refill_statistics(world):
    """Refill-RMS scoring with the experts split over the ranks: each rank's
    k + 1 routed rows per token travel and come back, the statistics are added
    at the tokens' home, and after the all-reduce every rank holds the sums and
    counts of all ranks' tokens, as the oracle's single-process pass gives."""
    from oracle import moe, razor

    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_refill_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    w = {n: t.numpy() for n, t in _weights(E, H, I, 7).items()}
    ew = lambda e: (w["w_gate_up"][e, :I], w["w_gate_up"][e, I:], w["w_down"][e])
    sh = (w["w_sh_gate_up"][:I], w["w_sh_gate_up"][I:], w["w_sh_down"])
    s_ref, c_ref = np.zeros(E), np.zeros(E, np.int64)
    for rank in range(world):
        T = 20 + 7 * rank
        for step in range(2):
            x = _tokens(rank + 10 * step, T, H).numpy()
            ref = moe.moe_layer(x, w["w_router"], w["bias"], K, ew, sh, extra=1)
            r = ref["route"]
            d = razor.refill_deltas_closed_form(ref["f"], ref["perm"]["slot_row"], r["idx"], r["p"], K)
            razor.accumulate(s_ref, c_ref, d, r["idx"], K)
            assert np.allclose(res[f"y{rank}_{step}"], ref["y"], rtol=1e-12, atol=1e-12), (rank, step)
    assert c_ref.sum() > 0
    for rank in range(world):
        assert np.array_equal(res[f"c{rank}"], c_ref), rank
        assert np.allclose(res[f"s{rank}"], s_ref, rtol=1e-12, atol=0), rank


def test_expert_parallel_rejects_bad_splits():
    # the contiguous expert ranges need E % world == 0; extra is 0 or 1; a
    # rank's slice of the expert weights must hold E / world experts
    from bit_expert_gemm_b200 import ep

    w = _weights(E, H, I, 7)
    with pytest.raises(ValueError, match="multiple"):
        ep.ExpertParallelLayer(w, K, 0, 3, T_max=8, ops=OracleOps(), device=torch.device("cpu"))
    with pytest.raises(ValueError, match="extra"):
        ep.ExpertParallelLayer(w, K, 0, 2, T_max=8, ops=OracleOps(), device=torch.device("cpu"), extra=2)
    part = dict(w, w_gate_up=w["w_gate_up"][:3], w_down=w["w_down"][:3])
    with pytest.raises(ValueError, match="E/world"):
        ep.ExpertParallelLayer(part, K, 0, 2, T_max=8, ops=OracleOps(), device=torch.device("cpu"))
    # a rank given only its own slice keeps it as is
    own = dict(w, w_gate_up=w["w_gate_up"][8:16], w_down=w["w_down"][8:16])
    layer = ep.ExpertParallelLayer(own, K, 1, 2, T_max=8, ops=OracleOps(), device=torch.device("cpu"))
    assert torch.equal(layer.w["w_gate_up"], w["w_gate_up"][8:16])
