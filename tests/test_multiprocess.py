"""Multi-process host logic on CPU (gloo, world size 2): the bench's rank
helper (barrier, max over ranks of a timing) and the combination of Refill-RMS
statistics across ranks, against the oracle run over all tokens in one
process."""

import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

from oracle import razor

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _stats(seed: int, T: int, E: int, k: int):
    """Synthetic routing (k distinct experts per token) and per-assignment
    squared deltas, accumulated by the oracle."""
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, k + 1, replace=False) for _ in range(T)])
    d = rng.standard_normal((T, k, 8)) * rng.random((T, 1, 1)) * 3.0  # delta vectors (H = 8)
    s = np.zeros(E)
    c = np.zeros(E, np.int64)
    razor.accumulate(s, c, d, idx, k)
    return s, c


def _worker(rank: int, port: int, E: int, k: int, keep: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD),
                      LOCAL_RANK=str(rank))
    import importlib.util
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from bit_expert_gemm_b200.layer import refill_allreduce

    d = bench.Dist(backend="gloo")
    try:
        d.barrier()
        out[f"max{rank}"] = d.max(1.5 + rank)  # every rank sees the slowest rank's time
        s, c = _stats(100 + rank, 300 + 50 * rank, E, k)  # this rank's share of the tokens
        ts, tc = torch.from_numpy(s.copy()), torch.from_numpy(c.copy())
        refill_allreduce(ts, tc)
        out[f"s{rank}"] = ts.numpy().copy()
        out[f"c{rank}"] = tc.numpy().copy()
        kept, ranking, score = razor.select(ts.numpy(), tc.numpy(), keep)
        out[f"kept{rank}"] = kept
    finally:
        d.close()


def test_two_rank_timing_max_and_refill_statistics():
    E, k, keep = 64, 4, 32
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(port, E, k, keep, out), nprocs=WORLD, join=True, start_method="spawn")
        res = dict(out)
    assert res["max0"] == res["max1"] == 2.5
    # every rank holds the same combined statistics, equal to the two shares added in rank order
    s0, c0 = _stats(100, 300, E, k)
    s1, c1 = _stats(101, 350, E, k)
    for r in range(WORLD):
        assert np.array_equal(res[f"c{r}"], c0 + c1)
        assert np.array_equal(res[f"s{r}"], s0 + s1)
    assert np.array_equal(res["kept0"], res["kept1"])
    # and the selection matches one pass of the oracle over the statistics of all tokens
    kept_ref, _, _ = razor.select(s0 + s1, c0 + c1, keep)
    assert np.array_equal(res["kept0"], kept_ref)
