"""Expert parallelism across ranks on CPU, world size 2 over gloo: the
rank-level exchange of bit_moe_expert_sqrtsoftplus_b200.ep with stand-in
steps (routing, grouping and a per-expert transform in numpy), so that the
split of the pairs by owner rank, the send/receive counts, the rows each
rank receives and the order in which the outputs return are checked exactly
against a one-process computation.  The library's own kernels for the three
steps are covered on the GPU (tests/test_ep_gpu.py)."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

E, K, H = 16, 3, 8


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _routing(rank: int, T: int):
    """Seeded routing of a rank's tokens: k distinct experts per token in
    ascending id, weights; token rows."""
    rng = np.random.default_rng(100 + rank)
    idx = np.sort(np.stack([rng.choice(E, K, replace=False) for _ in range(T)]), axis=1).astype(np.int32)
    w = rng.uniform(0.1, 1.0, size=(T, K)).astype(np.float32)
    x = rng.standard_normal((T, H)).astype(np.float32)
    return x, idx, w


def _expert(e, xrow):
    """Stand-in expert e: an affine map that differs per expert."""
    return xrow.astype(np.float32) * np.float32(e + 1) + np.float32(0.25 * e)


def _shared(x):
    return x * np.float32(0.5)


def _reference(x, idx, w):
    """y[t] = shared + sum over slots (ascending expert id) of w * expert(x)."""
    y = _shared(x).copy()
    xs = x.astype(np.float16)
    for t in range(x.shape[0]):
        for q in range(K):
            y[t] += w[t, q] * _expert(int(idx[t, q]), xs[t])
    return y


class StandInOps:
    """The three steps in numpy on CPU tensors, with the library's data
    layout: pairs grouped by expert (stable), rows as f16."""

    def __init__(self, rank, world, T, log):
        import oracle
        self.oracle = oracle
        self.E, self.k, self.H = E, K, H
        self.rank, self.world = rank, world
        self.x, self.idx, self.w = _routing(rank, T)
        self.log = log

    def dispatch(self, x, token_ids=None):
        import torch
        offsets, perm = self.oracle.permutation(self.idx, E)
        xs = self.x.astype(np.float16)
        x_send = torch.from_numpy(xs[perm // K].copy())
        e_send = torch.from_numpy(self.idx.ravel()[perm].astype(np.int32))
        w_send = torch.from_numpy(self.w.ravel()[perm].astype(np.float32))
        self.log["offsets"] = offsets
        return torch.from_numpy(offsets), torch.from_numpy(perm), x_send, e_send, w_send

    def experts(self, x_recv, e_recv, w_recv):
        import torch
        per = E // self.world
        e = e_recv.numpy()
        self.log["e_recv"] = e.copy()
        assert np.all((e >= self.rank * per) & (e < (self.rank + 1) * per))
        xr = x_recv.numpy()
        out = np.stack([w_recv.numpy()[i] * _expert(int(e[i]), xr[i]) for i in range(len(e))]) if len(e) else \
            np.zeros((0, H), np.float32)
        return torch.from_numpy(out.astype(np.float32))

    def combine(self, x, perm, out_back, y=None):
        import torch
        p = perm.numpy()
        pos = np.empty_like(p)
        pos[p] = np.arange(len(p))
        ob = out_back.numpy()
        yy = _shared(self.x).copy()
        for t in range(self.x.shape[0]):
            for q in range(K):
                yy[t] += ob[pos[t * K + q]]
        return torch.from_numpy(yy)


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    import datetime
    import json

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from bit_moe_expert_sqrtsoftplus_b200 import ep

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        T = [7, 5][rank]
        log = {}
        ops = StandInOps(rank, world, T, log)
        layer = ep.ExpertParallelLayer(ops, world, rank)
        y = layer.forward(torch.from_numpy(ops.x)).numpy()
        ref = _reference(ops.x, ops.idx, ops.w)
        send = ep.rank_splits(log["offsets"], world, E)
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y)
        np.save(os.path.join(out_dir, f"ref{rank}.npy"), ref)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"send": send, "e_recv": log["e_recv"].tolist()}, f)
    finally:
        dist.destroy_process_group()


def test_rank_splits_follow_the_expert_blocks():
    sys.path.insert(0, ROOT)
    from bit_moe_expert_sqrtsoftplus_b200 import ep
    offsets = np.array([0, 2, 2, 5, 9, 9, 9, 12, 20])  # E = 8
    assert ep.rank_splits(offsets, 2, 8) == [9, 11]
    assert ep.rank_splits(offsets, 4, 8) == [2, 7, 0, 11]
    assert [ep.rank_of_expert(e, 8, 4) for e in range(8)] == [0, 0, 1, 1, 2, 2, 3, 3]
    with pytest.raises(ValueError):
        ep.rank_splits(offsets, 3, 8)


def test_expert_parallel_exchange_gloo(tmp_path):
    import json

    import torch.multiprocessing as mp

    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    info = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in range(world):
        y = np.load(tmp_path / f"y{r}.npy")
        ref = np.load(tmp_path / f"ref{r}.npy")
        assert np.array_equal(y, ref), r
    # what rank r received is exactly the pairs every rank sent to it, in
    # source-rank order, each source's rows grouped by expert
    for r in range(world):
        want = []
        for src in range(world):
            _, idx, _ = _routing(src, [7, 5][src])
            ids = np.sort(idx.ravel(), kind="stable")
            want += [int(e) for e in ids if e // (E // world) == r]
        assert info[r]["e_recv"] == want
    sent = np.array([i["send"] for i in info])
    assert sent.sum() == (7 + 5) * K
