"""Expert parallelism for the MoE layer: the routed experts split over the
ranks of a process group (one GPU per rank, torch.distributed over NCCL).

Rank r owns the experts [r*E/G, (r+1)*E/G).  Every rank routes its own
tokens; the token rows travel to the ranks that own their experts and the
expert outputs come back in one all-to-all each way; the shared expert runs
where the tokens live.  Source for the split: ds4 runs one model over two
machines ("DeepSeek-V4-Flash one-token computation flow", section
"128GB にどう収めるか"); splitting by expert is this library's choice.

The arithmetic runs in the library's kernels (``moe_ep_dispatch``,
``moe_ep_experts``, ``moe_ep_combine``); this module only sizes the buffers
and calls the collectives.  The three steps are reached through an ``ops``
object so that the exchange logic can be exercised with stand-in steps on
CPU process groups; :class:`DeviceOps` is the one the layer uses.
"""
from __future__ import annotations

import bit_moe_expert_sqrtsoftplus_b200 as _moe


def rank_of_expert(e: int, n_experts: int, world: int) -> int:
    """The rank that owns global expert e (contiguous blocks of E/G)."""
    return e // (n_experts // world)


def rank_splits(offsets, world: int, n_experts: int) -> list[int]:
    """Dispatch rows per destination rank from the grouped offsets [E+1]:
    pairs are grouped by expert and experts by owner, so rank r's rows are
    the contiguous range offsets[r*E/G] .. offsets[(r+1)*E/G]."""
    if n_experts % world:
        raise ValueError(f"{n_experts} experts do not split evenly over {world} ranks")
    per = n_experts // world
    return [int(offsets[(r + 1) * per]) - int(offsets[r * per]) for r in range(world)]


class DeviceOps:
    """The three steps on this rank's GPU through the C ABI.

    front: a handle with the router (or token table) and the shared expert
           (made with MOE_FLAG_NO_ROUTED, or a whole-layer config)
    shard: a handle made with MOE_FLAG_EXPERTS_ONLY over this rank's experts
    first_expert: global id of the shard's first expert"""

    def __init__(self, front_cfg, front_weights: dict, shard_cfg, shard_weights: dict, first_expert: int,
                 max_tokens: int, max_recv_rows: int, device="cuda"):
        import torch
        self.H, self.k, self.E = front_cfg.hidden, front_cfg.top_k, front_cfg.n_experts
        self.first_expert = first_expert
        self.device = device
        self.front_cfg, self.shard_cfg = front_cfg, shard_cfg
        pb, _ = _moe.moe_workspace_size(front_cfg, 1)
        self.front_persist = torch.empty(max(pb, 16), dtype=torch.uint8, device=device)
        self._fw = _moe.make_weights(front_weights)
        self.front = _moe.moe_init(front_cfg, self._fw, self.front_persist)
        pb, _ = _moe.moe_workspace_size(shard_cfg, 1)
        self.shard_persist = torch.empty(max(pb, 16), dtype=torch.uint8, device=device)
        self._sw = _moe.make_weights(shard_weights)
        self.shard = _moe.moe_init(shard_cfg, self._sw, self.shard_persist)
        self.weights = (front_weights, shard_weights)  # kept alive with the handles
        d, _, c = _moe.moe_ep_workspace_size(front_cfg, max_tokens, 0)
        _, x, _ = _moe.moe_ep_workspace_size(shard_cfg, 0, max_recv_rows)
        self.scratch_dispatch = torch.empty(max(d, 16), dtype=torch.uint8, device=device)
        self.scratch_combine = torch.empty(max(c, 16), dtype=torch.uint8, device=device)
        self.scratch_experts = torch.empty(max(x, 16), dtype=torch.uint8, device=device)
        self.max_tokens, self.max_recv_rows = max_tokens, max_recv_rows

    def dispatch(self, x, token_ids=None):
        import torch
        T = x.shape[0]
        n = T * self.k
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=x.device)
        perm = torch.empty(n, dtype=torch.int32, device=x.device)
        x_send = torch.empty((n, self.H), dtype=torch.float16, device=x.device)
        e_send = torch.empty(n, dtype=torch.int32, device=x.device)
        w_send = torch.empty(n, dtype=torch.float32, device=x.device)
        _moe.moe_ep_dispatch(self.front, x, token_ids, T, offsets, perm, x_send, e_send, w_send,
                             self.scratch_dispatch)
        return offsets, perm, x_send, e_send, w_send

    def experts(self, x_recv, e_recv, w_recv):
        import torch
        N = x_recv.shape[0]
        out = torch.empty((N, self.H), dtype=torch.float32, device=x_recv.device)
        if N > self.max_recv_rows:
            raise _moe.MoeError(_moe.MOE_ERR_WORKSPACE_TOO_SMALL,
                                f"{N} received rows, the layer was sized for {self.max_recv_rows}")
        _moe.moe_ep_experts(self.shard, x_recv, e_recv, w_recv, N, self.first_expert, out, self.scratch_experts)
        return out

    def combine(self, x, perm, out_back, y=None):
        import torch
        if y is None:
            y = torch.empty_like(x)
        _moe.moe_ep_combine(self.front, x, x.shape[0], perm, out_back, y, self.scratch_combine)
        return y

    def poll(self):
        _moe.moe_poll_device_error(self.front)
        _moe.moe_poll_device_error(self.shard)

    def close(self):
        for h in ("front", "shard"):
            if getattr(self, h, None):
                _moe.moe_destroy(getattr(self, h))
                setattr(self, h, None)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ExpertParallelLayer:
    """One layer call split over the ranks of `group`: dispatch on this
    rank's tokens, one all-to-all of the rows (and their expert ids and
    weights) to the experts' owners, the shard's experts, one all-to-all of
    the outputs back, combine with the shared expert.  Every rank calls
    forward with its own tokens (any T, possibly different per rank); the
    collectives are the same on every rank and in the same order."""

    def __init__(self, ops, world: int, rank: int, group=None):
        self.ops, self.world, self.rank, self.group = ops, world, rank, group
        if ops.E % world:
            raise ValueError(f"{ops.E} experts do not split evenly over {world} ranks")

    def forward(self, x, token_ids=None, y=None):
        import torch
        import torch.distributed as dist
        offsets, perm, x_send, e_send, w_send = self.ops.dispatch(x, token_ids)
        send = rank_splits(offsets.cpu().tolist(), self.world, self.ops.E)
        send_t = torch.tensor(send, dtype=torch.int64, device=x.device)
        recv_t = torch.empty_like(send_t)
        dist.all_to_all_single(recv_t, send_t, group=self.group)
        recv = [int(v) for v in recv_t.cpu().tolist()]
        N = sum(recv)
        x_recv = x_send.new_empty((N, x_send.shape[1]))
        e_recv = e_send.new_empty(N)
        w_recv = w_send.new_empty(N)
        dist.all_to_all_single(x_recv, x_send, recv, send, group=self.group)
        dist.all_to_all_single(e_recv, e_send, recv, send, group=self.group)
        dist.all_to_all_single(w_recv, w_send, recv, send, group=self.group)
        out = self.ops.experts(x_recv, e_recv, w_recv)
        out_back = out.new_empty((x_send.shape[0], out.shape[1]))
        dist.all_to_all_single(out_back, out, send, recv, group=self.group)
        return self.ops.combine(x, perm, out_back, y)
