"""Expert parallelism on one GPU: the library's dispatch, shard-expert and
combine kernels (moe_ep_*) with the experts split into two shards, the
exchange between the shards done in-process (the rows for shard r are a
contiguous range of the dispatch order), checked against the single-GPU
layer and the fp64 oracle; and the torch.distributed driver of the
exchange on a one-rank NCCL group.  The two-rank exchange itself is tested
on CPU (tests/test_ep_multirank.py); this box runs one GPU per call."""
import numpy as np
import pytest

import synth
from tests import harness

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


@pytest.fixture(scope="module")
def moe():
    from bit_moe_expert_sqrtsoftplus_b200 import build
    build.build()
    import bit_moe_expert_sqrtsoftplus_b200 as m
    return m


def _cfg(moe, s, flags, n_experts=None, q4k=False, mode=None):
    return moe.make_config(s.hidden, s.inter, n_experts or s.n_experts, s.top_k, s.shared_inter, vocab=s.vocab,
                           routed_scaling=s.routed_scaling, rms_eps=1e-6,
                           mode=moe.MOE_ROUTE_ROUTER if mode is None else mode, flags=flags,
                           routed_format=moe.MOE_ROUTED_Q4K if q4k else moe.MOE_ROUTED_Q2)


def _ops(moe, s, W, shard, G, T, pre=0, q4k=False, mode=None):
    from bit_moe_expert_sqrtsoftplus_b200 import ep
    per = s.n_experts // G
    front_w = {k: W.get(k) for k in ("router_w", "bias", "tid2eid", "sh_gate", "sh_up", "sh_down", "grid")}
    front_w.update(gate=None, up=None, down=None)
    lo, hi = shard * per, (shard + 1) * per
    shard_w = {"gate": W["gate"][lo:hi], "up": W["up"][lo:hi], "down": W["down"][lo:hi], "grid": W["grid"],
               "sh_gate": None, "sh_up": None, "sh_down": None}
    return ep.DeviceOps(_cfg(moe, s, moe.MOE_FLAG_NO_ROUTED | pre, q4k=q4k, mode=mode), front_w,
                        _cfg(moe, s, moe.MOE_FLAG_EXPERTS_ONLY, n_experts=per, q4k=q4k, mode=mode), shard_w, lo,
                        max_tokens=T, max_recv_rows=T * s.top_k)


def _two_shards(moe, s, seed, layer, T, prenorm=False, q4k=False, router=True):
    from bit_moe_expert_sqrtsoftplus_b200 import ep
    G = 2
    mode = moe.MOE_ROUTE_ROUTER if router else moe.MOE_ROUTE_HASH
    W = harness.device_layer(s, seed, layer, router=router, q4k=q4k)
    pre = moe.MOE_FLAG_PRENORM_RESIDUAL if prenorm else 0
    ops = [_ops(moe, s, W, r, G, T, pre, q4k, mode) for r in range(G)]
    x_np = synth.activations(seed, T, s.hidden, stream=layer)
    tok_np = synth.token_ids(seed, T, s.vocab, stream=layer)
    x = torch.from_numpy(x_np).cuda()
    tok = torch.from_numpy(tok_np).cuda()
    offsets, perm, x_send, e_send, w_send = ops[0].dispatch(x, tok)
    send = ep.rank_splits(offsets.cpu().tolist(), G, s.n_experts)
    outs, r0 = [], 0
    for r in range(G):
        rows = slice(r0, r0 + send[r])
        outs.append(ops[r].experts(x_send[rows], e_send[rows], w_send[rows]))
        r0 += send[r]
    y = ops[0].combine(x, perm, torch.cat(outs))
    torch.cuda.synchronize()
    for o in ops:
        o.poll()
    # the single-GPU layer on the same weights and inputs
    L = moe.Layer(harness.config_for(s, mode, pre, q4k=q4k), W, max_tokens=T)
    y1 = L.forward(x, tok).cpu().numpy()
    L.poll()
    return x_np, tok_np, y.cpu().numpy(), y1, send


@pytest.mark.parametrize("T", [40, 300])
def test_two_shards_match_the_layer_and_the_oracle(moe, T):
    s = synth.workload("tiny", tokens=T)
    x, tok, y, y1, send = _two_shards(moe, s, 3, 2, T)
    assert sum(send) == T * s.top_k and min(send) > 0
    rel, mx = harness.errors(y, y1)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
    _, _, yref, _ = harness.oracle_layer(s, 3, 2, x)
    rel, mx = harness.errors(y, yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_two_shards_hash_routing_prenorm_residual(moe):
    s = synth.workload("tiny", tokens=64)
    x, tok, y, y1, _ = _two_shards(moe, s, 4, 1, 64, prenorm=True, router=False)
    _, _, yref, _ = harness.oracle_layer(s, 4, 1, x, tok, router=False, prenorm=True)
    rel, mx = harness.errors(y, yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_two_shards_q4k_experts(moe):
    s = synth.workload("tiny", tokens=96)
    x, tok, y, y1, _ = _two_shards(moe, s, 5, 0, 96, q4k=True)
    rel, mx = harness.errors(y, y1)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_two_shards_full_shape(moe):
    """V4-Flash shapes, 512 tokens with the skewed bias, 128 experts per shard."""
    s = synth.workload("prefill_t4096", tokens=512)
    x, tok, y, y1, send = _two_shards(moe, s, 6, 9, 512)
    rel, mx = harness.errors(y, y1)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
    _, _, yref, _ = harness.oracle_layer_dense(s, 6, 9, x)
    rel, mx = harness.errors(y, yref)
    assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)


def test_rows_outside_the_shard_are_reported(moe):
    s = synth.workload("tiny", tokens=40)
    W = harness.device_layer(s, 3, 2)
    ops = _ops(moe, s, W, 1, 2, 40)
    x16 = torch.zeros((3, s.hidden), dtype=torch.float16, device="cuda")
    e = torch.tensor([9, 3, 15], dtype=torch.int32, device="cuda")  # 3 is in shard 0
    w = torch.ones(3, dtype=torch.float32, device="cuda")
    out = ops.experts(x16, e, w)
    torch.cuda.synchronize()
    with pytest.raises(moe.MoeError) as ei:
        ops.poll()
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    assert torch.all(out[1] == 0)


def test_split_handles_do_not_serve_the_whole_layer(moe):
    s = synth.workload("tiny", tokens=4)
    W = harness.device_layer(s, 3, 2)
    ops = _ops(moe, s, W, 0, 2, 4)
    x = torch.zeros((4, s.hidden), device="cuda")
    y = torch.empty_like(x)
    for h in (ops.front, ops.shard):
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_ffn_forward(h, x, None, 4, y, ops.scratch_dispatch)
        assert ei.value.status in (moe.MOE_ERR_INVALID_ARG, moe.MOE_ERR_WORKSPACE_TOO_SMALL)


def test_expert_parallel_layer_on_a_one_rank_nccl_group(moe):
    """The torch.distributed driver (count exchange, three row all-to-alls
    out, one back) on a one-rank NCCL group: every row goes to this rank."""
    import datetime
    import os
    import socket

    import torch.distributed as dist

    from bit_moe_expert_sqrtsoftplus_b200 import ep
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        s = synth.workload("tiny", tokens=120)
        W = harness.device_layer(s, 7, 3)
        ops = _ops(moe, s, W, 0, 1, 120)
        layer = ep.ExpertParallelLayer(ops, 1, 0)
        x_np = synth.activations(7, 120, s.hidden, stream=3)
        y = layer.forward(torch.from_numpy(x_np).cuda()).cpu().numpy()
        ops.poll()
        _, _, yref, _ = harness.oracle_layer(s, 7, 3, x_np)
        rel, mx = harness.errors(y, yref)
        assert rel <= harness.MMA_REL_L2 and mx <= harness.MAX_ABS_FRAC, (rel, mx)
    finally:
        dist.destroy_process_group()
