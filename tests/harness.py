"""Shared helpers for the GPU parity tests: build device layers from the
seeded generator, run the oracle on the same inputs, compare."""
from __future__ import annotations

import numpy as np

import oracle
import synth

GEMV_REL_L2 = 1e-4        # decode (mma.sync int8 limbs) path
MMA_REL_L2 = 3e-3         # bf16 tensor-core path
MAX_ABS_FRAC = 2e-2       # max |err| <= 2e-2 * max |y|


def config_for(s: synth.LayerShape, mode=None, flags=0, q4k=False):
    import bit_moe_expert_sqrtsoftplus_b200 as moe
    if mode is None:
        mode = moe.MOE_ROUTE_ROUTER
    return moe.make_config(s.hidden, s.inter, s.n_experts, s.top_k, s.shared_inter, vocab=s.vocab,
                           routed_scaling=s.routed_scaling, rms_eps=1e-6, mode=mode, flags=flags,
                           routed_format=moe.MOE_ROUTED_Q4K if q4k else moe.MOE_ROUTED_Q2)


def device_layer(s: synth.LayerShape, seed: int, layer: int, router=True, q4k=False):
    return synth.device_layer(seed, layer, s, router=router, q4k=q4k)


def oracle_layer(s: synth.LayerShape, seed: int, layer: int, x: np.ndarray, token_ids=None, router=True,
                 prenorm=False, threads: int = 1, q4k=False):
    """fp64 oracle: returns (idx, w, y, margin)."""
    xin = x.astype(np.float64)
    if prenorm:
        xin = oracle.rmsnorm(xin, 1e-6)
    if router:
        Wr = synth.router_weight(seed, layer, s.n_experts, s.hidden)
        b = synth.bias(seed, layer, s.n_experts, s.skew)
        z = oracle.router_logits(xin, Wr)
        idx, w, margin = oracle.select(z, b, s.top_k, s.routed_scaling)
    else:
        tab = synth.tid2eid(seed, layer, s.vocab, s.n_experts, s.top_k)
        idx, w = oracle.hash_route(token_ids, tab, s.top_k, s.routed_scaling, n_experts=s.n_experts)
        margin = np.full(x.shape[0], np.inf)
    W = synth.host_layer(seed, layer, s, experts=np.unique(idx), router=router, q4k=q4k)
    y = oracle.layer(W, s, xin, idx, w, threads=threads)
    if prenorm:
        y = y + x.astype(np.float64)
    return idx, w, y, margin


def oracle_layer_dense(s: synth.LayerShape, seed: int, layer: int, x: np.ndarray, token_ids=None, router=True,
                       prenorm=False, q4k=False):
    """As oracle_layer, with the layer computed by oracle.layer_dense (decode
    each used matrix once, fp64 matrix products): for checking every row of
    full-size calls."""
    xin = x.astype(np.float64)
    if prenorm:
        xin = oracle.rmsnorm(xin, 1e-6)
    if router:
        Wr = synth.router_weight(seed, layer, s.n_experts, s.hidden)
        b = synth.bias(seed, layer, s.n_experts, s.skew)
        idx, w, margin = oracle.select(oracle.router_logits(xin, Wr), b, s.top_k, s.routed_scaling)
    else:
        tab = synth.tid2eid(seed, layer, s.vocab, s.n_experts, s.top_k)
        idx, w = oracle.hash_route(token_ids, tab, s.top_k, s.routed_scaling, n_experts=s.n_experts)
        margin = np.full(x.shape[0], np.inf)
    W = synth.host_layer(seed, layer, s, experts=np.unique(idx), router=router, q4k=q4k)
    y = oracle.layer_dense(W, s, xin, idx, w)
    if prenorm:
        y = y + x.astype(np.float64)
    return idx, w, y, margin


def errors(y: np.ndarray, ref: np.ndarray):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rel_l2 = float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))
    max_abs = float(np.abs(y - ref).max() / max(np.abs(ref).max(), 1e-300))
    return rel_l2, max_abs
