"""Seeded synthetic inputs for the MoE FFN layer.

This package is the one input source that the oracle and the CUDA layer share.
It draws activations, router weights, bias, codebook, hash table and the
packed expert blocks; it holds none of the layer's arithmetic (no decoding, no
routing, no expert math).  Packed blocks and the small integer tables come
from the counter-based generator in ``synth.h`` (host library via ctypes,
device kernels for multi-gigabyte sets, byte-identical); the Gaussian inputs
(activations and F16 router weights) come from numpy's seeded PCG64 generator.

Workloads (sizes from the DeepSeek-V4-Flash config table: hidden 4096, expert
intermediate 2048, 256 routed experts, top-6, one shared expert, vocabulary
129,280, 43 layers of which the first 3 are hash-routed):

=================  =====  ====  ====  ===  ==  =====  ======================
name               H      I     Is    E    k   T      notes
=================  =====  ====  ====  ===  ==  =====  ======================
tiny               256    256   256   16   2   4      oracle runs in ms
decode_t1          4096   2048  2048  256  6   1      8 rotating weight sets
decode_t32         4096   2048  2048  256  6   32     bias +0.5 on e % 8 == 0
prefill_t4096      4096   2048  2048  256  6   4096   bias +0.5 on e % 8 == 0
stack43_t8         4096   2048  2048  256  6   8      43 layers, 0-2 hashed
decode_t1_q4k      4096   2048  2048  256  6   1      Q4_K routed experts
stack43_t8_q2q4    4096   2048  2048  256  6   8      stack43_t8, layers 37-42 Q4_K
=================  =====  ====  ====  ===  ==  =====  ======================
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "_synth_host.so")
_DEV_SO = os.path.join(_HERE, "_synth_dev.so")

KIND_IQ2XXS, KIND_Q2K, KIND_Q80, KIND_Q4K = 0, 1, 2, 3
T_BIAS, T_GATE, T_UP, T_DOWN, T_SH_GATE, T_SH_UP, T_SH_DOWN, T_GRID, T_TID2EID = 2, 3, 4, 5, 6, 7, 8, 9, 10
BLOCK_BYTES = {KIND_IQ2XXS: 66, KIND_Q2K: 84, KIND_Q80: 34, KIND_Q4K: 144}
BLOCK_ELEMS = {KIND_IQ2XXS: 256, KIND_Q2K: 256, KIND_Q80: 32, KIND_Q4K: 256}


@dataclass(frozen=True)
class LayerShape:
    hidden: int
    inter: int
    shared_inter: int
    n_experts: int
    top_k: int
    tokens: int
    vocab: int = 129280
    routed_scaling: float = 1.5
    skew: bool = False
    layers: int = 1
    hash_layers: int = 0
    weight_sets: int = 1
    q4k: bool = False  # routed experts in Q4_K (the q2-q4 build's upgraded layers)
    q4k_layers: int = 0  # in a stack: the last q4k_layers layers have Q4_K routed experts

    def layer_shape(self, layer: int) -> "LayerShape":
        """The shape of one layer of a stack (its routed format included)."""
        q4k = self.q4k or layer >= self.layers - self.q4k_layers
        return replace(self, q4k=q4k, q4k_layers=0)

    def row_bytes(self, kind: int, cols: int) -> int:
        return cols // BLOCK_ELEMS[kind] * BLOCK_BYTES[kind]

    @property
    def gate_kind(self) -> int:
        return KIND_Q4K if self.q4k else KIND_IQ2XXS

    @property
    def down_kind(self) -> int:
        return KIND_Q4K if self.q4k else KIND_Q2K

    @property
    def gate_bytes_per_expert(self) -> int:
        return self.inter * self.row_bytes(self.gate_kind, self.hidden)

    @property
    def down_bytes_per_expert(self) -> int:
        return self.hidden * self.row_bytes(self.down_kind, self.inter)

    @property
    def expert_bytes(self) -> int:
        return 2 * self.gate_bytes_per_expert + self.down_bytes_per_expert

    @property
    def shared_bytes(self) -> int:
        return 2 * self.shared_inter * self.row_bytes(KIND_Q80, self.hidden) + self.hidden * self.row_bytes(
            KIND_Q80, self.shared_inter)


WORKLOADS = {
    "tiny": LayerShape(256, 256, 256, 16, 2, 4, vocab=1024),
    "decode_t1": LayerShape(4096, 2048, 2048, 256, 6, 1, weight_sets=8),
    "decode_t32": LayerShape(4096, 2048, 2048, 256, 6, 32, skew=True),
    "prefill_t4096": LayerShape(4096, 2048, 2048, 256, 6, 4096, skew=True),
    "stack43_t8": LayerShape(4096, 2048, 2048, 256, 6, 8, layers=43, hash_layers=3),
    "decode_t1_q4k": LayerShape(4096, 2048, 2048, 256, 6, 1, weight_sets=8, q4k=True),
    "stack43_t8_q2q4": LayerShape(4096, 2048, 2048, 256, 6, 8, layers=43, hash_layers=3, q4k_layers=6),
}


def workload(name: str, **over) -> LayerShape:
    return replace(WORKLOADS[name], **over)


# --------------------------------------------------------------------------- build

def _build_host():
    src = os.path.join(_HERE, "synth_host.c")
    if os.path.exists(_HOST_SO) and os.path.getmtime(_HOST_SO) >= max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "synth.h"))):
        return
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                           "-o", _HOST_SO, src])


def _build_dev():
    src = os.path.join(_HERE, "synth_dev.cu")
    if os.path.exists(_DEV_SO) and os.path.getmtime(_DEV_SO) >= max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "synth.h"))):
        return
    subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-Xcompiler", "-fPIC", "-shared", "-o", _DEV_SO, src])


def build(device: bool = True) -> None:
    _build_host()
    if device:
        _build_dev()


_host = None
_dev = None


def _hostlib():
    global _host
    if _host is None:
        _build_host()
        lib = ctypes.CDLL(_HOST_SO)
        u64, u32, i32, vp = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_void_p
        lib.synth_fill_routed.argtypes = [u64, u32, u32, i32, i32, i32, i32, i32, vp, i32]
        lib.synth_fill_grid.argtypes = [u64, u32, vp]
        lib.synth_fill_bias.argtypes = [u64, u32, i32, i32, vp]
        lib.synth_fill_tid2eid.argtypes = [u64, u32, i32, i32, i32, vp]
        lib.synth_f16_of.argtypes = [ctypes.c_float]
        lib.synth_f16_of.restype = ctypes.c_uint16
        _host = lib
    return _host


def _devlib():
    global _dev
    if _dev is None:
        _build_dev()
        lib = ctypes.CDLL(_DEV_SO)
        u64, u32, i32, vp = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_void_p
        lib.synth_dev_fill_routed.argtypes = [u64, u32, u32, i32, i32, i32, i32, i32, vp, vp]
        lib.synth_dev_fill_routed.restype = i32
        _dev = lib
    return _dev


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


# --------------------------------------------------------------------------- host draws

def activations(seed: int, tokens: int, hidden: int, stream: int = 0) -> np.ndarray:
    """x ~ N(0, 1) fp32, [tokens][hidden]."""
    rng = np.random.default_rng([seed, 0xA11, stream])
    return rng.standard_normal((tokens, hidden), dtype=np.float32)


def router_weight(seed: int, layer: int, n_experts: int, hidden: int) -> np.ndarray:
    """W_r = f16(N(0, 0.02^2)), [n_experts][hidden] float16."""
    rng = np.random.default_rng([seed, 0x707, layer])
    return (rng.standard_normal((n_experts, hidden), dtype=np.float32) * np.float32(0.02)).astype(np.float16)


def token_ids(seed: int, tokens: int, vocab: int, stream: int = 0) -> np.ndarray:
    rng = np.random.default_rng([seed, 0x71D, stream])
    return rng.integers(0, vocab, size=tokens, dtype=np.int32)


def bias(seed: int, layer: int, n_experts: int, skew: bool) -> np.ndarray:
    out = np.empty(n_experts, dtype=np.float32)
    _hostlib().synth_fill_bias(seed, layer, n_experts, int(skew), out.ctypes.data)
    return out


def grid(seed: int, layer: int = 0) -> np.ndarray:
    out = np.empty((256, 8), dtype=np.uint8)
    _hostlib().synth_fill_grid(seed, layer, out.ctypes.data)
    return out


def tid2eid(seed: int, layer: int, vocab: int, n_experts: int, k: int) -> np.ndarray:
    out = np.empty((vocab, k), dtype=np.int32)
    _hostlib().synth_fill_tid2eid(seed, layer, vocab, n_experts, k, out.ctypes.data)
    return out


def routed(seed: int, layer: int, tensor: int, kind: int, e0: int, ne: int, rows: int, cols: int) -> np.ndarray:
    """Packed routed tensor for experts [e0, e0+ne): uint8 [ne][rows][row_bytes]."""
    rb = cols // BLOCK_ELEMS[kind] * BLOCK_BYTES[kind]
    out = np.empty((ne, rows, rb), dtype=np.uint8)
    _hostlib().synth_fill_routed(seed, layer, tensor, kind, e0, ne, rows, cols, out.ctypes.data, _threads())
    return out


def shared(seed: int, layer: int, tensor: int, rows: int, cols: int) -> np.ndarray:
    """Packed Q8_0 shared-expert tensor: uint8 [rows][row_bytes]."""
    return routed(seed, layer, tensor, KIND_Q80, 0, 1, rows, cols)[0]


def host_layer(seed: int, layer: int, s: LayerShape, experts=None, router: bool = True, q4k: bool = False) -> dict:
    """All inputs of one layer on the host.  ``experts`` limits the routed
    tensors to the listed expert ids (returned as dicts id -> array).  With
    ``q4k`` the routed gate, up and down tensors are Q4_K (the q2-q4 build's
    upgraded layers) and the dict names their formats."""
    ids = range(s.n_experts) if experts is None else sorted(set(int(e) for e in experts))
    out = {
        "grid": grid(seed, layer),
        "sh_gate": shared(seed, layer, T_SH_GATE, s.shared_inter, s.hidden),
        "sh_up": shared(seed, layer, T_SH_UP, s.shared_inter, s.hidden),
        "sh_down": shared(seed, layer, T_SH_DOWN, s.hidden, s.shared_inter),
    }
    if router:
        out["router_w"] = router_weight(seed, layer, s.n_experts, s.hidden)
        out["bias"] = bias(seed, layer, s.n_experts, s.skew)
    else:
        out["tid2eid"] = tid2eid(seed, layer, s.vocab, s.n_experts, s.top_k)
    kg, kd = (KIND_Q4K, KIND_Q4K) if q4k else (KIND_IQ2XXS, KIND_Q2K)
    out["gate_kind"], out["down_kind"] = kg, kd
    if experts is None:
        out["gate"] = routed(seed, layer, T_GATE, kg, 0, s.n_experts, s.inter, s.hidden)
        out["up"] = routed(seed, layer, T_UP, kg, 0, s.n_experts, s.inter, s.hidden)
        out["down"] = routed(seed, layer, T_DOWN, kd, 0, s.n_experts, s.hidden, s.inter)
    else:
        out["gate"] = {e: routed(seed, layer, T_GATE, kg, e, 1, s.inter, s.hidden)[0] for e in ids}
        out["up"] = {e: routed(seed, layer, T_UP, kg, e, 1, s.inter, s.hidden)[0] for e in ids}
        out["down"] = {e: routed(seed, layer, T_DOWN, kd, e, 1, s.hidden, s.inter)[0] for e in ids}
    return out


# --------------------------------------------------------------------------- device draws

def device_routed(out_tensor, seed: int, layer: int, tensor: int, kind: int, e0: int, ne: int, rows: int,
                  cols: int, stream_ptr: int = 0) -> None:
    """Fill a CUDA uint8 tensor in place (byte-identical to :func:`routed`)."""
    rc = _devlib().synth_dev_fill_routed(seed, layer, tensor, kind, e0, ne, rows, cols, out_tensor.data_ptr(),
                                         stream_ptr)
    if rc != 0:
        raise RuntimeError(f"synth_dev_fill_routed failed ({rc})")


def device_layer(seed: int, layer: int, s: LayerShape, router: bool = True, device="cuda", q4k: bool = False) -> dict:
    """All inputs of one layer as CUDA tensors (packed weights generated on
    the GPU); ``q4k`` as in :func:`host_layer`."""
    import torch

    stream = torch.cuda.current_stream().cuda_stream
    kg, kd = (KIND_Q4K, KIND_Q4K) if q4k else (KIND_IQ2XXS, KIND_Q2K)
    rb_g = s.row_bytes(kg, s.hidden)
    rb_d = s.row_bytes(kd, s.inter)
    out = {"gate_kind": kg, "down_kind": kd}
    out["gate"] = torch.empty((s.n_experts, s.inter, rb_g), dtype=torch.uint8, device=device)
    out["up"] = torch.empty((s.n_experts, s.inter, rb_g), dtype=torch.uint8, device=device)
    out["down"] = torch.empty((s.n_experts, s.hidden, rb_d), dtype=torch.uint8, device=device)
    device_routed(out["gate"], seed, layer, T_GATE, kg, 0, s.n_experts, s.inter, s.hidden, stream)
    device_routed(out["up"], seed, layer, T_UP, kg, 0, s.n_experts, s.inter, s.hidden, stream)
    device_routed(out["down"], seed, layer, T_DOWN, kd, 0, s.n_experts, s.hidden, s.inter, stream)
    for name, t, rows, cols in (("sh_gate", T_SH_GATE, s.shared_inter, s.hidden),
                                ("sh_up", T_SH_UP, s.shared_inter, s.hidden),
                                ("sh_down", T_SH_DOWN, s.hidden, s.shared_inter)):
        out[name] = torch.empty((rows, s.row_bytes(KIND_Q80, cols)), dtype=torch.uint8, device=device)
        device_routed(out[name], seed, layer, t, KIND_Q80, 0, 1, rows, cols, stream)
    out["grid"] = torch.from_numpy(grid(seed, layer)).to(device)
    if router:
        out["router_w"] = torch.from_numpy(router_weight(seed, layer, s.n_experts, s.hidden)).to(device)
        out["bias"] = torch.from_numpy(bias(seed, layer, s.n_experts, s.skew)).to(device)
    else:
        out["tid2eid"] = torch.from_numpy(tid2eid(seed, layer, s.vocab, s.n_experts, s.top_k)).to(device)
    return out
