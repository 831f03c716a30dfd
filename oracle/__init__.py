"""Plain fp64 CPU oracle for the MoE FFN layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never reaches it: the
CUDA layer in ``bit_moe_expert_sqrtsoftplus_b200`` has no CPU fallback and
shares no code with this C oracle (``oracle.c``), which this module loads
through ctypes.  Sources and readings are documented in ``oracle.h`` and
``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_oracle.so")
_lib = None

KIND_IQ2XXS, KIND_Q2K, KIND_Q80, KIND_Q4K = 0, 1, 2, 3
_BB = {0: 66, 1: 84, 2: 34, 3: 144}
_BE = {0: 256, 1: 256, 2: 32, 3: 256}


def build() -> None:
    srcs = [os.path.join(_HERE, f) for f in ("oracle.c", "oracle.h")]
    if os.path.exists(_SO) and os.path.getmtime(_SO) >= max(os.path.getmtime(s) for s in srcs):
        return
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                           "-o", _SO, srcs[0], "-lm", "-pthread"])


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        d, i32, vp = ctypes.c_double, ctypes.c_int, ctypes.c_void_p
        L.oracle_f16.argtypes = [ctypes.c_uint16]
        L.oracle_f16.restype = d
        for name in ("oracle_iq2xxs_elem",):
            getattr(L, name).argtypes = [vp, vp, i32]
            getattr(L, name).restype = d
        for name in ("oracle_q2k_elem", "oracle_q80_elem", "oracle_q4k_elem"):
            getattr(L, name).argtypes = [vp, i32]
            getattr(L, name).restype = d
        L.oracle_row_iq2xxs.argtypes = [vp, i32, vp, vp]
        L.oracle_row_q2k.argtypes = [vp, i32, vp]
        L.oracle_row_q80.argtypes = [vp, i32, vp]
        L.oracle_row_q4k.argtypes = [vp, i32, vp]
        L.oracle_matvec.argtypes = [i32, vp, i32, i32, vp, vp, vp]
        L.oracle_decode_matrix.argtypes = [i32, vp, i32, i32, vp, vp]
        L.oracle_sqrtsoftplus.argtypes = [d]
        L.oracle_sqrtsoftplus.restype = d
        L.oracle_silu.argtypes = [d]
        L.oracle_silu.restype = d
        L.oracle_router_logits.argtypes = [vp, i32, i32, vp, i32, vp]
        L.oracle_select.argtypes = [vp, vp, i32, i32, i32, d, vp, vp, vp]
        L.oracle_hash_select.argtypes = [vp, i32, vp, i32, i32, i32, d, vp, vp]
        L.oracle_hash_select.restype = i32
        L.oracle_swiglu_expert.argtypes = [i32, i32, vp, vp, vp, i32, i32, vp, vp, vp]
        L.oracle_layer.argtypes = [vp, vp, i32, vp, vp, vp]
        L.oracle_layer.restype = i32
        L.oracle_layer_mt.argtypes = [vp, vp, i32, vp, vp, vp, i32]
        L.oracle_layer_mt.restype = i32
        L.oracle_permutation.argtypes = [vp, i32, i32, i32, vp, vp]
        L.oracle_rmsnorm.argtypes = [vp, i32, d, vp]
        L.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_f16.restype = ctypes.c_uint16
        for name in ("oracle_quantize_q80", "oracle_quantize_q2k", "oracle_quantize_q4k"):
            getattr(L, name).argtypes = [vp, i32, vp]
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


# ------------------------------------------------------------------ decoders

def f16(bits: int) -> float:
    return lib().oracle_f16(int(bits) & 0xFFFF)


def iq2xxs_elem(block: np.ndarray, grid: np.ndarray, e: int) -> float:
    b, pb = _c(block, np.uint8)
    g, pg = _c(grid, np.uint8)
    return lib().oracle_iq2xxs_elem(pb, pg, int(e))


def q2k_elem(block: np.ndarray, e: int) -> float:
    b, pb = _c(block, np.uint8)
    return lib().oracle_q2k_elem(pb, int(e))


def q80_elem(block: np.ndarray, e: int) -> float:
    b, pb = _c(block, np.uint8)
    return lib().oracle_q80_elem(pb, int(e))


def q4k_elem(block: np.ndarray, e: int) -> float:
    b, pb = _c(block, np.uint8)
    return lib().oracle_q4k_elem(pb, int(e))


def decode_row(kind: int, row: np.ndarray, cols: int, grid: np.ndarray | None = None) -> np.ndarray:
    r, pr = _c(row, np.uint8)
    out = np.empty(cols, dtype=np.float64)
    if kind == KIND_IQ2XXS:
        g, pg = _c(grid, np.uint8)
        lib().oracle_row_iq2xxs(pr, cols, pg, out.ctypes.data)
    elif kind == KIND_Q2K:
        lib().oracle_row_q2k(pr, cols, out.ctypes.data)
    elif kind == KIND_Q4K:
        lib().oracle_row_q4k(pr, cols, out.ctypes.data)
    else:
        lib().oracle_row_q80(pr, cols, out.ctypes.data)
    return out


def decode_matrix(kind: int, W: np.ndarray, rows: int, cols: int, grid=None) -> np.ndarray:
    """All rows of a packed [rows][cols] matrix decoded to fp64 by the scalar C
    decoders (one call; the GIL is released while it runs)."""
    w, pw = _c(np.asarray(W).reshape(rows, -1), np.uint8)
    g, pg = (None, None) if grid is None else _c(grid, np.uint8)
    out = np.empty((rows, cols), dtype=np.float64)
    lib().oracle_decode_matrix(kind, pw, rows, cols, pg, out.ctypes.data)
    return out


def matvec(kind: int, W: np.ndarray, rows: int, cols: int, x: np.ndarray, grid=None) -> np.ndarray:
    w, pw = _c(W, np.uint8)
    xx, px = _c(x, np.float64)
    g, pg = (None, None) if grid is None else _c(grid, np.uint8)
    y = np.empty(rows, dtype=np.float64)
    lib().oracle_matvec(kind, pw, rows, cols, pg, px, y.ctypes.data)
    return y


# -------------------------------------------------------------------- router

def sqrtsoftplus(z: float) -> float:
    return lib().oracle_sqrtsoftplus(float(z))


def silu(u: float) -> float:
    return lib().oracle_silu(float(u))


def router_logits(x: np.ndarray, Wr: np.ndarray) -> np.ndarray:
    """z = W_r x in fp64 (fp32 inputs convert exactly)."""
    xx, px = _c(x, np.float64)
    T, H = xx.shape
    E = Wr.shape[0]
    w, pw = _c(np.asarray(Wr).view(np.uint16) if np.asarray(Wr).dtype == np.float16 else Wr, np.uint16)
    z = np.empty((T, E), dtype=np.float64)
    lib().oracle_router_logits(px, T, H, pw, E, z.ctypes.data)
    return z


def select(z: np.ndarray, bias: np.ndarray, k: int, scaling: float = 1.5):
    zz, pz = _c(z, np.float64)
    T, E = zz.shape
    b, pb = _c(bias, np.float32)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    margin = np.empty(T, dtype=np.float64)
    lib().oracle_select(pz, pb, T, E, k, float(scaling), idx.ctypes.data, w.ctypes.data, margin.ctypes.data)
    return idx, w, margin


def route(x: np.ndarray, Wr: np.ndarray, bias: np.ndarray, k: int, scaling: float = 1.5):
    """Returns (idx [T][k] ascending ids, w [T][k], margin [T] = key_k - key_{k+1})."""
    return select(router_logits(x, Wr), bias, k, scaling)


def hash_route(token_ids: np.ndarray, tid2eid: np.ndarray, k: int, scaling: float = 1.5, n_experts: int = 256):
    """Hash routing through the table; raises ValueError for a token id outside
    the table or a used table row that does not hold k distinct ids in
    [0, n_experts)."""
    t, pt = _c(token_ids, np.int32)
    tab, ptab = _c(tid2eid, np.int32)
    T = t.shape[0]
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    rc = lib().oracle_hash_select(pt, T, ptab, tab.shape[0], int(n_experts), k, float(scaling), idx.ctypes.data,
                                  w.ctypes.data)
    if rc == -1:
        raise ValueError("hash routing: token id outside the table")
    if rc != 0:
        raise ValueError("hash routing: a table row does not hold distinct expert ids in range")
    return idx, w


# --------------------------------------------------------------------- layer

class _LayerW(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("shared_inter", ctypes.c_int),
                ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("gate", ctypes.POINTER(ctypes.c_void_p)), ("up", ctypes.POINTER(ctypes.c_void_p)),
                ("down", ctypes.POINTER(ctypes.c_void_p)), ("sh_gate", ctypes.c_void_p),
                ("sh_up", ctypes.c_void_p), ("sh_down", ctypes.c_void_p), ("grid", ctypes.c_void_p),
                ("gate_kind", ctypes.c_int), ("down_kind", ctypes.c_int)]


def _expert_ptrs(src, E, keep):
    arr = (ctypes.c_void_p * E)()
    for e in range(E):
        if isinstance(src, dict):
            a = src.get(e)
        else:
            a = src[e]
        if a is None:
            arr[e] = None
        else:
            a = np.ascontiguousarray(a, dtype=np.uint8)
            keep.append(a)
            arr[e] = a.ctypes.data
    return arr


def swiglu_expert(gate, up, down, hidden, inter, x, grid=None, gate_kind=KIND_IQ2XXS, down_kind=KIND_Q2K):
    keep = []
    ptr = []
    for a in (gate, up, down):
        a = np.ascontiguousarray(a, dtype=np.uint8)
        keep.append(a)
        ptr.append(a.ctypes.data)
    xx, px = _c(x, np.float64)
    g, pg = (None, None) if grid is None else _c(grid, np.uint8)
    out = np.empty(hidden, dtype=np.float64)
    lib().oracle_swiglu_expert(gate_kind, down_kind, ptr[0], ptr[1], ptr[2], hidden, inter, pg, px,
                               out.ctypes.data)
    return out


def layer(weights: dict, shape, x: np.ndarray, idx: np.ndarray, w: np.ndarray, threads: int = 1) -> np.ndarray:
    """y [T][H] fp64 for the given routing.  ``weights`` as returned by
    ``synth.host_layer`` (routed tensors as full arrays or dicts by id;
    optional "gate_kind" / "down_kind" name the routed formats, IQ2_XXS and
    Q2_K when absent)."""
    keep = []
    E = shape.n_experts
    lw = _LayerW()
    lw.hidden, lw.inter, lw.shared_inter, lw.n_experts, lw.top_k = (shape.hidden, shape.inter,
                                                                     shape.shared_inter, E, shape.top_k)
    garr = _expert_ptrs(weights["gate"], E, keep)
    uarr = _expert_ptrs(weights["up"], E, keep)
    darr = _expert_ptrs(weights["down"], E, keep)
    lw.gate = ctypes.cast(garr, ctypes.POINTER(ctypes.c_void_p))
    lw.up = ctypes.cast(uarr, ctypes.POINTER(ctypes.c_void_p))
    lw.down = ctypes.cast(darr, ctypes.POINTER(ctypes.c_void_p))
    # routed formats: the q2 build by default, Q4_K for the q2-q4 layers
    lw.gate_kind = int(weights.get("gate_kind", KIND_IQ2XXS))
    lw.down_kind = int(weights.get("down_kind", KIND_Q2K))
    for name in ("sh_gate", "sh_up", "sh_down", "grid"):
        a = np.ascontiguousarray(weights[name], dtype=np.uint8)
        keep.append(a)
        setattr(lw, name, a.ctypes.data)
    xx, px = _c(x, np.float64)
    T = xx.shape[0]
    ii, pi = _c(idx, np.int32)
    ww, pw = _c(w, np.float64)
    y = np.zeros((T, shape.hidden), dtype=np.float64)
    if threads > 1:
        rc = lib().oracle_layer_mt(ctypes.byref(lw), px, T, pi, pw, y.ctypes.data, int(threads))
    else:
        rc = lib().oracle_layer(ctypes.byref(lw), px, T, pi, pw, y.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_layer: a selected expert has no weights")
    return y


def layer_dense(weights: dict, shape, x: np.ndarray, idx: np.ndarray, w: np.ndarray, threads: int = 0) -> np.ndarray:
    """The same layer as :func:`layer`, computed as dequantise-then-multiply:
    every matrix a call uses is decoded once to fp64 by the scalar C decoders
    (``decode_matrix``) and the products are numpy fp64 matrix products, the
    textbook reduction of the fused route.  y = shared(x) + the selected
    experts' weighted outputs added in ascending expert id, as in ``layer``;
    results agree with ``layer`` up to the order of the fp64 additions inside
    each dot product.  Meant for checking many tokens of a full-size call,
    where the row-by-row route is too slow.  ``threads`` decodes that many
    experts at once (0: the host's cores)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    H, I, Is, E = shape.hidden, shape.inter, shape.shared_inter, shape.n_experts
    gk = int(weights.get("gate_kind", KIND_IQ2XXS))
    dk = int(weights.get("down_kind", KIND_Q2K))
    grid = weights["grid"]
    x = np.ascontiguousarray(x, dtype=np.float64)
    idx = np.asarray(idx)
    w = np.asarray(w, dtype=np.float64)

    def silu(u):
        return u / (1.0 + np.exp(-u))

    def expert_of(src, e):
        a = src.get(e) if isinstance(src, dict) else src[e]
        if a is None:
            raise ValueError("layer_dense: a selected expert has no weights")
        return a

    def run_expert(e):
        rows_t, slots = np.nonzero(idx == e)
        Wg = decode_matrix(gk, expert_of(weights["gate"], e), I, H, grid)
        Wu = decode_matrix(gk, expert_of(weights["up"], e), I, H, grid)
        Wd = decode_matrix(dk, expert_of(weights["down"], e), H, I, grid)
        xe = x[rows_t]
        h = silu(xe @ Wg.T) * (xe @ Wu.T)
        return rows_t, slots, h @ Wd.T

    Wsg = decode_matrix(KIND_Q80, weights["sh_gate"], Is, H)
    Wsu = decode_matrix(KIND_Q80, weights["sh_up"], Is, H)
    Wsd = decode_matrix(KIND_Q80, weights["sh_down"], H, Is)
    y = (silu(x @ Wsg.T) * (x @ Wsu.T)) @ Wsd.T
    experts = [int(e) for e in np.unique(idx)]
    n = threads if threads > 0 else max(1, min(8, os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=n) as pool:
        # results are added in ascending expert id, whatever order they finish in
        for rows_t, slots, o in pool.map(run_expert, experts):
            y[rows_t] += w[rows_t, slots][:, None] * o
    return y


def permutation(idx: np.ndarray, n_experts: int):
    ii, pi = _c(idx, np.int32)
    T, k = ii.shape
    offsets = np.empty(n_experts + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    lib().oracle_permutation(pi, T, k, n_experts, offsets.ctypes.data, perm.ctypes.data)
    return offsets, perm


def rmsnorm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    xx = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(xx)
    for t in range(xx.shape[0]):
        lib().oracle_rmsnorm(xx[t].ctypes.data, xx.shape[1], float(eps), out[t].ctypes.data)
    return out


# -------------------------------------------------------------------- encoders

def f32_to_f16(f: float) -> int:
    """Bits of the nearest binary16 (ties to even) of the binary32 value f."""
    return int(lib().oracle_f32_to_f16(float(np.float32(f))))


def quantize(kind: int, x: np.ndarray) -> np.ndarray:
    """Encode fp32 values (a multiple of the block size) into Q8_0, Q2_K or
    Q4_K blocks: uint8 [n_blocks][block_bytes].  Raises on non-finite input."""
    if kind not in (KIND_Q80, KIND_Q2K, KIND_Q4K):
        raise ValueError("only the Q8_0, Q2_K and Q4_K encoders exist")
    xx, px = _c(np.asarray(x, dtype=np.float32).ravel(), np.float32)
    n = xx.size
    if n % _BE[kind]:
        raise ValueError(f"{n} values is not a multiple of {_BE[kind]}")
    out = np.zeros((n // _BE[kind], _BB[kind]), dtype=np.uint8)
    fn = {KIND_Q80: lib().oracle_quantize_q80, KIND_Q2K: lib().oracle_quantize_q2k,
          KIND_Q4K: lib().oracle_quantize_q4k}[kind]
    rc = fn(px, n, out.ctypes.data)
    if rc != 0:
        raise ValueError("non-finite input" if rc == -1 else f"encoder error {rc}")
    return out
