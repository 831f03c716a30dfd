"""Python binding of the MoE FFN layer's C ABI (include/moe.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels
of ``libmoe_b200.so``.  PyTorch supplies device memory and streams.  There is
no CPU fallback: importing this module without the built library raises.

The functions keep the C names (``moe_workspace_size``, ``moe_init``,
``moe_route``, ``moe_ffn_forward``, ``moe_poll_device_error``,
``moe_last_error``, ``moe_destroy``); :class:`Layer` bundles a handle with
its persistent buffer and a scratch buffer.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_MISALIGNED = -3
MOE_ERR_WORKSPACE_TOO_SMALL = -4
MOE_ERR_CUDA = -5
MOE_ERR_TIMEOUT = -6
MOE_ERR_DEVICE_FAULT = -7
MOE_ROUTE_ROUTER = 0
MOE_ROUTE_HASH = 1
MOE_FLAG_PRENORM_RESIDUAL = 1
MOE_FLAG_EXPERTS_ONLY = 2
MOE_FLAG_NO_ROUTED = 4
MOE_FLAG_DETERMINISTIC = 8
MOE_SMALL_T_MAX = 32  # calls with T <= this run the small-token kernels
MOE_CHUNKED_T_MAX = 64  # q2 layers up to this T: the small-token kernels on 32 tokens, then the rest
MOE_QUANT_Q8_0 = 0
MOE_QUANT_Q2_K = 1
MOE_QUANT_Q4_K = 2
_QUANT_BLOCK = {MOE_QUANT_Q8_0: (32, 34), MOE_QUANT_Q2_K: (256, 84), MOE_QUANT_Q4_K: (256, 144)}
MOE_ROUTED_Q2 = 0
MOE_ROUTED_Q4K = 1

EXPORTED = ("moe_workspace_size", "moe_init", "moe_route", "moe_ffn_forward", "moe_poll_device_error",
            "moe_last_error", "moe_set_timing_events", "moe_set_next_layer", "moe_set_wait_limit", "moe_ffn_forward_noalloc", "moe_quantize",
            "moe_ep_workspace_size", "moe_ep_dispatch", "moe_ep_experts", "moe_ep_combine", "moe_destroy")


class moe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("shared_inter", ctypes.c_int), ("vocab", ctypes.c_int),
                ("routed_scaling", ctypes.c_float), ("rms_eps", ctypes.c_float), ("mode", ctypes.c_int),
                ("flags", ctypes.c_int), ("routed_format", ctypes.c_int)]


class moe_weights(ctypes.Structure):
    _fields_ = [("router_w_f16", ctypes.c_void_p), ("router_bias", ctypes.c_void_p), ("tid2eid", ctypes.c_void_p),
                ("gate_iq2xxs", ctypes.c_void_p), ("up_iq2xxs", ctypes.c_void_p), ("down_q2k", ctypes.c_void_p),
                ("sh_gate_q80", ctypes.c_void_p), ("sh_up_q80", ctypes.c_void_p), ("sh_down_q80", ctypes.c_void_p),
                ("iq2_grid", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"moe status {status}: {message}")
        self.status = status


_lib = None


def lib():
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with python -m bit_moe_expert_sqrtsoftplus_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.moe_workspace_size.argtypes = [ctypes.POINTER(moe_config), i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.moe_init.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights), vp, sz, vp,
                               ctypes.POINTER(vp)]
        L.moe_route.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.moe_ffn_forward.argtypes = [vp, vp, vp, i32, vp, vp, sz, vp]
        L.moe_ffn_forward_noalloc.argtypes = [vp, vp, vp, i32, vp, vp]
        L.moe_ffn_forward_noalloc.restype = i32
        L.moe_poll_device_error.argtypes = [vp, vp]
        L.moe_last_error.restype = ctypes.c_char_p
        L.moe_set_timing_events.argtypes = [vp, vp, vp]
        L.moe_set_timing_events.restype = i32
        L.moe_set_next_layer.argtypes = [vp, vp]
        L.moe_set_next_layer.restype = i32
        L.moe_set_wait_limit.argtypes = [vp, ctypes.c_longlong]
        L.moe_set_wait_limit.restype = i32
        L.moe_quantize.argtypes = [i32, vp, ctypes.c_int64, vp, vp, vp]
        L.moe_quantize.restype = i32
        L.moe_ep_workspace_size.argtypes = [ctypes.POINTER(moe_config), i32, i32, ctypes.POINTER(sz),
                                            ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.moe_ep_dispatch.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_ep_experts.argtypes = [vp, vp, vp, vp, i32, i32, vp, vp, sz, vp]
        L.moe_ep_combine.argtypes = [vp, vp, i32, vp, vp, vp, vp, sz, vp]
        for name in ("moe_ep_workspace_size", "moe_ep_dispatch", "moe_ep_experts", "moe_ep_combine"):
            getattr(L, name).restype = i32
        L.moe_destroy.argtypes = [vp]
        L.moe_destroy.restype = None
        for name in ("moe_workspace_size", "moe_init", "moe_route", "moe_ffn_forward", "moe_poll_device_error"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def moe_last_error() -> str:
    return lib().moe_last_error().decode()


def _check(status: int):
    if status != MOE_OK:
        raise MoeError(status, moe_last_error())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def make_config(hidden, inter, n_experts, top_k, shared_inter, vocab=0, routed_scaling=1.5, rms_eps=1e-6,
                mode=MOE_ROUTE_ROUTER, flags=0, routed_format=MOE_ROUTED_Q2) -> moe_config:
    return moe_config(hidden, inter, n_experts, top_k, shared_inter, vocab, routed_scaling, rms_eps, mode, flags,
                      routed_format)


def moe_workspace_size(cfg: moe_config, max_tokens: int):
    p, s = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(cfg), max_tokens, ctypes.byref(p), ctypes.byref(s)))
    return p.value, s.value


def make_weights(w: dict) -> moe_weights:
    return moe_weights(_ptr(w.get("router_w")), _ptr(w.get("bias")), _ptr(w.get("tid2eid")), _ptr(w["gate"]),
                       _ptr(w["up"]), _ptr(w["down"]), _ptr(w["sh_gate"]), _ptr(w["sh_up"]), _ptr(w["sh_down"]),
                       _ptr(w.get("grid")))


def moe_init(cfg: moe_config, weights: moe_weights, persist, stream=None) -> int:
    h = ctypes.c_void_p(None)
    _check(lib().moe_init(ctypes.byref(cfg), ctypes.byref(weights), _ptr(persist),
                          persist.numel() * persist.element_size(), _stream(stream), ctypes.byref(h)))
    return h.value


def moe_route(handle, x, token_ids, T, idx, w, expert_offsets=None, perm=None, scratch=None, stream=None):
    _check(lib().moe_route(handle, _ptr(x), _ptr(token_ids), T, _ptr(idx), _ptr(w), _ptr(expert_offsets), _ptr(perm),
                           _ptr(scratch), 0 if scratch is None else scratch.numel() * scratch.element_size(),
                           _stream(stream)))


def moe_ffn_forward(handle, x, token_ids, T, y, scratch, stream=None):
    _check(lib().moe_ffn_forward(handle, _ptr(x), _ptr(token_ids), T, _ptr(y), _ptr(scratch),
                                 0 if scratch is None else scratch.numel() * scratch.element_size(), _stream(stream)))


def moe_ffn_forward_noalloc(handle, x, token_ids, T, y, stream=None):
    """Forward without a scratch buffer (small T only; see include/moe.h)."""
    _check(lib().moe_ffn_forward_noalloc(handle, _ptr(x), _ptr(token_ids), T, _ptr(y), _stream(stream)))


def moe_poll_device_error(handle, stream=None):
    _check(lib().moe_poll_device_error(handle, _stream(stream)))


def moe_set_timing_events(handle, ev_begin=None, ev_end=None):
    """ev_begin / ev_end: torch.cuda.Event objects (or None to stop)."""
    _check(lib().moe_set_timing_events(handle, None if ev_begin is None else ev_begin.cuda_event,
                                       None if ev_end is None else ev_end.cuda_event))


def moe_set_next_layer(handle, next_handle):
    """Stacked layers: forwards on `handle` prefetch into L2 the weights the
    next layer reads first (None clears)."""
    _check(lib().moe_set_next_layer(handle, next_handle))


def moe_set_wait_limit(handle, cycles: int):
    """Test hook: bound of the device waits on other warps' results, in SM
    clock cycles (0 restores the default of about 2 s)."""
    _check(lib().moe_set_wait_limit(handle, int(cycles)))


def moe_quantize(fmt, x, out, nonfinite=None, stream=None):
    """Encode the fp32 CUDA tensor x (numel a multiple of the block size) into
    the uint8 CUDA tensor out (numel/32 * 34, numel/256 * 84 or numel/256 *
    144 bytes)."""
    per, nbytes = _QUANT_BLOCK.get(fmt, (32, 34))
    if out.numel() * out.element_size() < x.numel() // per * nbytes:
        raise MoeError(MOE_ERR_WORKSPACE_TOO_SMALL, "out is too small for the encoded blocks")
    _check(lib().moe_quantize(fmt, _ptr(x), x.numel(), _ptr(out), _ptr(nonfinite), _stream(stream)))


def quantize(fmt, x, stream=None):
    """Encoded blocks of x as a uint8 CUDA tensor [n_blocks][block_bytes] and a
    device int32 count of blocks that held a non-finite value."""
    import torch
    per, nbytes = _QUANT_BLOCK.get(fmt, (32, 34))
    x = x.contiguous()
    out = torch.empty((x.numel() // per, nbytes), dtype=torch.uint8, device=x.device)
    bad = torch.zeros(1, dtype=torch.int32, device=x.device)
    moe_quantize(fmt, x, out, bad, stream)
    return out, bad


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def moe_ep_workspace_size(cfg: moe_config, max_tokens: int, max_recv_rows: int):
    a, b, c = ctypes.c_size_t(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib().moe_ep_workspace_size(ctypes.byref(cfg), max_tokens, max_recv_rows, ctypes.byref(a),
                                       ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def moe_ep_dispatch(handle, x, token_ids, T, offsets, perm, x_send, e_send, w_send, scratch, stream=None):
    _check(lib().moe_ep_dispatch(handle, _ptr(x), _ptr(token_ids), T, _ptr(offsets), _ptr(perm), _ptr(x_send),
                                 _ptr(e_send), _ptr(w_send), _ptr(scratch), _nbytes(scratch), _stream(stream)))


def moe_ep_experts(handle, x_recv, e_recv, w_recv, N, first_expert, out, scratch, stream=None):
    _check(lib().moe_ep_experts(handle, _ptr(x_recv), _ptr(e_recv), _ptr(w_recv), N, first_expert, _ptr(out),
                                _ptr(scratch), _nbytes(scratch), _stream(stream)))


def moe_ep_combine(handle, x, T, perm, out_back, y, scratch, stream=None):
    _check(lib().moe_ep_combine(handle, _ptr(x), T, _ptr(perm), _ptr(out_back), _ptr(y), _ptr(scratch),
                                _nbytes(scratch), _stream(stream)))


def moe_destroy(handle):
    if handle:
        lib().moe_destroy(handle)


class Stack:
    """Layers applied in order to the same tokens, each as x <- x +
    MoE_l(RMSNorm(x)) in place (every layer's config must carry
    MOE_FLAG_PRENORM_RESIDUAL).  Each layer prefetches the next one's router
    and shared-expert gate/up weights into L2 (moe_set_next_layer).  With
    ``graph=True`` the first forward captures the whole pass into a CUDA
    graph on a side stream and later forwards replay it (the input and
    token-id buffers are then fixed: forward copies into them)."""

    def __init__(self, layers, graph: bool = False):
        self.layers = list(layers)
        for L in self.layers:
            if not (L.cfg.flags & MOE_FLAG_PRENORM_RESIDUAL):
                raise MoeError(MOE_ERR_INVALID_ARG, "stacked layers need MOE_FLAG_PRENORM_RESIDUAL")
        for a, b in zip(self.layers, self.layers[1:]):
            moe_set_next_layer(a.handle, b.handle)
        self.graph = graph
        self._g = None

    def _run(self, x, token_ids):
        for L in self.layers:
            L.forward(x, token_ids, y=x)

    def forward(self, x, token_ids=None):
        """x [T][H] fp32 CUDA tensor, updated in place and returned."""
        import torch
        if not self.graph:
            self._run(x, token_ids)
            return x
        if self._g is None:
            self._x = x.clone()
            self._tok = None if token_ids is None else token_ids.clone()
            self._run(self._x, self._tok)  # first pass outside capture (lazy set-up)
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            self._g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                with torch.cuda.graph(self._g, stream=s):
                    self._run(self._x, self._tok)
            torch.cuda.current_stream().wait_stream(s)
        self._x.copy_(x)
        if self._tok is not None:
            self._tok.copy_(token_ids)
        self._g.replay()
        x.copy_(self._x)
        return x

    def close(self):
        self._g = None
        for L in self.layers:
            if L.handle:
                moe_set_next_layer(L.handle, None)


class Layer:
    """One layer: a handle, its persistent buffer and a scratch buffer sized
    for ``max_tokens``.  ``weights`` holds CUDA tensors keyed like
    ``synth.device_layer`` (router_w, bias | tid2eid, gate, up, down,
    sh_gate, sh_up, sh_down, grid); they must outlive the layer."""

    def __init__(self, cfg: moe_config, weights: dict, max_tokens: int, device="cuda", stream=None, scratch=None):
        import torch
        self.cfg = cfg
        self.weights = weights
        pbytes, sbytes = moe_workspace_size(cfg, max_tokens)
        self.persist = torch.zeros(max(pbytes, 16), dtype=torch.uint8, device=device)
        if scratch is not None and _nbytes(scratch) < sbytes:
            raise MoeError(MOE_ERR_WORKSPACE_TOO_SMALL,
                           f"shared scratch has {_nbytes(scratch)} bytes, this layer needs {sbytes}")
        self.scratch = scratch if scratch is not None else torch.empty(max(sbytes, 16), dtype=torch.uint8,
                                                                       device=device)
        self.scratch_bytes = sbytes
        self._w = make_weights(weights)
        self.handle = moe_init(cfg, self._w, self.persist, stream)

    def forward(self, x, token_ids=None, y=None, stream=None):
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        moe_ffn_forward(self.handle, x, token_ids, T, y, self.scratch, stream)
        return y

    def route(self, x, token_ids=None, with_perm=False, stream=None):
        import torch
        T = x.shape[0]
        k, E = self.cfg.top_k, self.cfg.n_experts
        idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, k), dtype=torch.float32, device=x.device)
        off = torch.empty(E + 1, dtype=torch.int32, device=x.device) if with_perm else None
        perm = torch.empty(T * k, dtype=torch.int32, device=x.device) if with_perm else None
        moe_route(self.handle, x, token_ids, T, idx, w, off, perm, self.scratch, stream)
        return (idx, w, off, perm) if with_perm else (idx, w)

    def poll(self, stream=None):
        moe_poll_device_error(self.handle, stream)

    def close(self):
        if getattr(self, "handle", None):
            moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
