"""The C-ABI library: it builds, loads without a GPU, exports every function
declared in include/moe.h, and rejects bad arguments before touching the
device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def moe():
    from bit_moe_expert_sqrtsoftplus_b200 import build
    build.build()
    import bit_moe_expert_sqrtsoftplus_b200 as m
    return m


def test_exports_every_declared_function(moe):
    declared = _declared()
    assert {"moe_workspace_size", "moe_init", "moe_route", "moe_ffn_forward", "moe_poll_device_error",
            "moe_last_error", "moe_destroy"} <= set(declared)
    lib = ctypes.CDLL(moe.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def test_binding_constants_match_the_header(moe):
    src = ""
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src += open(os.path.join(ROOT, "include", h)).read()
    values = {n: int(v) for n, v in re.findall(r"#define\s+(MOE_[A-Z0-9_]+)\s+(-?\d+)", src)}
    values.update({n: int(v) for n, v in re.findall(r"\b(MOE_[A-Z0-9_]+)\s*=\s*(-?\d+)", src)})
    assert {"MOE_OK", "MOE_ERR_TIMEOUT", "MOE_ROUTE_HASH", "MOE_FLAG_PRENORM_RESIDUAL", "MOE_SMALL_T_MAX"} <= set(values)
    for name, v in values.items():
        assert getattr(moe, name) == v, name


def test_the_abi_from_plain_c(moe, tmp_path):
    """A C program (tests/c_abi_check.c) includes include/moe.h, links the
    library and runs its host-side checks: the boundary needs no Python."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    exe = tmp_path / "c_abi_check"
    lib_dir = os.path.dirname(moe.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe), "-L", lib_dir, "-lmoe_b200",
                    f"-Wl,-rpath,{lib_dir}"], check=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert p.returncode == 0, p.stdout + p.stderr
    assert "C ABI checks passed" in p.stdout


def _cfg(moe, **over):
    base = dict(hidden=4096, inter=2048, n_experts=256, top_k=6, shared_inter=2048, vocab=129280)
    base.update(over)
    return moe.make_config(**base)


def test_workspace_size_and_shape_checks(moe):
    p, s = moe.moe_workspace_size(_cfg(moe), 1)
    assert p >= 4 and s > 0
    _, s32 = moe.moe_workspace_size(_cfg(moe), 4096)
    assert s32 > s
    for bad, status in ((dict(hidden=4000), moe.MOE_ERR_UNSUPPORTED_SHAPE),
                        (dict(inter=100), moe.MOE_ERR_UNSUPPORTED_SHAPE),
                        (dict(shared_inter=96), moe.MOE_ERR_UNSUPPORTED_SHAPE),
                        (dict(top_k=0), moe.MOE_ERR_UNSUPPORTED_SHAPE),
                        (dict(top_k=9), moe.MOE_ERR_UNSUPPORTED_SHAPE),
                        (dict(n_experts=300), moe.MOE_ERR_UNSUPPORTED_SHAPE),
                        (dict(n_experts=4, top_k=6), moe.MOE_ERR_UNSUPPORTED_SHAPE),
                        (dict(mode=7), moe.MOE_ERR_INVALID_ARG),
                        (dict(mode=1, vocab=0), moe.MOE_ERR_INVALID_ARG),
                        (dict(flags=16), moe.MOE_ERR_INVALID_ARG),
                        (dict(flags=6), moe.MOE_ERR_INVALID_ARG),
                        (dict(routed_format=5), moe.MOE_ERR_INVALID_ARG)):
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_workspace_size(_cfg(moe, **bad), 1)
        assert ei.value.status == status, bad
        assert moe.moe_last_error()


def test_scratch_size_never_shrinks_with_more_tokens(moe):
    """A scratch buffer sized for max_tokens serves every call with fewer
    tokens, so the size must not decrease as max_tokens grows (the small-T
    layout changes with the unit width, the large-T one starts above 32)."""
    for shape in (dict(), dict(hidden=256, inter=256, n_experts=16, top_k=2, shared_inter=256),
                  dict(routed_format=moe.MOE_ROUTED_Q4K)):
        prev = 0
        for T in list(range(1, 70)) + [128, 4096]:
            _, s = moe.moe_workspace_size(_cfg(moe, **shape), T)
            assert s >= prev, (shape, T, s, prev)
            prev = s


def test_q4k_layers_take_more_scratch_up_to_32_tokens(moe):
    """The Q4_K forward keeps its expert buffers beside the routing scratch."""
    for T in (1, 8, 32):
        _, q2 = moe.moe_workspace_size(_cfg(moe), T)
        _, q4 = moe.moe_workspace_size(_cfg(moe, routed_format=moe.MOE_ROUTED_Q4K), T)
        assert q4 >= q2 + 4 * T * (4096 + 6 * 2048 + 2048)


def test_quantize_argument_checks(moe):
    """moe_quantize rejects bad arguments before it touches a device."""
    L = moe.lib()
    ok = 0x20000000
    cases = [((7, ok, 256, ok), moe.MOE_ERR_INVALID_ARG),
             ((moe.MOE_QUANT_Q2_K, ok, -256, ok), moe.MOE_ERR_INVALID_ARG),
             ((moe.MOE_QUANT_Q2_K, ok, 300, ok), moe.MOE_ERR_UNSUPPORTED_SHAPE),
             ((moe.MOE_QUANT_Q8_0, ok, 48, ok), moe.MOE_ERR_UNSUPPORTED_SHAPE),
             ((moe.MOE_QUANT_Q4_K, ok, 512 + 32, ok), moe.MOE_ERR_UNSUPPORTED_SHAPE),
             ((moe.MOE_QUANT_Q8_0, None, 64, ok), moe.MOE_ERR_INVALID_ARG),
             ((moe.MOE_QUANT_Q2_K, ok, 256, None), moe.MOE_ERR_INVALID_ARG),
             ((moe.MOE_QUANT_Q2_K, ok + 4, 256, ok), moe.MOE_ERR_MISALIGNED),
             ((moe.MOE_QUANT_Q8_0, ok, 32, ok + 2), moe.MOE_ERR_MISALIGNED)]
    for (fmt, x, n, out), status in cases:
        assert L.moe_quantize(fmt, x, n, out, None, None) == status, (fmt, x, n, out)
        assert moe.moe_last_error()
    assert L.moe_quantize(moe.MOE_QUANT_Q2_K, None, 0, None, None, None) == moe.MOE_OK  # n = 0: no-op


def _fake_weights(moe, base=0x10000000, step=0x1000000, misalign=None, null=None):
    names = [f for f, _ in moe.moe_weights._fields_]
    vals = {}
    for i, n in enumerate(names):
        vals[n] = base + i * step
    if misalign:
        vals[misalign] += 8
    if null:
        vals[null] = None
    return moe.moe_weights(**vals)


class _FakeTensor:
    def __init__(self, ptr, n):
        self.ptr, self.n = ptr, n

    def data_ptr(self):
        return self.ptr

    def numel(self):
        return self.n

    def element_size(self):
        return 1


def _init(moe, cfg, w, persist_ptr=0x7000000, persist_bytes=1 << 20):
    h = ctypes.c_void_p(None)
    st = moe.lib().moe_init(ctypes.byref(cfg), ctypes.byref(w), persist_ptr, persist_bytes, None, ctypes.byref(h))
    return st, h.value


def test_init_validates_before_touching_the_device(moe):
    cfg = _cfg(moe)
    assert _init(moe, cfg, _fake_weights(moe, null="gate_iq2xxs"))[0] == moe.MOE_ERR_INVALID_ARG
    assert "gate_iq2xxs" in moe.moe_last_error()
    assert _init(moe, cfg, _fake_weights(moe, misalign="down_q2k"))[0] == moe.MOE_ERR_MISALIGNED
    assert _init(moe, cfg, _fake_weights(moe, null="router_w_f16"))[0] == moe.MOE_ERR_INVALID_ARG
    hcfg = _cfg(moe, mode=moe.MOE_ROUTE_HASH)
    assert _init(moe, hcfg, _fake_weights(moe, null="tid2eid"))[0] == moe.MOE_ERR_INVALID_ARG
    assert _init(moe, cfg, _fake_weights(moe), persist_ptr=0)[0] == moe.MOE_ERR_INVALID_ARG
    assert _init(moe, cfg, _fake_weights(moe), persist_ptr=0x7000004)[0] == moe.MOE_ERR_MISALIGNED
    assert _init(moe, cfg, _fake_weights(moe), persist_bytes=8)[0] == moe.MOE_ERR_WORKSPACE_TOO_SMALL


def test_calls_reject_null_handle(moe):
    L = moe.lib()
    assert L.moe_ffn_forward(None, None, None, 1, None, None, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route(None, None, None, 1, None, None, None, None, None, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_poll_device_error(None, None) == moe.MOE_ERR_INVALID_ARG
    L.moe_destroy(None)
