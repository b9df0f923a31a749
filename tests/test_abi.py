"""The C ABI library: builds, loads without a GPU, exports what include/moe.h
declares, and rejects bad arguments before touching CUDA."""

import ctypes
import os
import re

import pytest

from sparse_moe_transformer_gemm_b200 import build as moe_build
from sparse_moe_transformer_gemm_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_binding_surface():
    assert declared_functions() == sorted(moe.EXPORTED)


def test_header_constants_match_the_binding():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    m = re.search(r"#define MOE_GATHER_MAX_SLOTS (\d+)", text)
    assert m and int(m.group(1)) == moe.MOE_GATHER_MAX_SLOTS
    m = re.search(r"#define MOE_EP_MAX_SEGMENTS (\d+)", text)
    assert m and int(m.group(1)) == moe.MOE_EP_MAX_SEGMENTS
    m = re.search(r"#define MOE_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == moe.MOE_NOALLOC_SCRATCH_BYTES
    for name in ("MOE_FLAG_FP8_WEIGHTS", "MOE_FLAG_STREAM_PATH", "MOE_FLAG_GEMM_PATH",
                 "MOE_FLAG_PACKED_WEIGHTS", "MOE_FLAG_SHARED_EXPERT", "MOE_FLAG_FP4_WEIGHTS"):
        m = re.search(r"#define %s (0x[0-9a-f]+)u" % name, text)
        assert m and int(m.group(1), 16) == getattr(moe, name), name
    for name in ("MOE_WEIGHTS_GATE_UP", "MOE_WEIGHTS_DOWN", "MOE_SCORE_SIGMOID",
                 "MOE_SCORE_SQRT_SOFTPLUS"):
        m = re.search(r"#define %s (\d+)" % name, text)
        assert m and int(m.group(1)) == getattr(moe, name), name


def test_packed_weights_flag_rules(lib):
    assert moe.moe_workspace_size(moe.config(**HY3, packed=True)) > 0
    assert moe.moe_workspace_size(moe.config(**HY3, packed=True, fp8=True)) == 0
    assert moe.moe_workspace_size(moe.config(**HY3, packed=True, path="stream")) == 0
    assert moe.moe_workspace_size(moe.config(**HY3, packed=True, path="gemm")) > 0
    # the tensor-core pair kernels need d and d_ff multiples of 256
    assert moe.moe_workspace_size(moe.config(**{**HY3, "d": 384}, packed=True)) == 0
    assert moe.moe_workspace_size(moe.config(**{**HY3, "d": 384})) > 0


def test_shared_expert_flag_rules(lib):
    plain = moe.moe_workspace_size(moe.config(**HY3))
    shared = moe.moe_workspace_size(moe.config(**HY3, shared=True))
    assert shared > plain  # one more slot per token in the grouped buffers
    assert moe.moe_workspace_size(moe.config(**{**HY3, "E": 255}, shared=True)) > 0
    assert moe.moe_workspace_size(moe.config(**{**HY3, "E": 256}, shared=True)) == 0
    assert moe.moe_workspace_size(moe.config(**{**HY3, "E": 256})) > 0


def test_fp4_weights_flag_rules(lib):
    assert moe.moe_workspace_size(moe.config(**HY3, fp4=True)) > 0
    assert moe.moe_workspace_size(moe.config(**HY3, fp4=True, path="stream")) > 0
    # the tensor-core pair kernels take FP4 too (d, d_ff multiples of 256)
    assert moe.moe_workspace_size(moe.config(**HY3, fp4=True, path="gemm")) > 0
    for bad in (dict(fp8=True), dict(packed=True), dict(shared=True)):
        assert moe.moe_workspace_size(moe.config(**HY3, fp4=True, **bad)) == 0, bad
    # FP4 weights need their block scales
    cfg = moe.config(**HY3, fp4=True)
    P = ctypes.c_void_p
    rc = _call("moe_expert_down", ctypes.byref(cfg), P(FAKE), P(FAKE), P(FAKE), None, P(FAKE),
               P(FAKE), moe.moe_workspace_size(cfg), None)
    assert rc == moe.MOE_ERR_INVALID_ARG


def test_route_options_struct_matches_the_header():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    body = re.search(r"typedef struct moe_route_options \{(.*?)\} moe_route_options;", text,
                     re.S).group(1)
    fields = re.findall(r"(\w+);", body)
    assert fields == [f for f, _ in moe.MoeRouteOptions._fields_]
    assert ctypes.sizeof(moe.MoeRouteOptions) == 24


def test_route_options_are_checked_before_any_launch(lib):
    cfg = moe.config(**HY3)
    ws_n = moe.moe_workspace_size(cfg)
    P = ctypes.c_void_p
    bad = moe.MoeRouteOptions(None, FAKE, 0.0)      # a norm weight needs eps > 0
    rc = _call("moe_route3", ctypes.byref(cfg), P(FAKE), P(FAKE), None, ctypes.byref(bad),
               P(FAKE), P(FAKE), P(FAKE), ws_n, None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    bad = moe.MoeRouteOptions(None, FAKE, float("nan"))
    rc = _call("moe_forward3", ctypes.byref(cfg), P(FAKE), P(FAKE), None, ctypes.byref(bad),
               P(FAKE), None, P(FAKE), None, P(FAKE), P(FAKE), ws_n, None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    for fn in (-1, 2):  # no such score function
        bad = moe.MoeRouteOptions(None, None, 0.0, fn)
        rc = _call("moe_route3", ctypes.byref(cfg), P(FAKE), P(FAKE), None, ctypes.byref(bad),
                   P(FAKE), P(FAKE), P(FAKE), ws_n, None)
        assert rc == moe.MOE_ERR_INVALID_ARG
    assert moe.route_options(score_fn="sqrtsoftplus").score_fn == moe.MOE_SCORE_SQRT_SOFTPLUS


def test_pack_weights_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    cfg = moe.config(**HY3)
    n = 192 * 2 * 1536 * 4096 * 2
    call = lambda c, which, a, b: _call("moe_pack_weights", ctypes.byref(c), which, a, b, None)  # noqa: E731
    assert call(cfg, 2, P(FAKE), P(FAKE + n)) == moe.MOE_ERR_INVALID_ARG
    assert call(cfg, moe.MOE_WEIGHTS_GATE_UP, None, P(FAKE + n)) == moe.MOE_ERR_INVALID_ARG
    assert call(cfg, moe.MOE_WEIGHTS_GATE_UP, P(FAKE), P(FAKE + 8)) == moe.MOE_ERR_INVALID_ARG
    assert call(cfg, moe.MOE_WEIGHTS_GATE_UP, P(FAKE), P(FAKE + n - 16)) == moe.MOE_ERR_INVALID_ARG
    assert call(moe.config(**HY3, fp8=True), moe.MOE_WEIGHTS_DOWN, P(FAKE), P(FAKE + n)) == \
        moe.MOE_ERR_INVALID_ARG
    assert call(moe.config(**{**HY3, "d_ff": 384}), moe.MOE_WEIGHTS_DOWN, P(FAKE),
                P(FAKE + n)) == moe.MOE_ERR_UNSUPPORTED_SHAPE


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_only_the_abi_is_exported():
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert syms == set(moe.EXPORTED)


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5):
        assert moe.moe_status_string(code) and moe.moe_status_string(code) != "unknown status code"
    assert moe.moe_status_string(-99) == "unknown status code"


HY3 = dict(T=64, d=4096, E=192, k=8, d_ff=1536)


@pytest.mark.parametrize("bad", [
    dict(T=0), dict(d=100), dict(d=4096 + 64), dict(d_ff=1000), dict(E=0), dict(E=257),
    dict(k=0), dict(k=9, E=8), dict(k=33, E=64), dict(d=8320), dict(T=1 << 20, d_ff=4096),
])
def test_workspace_size_rejects_unsupported_shapes(lib, bad):
    cfg = moe.config(**{**HY3, **bad})
    assert moe.moe_workspace_size(cfg) == 0


def test_workspace_size_covers_the_intermediates(lib):
    cfg = moe.config(**HY3)
    n = moe.moe_workspace_size(cfg)
    R = 64 * 8
    assert n >= R * 4096 * 2 * 2 + R * 1536 * 2   # x_perm + y + h
    big = moe.config(**{**HY3, "T": 4096})
    assert moe.moe_workspace_size(big) > 60 * n


FAKE = 0x10000  # an aligned address that is never dereferenced: every call below fails first


def _call(fn, *args):
    return getattr(moe.lib(), fn)(*args)


def test_null_pointers_and_bad_flags_are_invalid_args(lib):
    cfg = moe.config(**HY3)
    ws_n = moe.moe_workspace_size(cfg)
    P = ctypes.c_void_p
    # moe_route with a NULL x
    rc = _call("moe_route", ctypes.byref(cfg), None, P(FAKE), None, P(FAKE), P(FAKE), P(FAKE),
               ws_n, None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    # misaligned x
    rc = _call("moe_route", ctypes.byref(cfg), P(FAKE + 2), P(FAKE), None, P(FAKE), P(FAKE),
               P(FAKE), ws_n, None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    # both path flags
    both = moe.config(**HY3)
    both.flags = moe.MOE_FLAG_STREAM_PATH | moe.MOE_FLAG_GEMM_PATH
    assert moe.moe_workspace_size(both) == 0
    # unknown flag bit
    unk = moe.config(**HY3)
    unk.flags = 0x100
    assert moe.moe_workspace_size(unk) == 0
    # bf16 weights given scales, FP8 weights without scales
    rc = _call("moe_expert_gate_up", ctypes.byref(cfg), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
               P(FAKE), P(FAKE), ws_n, None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    fp8 = moe.config(**HY3, fp8=True)
    rc = _call("moe_expert_gate_up", ctypes.byref(fp8), P(FAKE), P(FAKE), P(FAKE), None,
               P(FAKE), P(FAKE), ws_n, None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    # misaligned workspace
    rc = _call("moe_combine", ctypes.byref(cfg), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
               P(FAKE + 16), ws_n, None)
    assert rc == moe.MOE_ERR_INVALID_ARG


def test_small_workspace_is_reported(lib):
    cfg = moe.config(**HY3)
    ws_n = moe.moe_workspace_size(cfg)
    P = ctypes.c_void_p
    rc = _call("moe_forward", ctypes.byref(cfg), P(FAKE), P(FAKE), None, P(FAKE), None, P(FAKE),
               None, P(FAKE), P(FAKE), ws_n - 256, None)
    assert rc == moe.MOE_ERR_WORKSPACE


def test_unsupported_shape_is_reported_by_every_entry_point(lib):
    cfg = moe.config(**{**HY3, "d": 100})
    P = ctypes.c_void_p
    f = P(FAKE)
    cases = {
        "moe_route": (f, f, None, f, f, f, 1 << 30, None),
        "moe_permute": (f, f, f, f, f, f, f, 1 << 30, None),
        "moe_permute_index": (f, f, f, f, f, f, 1 << 30, None),
        "moe_expert_gate_up_gather": (f, f, f, f, None, f, f, 1 << 30, None),
        "moe_expert_gate_up": (f, f, f, None, f, f, 1 << 30, None),
        "moe_expert_down": (f, f, f, None, f, f, 1 << 30, None),
        "moe_experts": (f, f, f, None, f, None, f, f, 1 << 30, None),
        "moe_combine": (f, f, f, f, f, 1 << 30, None),
        "moe_forward": (f, f, None, f, None, f, None, f, f, 1 << 30, None),
        "moe_pack_weights": (moe.MOE_WEIGHTS_GATE_UP, f, P(FAKE + (1 << 34)), None),
        "moe_route2": (f, f, None, None, f, f, f, 1 << 30, None),
        "moe_forward2": (f, f, None, None, f, None, f, None, f, f, 1 << 30, None),
        "moe_route3": (f, f, None, None, f, f, f, 1 << 30, None),
        "moe_forward3": (f, f, None, None, f, None, f, None, f, f, 1 << 30, None),
    }
    for fn, args in cases.items():
        assert _call(fn, ctypes.byref(cfg), *args) == moe.MOE_ERR_UNSUPPORTED_SHAPE, fn


def test_ep_row_experts_rejects_bad_arguments_before_any_launch(lib):
    P = ctypes.c_void_p
    call = lambda c, n_src, el, out, n: _call("moe_ep_row_experts", c, n_src, el, out, n, None)  # noqa: E731
    assert call(None, 2, 24, P(FAKE), 10) == moe.MOE_ERR_INVALID_ARG
    assert call(P(FAKE), 2, 24, None, 10) == moe.MOE_ERR_INVALID_ARG
    assert call(P(FAKE), 0, 24, P(FAKE), 10) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert call(P(FAKE), 2, 257, P(FAKE), 10) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert call(P(FAKE), 2, 24, P(FAKE), 0) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert call(P(FAKE), 33, 256, P(FAKE), 10) == moe.MOE_ERR_UNSUPPORTED_SHAPE  # 8448 segments
