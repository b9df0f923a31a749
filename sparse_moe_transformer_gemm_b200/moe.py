"""ctypes binding of libmoe_b200.so (the C ABI of include/moe.h).

Argument marshalling only: every function here turns torch tensors into device
pointers, calls the C entry point of the same name on the current (or given)
CUDA stream and raises ``MoeError`` on a non-zero status. All arithmetic runs
in the library's CUDA kernels; there is no fallback. Loading fails loudly if
the library has not been built (``python -m sparse_moe_transformer_gemm_b200.build``).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

# MOE_B200_LIB selects another build of the same library (e.g. for A/B timing).
LIB_PATH = os.environ.get("MOE_B200_LIB") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5

MOE_FLAG_FP8_WEIGHTS = 0x1
MOE_FLAG_STREAM_PATH = 0x2
MOE_FLAG_GEMM_PATH = 0x4
MOE_FLAG_PACKED_WEIGHTS = 0x8
MOE_FLAG_SHARED_EXPERT = 0x10
MOE_FLAG_FP4_WEIGHTS = 0x20
MOE_WEIGHTS_GATE_UP = 0
MOE_WEIGHTS_DOWN = 1
MOE_SCORE_SIGMOID = 0
MOE_SCORE_SQRT_SOFTPLUS = 1
SCORE_FNS = {"sigmoid": MOE_SCORE_SIGMOID, "sqrtsoftplus": MOE_SCORE_SQRT_SOFTPLUS}

EXPORTED = ("moe_workspace_size", "moe_workspace_init", "moe_route", "moe_permute",
            "moe_permute_index", "moe_expert_gate_up", "moe_expert_gate_up_gather",
            "moe_expert_down", "moe_experts", "moe_combine", "moe_forward", "moe_read_status",
            "moe_status_string", "moe_route_noalloc", "moe_pack_weights", "moe_route2",
            "moe_forward2", "moe_route3", "moe_forward3", "moe_selftest_bounded_wait",
            "moe_ep_row_experts")

MOE_NOALLOC_SCRATCH_BYTES = 2 << 20
MOE_EP_MAX_SEGMENTS = 8192
# batches of at most this many token-slots (T*k) gather their token rows inside
# the gate_up GEMM; larger ones write the permuted copy (moe_forward's rule)
MOE_GATHER_MAX_SLOTS = 4096


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("scale", ctypes.c_float),
                ("flags", ctypes.c_uint32)]

    def __repr__(self):
        return (f"MoeConfig(T={self.T}, d={self.d}, E={self.E}, k={self.k}, d_ff={self.d_ff}, "
                f"scale={self.scale}, flags={self.flags:#x})")


class MoeRouteOptions(ctypes.Structure):
    """moe_route_options: score_bias [E], norm_weight [d] (device pointers), norm_eps,
    score_fn (MOE_SCORE_*)."""
    _fields_ = [("score_bias", ctypes.c_void_p), ("norm_weight", ctypes.c_void_p),
                ("norm_eps", ctypes.c_float), ("score_fn", ctypes.c_int32)]


def route_options(score_bias=None, norm_weight=None, norm_eps: float = 1e-6,
                  score_fn: str = "sigmoid"):
    """Router options; score_fn is "sigmoid" or "sqrtsoftplus" (or a MOE_SCORE_* value)."""
    fn = SCORE_FNS[score_fn] if isinstance(score_fn, str) else int(score_fn)
    return MoeRouteOptions(None if score_bias is None else score_bias.data_ptr(),
                           None if norm_weight is None else norm_weight.data_ptr(),
                           float(norm_eps), fn)


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {code} ({moe_status_string(code)})")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe_b200.so once, declaring the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_moe_transformer_gemm_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    C = ctypes.POINTER(MoeConfig)
    sig = {
        "moe_workspace_size": (S, [C]),
        "moe_workspace_init": (I, [C, P, S, P]),
        "moe_route": (I, [C, P, P, P, P, P, P, S, P]),
        "moe_permute": (I, [C, P, P, P, P, P, P, P, S, P]),
        "moe_permute_index": (I, [C, P, P, P, P, P, P, S, P]),
        "moe_expert_gate_up": (I, [C, P, P, P, P, P, P, S, P]),
        "moe_expert_gate_up_gather": (I, [C, P, P, P, P, P, P, P, S, P]),
        "moe_expert_down": (I, [C, P, P, P, P, P, P, S, P]),
        "moe_experts": (I, [C, P, P, P, P, P, P, P, P, S, P]),
        "moe_combine": (I, [C, P, P, P, P, P, S, P]),
        "moe_forward": (I, [C, P, P, P, P, P, P, P, P, P, S, P]),
        "moe_read_status": (I, [P, P]),
        "moe_status_string": (ctypes.c_char_p, [I]),
        "moe_route_noalloc": (I, [C, P, P, P, P, P, P]),
        "moe_pack_weights": (I, [C, I, P, P, P]),
        "moe_route2": (I, [C, P, P, P, P, P, P, P, S, P]),
        "moe_forward2": (I, [C, P, P, P, P, P, P, P, P, P, P, S, P]),
        "moe_route3": (I, [C, P, P, P, P, P, P, P, S, P]),
        "moe_forward3": (I, [C, P, P, P, P, P, P, P, P, P, P, S, P]),
        "moe_selftest_bounded_wait": (I, [P, ctypes.c_ulonglong, P]),
        "moe_ep_row_experts": (I, [P, ctypes.c_int32, ctypes.c_int32, P, ctypes.c_int32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def config(T: int, d: int, E: int, k: int, d_ff: int, scale: float = 2.826, fp8: bool = False,
           path: Optional[str] = None, packed: bool = False, shared: bool = False,
           fp4: bool = False) -> MoeConfig:
    """Build a moe_config. path: None (automatic), "stream" or "gemm"; packed: the
    bf16 expert weights are in moe_pack_weights' layout; shared: expert E of the
    weight arrays is a shared expert; fp4: E2M1 expert weights with E8M0 block
    scales."""
    flags = MOE_FLAG_FP8_WEIGHTS if fp8 else 0
    if fp4:
        flags |= MOE_FLAG_FP4_WEIGHTS
    if packed:
        flags |= MOE_FLAG_PACKED_WEIGHTS
    if shared:
        flags |= MOE_FLAG_SHARED_EXPERT
    if path == "stream":
        flags |= MOE_FLAG_STREAM_PATH
    elif path == "gemm":
        flags |= MOE_FLAG_GEMM_PATH
    elif path is not None:
        raise ValueError(f"unknown path {path!r}")
    return MoeConfig(T, d, E, k, d_ff, scale, flags)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def moe_workspace_size(cfg: MoeConfig) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(cfg)))


def moe_workspace_init(cfg: MoeConfig, ws: torch.Tensor, stream=None) -> None:
    _check("moe_workspace_init",
           lib().moe_workspace_init(ctypes.byref(cfg), _p(ws), ws.numel(), _s(stream)))


def workspace(cfg: MoeConfig, device="cuda", stream=None) -> torch.Tensor:
    """Allocate (through torch) and initialise a workspace for cfg."""
    n = moe_workspace_size(cfg)
    if n == 0:
        raise MoeError("moe_workspace_size", MOE_ERR_UNSUPPORTED_SHAPE)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_workspace_init(cfg, ws, stream)
    return ws


def moe_route(cfg, x, w_gate, gate_bias, topk_idx, topk_w, ws, stream=None) -> None:
    _check("moe_route", lib().moe_route(ctypes.byref(cfg), _p(x), _p(w_gate), _p(gate_bias),
                                        _p(topk_idx), _p(topk_w), _p(ws), ws.numel(), _s(stream)))


def moe_permute(cfg, topk_idx, x, counts, offsets, row_of, x_perm, ws, stream=None) -> None:
    _check("moe_permute", lib().moe_permute(ctypes.byref(cfg), _p(topk_idx), _p(x), _p(counts),
                                            _p(offsets), _p(row_of), _p(x_perm), _p(ws),
                                            ws.numel(), _s(stream)))


def moe_permute_index(cfg, topk_idx, counts, offsets, row_of, token_of_row, ws,
                      stream=None) -> None:
    _check("moe_permute_index",
           lib().moe_permute_index(ctypes.byref(cfg), _p(topk_idx), _p(counts), _p(offsets),
                                   _p(row_of), _p(token_of_row), _p(ws), ws.numel(), _s(stream)))


def moe_expert_gate_up_gather(cfg, x, token_of_row, offsets, w_gate_up, s_gate_up, h, ws,
                              stream=None) -> None:
    _check("moe_expert_gate_up_gather",
           lib().moe_expert_gate_up_gather(ctypes.byref(cfg), _p(x), _p(token_of_row),
                                           _p(offsets), _p(w_gate_up), _p(s_gate_up), _p(h),
                                           _p(ws), ws.numel(), _s(stream)))


def moe_expert_gate_up(cfg, x_perm, offsets, w_gate_up, s_gate_up, h, ws, stream=None) -> None:
    _check("moe_expert_gate_up",
           lib().moe_expert_gate_up(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(w_gate_up),
                                    _p(s_gate_up), _p(h), _p(ws), ws.numel(), _s(stream)))


def moe_expert_down(cfg, h, offsets, w_down, s_down, y, ws, stream=None) -> None:
    _check("moe_expert_down",
           lib().moe_expert_down(ctypes.byref(cfg), _p(h), _p(offsets), _p(w_down), _p(s_down),
                                 _p(y), _p(ws), ws.numel(), _s(stream)))


def moe_experts(cfg, x_perm, offsets, w_gate_up, s_gate_up, w_down, s_down, y, ws,
                stream=None) -> None:
    _check("moe_experts",
           lib().moe_experts(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(w_gate_up),
                             _p(s_gate_up), _p(w_down), _p(s_down), _p(y), _p(ws), ws.numel(),
                             _s(stream)))


def moe_combine(cfg, y, row_of, topk_w, out, ws, stream=None) -> None:
    _check("moe_combine", lib().moe_combine(ctypes.byref(cfg), _p(y), _p(row_of), _p(topk_w),
                                            _p(out), _p(ws), ws.numel(), _s(stream)))


def moe_forward(cfg, x, w_gate, gate_bias, w_gate_up, s_gate_up, w_down, s_down, out, ws,
                stream=None) -> None:
    _check("moe_forward",
           lib().moe_forward(ctypes.byref(cfg), _p(x), _p(w_gate), _p(gate_bias), _p(w_gate_up),
                             _p(s_gate_up), _p(w_down), _p(s_down), _p(out), _p(ws), ws.numel(),
                             _s(stream)))


def moe_route2(cfg, x, w_gate, gate_bias, score_bias, topk_idx, topk_w, ws, stream=None) -> None:
    _check("moe_route2", lib().moe_route2(ctypes.byref(cfg), _p(x), _p(w_gate), _p(gate_bias),
                                          _p(score_bias), _p(topk_idx), _p(topk_w), _p(ws),
                                          ws.numel(), _s(stream)))


def moe_forward2(cfg, x, w_gate, gate_bias, score_bias, w_gate_up, s_gate_up, w_down, s_down,
                 out, ws, stream=None) -> None:
    _check("moe_forward2",
           lib().moe_forward2(ctypes.byref(cfg), _p(x), _p(w_gate), _p(gate_bias),
                              _p(score_bias), _p(w_gate_up), _p(s_gate_up), _p(w_down),
                              _p(s_down), _p(out), _p(ws), ws.numel(), _s(stream)))


def moe_route3(cfg, x, w_gate, gate_bias, opt, topk_idx, topk_w, ws, stream=None) -> None:
    _check("moe_route3", lib().moe_route3(ctypes.byref(cfg), _p(x), _p(w_gate), _p(gate_bias),
                                          None if opt is None else ctypes.byref(opt),
                                          _p(topk_idx), _p(topk_w), _p(ws), ws.numel(),
                                          _s(stream)))


def moe_forward3(cfg, x, w_gate, gate_bias, opt, w_gate_up, s_gate_up, w_down, s_down, out, ws,
                 stream=None) -> None:
    _check("moe_forward3",
           lib().moe_forward3(ctypes.byref(cfg), _p(x), _p(w_gate), _p(gate_bias),
                              None if opt is None else ctypes.byref(opt), _p(w_gate_up),
                              _p(s_gate_up), _p(w_down), _p(s_down), _p(out), _p(ws), ws.numel(),
                              _s(stream)))


def moe_route_noalloc(cfg, x, w_gate, gate_bias, topk_idx, topk_w, stream=None) -> None:
    """moe_route without a workspace, for callers that cannot allocate device
    memory; the scratch is a fixed 2 MiB device array inside the library."""
    _check("moe_route_noalloc",
           lib().moe_route_noalloc(ctypes.byref(cfg), _p(x), _p(w_gate), _p(gate_bias),
                                   _p(topk_idx), _p(topk_w), _s(stream)))


def moe_pack_weights(cfg, which, w, w_packed, stream=None) -> None:
    """Rearrange one bf16 expert weight into the packed 128 x 64 block layout."""
    _check("moe_pack_weights", lib().moe_pack_weights(ctypes.byref(cfg), int(which), _p(w),
                                                      _p(w_packed), _s(stream)))


def moe_selftest_bounded_wait(ws, limit_ns: int, stream=None) -> None:
    """Run the bounded-wait self-test; its MOE_ERR_TIMEOUT lands in ws's status word."""
    _check("moe_selftest_bounded_wait",
           lib().moe_selftest_bounded_wait(_p(ws), int(limit_ns), _s(stream)))


def moe_ep_row_experts(counts, n_src: int, e_local: int, expert_of_row, stream=None) -> None:
    """Local expert of every received row (expert parallelism): counts [n_src, e_local]
    int32, expert_of_row [n_rows] int32, both on the device."""
    _check("moe_ep_row_experts",
           lib().moe_ep_row_experts(_p(counts), int(n_src), int(e_local), _p(expert_of_row),
                                    int(expert_of_row.numel()), _s(stream)))


def moe_read_status(ws, stream=None) -> int:
    return int(lib().moe_read_status(_p(ws), _s(stream)))


def layer_args(layer: dict):
    """(w_gate_up, s_gate_up, w_down, s_down) of a synthetic layer dict, FP4, FP8 or
    bf16; with a shared expert, its weights follow the routed ones as expert E."""
    cfg = layer["cfg"]
    if getattr(cfg, "fp4", False):
        return (layer["q4_gate_up"], layer["s4_gate_up"], layer["q4_down"], layer["s4_down"])
    if cfg.fp8:
        args = [layer["q_gate_up"], layer["s_gate_up"], layer["q_down"], layer["s_down"]]
        sh = ("q_shared_gate_up", "s_shared_gate_up", "q_shared_down", "s_shared_down")
    else:
        args = [layer["w_gate_up"], None, layer["w_down"], None]
        sh = ("w_shared_gate_up", None, "w_shared_down", None)
    if getattr(cfg, "shared", False):
        args = [a if n is None else torch.cat([a, layer[n][None]]) for a, n in zip(args, sh)]
    return tuple(args)


def config_of(shape, path: Optional[str] = None, packed: bool = False) -> MoeConfig:
    """moe_config for a synthetic LayerShape."""
    return config(shape.T, shape.d, shape.E, shape.k, shape.F, shape.scale, shape.fp8, path,
                  packed, getattr(shape, "shared", False), getattr(shape, "fp4", False))


def pack_layer_weights(cfg: MoeConfig, w_gate_up: torch.Tensor, w_down: torch.Tensor,
                       stream=None):
    """(packed w_gate_up, packed w_down): new tensors in moe_pack_weights' layout."""
    gu = torch.empty_like(w_gate_up)
    dn = torch.empty_like(w_down)
    moe_pack_weights(cfg, MOE_WEIGHTS_GATE_UP, w_gate_up, gu, stream)
    moe_pack_weights(cfg, MOE_WEIGHTS_DOWN, w_down, dn, stream)
    return gu, dn
