"""ctypes wrapper of the C oracle (moe_oracle.c) plus its build step.

TEST INFRASTRUCTURE ONLY (see the package docstring). Arrays cross as numpy
buffers: bf16 tensors as their uint16 bit patterns, e4m3 as uint8 codes.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (fp64, OpenMP) into libmoe_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # MOE_ORACLE_LIB points the wrapper at another build of moe_oracle.c; the
        # mutation test uses it to check that the pins catch planted mistakes.
        path = os.environ.get("MOE_ORACLE_LIB")
        if not path:
            path = build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        L = ctypes.c_long
        lib.oracle_num_threads.restype = I
        lib.oracle_set_num_threads.argtypes = [I]
        lib.oracle_bf16_from_double.argtypes = [P, P, L]
        lib.oracle_double_from_bf16.argtypes = [P, P, L]
        lib.oracle_double_from_e4m3.argtypes = [P, P, L]
        lib.oracle_route.argtypes = [I, I, I, I, D, P, P, P, P, P, P, P, P]
        lib.oracle_route.restype = I
        lib.oracle_route2.argtypes = [I, I, I, I, D, P, P, P, P, P, D, I, P, P, P, P, P]
        lib.oracle_route2.restype = I
        lib.oracle_expert_rows.argtypes = [I, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_expert_rows.restype = I
        lib.oracle_forward_tokens.argtypes = [I, I, I, I, I, D, P, P, P, P, P, P, P, P, I, P, P,
                                              P, P, P]
        lib.oracle_forward_tokens.restype = I
        lib.oracle_forward_tokens2.argtypes = [I, I, I, I, I, D, P, P, P, P, P, D, I, P, P, P, P,
                                               P, P, P, P, P, I, P, P, P, P, P]
        lib.oracle_forward_tokens2.restype = I
        lib.oracle_combine.argtypes = [I, I, I, P, P, P]
        lib.oracle_double_from_e2m1.argtypes = [P, P, L]
        lib.oracle_double_from_e8m0.argtypes = [P, P, L]
        lib.oracle_expert_rows_fp4.argtypes = [I, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_expert_rows_fp4.restype = I
        lib.oracle_forward_tokens_fp4.argtypes = [I, I, I, I, I, D, P, P, P, P, I, P, P, P, P, P,
                                                  I, P, P, P, P, P]
        lib.oracle_forward_tokens_fp4.restype = I
        lib.oracle_permute.argtypes = [I, I, I, P, P, P, P]
        lib.oracle_permute.restype = I
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def bf16_bits(t) -> np.ndarray:
    """uint16 bit patterns of a bf16 torch tensor (any device), as numpy."""
    import torch

    return np.ascontiguousarray(t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def bf16_from_double(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_bf16_from_double(_ptr(v), _ptr(out), v.size)
    return out


def double_from_bf16(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    _load().oracle_double_from_bf16(_ptr(b), _ptr(out), b.size)
    return out


def double_from_e4m3(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    out = np.empty(q.shape, dtype=np.float64)
    _load().oracle_double_from_e4m3(_ptr(q), _ptr(out), q.size)
    return out


SCORE_FNS = {"sigmoid": 0, "sqrtsoftplus": 1}


def route(x, wg, k: int, scale: float, gate_bias=None, want_scores: bool = False,
          score_bias=None, norm_w=None, norm_eps: float = 1e-6, score_fn: str = "sigmoid"):
    """Steps 1-4 for all tokens. x [T,d] / wg [E,d] uint16 bf16 bits.

    gate_bias [E] is added to the logits (before the sigmoid); score_bias [E]
    (e_score_correction_bias) to the scores for the choice only; norm_w [d]
    turns on route_norm (the router scores the token's RMSNorm with that weight
    and norm_eps); score_fn "sqrtsoftplus" scores sqrt(softplus(logit)) instead of
    the sigmoid. Returns
    dict(idx int32 [T,k], w f64 [T,k], gap f64 [T] -- between the k-th and
    (k+1)-th ranked value -- and with want_scores also logits/scores f64 [T,E]).
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    wg = np.ascontiguousarray(wg, dtype=np.uint16)
    T, d = x.shape
    E = wg.shape[0]
    gb = None if gate_bias is None else np.ascontiguousarray(gate_bias, dtype=np.float32)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    gap = np.empty((T,), dtype=np.float64)
    logits = np.empty((T, E), dtype=np.float64) if want_scores else None
    scores = np.empty((T, E), dtype=np.float64) if want_scores else None
    sb = None if score_bias is None else np.ascontiguousarray(score_bias, dtype=np.float32)
    nw = None if norm_w is None else np.ascontiguousarray(norm_w, dtype=np.float32)
    rc = _load().oracle_route2(T, d, E, k, float(scale), _ptr(x), _ptr(wg), _ptr(gb), _ptr(sb),
                               _ptr(nw), float(norm_eps), SCORE_FNS[score_fn], _ptr(idx), _ptr(w),
                               _ptr(logits), _ptr(scores), _ptr(gap))
    if rc != 0:
        raise ValueError("oracle_route: bad arguments")
    out = {"idx": idx, "w": w, "gap": gap}
    if want_scores:
        out.update(logits=logits, scores=scores)
    return out


def expert_rows(xrows, experts, wgu, wd, s_gu=None, s_d=None, want_h: bool = False):
    """Step 5 for (row, expert) pairs. xrows [n,d] bf16 bits; experts [n] int32.

    wgu [E,2F,d] / wd [E,d,F]: uint16 bf16 bits, or uint8 e4m3 codes with
    fp32 row scales s_gu [E,2F] / s_d [E,d]. Returns y [n,d] (and h [n,F]).
    """
    xrows = np.ascontiguousarray(xrows, dtype=np.uint16)
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    n, d = xrows.shape
    F = wd.shape[2]
    fp8 = s_gu is not None
    wgu = np.ascontiguousarray(wgu, dtype=np.uint8 if fp8 else np.uint16)
    wd = np.ascontiguousarray(wd, dtype=np.uint8 if fp8 else np.uint16)
    s_gu = None if s_gu is None else np.ascontiguousarray(s_gu, dtype=np.float32)
    s_d = None if s_d is None else np.ascontiguousarray(s_d, dtype=np.float32)
    h = np.empty((n, F), dtype=np.float64) if want_h else None
    y = np.empty((n, d), dtype=np.float64)
    _load().oracle_expert_rows(n, d, F, _ptr(xrows), _ptr(experts), _ptr(wgu), _ptr(s_gu),
                               _ptr(wd), _ptr(s_d), _ptr(h), _ptr(y))
    return (y, h) if want_h else y


def double_from_e2m1(nibbles: np.ndarray) -> np.ndarray:
    nb = np.ascontiguousarray(nibbles, dtype=np.uint8)
    out = np.empty(nb.shape, dtype=np.float64)
    _load().oracle_double_from_e2m1(_ptr(nb), _ptr(out), nb.size)
    return out


def double_from_e8m0(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(b.shape, dtype=np.float64)
    _load().oracle_double_from_e8m0(_ptr(b), _ptr(out), b.size)
    return out


def expert_rows_fp4(xrows, experts, wgu4, sgu8, wd4, sd8, want_h: bool = False):
    """Step 5 with FP4 experts: packed E2M1 codes wgu4 [E,2F,d/2] / wd4 [E,d,F/2]
    and E8M0 block-32 scales sgu8 [E,2F,d/32] / sd8 [E,d,F/32]."""
    xrows = np.ascontiguousarray(xrows, dtype=np.uint16)
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    n, d = xrows.shape
    F = wd4.shape[2] * 2
    arrs = [np.ascontiguousarray(a, dtype=np.uint8) for a in (wgu4, sgu8, wd4, sd8)]
    h = np.empty((n, F), dtype=np.float64) if want_h else None
    y = np.empty((n, d), dtype=np.float64)
    if _load().oracle_expert_rows_fp4(n, d, F, _ptr(xrows), _ptr(experts), *map(_ptr, arrs),
                                      _ptr(h), _ptr(y)) != 0:
        raise ValueError("oracle_expert_rows_fp4: bad arguments")
    return (y, h) if want_h else y


def forward_tokens(layer: "OracleLayer", tokens=None):
    """Steps 1-6 for the listed tokens (all tokens when None)."""
    L = layer
    if tokens is None:
        tokens = np.arange(L.T, dtype=np.int32)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    n = tokens.shape[0]
    out_f64 = np.empty((n, L.d), dtype=np.float64)
    out_bf16 = np.empty((n, L.d), dtype=np.uint16)
    idx = np.empty((n, L.k), dtype=np.int32)
    w = np.empty((n, L.k), dtype=np.float64)
    gap = np.empty((n,), dtype=np.float64)
    if L.fp4:
        rc = _load().oracle_forward_tokens_fp4(
            L.T, L.d, L.E, L.k, L.F, float(L.scale), _ptr(L.x), _ptr(L.wg), _ptr(L.gate_bias),
            _ptr(L.score_bias), SCORE_FNS[L.score_fn], _ptr(L.wgu4), _ptr(L.sgu8), _ptr(L.wd4),
            _ptr(L.sd8), _ptr(tokens), n, _ptr(out_f64), _ptr(out_bf16), _ptr(idx), _ptr(w),
            _ptr(gap))
        if rc != 0:
            raise ValueError("oracle_forward_tokens_fp4: bad arguments")
        return {"out_f64": out_f64, "out_bf16": out_bf16, "idx": idx, "w": w, "gap": gap,
                "tokens": tokens}
    rc = _load().oracle_forward_tokens2(L.T, L.d, L.E, L.k, L.F, float(L.scale), _ptr(L.x),
                                        _ptr(L.wg), _ptr(L.gate_bias), _ptr(L.score_bias),
                                        _ptr(L.norm_w), float(L.norm_eps),
                                        SCORE_FNS[L.score_fn], _ptr(L.wgu), _ptr(L.s_gu),
                                        _ptr(L.wd), _ptr(L.s_d),
                                        _ptr(L.sh_wgu), _ptr(L.sh_s_gu), _ptr(L.sh_wd),
                                        _ptr(L.sh_s_d), _ptr(tokens), n, _ptr(out_f64),
                                        _ptr(out_bf16), _ptr(idx), _ptr(w), _ptr(gap))
    if rc != 0:
        raise ValueError("oracle_forward_tokens: bad arguments")
    return {"out_f64": out_f64, "out_bf16": out_bf16, "idx": idx, "w": w, "gap": gap,
            "tokens": tokens}


def combine(y, w) -> np.ndarray:
    """Step 6: y [n,k,d] f64, w [n,k] f64 -> bf16 bits [n,d]."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    n, k, d = y.shape
    out = np.empty((n, d), dtype=np.uint16)
    _load().oracle_combine(n, k, d, _ptr(y), _ptr(w), _ptr(out))
    return out


def permute(idx, E: int):
    """The library's grouping of token-slots by expert, from its definition."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.empty((E,), dtype=np.int32)
    offsets = np.empty((E + 1,), dtype=np.int32)
    row_of = np.empty((T * k,), dtype=np.int32)
    if _load().oracle_permute(T, k, E, _ptr(idx), _ptr(counts), _ptr(offsets), _ptr(row_of)) != 0:
        raise ValueError("oracle_permute: expert index out of range")
    return {"counts": counts, "offsets": offsets, "row_of": row_of}


class OracleLayer:
    """Host copies (numpy bit patterns) of one layer's inputs for the oracle.

    ``layer`` is the dict the synthetic generator returns (tensors on any
    device). FP8 layers use the e4m3 codes and scales.
    """

    def __init__(self, layer: dict, scale: Optional[float] = None, k: Optional[int] = None):
        cfg = layer["cfg"]
        self.cfg = cfg
        self.T, self.d, self.E, self.F = cfg.T, cfg.d, cfg.E, cfg.F
        self.k = cfg.k if k is None else k
        self.scale = cfg.scale if scale is None else scale
        self.x = bf16_bits(layer["x"])
        self.wg = bf16_bits(layer["w_gate"])
        gb = layer.get("gate_bias")
        self.gate_bias = None if gb is None else np.ascontiguousarray(gb.detach().cpu().numpy(),
                                                                      dtype=np.float32)
        nw = layer.get("route_norm_weight")
        self.norm_w = None if nw is None else np.ascontiguousarray(nw.detach().cpu().numpy(),
                                                                   dtype=np.float32)
        self.norm_eps = float(getattr(cfg, "route_norm_eps", 1e-6))
        self.score_fn = getattr(cfg, "score_fn", "sigmoid")
        self.fp4 = bool(getattr(cfg, "fp4", False))
        if self.fp4:
            self.wgu4 = np.ascontiguousarray(layer["q4_gate_up"].cpu().numpy())
            self.sgu8 = np.ascontiguousarray(layer["s4_gate_up"].cpu().numpy())
            self.wd4 = np.ascontiguousarray(layer["q4_down"].cpu().numpy())
            self.sd8 = np.ascontiguousarray(layer["s4_down"].cpu().numpy())
        sb = layer.get("score_bias")
        self.score_bias = None if sb is None else np.ascontiguousarray(
            sb.detach().cpu().numpy(), dtype=np.float32)
        if cfg.fp8:
            self.wgu = np.ascontiguousarray(layer["q_gate_up"].cpu().numpy())
            self.wd = np.ascontiguousarray(layer["q_down"].cpu().numpy())
            self.s_gu = np.ascontiguousarray(layer["s_gate_up"].cpu().numpy(), dtype=np.float32)
            self.s_d = np.ascontiguousarray(layer["s_down"].cpu().numpy(), dtype=np.float32)
        elif self.fp4:  # the FP4 codes above are the experts' weights
            self.wgu = self.wd = self.s_gu = self.s_d = None
        else:
            self.wgu = bf16_bits(layer["w_gate_up"])
            self.wd = bf16_bits(layer["w_down"])
            self.s_gu = None
            self.s_d = None
        # the shared expert (optional), in the routed experts' format
        self.sh_wgu = self.sh_wd = self.sh_s_gu = self.sh_s_d = None
        if cfg.fp8 and layer.get("q_shared_gate_up") is not None:
            self.sh_wgu = np.ascontiguousarray(layer["q_shared_gate_up"].cpu().numpy())
            self.sh_wd = np.ascontiguousarray(layer["q_shared_down"].cpu().numpy())
            self.sh_s_gu = np.ascontiguousarray(layer["s_shared_gate_up"].cpu().numpy(),
                                                dtype=np.float32)
            self.sh_s_d = np.ascontiguousarray(layer["s_shared_down"].cpu().numpy(),
                                               dtype=np.float32)
        elif not cfg.fp8 and layer.get("w_shared_gate_up") is not None:
            self.sh_wgu = bf16_bits(layer["w_shared_gate_up"])
            self.sh_wd = bf16_bits(layer["w_shared_down"])
