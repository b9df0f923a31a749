"""Algorithmic work of one routed-MoE layer call, for roofline accounting.

"Algorithmic" is what the layer must move or compute, independent of how the
kernels are tiled:

* bytes  = weights of the experts that at least one token selects (plus their
  fp32 row scales for FP8 weights, their E8M0 block scales for FP4 weights) +
  router weight + x read + out write;
* flops  = 2*T*d*E (router) + 6*T*k*d*F (gate, up and down projections of the
  k selected experts; 6*d*F per token per expert is the per-expert count of
  "Tencent Hy3-Flash QA", Q2.4).

The expert steps alone: gate_up must read the touched experts' [2F, d]
weights and the batch's tokens (T rows of x, once); down must read the
touched experts' [d, F] weights. The intermediates between the steps (the
permuted token rows, h [R, F], y [R, d]) and any re-read of a token row are
implementation traffic, reported apart as ``implementation_bytes``.
"""

from __future__ import annotations


def weight_bytes(rows: int, cols: int, fp8: bool = False, fp4: bool = False) -> int:
    """Bytes of one [rows, cols] expert weight with its scales: bf16 2 bytes per
    element; FP8 1 byte + an fp32 scale per row; FP4 half a byte + an E8M0 byte
    per 32 elements of a row."""
    if fp4:
        return rows * cols // 2 + rows * (cols // 32)
    if fp8:
        return rows * cols + rows * 4
    return rows * cols * 2


def expert_bytes(d: int, F: int, fp8: bool = False, fp4: bool = False) -> int:
    """Weight bytes of one expert: gate_up [2F, d] and down [d, F] with their scales."""
    return weight_bytes(2 * F, d, fp8, fp4) + weight_bytes(d, F, fp8, fp4)


def expert_flops_per_token(d: int, F: int) -> int:
    return 6 * d * F


def layer_work(T: int, d: int, E: int, k: int, F: int, touched: int, fp8: bool = False,
               fp4: bool = False) -> dict:
    byts = touched * expert_bytes(d, F, fp8, fp4) + E * d * 2 + 2 * T * d * 2
    flops = 2 * T * d * E + T * k * expert_flops_per_token(d, F)
    return {"bytes": byts, "flops": flops}


def gate_up_work(T: int, n_rows: int, touched: int, d: int, F: int, fp8: bool = False,
                 fp4: bool = False) -> dict:
    """The gate_up step alone: the touched experts' [2F, d] weights and the T
    token rows of x (algorithmic); the n_rows grouped token rows beyond those T
    and the h [n_rows, F] write (implementation)."""
    return {"bytes": touched * weight_bytes(2 * F, d, fp8, fp4) + T * d * 2,
            "flops": 4 * n_rows * d * F,
            "implementation_bytes": (n_rows - T) * d * 2 + n_rows * F * 2}


def down_work(n_rows: int, touched: int, d: int, F: int, fp8: bool = False,
              fp4: bool = False) -> dict:
    """The down step alone: the touched experts' [d, F] weights (algorithmic);
    the h read and the y [n_rows, d] write (implementation)."""
    return {"bytes": touched * weight_bytes(d, F, fp8, fp4),
            "flops": 2 * n_rows * d * F,
            "implementation_bytes": n_rows * F * 2 + n_rows * d * 2}
