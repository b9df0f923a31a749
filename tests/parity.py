"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle.

Tolerances (fixed by the layer's parity specification):
  * routing: selected expert sets equal, bit-exact, for every token whose gap
    between the k-th and (k+1)-th oracle score is >= 1e-5; tokens below that
    gap are reported and their selection only has to be a valid top-k within
    the gap; routing weights within 2e-5 relative (fp32 logits, sigmoid and
    renormalisation against fp64);
  * layer output (bf16): relative L2 <= 1e-2 and max-abs <= 5e-2.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_moe_transformer_gemm_b200 import moe

NEAR_TIE = 1e-5
REL_L2 = 1e-2
MAX_ABS = 5e-2
W_RTOL = 2e-5


def route_options(layer):
    """The layer's router options (score bias, route_norm, score function)."""
    cfg = layer["cfg"]
    return moe.route_options(layer.get("score_bias"), layer.get("route_norm_weight"),
                             getattr(cfg, "route_norm_eps", 1e-6),
                             getattr(cfg, "score_fn", "sigmoid"))


def gpu_route(layer, path=None):
    cfg = moe.config_of(layer["cfg"], path)
    T, k = layer["cfg"].T, layer["cfg"].k
    ws = moe.workspace(cfg)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    opt = route_options(layer)
    moe.moe_route3(cfg, layer["x"], layer["w_gate"], layer.get("gate_bias"), opt, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    return idx.cpu().numpy(), w.cpu().numpy()


def gpu_forward(layer, path=None, ws=None, out=None):
    cfg = moe.config_of(layer["cfg"], path)
    T, d = layer["cfg"].T, layer["cfg"].d
    if ws is None:
        ws = moe.workspace(cfg)
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    opt = route_options(layer)
    moe.moe_forward3(cfg, layer["x"], layer["w_gate"], layer.get("gate_bias"), opt,
                     *moe.layer_args(layer), out, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    return out


def check_route(gpu_idx, gpu_w, ref):
    """Compare the GPU routing with the oracle's (all tokens). Returns near-tie token ids."""
    T, k = gpu_idx.shape
    near = np.nonzero(ref["gap"] < NEAR_TIE)[0]
    mism = []
    for t in range(T):
        g, o = set(gpu_idx[t].tolist()), set(ref["idx"][t].tolist())
        if g != o:
            if t in near:
                continue
            mism.append(t)
    assert not mism, f"routing differs on {len(mism)} tokens (first {mism[:8]})"
    # weights by matched expert id, tokens with equal sets
    for t in range(T):
        o_ids = ref["idx"][t].tolist()
        if set(gpu_idx[t].tolist()) != set(o_ids):
            continue
        o_w = dict(zip(o_ids, ref["w"][t].tolist()))
        for j, e in enumerate(gpu_idx[t].tolist()):
            assert abs(gpu_w[t, j] - o_w[e]) <= W_RTOL * abs(o_w[e]) + 1e-7, (t, e)
    return near


def check_near_tie_selection(gpu_idx, scores, t, k):
    """A near-tie token's GPU set is a valid top-k of the oracle scores within the gap."""
    s = scores[t]
    kth = np.sort(s)[::-1][k - 1]
    assert all(s[e] >= kth - NEAR_TIE for e in gpu_idx[t]), t


def oracle_out_with_selection(O, t, experts):
    """Oracle output of token t when it is routed to ``experts`` (weights from the
    oracle's fp64 scores, renormalised over that set; the shared expert, if any,
    added last with weight 1)."""
    scores = oracle.route(O.x[t:t + 1], O.wg, O.k, O.scale, O.gate_bias, want_scores=True,
                          norm_w=O.norm_w, norm_eps=O.norm_eps, score_fn=O.score_fn)["scores"]
    experts = np.asarray(experts, np.int32)
    xrows = np.repeat(O.x[t:t + 1], len(experts), axis=0)
    if O.fp4:
        y = oracle.expert_rows_fp4(xrows, experts, O.wgu4, O.sgu8, O.wd4, O.sd8)
    else:
        y = oracle.expert_rows(xrows, experts, O.wgu, O.wd, O.s_gu, O.s_d)
    s = scores[0, experts]
    w = O.scale * s / s.sum()
    if O.sh_wgu is not None:
        y_sh = oracle.expert_rows(O.x[t:t + 1], np.zeros(1, np.int32), O.sh_wgu[None],
                                  O.sh_wd[None], None if O.sh_s_gu is None else O.sh_s_gu[None],
                                  None if O.sh_s_d is None else O.sh_s_d[None])
        y = np.concatenate([y, y_sh])
        w = np.concatenate([w, [1.0]])
    return oracle.combine(y[None], w[None])[0]


def compare_out(gpu_bits: np.ndarray, ref_bits: np.ndarray):
    g = oracle.double_from_bf16(gpu_bits)
    o = oracle.double_from_bf16(ref_bits)
    rel = float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30))
    mx = float(np.max(np.abs(g - o))) if g.size else 0.0
    return rel, mx


def check_forward(layer, out_gpu, tokens=None, route_gpu=None):
    """Oracle forward on ``tokens`` (all when None) and element-wise comparison.

    Near-tie tokens whose GPU selection differs from the oracle's are compared
    against the oracle evaluated on the GPU's selection.
    """
    O = oracle.OracleLayer(layer)
    ref = oracle.forward_tokens(O, tokens)
    toks = ref["tokens"]
    gpu_bits = oracle.bf16_bits(out_gpu)[toks]
    want = ref["out_bf16"].copy()
    swapped = []
    if route_gpu is not None:
        gi = route_gpu[0][toks]
        for r, t in enumerate(toks):
            if set(gi[r].tolist()) != set(ref["idx"][r].tolist()):
                assert ref["gap"][r] < NEAR_TIE, f"token {t} routed differently without a near tie"
                want[r] = oracle_out_with_selection(O, t, gi[r])
                swapped.append(int(t))
    rel, mx = compare_out(gpu_bits, want)
    assert rel <= REL_L2, f"rel-L2 {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS, f"max-abs {mx:.3e} > {MAX_ABS}"
    return {"rel_l2": rel, "max_abs": mx, "n_tokens": int(len(toks)), "swapped": swapped}


def sample_tokens(T: int, n: int = 48, seed: int = 0) -> np.ndarray:
    """First 8, last 8 and a seeded random sample of the rest."""
    if T <= n + 16:
        return np.arange(T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(8, T - 8), size=n, replace=False)
    return np.unique(np.concatenate([np.arange(8), mid, np.arange(T - 8, T)])).astype(np.int32)


NMAX = 256       # token rows per tile of the bf16 and FP4 SM-pair GEMMs
FP8_NMAX = 192   # FP8 and FP4: the widened weights share tensor memory with the accumulators


def gemm_tiles(counts, nmax: int = NMAX, unit: int = 32):
    """The token tiles of the SM-pair grouped GEMMs: expert e's n_e grouped rows
    split into nt = ceil(n_e / nmax) tiles, all but the last of unit*q rows
    (q = ceil(ceil(n_e / unit) / nt), or nmax / unit if that left the last tile
    empty). Yields (e, first row, length) with rows counted from the expert's
    first grouped row."""
    for e, n in enumerate(np.asarray(counts).tolist()):
        if n == 0:
            continue
        nt = (n + nmax - 1) // nmax
        q = (-(-n // unit) + nt - 1) // nt
        if unit * q * (nt - 1) >= n:
            q = nmax // unit
        for j in range(nt):
            yield e, j * unit * q, unit * q if j < nt - 1 else n - unit * q * (nt - 1)


FP8_SUB = 192    # FP8 down with two token sub-tiles: rows per accumulator


def fp8_down_tiles(counts, T: int, k: int, E: int):
    """The token tiles of the FP8 SM-pair down GEMM, as (e, first row, length):
    once the experts average at least 128 grouped rows (T*k >= 128 E) a pair
    tile holds up to 2*FP8_SUB rows (gemm_tiles with that maximum) and its two
    accumulators take rows [0, FP8_SUB) and [FP8_SUB, length); below that the
    tiles hold up to FP8_NMAX rows, as gate_up's always do."""
    if T * k < 128 * E:
        yield from gemm_tiles(counts, FP8_NMAX)
        return
    for e, start, n in gemm_tiles(counts, 2 * FP8_SUB):
        yield e, start, min(n, FP8_SUB)
        if n > FP8_SUB:
            yield e, start + FP8_SUB, n - FP8_SUB


def tile_cover_tokens(idx: np.ndarray, E: int, edge: int = 32, nmax: int = NMAX,
                      tiles=None) -> np.ndarray:
    """Tokens that put a grouped row into the first and into the last ``edge``
    rows of every (expert, token tile) of the grouped GEMMs (``tiles``, else
    gemm_tiles with ``nmax``), chosen greedily
    (each token brings k rows). The grouping is the oracle's (row_of), so the
    rows are those the GPU's GEMMs compute for the same routing."""
    T, k = idx.shape
    g = oracle.permute(idx, E)
    offsets, row_of = g["offsets"], g["row_of"]
    token_of_row = np.empty(T * k, dtype=np.int64)
    token_of_row[row_of] = np.arange(T * k) // k
    targets = {}   # target id -> set of candidate tokens
    for e, start, n in (gemm_tiles(g["counts"], nmax) if tiles is None else tiles):
        r0 = offsets[e] + start
        for lo, hi in ((r0, r0 + min(edge, n)), (r0 + n - min(edge, n), r0 + n)):
            targets[len(targets)] = set(token_of_row[lo:hi].tolist())
    covers = {}
    for tid, toks in targets.items():
        for t in toks:
            covers.setdefault(t, set()).add(tid)
    left, chosen = set(targets), []
    while left:
        t = max(covers, key=lambda c: (len(covers[c] & left), -c))
        chosen.append(t)
        left -= covers[t]
    return np.array(sorted(chosen), dtype=np.int32)
