"""Seeded synthetic inputs for the routed-MoE FFN layer (Hy3 shapes).

Workloads (all synthetic; the pages publish no dataset or trained weight for
this layer):

=========  =====  ====  ===  ==  ====  ===============================================
name         T      d    E   k    F    structure
=========  =====  ====  ===  ==  ====  ===============================================
tiny          64   256   16   4   128  x ~ N(0,1), W ~ N(0, 0.02^2)
decode        64  4096  192   8  1536  as tiny: logit std 0.02*sqrt(4096) = 1.28
prefill     4096  4096  192   8  1536  as decode, ~170.7 rows per expert
skewed     16384  4096  192   8  1536  + per-expert logit bias 0.5*ln(Zipf(1.1) rank weight)
fp8         8192  4096  192   8  1536  expert weights e4m3 + fp32 scale per output row
fp4_decode    64  4096  192   6  1536  sqrt-softplus scores, scale 1.5; experts E2M1 +
                                       E8M0 scale per 32 row elements (from the bf16 draw)
=========  =====  ====  ===  ==  ====  ===============================================

The Hy3 sizes (d=4096, 192 routed experts, top-8, expert d_ff=1536, router
scaling 2.826) are those of "Tencent Hy3-295B 架构深度拆解" (pillumina.github.io),
§2.1 hyper-parameter table and §2.3 parameter breakdown.

Draw order, from one torch.Generator seeded with ``seed``: x, W_gate,
W_gate_up (expert by expert), W_down (expert by expert), then -- only for
shapes that ask for them -- the shared expert's W_gate_up and W_down, the
e_score_correction_bias and the route_norm weight. Each weight is drawn as fp32 N(0,1), multiplied by
its standard deviation and rounded to bf16 (round-to-nearest-even, torch's
cast); the score bias stays fp32. The bf16 bit patterns are what both the
oracle and the CUDA path consume.

Layouts (row-major, contiguous):
  x          [T, d]        bf16
  w_gate     [E, d]        bf16
  w_gate_up  [E, 2F, d]    bf16   rows [0, F) are the gate rows, [F, 2F) the up rows
  w_down     [E, d, F]     bf16
  gate_bias  [E]           fp32 or None (added to the router logits)
  score_bias [E]           fp32 or None (e_score_correction_bias: added to the
                           sigmoid scores for the choice of experts only)
  w_shared_gate_up [2F, d], w_shared_down [d, F]   bf16, when the shape has a
                           shared expert (q_/s_shared_* for FP8 shapes)
  route_norm_weight [d]    fp32 or None (the RMSNorm weight of the router input)
FP8 workloads add ``q_gate_up`` [E, 2F, d] / ``q_down`` [E, d, F] as uint8
e4m3 codes and ``s_gate_up`` [E, 2F] / ``s_down`` [E, d] fp32 scales, with the
weight meaning q * s.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class LayerShape:
    T: int
    d: int
    E: int
    k: int
    F: int
    scale: float = 2.826
    x_std: float = 1.0
    w_std: float = 0.02
    zipf_bias: bool = False
    fp8: bool = False
    shared: bool = False          # one shared expert (SwiGLU, d_ff = F), weight 1
    score_bias_std: float = 0.0   # e_score_correction_bias ~ N(0, std^2) when > 0
    route_norm: bool = False      # RMSNorm of the router's input, weight 1 + N(0, 0.1^2)
    route_norm_eps: float = 1e-6
    fp4: bool = False             # routed experts as E2M1 codes + E8M0 block-32 scales
    score_fn: str = "sigmoid"     # or "sqrtsoftplus" (the second routing variant)

    @property
    def R(self) -> int:
        """Routed rows: one per (token, slot)."""
        return self.T * self.k


CONFIGS = {
    "tiny": LayerShape(T=64, d=256, E=16, k=4, F=128),
    "decode": LayerShape(T=64, d=4096, E=192, k=8, F=1536),
    "prefill": LayerShape(T=4096, d=4096, E=192, k=8, F=1536),
    "skewed": LayerShape(T=16384, d=4096, E=192, k=8, F=1536, zipf_bias=True),
    "fp8": LayerShape(T=8192, d=4096, E=192, k=8, F=1536, fp8=True),
    # the second routing and precision variant at the decode shape: top-6
    # sqrt-softplus scores with scale 1.5, FP4 E2M1 experts (block-32 E8M0 scales)
    "fp4_decode": LayerShape(T=64, d=4096, E=192, k=6, F=1536, scale=1.5, fp4=True,
                             score_fn="sqrtsoftplus"),
}


def shape_of(name_or_shape) -> LayerShape:
    if isinstance(name_or_shape, LayerShape):
        return name_or_shape
    return CONFIGS[name_or_shape]


def zipf_logit_bias(E: int, s: float = 1.1) -> torch.Tensor:
    """Per-expert logit bias 0.5*ln(p_r), p_r = r^-s / sum_r' r'^-s, rank r = e+1.

    Expert e takes rank e+1 (identity mapping), so expert 0 is the hottest.
    """
    r = torch.arange(1, E + 1, dtype=torch.float64)
    w = r.pow(-s)
    p = w / w.sum()
    return (0.5 * torch.log(p)).to(torch.float32)


def _normal(gen: torch.Generator, shape, std: float, device) -> torch.Tensor:
    t = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def encode_e4m3_rows(w: torch.Tensor):
    """Per-output-row FP8 (e4m3) encoding of a bf16 weight block [..., rows, cols].

    s_row = max_c |w[row, c]| / 448 (1.0 for an all-zero row);
    q = e4m3(w / s_row) with round-to-nearest-even (torch's cast). Returns the
    uint8 codes and the fp32 scales.
    """
    wf = w.float()
    s = wf.abs().amax(dim=-1) / 448.0
    s = torch.where(s == 0, torch.ones_like(s), s)
    q = (wf / s.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    return q, s.to(torch.float32)


E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # magnitudes of codes 0..7


def encode_e2m1_blocks(w: torch.Tensor):
    """FP4 (OCP MX E2M1) encoding of a bf16 weight block [..., rows, cols], one
    E8M0 scale per 32 consecutive elements of a row (cols % 32 == 0).

    Scale 2^e with e = ceil(log2(amax / 6)) (so every |w| / scale <= 6; e = -127
    for an all-zero block), stored as the byte e + 127; codes round |w| / scale
    to the nearest E2M1 magnitude, ties to the even code, with the sign in bit
    3; two codes per byte, the even element in the low nibble. Returns
    (packed uint8 [..., rows, cols/2], scales uint8 [..., rows, cols/32]).
    """
    wf = w.float()
    *lead, rows, cols = wf.shape
    blk = wf.reshape(*lead, rows, cols // 32, 32)
    amax = blk.abs().amax(dim=-1)
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 6.0)), torch.full_like(amax, -127.0))
    e = e.clamp(-127, 127)
    scale = torch.pow(2.0, e)
    v = (blk / scale.unsqueeze(-1)).clamp(-6.0, 6.0)
    grid = torch.tensor(E2M1_GRID, dtype=torch.float32, device=w.device)
    a = v.abs().contiguous()
    hi = torch.searchsorted(grid, a).clamp(max=7)     # first grid value >= a
    lo = (hi - 1).clamp(min=0)
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = torch.where(take_hi, hi, lo)
    code = torch.where(a == grid[hi], hi, code)      # exact grid values
    nib = (code + ((v < 0) & (code > 0)).to(code.dtype) * 8).to(torch.uint8)
    nib = nib.reshape(*lead, rows, cols)
    packed = (nib[..., 0::2] | (nib[..., 1::2] << 4)).to(torch.uint8)
    return packed, (e + 127).to(torch.uint8)


def tensor_shapes(cfg) -> dict:
    """Shapes of the layer's tensors (the layouts listed in the module docstring)."""
    cfg = shape_of(cfg)
    T, d, E, F = cfg.T, cfg.d, cfg.E, cfg.F
    return {"x": (T, d), "w_gate": (E, d), "w_gate_up": (E, 2 * F, d), "w_down": (E, d, F),
            "gate_bias": (E,), "s_gate_up": (E, 2 * F), "s_down": (E, d)}


def make_layer(cfg, seed: int = 0, device="cpu", T: Optional[int] = None,
               with_experts: bool = True) -> dict:
    """Draw one layer's inputs. ``T`` overrides the token count of ``cfg``.

    ``with_experts=False`` stops after x and W_gate (the first two draws), for
    router-only work; those two tensors are identical to the full draw's.
    """
    cfg = shape_of(cfg)
    if T is not None:
        cfg = dataclasses.replace(cfg, T=T)
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    shp = tensor_shapes(cfg)
    E = cfg.E

    x = _normal(gen, shp["x"], cfg.x_std, dev)
    w_gate = _normal(gen, shp["w_gate"], cfg.w_std, dev)
    if not with_experts:
        return {"cfg": cfg, "seed": seed, "x": x, "w_gate": w_gate,
                "gate_bias": zipf_logit_bias(E).to(dev) if cfg.zipf_bias else None}
    w_gate_up = torch.empty(shp["w_gate_up"], dtype=torch.bfloat16, device=dev)
    for e in range(E):
        w_gate_up[e] = _normal(gen, shp["w_gate_up"][1:], cfg.w_std, dev)
    w_down = torch.empty(shp["w_down"], dtype=torch.bfloat16, device=dev)
    for e in range(E):
        w_down[e] = _normal(gen, shp["w_down"][1:], cfg.w_std, dev)

    out = {
        "cfg": cfg,
        "seed": seed,
        "x": x,
        "w_gate": w_gate,
        "w_gate_up": w_gate_up,
        "w_down": w_down,
        "gate_bias": zipf_logit_bias(E).to(dev) if cfg.zipf_bias else None,
        "score_bias": None,
    }
    if cfg.shared:
        out["w_shared_gate_up"] = _normal(gen, shp["w_gate_up"][1:], cfg.w_std, dev)
        out["w_shared_down"] = _normal(gen, shp["w_down"][1:], cfg.w_std, dev)
    if cfg.score_bias_std > 0:
        out["score_bias"] = torch.randn((E,), generator=gen, dtype=torch.float32,
                                        device=dev) * cfg.score_bias_std
    if cfg.fp4:
        # one expert at a time (blocks are independent): bounded temporaries at
        # the full Hy3 sizes
        d, F = cfg.d, cfg.F
        q4_gu = torch.empty((E, 2 * F, d // 2), dtype=torch.uint8, device=dev)
        s4_gu = torch.empty((E, 2 * F, d // 32), dtype=torch.uint8, device=dev)
        q4_d = torch.empty((E, d, F // 2), dtype=torch.uint8, device=dev)
        s4_d = torch.empty((E, d, F // 32), dtype=torch.uint8, device=dev)
        for e in range(E):
            q4_gu[e], s4_gu[e] = encode_e2m1_blocks(w_gate_up[e])
            q4_d[e], s4_d[e] = encode_e2m1_blocks(w_down[e])
        out.update(q4_gate_up=q4_gu, s4_gate_up=s4_gu, q4_down=q4_d, s4_down=s4_d)
    out["route_norm_weight"] = None
    if cfg.route_norm:
        out["route_norm_weight"] = 1.0 + 0.1 * torch.randn((cfg.d,), generator=gen,
                                                           dtype=torch.float32, device=dev)
    if cfg.fp8:
        q_gu = torch.empty(shp["w_gate_up"], dtype=torch.uint8, device=dev)
        s_gu = torch.empty(shp["s_gate_up"], dtype=torch.float32, device=dev)
        q_d = torch.empty(shp["w_down"], dtype=torch.uint8, device=dev)
        s_d = torch.empty(shp["s_down"], dtype=torch.float32, device=dev)
        for e in range(E):
            q_gu[e], s_gu[e] = encode_e4m3_rows(w_gate_up[e])
            q_d[e], s_d[e] = encode_e4m3_rows(w_down[e])
        out.update(q_gate_up=q_gu, s_gate_up=s_gu, q_down=q_d, s_down=s_d)
        if cfg.shared:
            qs_gu, ss_gu = encode_e4m3_rows(out["w_shared_gate_up"])
            qs_d, ss_d = encode_e4m3_rows(out["w_shared_down"])
            out.update(q_shared_gate_up=qs_gu, s_shared_gate_up=ss_gu, q_shared_down=qs_d,
                       s_shared_down=ss_d)
    return out
