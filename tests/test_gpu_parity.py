"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small shapes are compared on every token; the full Hy3 shapes route every
token through both sides and compare the layer output on a seeded sample of
tokens, in the launch configuration the benchmark uses (moe_forward with the
automatic path choice). Tolerances are in tests/parity.py.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
import parity
from sparse_moe_transformer_gemm_b200 import build as moe_build
from sparse_moe_transformer_gemm_b200 import moe
from synthetic import CONFIGS, LayerShape, make_layer

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": CONFIGS["tiny"],
    # several 128-row weight tiles, ~75 rows per expert, ragged token tiles
    "ragged": LayerShape(T=300, d=512, E=32, k=8, F=384),
    "single_token": LayerShape(T=1, d=256, E=16, k=4, F=128),
    "k_equals_E": LayerShape(T=20, d=256, E=8, k=8, F=128),
    "top1": LayerShape(T=50, d=256, E=16, k=1, F=128),
    "tiny_fp8": dataclasses.replace(CONFIGS["tiny"], fp8=True),
    # FP8 weights on the pair-of-SMs tensor-core path (d, d_ff multiples of 256)
    "pair_fp8": LayerShape(T=333, d=768, E=24, k=6, F=512, fp8=True),
    # FP8 down with two token sub-tiles per pair tile (T*k >= 128 E): Zipf-hot
    # experts take more than one pair tile, the rest one or two sub-tiles
    "pair_fp8_subtiles": LayerShape(T=700, d=768, E=8, k=2, F=256, fp8=True, zipf_bias=True),
    "ragged_skewed": LayerShape(T=300, d=512, E=32, k=8, F=384, zipf_bias=True),
    # d and d_ff multiples of 256: the pair-of-SMs GEMMs (several tiles, ragged tokens)
    "pair_small": LayerShape(T=200, d=512, E=16, k=4, F=512),
    "pair_ragged": LayerShape(T=333, d=768, E=24, k=6, F=256, zipf_bias=True),
    # ~375 rows per expert: two token tiles each (256 + a ragged tail), rows
    # gathered by index with cp.async in the gate_up GEMM
    "pair_multi": LayerShape(T=1500, d=512, E=8, k=2, F=256),
    # fewer grouped rows (6) than the smallest token box (16 rows)
    "pair_tiny": LayerShape(T=3, d=512, E=8, k=2, F=256),
    # the CUDA-core router (k > 8, or E not a multiple of 4)
    "k12": LayerShape(T=100, d=256, E=32, k=12, F=128),
    "e18": LayerShape(T=90, d=256, E=18, k=4, F=128),
}


@pytest.fixture(scope="module", autouse=True)
def _built():
    moe_build.build()
    oracle.build()
    assert torch.cuda.is_available()
    torch.cuda.init()


def _free(*objs):
    for o in objs:
        del o
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("path", [None, "stream", "gemm"])
def test_small_shapes_every_token(name, path):
    sh = SMALL[name]
    if path == "gemm" and sh.fp8 and (sh.d % 256 or sh.F % 256):
        pytest.skip("FP8 weights on the tensor cores need d and d_ff multiples of 256")
    layer = make_layer(SMALL[name], seed=1, device="cuda")
    route = parity.gpu_route(layer, path)
    O = oracle.OracleLayer(layer)
    ref = oracle.route(O.x, O.wg, O.k, O.scale, O.gate_bias)
    parity.check_route(*route, ref)
    out = parity.gpu_forward(layer, path)
    res = parity.check_forward(layer, out, None, route)
    print(name, path, res)


@pytest.mark.parametrize("path", ["stream", "gemm"])
def test_decode_shape_every_token_on_both_expert_paths(path):
    """The Hy3 decode shape (T=64) with the experts forced onto the
    weight-streaming kernels or the tensor-core GEMMs: every token's routing
    and layer output against the oracle."""
    layer = make_layer(CONFIGS["decode"], seed=0, device="cuda")
    route = parity.gpu_route(layer, path)
    O = oracle.OracleLayer(layer)
    parity.check_route(*route, oracle.route(O.x, O.wg, O.k, O.scale, O.gate_bias))
    out = parity.gpu_forward(layer, path)
    res = parity.check_forward(layer, out, None, route)
    print("decode", path, res)
    _free(layer, out)


@pytest.mark.parametrize("name", ["decode", "prefill", "skewed", "fp8"])
def test_hy3_shapes(name):
    shape = CONFIGS[name]
    layer = make_layer(shape, seed=0, device="cuda")
    route = parity.gpu_route(layer)
    O = oracle.OracleLayer(layer)
    ref = oracle.route(O.x, O.wg, O.k, O.scale, O.gate_bias)
    near = parity.check_route(*route, ref)
    out = parity.gpu_forward(layer)
    # a seeded sample, the first near ties, and tokens that put a checked row
    # at the head and at the tail of every (expert, token tile) of the grouped
    # GEMMs under the GPU's routing
    toks = parity.sample_tokens(shape.T, n=48 if shape.T > 64 else 64)
    counts = np.bincount(route[0].ravel(), minlength=shape.E)
    # FP8: gate_up's tiles and down's (two sub-tiles per pair tile at this shape)
    tiles = (list(parity.gemm_tiles(counts, parity.FP8_NMAX)) +
             list(parity.fp8_down_tiles(counts, shape.T, shape.k, shape.E)) if shape.fp8 else
             list(parity.gemm_tiles(counts, parity.NMAX)))
    cover = parity.tile_cover_tokens(route[0], shape.E, tiles=tiles)
    toks = np.unique(np.concatenate([toks, near[:8].astype(np.int32), cover]))
    res = parity.check_forward(layer, out, toks, route)
    n_tiles = len(tiles)
    print(name, "near-tie tokens:", len(near), near[:16].tolist(),
          f"checked tokens {len(toks)} (rows {len(toks) * shape.k}), tiles covered {n_tiles}",
          res)
    _free(layer, out)


@pytest.mark.parametrize("fmt", ["fp8", "fp4"])
@pytest.mark.parametrize("T", [193, 700])
def test_quantised_all_tokens_to_the_same_experts(T, fmt):
    """FP8 / FP4 weights on the pair GEMMs with every token on experts 0..3: T
    rows each, in token tiles of at most 192 rows (193 as 128 + 65, 700 as
    3 x 192 + 124); FP8 down at T=700 (T*k >= 128 E) in two pair tiles of 352
    and 348 rows, each split 192 + the rest between its accumulators; every
    token against the oracle."""
    shape = LayerShape(T=T, d=512, E=16, k=4, F=256, fp8=fmt == "fp8", fp4=fmt == "fp4")
    layer = make_layer(shape, seed=5, device="cuda")
    b = torch.zeros(shape.E, dtype=torch.float32, device="cuda")
    b[:4] = 40.0
    layer["gate_bias"] = b
    route = parity.gpu_route(layer)
    assert np.all(np.sort(route[0], axis=1) == np.arange(4))
    counts = np.bincount(route[0].ravel())
    tiles = parity.gemm_tiles(counts, parity.FP8_NMAX)
    assert [n for e, _, n in tiles if e == 0] == ([128, 65] if T == 193 else [192, 192, 192, 124])
    if fmt == "fp8":
        down = parity.fp8_down_tiles(counts, T, shape.k, shape.E)
        assert [n for e, _, n in down if e == 0] == ([128, 65] if T == 193 else
                                                    [192, 160, 192, 156])
    out = parity.gpu_forward(layer, "gemm")
    parity.check_forward(layer, out, None, route)


@pytest.mark.parametrize("T", [1, 7, 64, 128, 129, 300])
def test_hy3_router_on_both_kernels(T):
    """The Hy3 router shape (d=4096, E=192, k=8, zipf bias) at batch sizes on
    both sides of the switch between the K-split CUDA-core router (T <= 128)
    and the tensor-core one (T >= 129)."""
    shape = dataclasses.replace(CONFIGS["decode"], T=T, zipf_bias=True)
    layer = make_layer(shape, seed=T, device="cuda", with_experts=False)
    route = parity.gpu_route(layer)
    ref = oracle.route(oracle.bf16_bits(layer["x"]), oracle.bf16_bits(layer["w_gate"]), shape.k,
                       shape.scale, layer["gate_bias"].cpu().numpy())
    parity.check_route(*route, ref)


@pytest.mark.parametrize("T,F", [(64, 128), (700, 128), (700, 256)])
def test_all_tokens_to_the_same_experts(T, F):
    """A logit bias of +40 on experts 0..3 sends every token to them (T rows each,
    split into several token tiles when T > 256); the other twelve are empty.
    F = 256 runs the pair-of-SMs GEMMs, F = 128 the single-SM ones."""
    shape = dataclasses.replace(CONFIGS["tiny"], T=T, F=F)
    layer = make_layer(shape, seed=2, device="cuda")
    b = torch.zeros(shape.E, dtype=torch.float32, device="cuda")
    b[:4] = 40.0
    layer["gate_bias"] = b
    route = parity.gpu_route(layer)
    assert np.all(np.sort(route[0], axis=1) == np.arange(4))
    for path in (None, "stream", "gemm"):
        out = parity.gpu_forward(layer, path)
        parity.check_forward(layer, out, None, route)


def test_permute_is_bit_exact():
    shape = LayerShape(T=3000, d=256, E=64, k=8, F=128)
    layer = make_layer(shape, seed=3, device="cuda", with_experts=False)
    cfg = moe.config_of(shape)
    ws = moe.workspace(cfg)
    T, k, E, d = shape.T, shape.k, shape.E, shape.d
    idx, _ = parity.gpu_route(layer)
    idx_d = torch.from_numpy(idx).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    xp = torch.empty((T * k, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(cfg, idx_d, layer["x"], counts, offsets, row_of, xp, ws)
    torch.cuda.synchronize()
    ref = oracle.permute(idx, E)
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    assert np.array_equal(offsets.cpu().numpy(), ref["offsets"])
    assert np.array_equal(row_of.cpu().numpy(), ref["row_of"])
    xb = oracle.bf16_bits(layer["x"])
    xpb = oracle.bf16_bits(xp)
    rows = ref["row_of"].reshape(T, k)
    for j in range(k):
        assert np.array_equal(xpb[rows[:, j]], xb)


@pytest.mark.parametrize("T,E", [(3000, 64), (512, 64), (500, 256), (1, 16)])
def test_permute_index_is_bit_exact(T, E):
    """moe_permute_index: the same grouping as moe_permute, plus token_of_row,
    the inverse of row_of (token of each grouped row). At most 4096 slots run
    the one-CTA kernel, more the rank/scan/scatter launches."""
    shape = LayerShape(T=T, d=256, E=E, k=8, F=128)
    layer = make_layer(shape, seed=3, device="cuda", with_experts=False)
    cfg = moe.config_of(shape)
    ws = moe.workspace(cfg)
    T, k, E = shape.T, shape.k, shape.E
    idx, _ = parity.gpu_route(layer)
    idx_d = torch.from_numpy(idx).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    tok = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    moe.moe_permute_index(cfg, idx_d, counts, offsets, row_of, tok, ws)
    torch.cuda.synchronize()
    ref = oracle.permute(idx, E)
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    assert np.array_equal(offsets.cpu().numpy(), ref["offsets"])
    assert np.array_equal(row_of.cpu().numpy(), ref["row_of"])
    want = np.empty(T * k, dtype=np.int32)
    want[ref["row_of"]] = np.arange(T * k) // k
    assert np.array_equal(tok.cpu().numpy(), want)


@pytest.mark.parametrize("name,path", [
    ("pair_small", None), ("pair_ragged", None), ("pair_multi", None), ("pair_ragged", "gemm"),
    ("ragged", None),
    ("tiny", "stream"), ("pair_fp8", None), ("single_token", None)])
def test_gate_up_gather_equals_permuted_copy_bitwise(name, path):
    """moe_expert_gate_up_gather (rows of x read by index inside the GEMM on the
    bf16 SM-pair path, a row-gather kernel elsewhere) gives the same bits as
    moe_permute + moe_expert_gate_up."""
    shape = SMALL[name]
    layer = make_layer(shape, seed=11, device="cuda")
    cfg = moe.config_of(shape, path)
    ws = moe.workspace(cfg)
    T, k, E, d, F = shape.T, shape.k, shape.E, shape.d, shape.F
    R = T * k
    idx, _ = parity.gpu_route(layer)
    idx_d = torch.from_numpy(idx).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    row_of = torch.empty(R, dtype=torch.int32, device="cuda")
    tok = torch.empty(R, dtype=torch.int32, device="cuda")
    xp = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    h_copy = torch.empty((R, F), dtype=torch.bfloat16, device="cuda")
    h_gather = torch.empty((R, F), dtype=torch.bfloat16, device="cuda")
    wgu, sgu, _, _ = moe.layer_args(layer)
    moe.moe_permute(cfg, idx_d, layer["x"], counts, offsets, row_of, xp, ws)
    moe.moe_expert_gate_up(cfg, xp, offsets, wgu, sgu, h_copy, ws)
    moe.moe_permute_index(cfg, idx_d, counts, offsets, row_of, tok, ws)
    moe.moe_expert_gate_up_gather(cfg, layer["x"], tok, offsets, wgu, sgu, h_gather, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    assert torch.equal(h_copy, h_gather)


def test_pack_weights_is_a_block_permutation():
    """moe_pack_weights: 128-row x 64-column blocks, ordered by expert, row block,
    column block, row-major inside -- checked against torch's view/permute."""
    E, F, d = 3, 256, 512
    cfg = moe.config(T=1, d=d, E=E, k=1, d_ff=F)
    g = torch.Generator(device="cpu").manual_seed(9)
    for which, rows, cols in ((moe.MOE_WEIGHTS_GATE_UP, 2 * F, d), (moe.MOE_WEIGHTS_DOWN, d, F)):
        w = torch.randn((E, rows, cols), generator=g).to(torch.bfloat16).cuda()
        wp = torch.empty_like(w)
        moe.moe_pack_weights(cfg, which, w, wp)
        torch.cuda.synchronize()
        want = w.view(E, rows // 128, 128, cols // 64, 64).permute(0, 1, 3, 2, 4).contiguous()
        assert torch.equal(wp.view(-1), want.view(-1))


@pytest.mark.parametrize("shape", [
    SMALL["pair_small"], SMALL["pair_ragged"],
    LayerShape(T=700, d=512, E=16, k=8, F=256),   # 5600 slots: the permuted-copy path
    CONFIGS["decode"],
], ids=["pair_small", "pair_ragged", "copy_path", "hy3_decode"])
def test_packed_weights_give_identical_outputs(shape):
    """MOE_FLAG_PACKED_WEIGHTS changes only where the weight tiles are read from:
    moe_forward's output is bitwise the same as with the row-major weights."""
    layer = make_layer(shape, seed=13, device="cuda")
    want = parity.gpu_forward(layer).clone()
    cfg = moe.config_of(shape, packed=True)
    gu, dn = moe.pack_layer_weights(cfg, layer["w_gate_up"], layer["w_down"])
    ws = moe.workspace(cfg)
    out = torch.empty_like(want)
    moe.moe_forward(cfg, layer["x"], layer["w_gate"], layer.get("gate_bias"), gu, None, dn, None,
                    out, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    assert torch.equal(out, want)
    _free(layer, gu, dn)


# The complete Hy3 MoE block: e_score_correction_bias (choice only) and one
# shared expert (expert E of the weights, weight 1, added last in the combine).
BLOCK = {
    # pair GEMMs, tensor-core router
    "block_pair": LayerShape(T=200, d=512, E=16, k=4, F=512, shared=True, score_bias_std=0.05),
    # single-SM GEMMs (d_ff % 256 != 0), tensor-core router
    "block_ragged": LayerShape(T=300, d=512, E=32, k=8, F=384, shared=True,
                               score_bias_std=0.05),
    # CUDA-core router (k > 8)
    "block_k12": LayerShape(T=100, d=256, E=32, k=12, F=128, shared=True, score_bias_std=0.05),
    # FP8 weights for the routed and the shared expert
    "block_fp8": LayerShape(T=333, d=768, E=24, k=6, F=512, fp8=True, shared=True,
                            score_bias_std=0.05),
    # T*(k+1) = 6300 slots: the permuted-copy grouping
    "block_copy": LayerShape(T=700, d=512, E=16, k=8, F=256, shared=True, score_bias_std=0.05),
}


@pytest.mark.parametrize("name", sorted(BLOCK))
@pytest.mark.parametrize("path", [None, "stream", "gemm"])
def test_complete_block_every_token(name, path):
    sh = BLOCK[name]
    if path == "gemm" and sh.fp8 and (sh.d % 256 or sh.F % 256):
        pytest.skip("FP8 weights on the tensor cores need d and d_ff multiples of 256")
    layer = make_layer(sh, seed=31, device="cuda")
    route = parity.gpu_route(layer, path)
    O = oracle.OracleLayer(layer)
    ref = oracle.route(O.x, O.wg, O.k, O.scale, O.gate_bias, score_bias=O.score_bias)
    parity.check_route(*route, ref)
    out = parity.gpu_forward(layer, path)
    res = parity.check_forward(layer, out, None, route)
    print(name, path, res)


def test_complete_hy3_block_decode():
    """Hy3 shapes with the shared expert and a score bias: every token's routing
    and output (decode, so the in-GEMM row gather on 193 experts)."""
    shape = dataclasses.replace(CONFIGS["decode"], shared=True, score_bias_std=0.05)
    layer = make_layer(shape, seed=3, device="cuda")
    route = parity.gpu_route(layer)
    O = oracle.OracleLayer(layer)
    ref = oracle.route(O.x, O.wg, O.k, O.scale, O.gate_bias, score_bias=O.score_bias)
    near = parity.check_route(*route, ref)
    out = parity.gpu_forward(layer)
    res = parity.check_forward(layer, out, None, route)
    print("hy3 block decode, near ties:", len(near), res)
    _free(layer, out)


def test_route2_without_score_bias_is_moe_route_bitwise():
    layer = make_layer(SMALL["pair_small"], seed=6, device="cuda", with_experts=False)
    a = parity.gpu_route(layer)
    cfg = moe.config_of(layer["cfg"])
    ws = moe.workspace(cfg)
    T, k = layer["cfg"].T, layer["cfg"].k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, layer["x"], layer["w_gate"], None, idx, w, ws)
    torch.cuda.synchronize()
    assert np.array_equal(a[0], idx.cpu().numpy()) and np.array_equal(a[1], w.cpu().numpy())


def test_complete_block_with_packed_weights_is_bitwise_the_same():
    shape = BLOCK["block_pair"]
    layer = make_layer(shape, seed=8, device="cuda")
    want = parity.gpu_forward(layer).clone()
    cfg = moe.config_of(shape, packed=True)
    wgu, _, wd, _ = moe.layer_args(layer)
    gu, dn = moe.pack_layer_weights(cfg, wgu, wd)
    ws = moe.workspace(cfg)
    out = torch.empty_like(want)
    moe.moe_forward2(cfg, layer["x"], layer["w_gate"], None, layer["score_bias"], gu, None, dn,
                     None, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    assert torch.equal(out, want)


# route_norm (RMSNorm of the router's input; the experts take x)
NORM = {
    "norm_decode": dataclasses.replace(CONFIGS["decode"], route_norm=True),
    "norm_tc_sized": LayerShape(T=300, d=512, E=32, k=8, F=256, route_norm=True),
    "norm_block": LayerShape(T=200, d=512, E=16, k=4, F=512, shared=True, score_bias_std=0.05,
                             route_norm=True),
}


@pytest.mark.parametrize("name", sorted(NORM))
def test_route_norm_every_token(name):
    sh = NORM[name]
    layer = make_layer(sh, seed=51, device="cuda")
    route = parity.gpu_route(layer)
    O = oracle.OracleLayer(layer)
    ref = oracle.route(O.x, O.wg, O.k, O.scale, O.gate_bias, score_bias=O.score_bias,
                       norm_w=O.norm_w, norm_eps=O.norm_eps)
    parity.check_route(*route, ref)
    out = parity.gpu_forward(layer)
    res = parity.check_forward(layer, out, None, route)
    print(name, res)
    _free(layer, out)


def test_fp32_combine_keeps_small_terms():
    """Hy3 commentary §2.3 example: one branch output 8.2 and seven of 0.03 (all
    already bf16). An fp32 sum gives 8.375 after the cast; a bf16 running sum
    would stay at 8.1875."""
    cfg = moe.config(T=1, d=128, E=8, k=8, d_ff=128)
    ws = moe.workspace(cfg)
    y = torch.full((8, 128), 0.030029296875, dtype=torch.bfloat16, device="cuda")
    y[0] = 8.1875
    row_of = torch.arange(8, dtype=torch.int32, device="cuda")
    w = torch.ones(8, dtype=torch.float32, device="cuda")
    out = torch.empty((1, 128), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(cfg, y, row_of, w, out, ws)
    torch.cuda.synchronize()
    assert torch.all(out.float() == 8.375)


def test_stage_calls_match_moe_forward_bitwise():
    shape = SMALL["ragged"]
    layer = make_layer(shape, seed=4, device="cuda")
    cfg = moe.config_of(shape)
    ws = moe.workspace(cfg)
    T, k, E, d, F = shape.T, shape.k, shape.E, shape.d, shape.F
    R = T * k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    row_of = torch.empty(R, dtype=torch.int32, device="cuda")
    xp = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    h = torch.empty((R, F), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    wgu, sgu, wd, sd = moe.layer_args(layer)
    moe.moe_route(cfg, layer["x"], layer["w_gate"], None, idx, w, ws)
    moe.moe_permute(cfg, idx, layer["x"], counts, offsets, row_of, xp, ws)
    moe.moe_expert_gate_up(cfg, xp, offsets, wgu, sgu, h, ws)
    moe.moe_expert_down(cfg, h, offsets, wd, sd, y, ws)
    moe.moe_combine(cfg, y, row_of, w, out, ws)
    full = parity.gpu_forward(layer)
    assert torch.equal(out, full)
    # the expert pieces against the oracle, row by row
    xpb = oracle.bf16_bits(xp)
    rows = np.arange(R)
    experts = np.searchsorted(offsets.cpu().numpy(), rows, side="right") - 1
    O = oracle.OracleLayer(layer)
    y_ref, h_ref = oracle.expert_rows(xpb, experts.astype(np.int32), O.wgu, O.wd, want_h=True)
    h_gpu = oracle.double_from_bf16(oracle.bf16_bits(h))
    rel_h = np.linalg.norm(h_gpu - h_ref) / np.linalg.norm(h_ref)
    assert rel_h < 4e-3, rel_h
    y_gpu = oracle.double_from_bf16(oracle.bf16_bits(y))
    rel_y = np.linalg.norm(y_gpu - y_ref) / np.linalg.norm(y_ref)
    assert rel_y < 8e-3, rel_y


def test_repeated_calls_are_bitwise_deterministic():
    layer = make_layer(SMALL["ragged_skewed"], seed=5, device="cuda")
    a = parity.gpu_forward(layer).clone()
    b = parity.gpu_forward(layer)
    assert torch.equal(a, b)


# The second routing and precision variant (the V4-Flash column of
# "Tencent Hy3-295B 架构深度拆解" §2.2): sqrt(softplus) scores (scale 1.5) and FP4
# E2M1 experts with E8M0 block-32 scales (the weight-streaming kernels).
F4 = {
    # the CUDA-core router (T <= 128) and the tensor-core one (T >= 129)
    "sqrtsp_small": LayerShape(T=100, d=256, E=32, k=6, F=128, scale=1.5,
                               score_fn="sqrtsoftplus"),
    "sqrtsp_tc": LayerShape(T=300, d=512, E=32, k=6, F=256, scale=1.5, score_fn="sqrtsoftplus"),
    "sqrtsp_bias": LayerShape(T=200, d=512, E=16, k=4, F=256, scale=1.5, score_fn="sqrtsoftplus",
                              score_bias_std=0.05),
    "fp4_tiny": LayerShape(T=64, d=256, E=16, k=4, F=128, scale=1.5, fp4=True,
                           score_fn="sqrtsoftplus"),
    # ~56 rows per expert: several passes of the streaming kernels' 8-row staging
    "fp4_ragged": LayerShape(T=300, d=512, E=32, k=6, F=384, scale=1.5, fp4=True,
                             score_fn="sqrtsoftplus", score_bias_std=0.05),
    "fp4_sigmoid": LayerShape(T=40, d=384, E=8, k=2, F=256, fp4=True),
    # d and d_ff multiples of 256: FP4 on the tensor-core SM-pair kernels
    "fp4_pair": LayerShape(T=333, d=768, E=24, k=6, F=512, scale=1.5, fp4=True,
                           score_fn="sqrtsoftplus", score_bias_std=0.05),
    "fp4_pair_tiny": LayerShape(T=3, d=512, E=8, k=2, F=256, fp4=True),
}


@pytest.mark.parametrize("name", sorted(F4))
@pytest.mark.parametrize("path", [None, "stream", "gemm"])
def test_second_variant_every_token(name, path):
    sh = F4[name]
    if path == "gemm" and (sh.d % 256 or sh.F % 256):
        pytest.skip("the tensor-core pair kernels need d and d_ff multiples of 256")
    if path is not None and not sh.fp4:
        pytest.skip("the expert path matters for the FP4 experts only")
    layer = make_layer(sh, seed=61, device="cuda")
    route = parity.gpu_route(layer, path)
    O = oracle.OracleLayer(layer)
    ref = oracle.route(O.x, O.wg, O.k, O.scale, O.gate_bias, score_bias=O.score_bias,
                       score_fn=O.score_fn)
    parity.check_route(*route, ref)
    out = parity.gpu_forward(layer, path)
    res = parity.check_forward(layer, out, None, route)
    print(name, path, res)
    _free(layer, out)


@pytest.mark.parametrize("T", [7, 300])
def test_sqrt_softplus_router_on_hy3_shape(T):
    """sqrt-softplus top-6 at d=4096, E=192 on both router kernels."""
    shape = dataclasses.replace(CONFIGS["decode"], T=T, k=6, scale=1.5, score_fn="sqrtsoftplus")
    layer = make_layer(shape, seed=T + 1, device="cuda", with_experts=False)
    route = parity.gpu_route(layer)
    ref = oracle.route(oracle.bf16_bits(layer["x"]), oracle.bf16_bits(layer["w_gate"]), shape.k,
                       shape.scale, score_fn="sqrtsoftplus")
    parity.check_route(*route, ref)


@pytest.mark.parametrize("path", [None, "stream", "gemm"])
def test_fp4_decode_hy3_shape(path):
    """FP4 experts at the Hy3 decode shape (T=64, d=4096, E=192, d_ff=1536), top-6
    sqrt-softplus routing, on the streaming kernels (the default at this batch)
    and on the tensor-core pair kernels: every token's routing and output."""
    shape = dataclasses.replace(CONFIGS["decode"], k=6, scale=1.5, fp4=True,
                                score_fn="sqrtsoftplus")
    layer = make_layer(shape, seed=5, device="cuda")
    route = parity.gpu_route(layer, path)
    O = oracle.OracleLayer(layer)
    ref = oracle.route(O.x, O.wg, O.k, O.scale, score_fn="sqrtsoftplus")
    near = parity.check_route(*route, ref)
    out = parity.gpu_forward(layer, path)
    res = parity.check_forward(layer, out, None, route)
    print("fp4 decode", path, "near ties:", len(near), res)
    _free(layer, out)


# The largest supported shapes: 256 experts with k = 32 (the CUDA-core router's
# 32 rounds, the one-CTA grouping over 256 experts, the 32-row combine), and
# d = d_ff = 8192 (128 KB of staged rows on the streaming path, 128 K blocks
# on the pair GEMMs). The d = 8192 draw takes weights N(0, 0.01^2): with the
# Hy3 configs' 0.02 its outputs reach ~27, where one bf16 ulp (0.125) already
# exceeds the 5e-2 max-abs bound set for outputs of the Hy3 range (below 8).
MAX = {
    "e256_k32": LayerShape(T=40, d=256, E=256, k=32, F=128),
    "d8192": LayerShape(T=16, d=8192, E=8, k=2, F=8192, w_std=0.01),
}


@pytest.mark.parametrize("name", sorted(MAX))
@pytest.mark.parametrize("path", [None, "stream", "gemm"])
def test_largest_supported_shapes_every_token(name, path):
    sh = MAX[name]
    layer = make_layer(sh, seed=81, device="cuda")
    route = parity.gpu_route(layer, path)
    O = oracle.OracleLayer(layer)
    ref = oracle.route(O.x, O.wg, O.k, O.scale, O.gate_bias)
    parity.check_route(*route, ref)
    out = parity.gpu_forward(layer, path)
    res = parity.check_forward(layer, out, None, route)
    print(name, path, res)
    _free(layer, out)


@pytest.mark.parametrize("T", [16, 200])
def test_router_at_d8192_on_both_kernels(T):
    shape = LayerShape(T=T, d=8192, E=256, k=8, F=128, zipf_bias=True)
    layer = make_layer(shape, seed=83, device="cuda", with_experts=False)
    route = parity.gpu_route(layer)
    ref = oracle.route(oracle.bf16_bits(layer["x"]), oracle.bf16_bits(layer["w_gate"]), shape.k,
                       shape.scale, layer["gate_bias"].cpu().numpy())
    parity.check_route(*route, ref)


@pytest.mark.parametrize("path", ["gemm", "stream"])
def test_fp8_weights_widen_exactly_for_every_code(path):
    """moe_expert_down with e4m3 weights of unit row scale and one-hot rows of h:
    y[r, i] = bf16(1.0 * value(W[e_r, i, f_r])) is each code's value itself
    (every e4m3 value is a bf16 value). The codes cover all 254 non-NaN e4m3
    patterns -- subnormals and both zeros included -- and each output is
    compared with the oracle's e4m3 decoding: equal values (a -0 weight
    gives +0, the sum of its -0 product and the other columns' +0 products)."""
    E, d, F, rows_e = 2, 256, 256, 128
    R = E * rows_e
    i = np.arange(d)[None, :, None]
    f = np.arange(F)[None, None, :]
    e = np.arange(E)[:, None, None]
    codes = ((i + 7 * f + 13 * e) % 256).astype(np.uint8)
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0x01   # no NaN weights
    f_of_row = (np.arange(R) * 5) % F
    h = torch.zeros((R, F), dtype=torch.bfloat16)
    h[torch.arange(R), torch.from_numpy(f_of_row)] = 1.0
    cfg = moe.config(T=R, d=d, E=E, k=1, d_ff=F, fp8=True, path=path)
    ws = moe.workspace(cfg)
    offsets = torch.tensor([0, rows_e, R], dtype=torch.int32, device="cuda")
    y = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_down(cfg, h.cuda(), offsets, torch.from_numpy(codes).cuda(),
                        torch.ones((E, d), dtype=torch.float32, device="cuda"), y, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    e_of_row = np.arange(R) // rows_e
    want_codes = codes[e_of_row[:, None], np.arange(d)[None, :], f_of_row[:, None]]
    want = oracle.double_from_e4m3(want_codes)
    assert len(np.unique(want_codes)) == 254
    got = oracle.double_from_bf16(oracle.bf16_bits(y))
    bad = np.nonzero(got != want)
    assert bad[0].size == 0, (f"{bad[0].size} outputs differ, first code "
                              f"{want_codes[bad][0]:#04x}: {got[bad][0]} vs {want[bad][0]}")


@pytest.mark.parametrize("path", ["gemm", "stream"])
def test_fp4_weights_widen_exactly_for_every_code_and_scale(path):
    """moe_expert_down with FP4 weights and one-hot rows of h: y[r, i] is the
    weight W[e_r, i, f_r] = E2M1 code value * 2^(b - 127) itself, exact in bf16.
    Rows cover all 16 codes (both signs, the subnormal 0.5 and both zeros) under
    block scales b from 0 to 252 -- on both sides of b = 128, where the tensor-core
    widening switches from one multiply by 2^(b-1) to two -- compared with the
    oracle's E2M1 and E8M0 decoding."""
    E, d, F, rows_e = 2, 256, 256, 128
    R = E * rows_e
    g = torch.Generator().manual_seed(17)
    codes = torch.randint(0, 256, (E, d, F // 2), generator=g, dtype=torch.uint8)
    bvals = torch.tensor([0, 1, 60, 110, 120, 126, 127, 128, 129, 130, 160, 200, 250, 252],
                         dtype=torch.uint8)
    scales = bvals[torch.randint(0, len(bvals), (E, d, F // 32), generator=g)]
    f_of_row = (np.arange(R) * 7 + 3) % F
    h = torch.zeros((R, F), dtype=torch.bfloat16)
    h[torch.arange(R), torch.from_numpy(f_of_row)] = 1.0
    cfg = moe.config(T=R, d=d, E=E, k=1, d_ff=F, fp4=True, path=path)
    ws = moe.workspace(cfg)
    offsets = torch.tensor([0, rows_e, R], dtype=torch.int32, device="cuda")
    y = torch.empty((R, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_down(cfg, h.cuda(), offsets, codes.cuda(), scales.cuda(), y, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    e_of_row = np.arange(R) // rows_e
    cn, sn = codes.numpy(), scales.numpy()
    ii = np.arange(d)[None, :]
    byte = cn[e_of_row[:, None], ii, (f_of_row // 2)[:, None]]
    nib = np.where((f_of_row % 2)[:, None] == 1, byte >> 4, byte & 0xF).astype(np.uint8)
    b = sn[e_of_row[:, None], ii, (f_of_row // 32)[:, None]]
    want = oracle.double_from_e2m1(nib) * oracle.double_from_e8m0(b)
    assert len(np.unique(nib)) == 16 and len(np.unique(b)) == len(bvals)
    got = oracle.double_from_bf16(oracle.bf16_bits(y))
    bad = np.nonzero(got != want)
    assert bad[0].size == 0, (f"{bad[0].size} outputs differ, first code {nib[bad][0]} scale "
                              f"{b[bad][0]}: {got[bad][0]} vs {want[bad][0]}")
