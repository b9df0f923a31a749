"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a value the
pages print, a closed form, a special case that reduces to a textbook routine
(numpy/torch), or brute force on tiny inputs. Together they are chosen so that
a dropped term, a wrong sign, a wrong index or a transposed operand anywhere
in the oracle fails at least one of them.
"""

import dataclasses
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from synthetic import LayerShape, make_layer, tensor_shapes
from sparse_moe_transformer_gemm_b200 import work


def _f64(t):
    """Exact widening of a bf16/fp32 torch tensor with torch (independent of the oracle)."""
    return t.detach().cpu().to(torch.float64).numpy()


def _layer(shape, seed=0, **kw):
    return make_layer(shape, seed=seed, **kw)


def _np_logits(L):
    return _f64(L["x"]) @ _f64(L["w_gate"]).T + (
        0.0 if L.get("gate_bias") is None else _f64(L["gate_bias"])[None, :])


def _np_expert(x64, wgu64, wd64, e, F):
    """Textbook SwiGLU MLP (no bias): down( SiLU(x Wg^T) * (x Wu^T) )."""
    g = x64 @ wgu64[e, :F, :].T
    u = x64 @ wgu64[e, F:, :].T
    h = g / (1.0 + np.exp(-g)) * u
    return h @ wd64[e].T


# ------------------------------------------------------------------ formats

def test_bf16_rounding_matches_torch_cast_on_random_fp32_bit_patterns():
    rng = np.random.default_rng(1)
    raw = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    # exact ties: low half 0x8000, with both parities of the kept half
    ties = (rng.integers(0, 2**16, size=20_000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    v = np.concatenate([raw, ties]).view(np.float32)
    v = v[np.isfinite(v)]
    want = oracle.bf16_bits(torch.from_numpy(v).to(torch.bfloat16))
    got = oracle.bf16_from_double(v.astype(np.float64))
    assert np.array_equal(got, want)


@pytest.mark.parametrize("value,expected", [
    (8.2, 8.1875),          # spacing 2^-4 at [8,16): 131.2 quanta -> 131
    (8.23, 8.25),           # 131.68 quanta -> 132
    (1.0 + 2.0**-8, 1.0),   # exact tie -> even mantissa (0)
    (1.0 + 3 * 2.0**-8, 1.0 + 2.0**-6),  # exact tie between mantissas 1 and 2 -> 2
    (2.0**-133, 2.0**-133),  # smallest subnormal
    (2.0**-134, 0.0),       # tie between 0 and the smallest subnormal -> 0
    (3 * 2.0**-134, 2.0**-132),  # tie between 1 and 2 subnormal quanta -> 2
    (-0.0, -0.0),
    ((2.0 - 2.0**-8) * 2.0**127, math.inf),  # tie at the top -> rounds up to infinity
    ((2.0 - 2.0**-7) * 2.0**127, (2.0 - 2.0**-7) * 2.0**127),  # largest finite bf16
])
def test_bf16_rounding_hand_cases(value, expected):
    got = oracle.double_from_bf16(oracle.bf16_from_double(np.array([value])))[0]
    assert got == expected and math.copysign(1, got) == math.copysign(1, expected)


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.double_from_e4m3(codes)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0**-9 and got[0x08] == 2.0**-6


# ------------------------------------------------------------------ combine

def test_fp32_combine_keeps_small_expert_outputs(golden):
    """The pages' example: a large branch output (8.2) next to small ones (0.03).

    With the outputs already in bf16 (8.1875 and 0.030029296875) a bf16
    running sum drops every small term; a wide sum keeps them.
    """
    ex = golden["fp32_combine_example"]
    big = oracle.double_from_bf16(oracle.bf16_from_double(np.array([ex["large_output"]])))[0]
    small = oracle.double_from_bf16(oracle.bf16_from_double(np.array([ex["small_output"]])))[0]
    assert (big, small) == (8.1875, 0.030029296875)
    y = np.array([[[big]] + [[small]] * 7], dtype=np.float64)  # [1, 8, 1]
    out = oracle.double_from_bf16(oracle.combine(y, np.ones((1, 8))))[0, 0]
    exact = big + 7 * small
    assert out == 8.375 and abs(out - exact) <= 2.0**-5
    # what a bf16 running sum would give, by hand: every partial sum rounds back
    running = big
    for _ in range(7):
        running = oracle.double_from_bf16(oracle.bf16_from_double(np.array([running + small])))[0]
    assert running == 8.1875 != out


# ------------------------------------------------------------------ routing

def test_selected_weights_sum_to_scale(golden):
    scale = golden["sum_of_selected_weights"]["value"]
    L = _layer("decode", with_experts=False, T=48)
    r = oracle.route(oracle.bf16_bits(L["x"]), oracle.bf16_bits(L["w_gate"]), 8, scale)
    assert np.allclose(r["w"].sum(axis=1), scale, rtol=1e-12, atol=0)
    assert np.all(np.diff(r["w"], axis=1) <= 0)  # descending score order


@pytest.mark.parametrize("k", [1, 2, 3, 5, 8])
def test_topk_is_the_best_subset_by_brute_force(k):
    shape = LayerShape(T=60, d=64, E=8, k=k, F=16, w_std=0.2)
    L = _layer(shape, seed=k)
    r = oracle.route(oracle.bf16_bits(L["x"]), oracle.bf16_bits(L["w_gate"]), k, 2.826)
    s = 1.0 / (1.0 + np.exp(-_np_logits(L)))
    checked = 0
    for t in range(shape.T):
        sums = sorted(((sum(s[t, list(c)]), c) for c in itertools.combinations(range(8), k)),
                      reverse=True)
        if len(sums) > 1 and sums[0][0] - sums[1][0] < 1e-12:
            continue
        assert set(r["idx"][t]) == set(sums[0][1])
        checked += 1
        # gap is the k-th minus the (k+1)-th largest score
        srt = np.sort(s[t])[::-1]
        want_gap = srt[k - 1] - srt[k] if k < 8 else math.inf
        assert r["gap"][t] == pytest.approx(want_gap, rel=1e-9, abs=1e-15)
    assert checked > 50


def test_k1_matches_softmax_argmax_and_takes_the_full_scale(golden):
    """k = 1: sigmoid top-1 = softmax top-1, and the single weight is the scale."""
    L = _layer("tiny", seed=3)
    r = oracle.route(oracle.bf16_bits(L["x"]), oracle.bf16_bits(L["w_gate"]), 1, 2.826)
    z = _np_logits(L)
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert np.array_equal(r["idx"][:, 0], p.argmax(axis=1))
    assert np.allclose(r["w"][:, 0], golden["router_scaling_factor"]["value"], rtol=1e-15, atol=0)


def test_equal_scores_take_lowest_indices_and_split_the_scale(golden):
    L = _layer("decode", with_experts=False, T=4)
    x0 = np.zeros((4, 4096), dtype=np.uint16)   # all logits 0 -> every score 0.5
    r = oracle.route(x0, oracle.bf16_bits(L["w_gate"]), 8, 2.826)
    assert np.array_equal(r["idx"], np.tile(np.arange(8, dtype=np.int32), (4, 1)))
    assert np.allclose(r["w"], 2.826 / 8, rtol=1e-15, atol=0)
    assert round(float(r["w"][0, 0]), 3) == golden["equal_split_weight"]["printed"]
    assert np.all(r["gap"] == 0.0)


def test_saturated_scores_rank_by_the_exact_order():
    """Logits 45 on expert 9 and 40 on expert 3 (a zero token and a logit bias):
    both sigmoids round to 1.0 in fp64, yet the exact scores put 9 before 3; the
    other experts (logit 0, score 0.5) follow by index. The weights use the
    rounded scores: 2.826 * (1, 1, 0.5 x 6) / 5."""
    assert 1.0 / (1.0 + math.exp(-40.0)) == 1.0
    x = np.zeros((1, 8), np.uint16)
    wg = np.zeros((12, 8), np.uint16)
    b = np.zeros(12, np.float32)
    b[9], b[3] = 45.0, 40.0
    r = oracle.route(x, wg, 1, 2.826, gate_bias=b)
    assert r["idx"][0, 0] == 9 and r["w"][0, 0] == 2.826
    r = oracle.route(x, wg, 8, 2.826, gate_bias=b)
    assert r["idx"][0].tolist() == [9, 3, 0, 1, 2, 4, 5, 6]
    want = 2.826 * np.array([1.0, 1.0] + [0.5] * 6) / 5.0
    assert np.allclose(r["w"][0], want, rtol=1e-15, atol=0)
    assert r["gap"][0] == 0.0   # scores 0.5 and 0.5 at the 8th and 9th places
    # the square root of the softplus does not saturate: the same order
    r = oracle.route(x, wg, 2, 1.5, gate_bias=b, score_fn="sqrtsoftplus")
    assert r["idx"][0].tolist() == [9, 3]


def test_scaled_weight_example(golden):
    """A normalised weight of 0.12 becomes 0.12 * 2.826 = 0.33912 (page prints 0.338)."""
    ex = golden["scaled_example"]
    s1, s2 = 0.12, 0.88
    bias = np.array([math.log(s1 / (1 - s1)), math.log(s2 / (1 - s2))], dtype=np.float32)
    r = oracle.route(np.zeros((1, 8), np.uint16), np.zeros((2, 8), np.uint16), 2, 2.826,
                     gate_bias=bias)
    w_small = r["w"][0, list(r["idx"][0]).index(0)]
    assert w_small == pytest.approx(ex["before"] * 2.826, abs=1e-6)
    assert abs(w_small - ex["printed_after"]) < 2e-3


def test_gate_bias_is_added_to_the_logits_before_the_sigmoid():
    rng = np.random.default_rng(7)
    E, k = 12, 4
    b = rng.normal(size=E).astype(np.float32)
    r = oracle.route(np.zeros((1, 16), np.uint16), np.zeros((E, 16), np.uint16), k, 2.826,
                     gate_bias=b)
    sig = [1.0 / (1.0 + math.exp(-float(v))) for v in b]
    want = sorted(range(E), key=lambda e: (-sig[e], e))[:k]
    assert list(r["idx"][0]) == want
    tot = sum(sig[e] for e in want)
    assert np.allclose(r["w"][0], [2.826 * sig[e] / tot for e in want], rtol=1e-14)


# ------------------------------------------------------------------ experts / layer

def test_k1_layer_is_the_textbook_swiglu_mlp_of_the_argmax_expert():
    shape = LayerShape(T=24, d=96, E=6, k=1, F=80)
    L = _layer(shape, seed=11)
    O = oracle.OracleLayer(L)
    r = oracle.forward_tokens(O)
    x64, wgu, wd = _f64(L["x"]), _f64(L["w_gate_up"]), _f64(L["w_down"])
    e_star = _np_logits(L).argmax(axis=1)
    for t in range(shape.T):
        want = 2.826 * _np_expert(x64[t:t + 1], wgu, wd, e_star[t], shape.F)[0]
        assert r["idx"][t, 0] == e_star[t]
        assert np.allclose(r["out_f64"][t], want, rtol=1e-9, atol=1e-12)
    assert np.array_equal(r["out_bf16"], oracle.bf16_from_double(r["out_f64"]))


def test_k_equals_E_is_the_dense_weighted_sum_over_all_experts():
    shape = LayerShape(T=16, d=64, E=5, k=5, F=48)
    L = _layer(shape, seed=5)
    r = oracle.forward_tokens(oracle.OracleLayer(L))
    x64, wgu, wd = _f64(L["x"]), _f64(L["w_gate_up"]), _f64(L["w_down"])
    s = 1.0 / (1.0 + np.exp(-_np_logits(L)))
    w = 2.826 * s / s.sum(axis=1, keepdims=True)
    want = sum(w[:, e:e + 1] * _np_expert(x64, wgu, wd, e, shape.F) for e in range(shape.E))
    assert np.allclose(r["out_f64"], want, rtol=1e-9, atol=1e-12)
    assert np.all(np.isinf(r["gap"]))


def test_zero_up_weights_give_zero_output():
    shape = LayerShape(T=10, d=64, E=4, k=2, F=32)
    L = _layer(shape, seed=2)
    L["w_gate_up"][:, shape.F:, :] = 0
    r = oracle.forward_tokens(oracle.OracleLayer(L))
    assert np.all(r["out_f64"] == 0.0)


def test_token_order_invariance_is_bitwise():
    L = _layer("tiny", seed=4)
    perm = torch.randperm(64, generator=torch.Generator().manual_seed(0))
    L2 = dict(L, x=L["x"][perm].contiguous())
    a = oracle.forward_tokens(oracle.OracleLayer(L))
    b = oracle.forward_tokens(oracle.OracleLayer(L2))
    assert np.array_equal(a["out_bf16"][perm.numpy()], b["out_bf16"])


def test_expert_relabelling_invariance_is_bitwise():
    L = _layer("tiny", seed=6)
    perm = torch.randperm(16, generator=torch.Generator().manual_seed(1))  # new e -> old perm[e]
    L2 = dict(L, w_gate=L["w_gate"][perm].contiguous(), w_gate_up=L["w_gate_up"][perm].contiguous(),
              w_down=L["w_down"][perm].contiguous())
    a = oracle.forward_tokens(oracle.OracleLayer(L))
    b = oracle.forward_tokens(oracle.OracleLayer(L2))
    assert np.array_equal(a["out_bf16"], b["out_bf16"])
    assert np.array_equal(perm.numpy()[b["idx"]], a["idx"])


def test_output_is_linear_in_the_scale():
    L = _layer("tiny", seed=8)
    one = oracle.forward_tokens(oracle.OracleLayer(L, scale=1.0))["out_f64"]
    big = oracle.forward_tokens(oracle.OracleLayer(L, scale=2.826))["out_f64"]
    assert np.allclose(big / 2.826, one, rtol=1e-12, atol=1e-18)


def test_fp8_expert_matches_textbook_mlp_on_decoded_weights():
    shape = LayerShape(T=6, d=64, E=3, k=1, F=32, fp8=True)
    L = _layer(shape, seed=9)
    dec = lambda q, s: (torch.from_numpy(q.cpu().numpy()).view(torch.float8_e4m3fn)  # noqa: E731
                        .to(torch.float64) * s.to(torch.float64)[..., None]).numpy()
    wgu = dec(L["q_gate_up"], L["s_gate_up"])
    wd = dec(L["q_down"], L["s_down"])
    x64 = _f64(L["x"])
    experts = np.array([0, 1, 2, 0, 1, 2], np.int32)
    y = oracle.expert_rows(oracle.bf16_bits(L["x"]), experts, L["q_gate_up"].numpy(),
                           L["q_down"].numpy(), L["s_gate_up"].numpy(), L["s_down"].numpy())
    for t in range(6):
        want = _np_expert(x64[t:t + 1], wgu, wd, experts[t], shape.F)[0]
        assert np.allclose(y[t], want, rtol=1e-9, atol=1e-13)


def test_fp8_layer_stays_within_quantisation_error_of_the_bf16_layer():
    shape = LayerShape(T=32, d=256, E=8, k=2, F=128, fp8=True)
    L = _layer(shape, seed=10)
    q = oracle.forward_tokens(oracle.OracleLayer(L))["out_f64"]
    ref = oracle.forward_tokens(oracle.OracleLayer(dict(L, cfg=dataclasses.replace(shape, fp8=False))))["out_f64"]
    rel = np.linalg.norm(q - ref) / np.linalg.norm(ref)
    assert 1e-4 < rel < 0.08   # e4m3: 3 mantissa bits, relative step <= 2^-3


# ------------------------------------------------------------------ sizes and work

def test_per_expert_parameter_count_matches_the_page(golden):
    g = golden["expert_shapes"]
    shp = tensor_shapes("decode")
    gu = math.prod(shp["w_gate_up"][1:])
    dn = math.prod(shp["w_down"][1:])
    assert (shp["w_gate_up"][0], shp["x"][1], shp["w_down"][2]) == (g["n_routed_experts"], g["d"],
                                                                    g["d_ff_expert"])
    assert gu + dn == 18_874_368
    assert round(gu / 1e6, 2) * 1e6 == g["gate_up_params"]
    assert round(dn / 1e6, 2) * 1e6 == g["down_params"]
    assert round((gu + dn) / 1e6, 2) * 1e6 == g["params_per_expert"]


def test_second_variant_shapes_match_the_page(golden):
    """The V4-Flash MoE column (the second routing and precision variant): the
    generator's tensors at its shape give the printed ~25.2M parameters per
    expert, and top-6 x 2048 covers the same intermediate width as Hy3's
    top-8 x 1536."""
    g = golden["v4_flash_moe"]
    shp = tensor_shapes(LayerShape(T=64, d=g["d"], E=g["n_routed_experts"], k=g["top_k"],
                                   F=g["d_ff_expert"], scale=g["routed_scaling_factor"],
                                   score_fn="sqrtsoftplus", fp4=True))
    per_expert = math.prod(shp["w_gate_up"][1:]) + math.prod(shp["w_down"][1:])
    assert per_expert == 3 * 4096 * 2048 == 25_165_824
    assert round(per_expert / 1e6, 1) * 1e6 == g["params_per_expert_printed"]
    assert g["top_k"] * g["d_ff_expert"] == g["total_intermediate_per_token"] == 8 * 1536
    assert shp["w_gate"] == (256, 4096)


def test_per_expert_flops_match_the_page(golden):
    f = work.expert_flops_per_token(4096, 1536)
    assert f == 37_748_736
    assert float(f"{f:.2e}") == golden["flops_per_token_per_expert"]["printed"]


# ------------------------------------------------------------------ permute definition

@pytest.mark.parametrize("T,k,E", [(100, 4, 16), (1, 8, 192), (257, 8, 192), (33, 1, 3)])
def test_permute_definition_matches_stable_argsort(T, k, E):
    rng = np.random.default_rng(T * 31 + k)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    r = oracle.permute(idx, E)
    flat = idx.ravel()
    order = np.argsort(flat, kind="stable")        # row -> slot
    want_row_of = np.empty_like(order)
    want_row_of[order] = np.arange(flat.size)
    assert np.array_equal(r["row_of"], want_row_of)
    assert np.array_equal(r["counts"], np.bincount(flat, minlength=E))
    assert np.array_equal(r["offsets"], np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))


# ------------------------------------------------------------------ the complete Hy3 block:
# e_score_correction_bias (choice only) and the shared expert (weight 1)

def _bits(t):
    return oracle.bf16_bits(t)


def _unit_router(logits):
    """x = e_0 and W_gate rows with the given first entries: the logits are exact."""
    E = len(logits)
    x = torch.zeros((1, 16), dtype=torch.bfloat16)
    x[0, 0] = 1.0
    wg = torch.zeros((E, 16), dtype=torch.bfloat16)
    wg[:, 0] = torch.tensor(logits, dtype=torch.float32).to(torch.bfloat16)
    assert [float(v) for v in wg[:, 0]] == list(map(float, logits))
    return _bits(x), _bits(wg)


def test_zero_score_bias_changes_nothing():
    L = _layer(LayerShape(T=40, d=64, E=12, k=4, F=32), seed=21)
    x, wg = _bits(L["x"]), _bits(L["w_gate"])
    a = oracle.route(x, wg, 4, 2.826)
    b = oracle.route(x, wg, 4, 2.826, score_bias=np.zeros(12, np.float32))
    for key in ("idx", "w", "gap"):
        assert np.array_equal(a[key], b[key]), key


def test_score_bias_chooses_but_does_not_weight(golden):
    """A large bias on four experts forces them into the top-4; their weights
    are the renormalised UNBIASED sigmoid scores (numpy, independent)."""
    assert "choice only" in golden["score_correction_bias"]["claim"]
    L = _layer(LayerShape(T=30, d=64, E=12, k=4, F=32), seed=22)
    forced = [2, 5, 7, 11]
    sb = np.zeros(12, np.float32)
    sb[forced] = 10.0
    r = oracle.route(_bits(L["x"]), _bits(L["w_gate"]), 4, 2.826, score_bias=sb)
    s = 1.0 / (1.0 + np.exp(-_np_logits(L)))
    for t in range(30):
        order = sorted(forced, key=lambda e: (-s[t, e], e))
        assert list(r["idx"][t]) == order
        assert np.allclose(r["w"][t], 2.826 * s[t, order] / s[t, order].sum(), rtol=1e-12)


def test_constant_score_bias_keeps_the_routing():
    L = _layer(LayerShape(T=50, d=64, E=16, k=4, F=32), seed=24)
    x, wg = _bits(L["x"]), _bits(L["w_gate"])
    a = oracle.route(x, wg, 4, 2.826)
    b = oracle.route(x, wg, 4, 2.826, score_bias=np.full(16, 0.37, np.float32))
    assert np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["w"], b["w"])


def test_score_bias_acts_after_the_sigmoid():
    """Logits 5 and 6 (a saturated sigmoid): +0.01 on expert 0's SCORE beats
    sigma(6) - sigma(5) = 0.0042, while +0.01 on its LOGIT does not."""
    x, wg = _unit_router([5.0, 6.0])
    r = oracle.route(x, wg, 1, 2.826, score_bias=np.array([0.01, 0.0], np.float32))
    assert r["idx"][0, 0] == 0 and r["w"][0, 0] == 2.826
    r = oracle.route(x, wg, 1, 2.826, gate_bias=np.array([0.01, 0.0], np.float32))
    assert r["idx"][0, 0] == 1


def test_gap_is_measured_on_the_ranked_value():
    """Logits 0, 1, 2 and a score bias of 0.5 on expert 0: the ranked values
    are 1.0, sigma(1), sigma(2); k=1 picks expert 0 with gap 1 - sigma(2)."""
    x, wg = _unit_router([0.0, 1.0, 2.0])
    r = oracle.route(x, wg, 1, 2.826, score_bias=np.array([0.5, 0.0, 0.0], np.float32))
    assert r["idx"][0, 0] == 0
    assert math.isclose(r["gap"][0], 1.0 - 1.0 / (1.0 + math.exp(-2.0)), rel_tol=1e-14)


def _np_shared(L):
    x64 = _f64(L["x"])
    F = L["cfg"].F
    gu, dn = _f64(L["w_shared_gate_up"]), _f64(L["w_shared_down"])
    return _np_expert(x64, gu[None], dn[None], 0, F)


def test_shared_expert_is_added_with_weight_one():
    L = _layer(LayerShape(T=12, d=64, E=6, k=2, F=32, shared=True), seed=23)
    O = oracle.OracleLayer(L)
    r = oracle.forward_tokens(O)
    O.sh_wgu = O.sh_wd = None
    r0 = oracle.forward_tokens(O)
    assert np.array_equal(r["idx"], r0["idx"])
    assert np.allclose(r["out_f64"] - r0["out_f64"], _np_shared(L), rtol=1e-9, atol=1e-12)


def test_shared_expert_alone_is_the_textbook_mlp():
    shape = LayerShape(T=10, d=64, E=4, k=2, F=32, shared=True)
    L = _layer(shape, seed=25)
    L["w_gate_up"][:, shape.F:, :] = 0          # every routed expert outputs 0
    r = oracle.forward_tokens(oracle.OracleLayer(L))
    assert np.allclose(r["out_f64"], _np_shared(L), rtol=1e-9, atol=1e-12)
    assert np.array_equal(r["out_bf16"], oracle.bf16_from_double(r["out_f64"]))


def test_fp8_shared_expert_uses_codes_times_row_scales():
    shape = LayerShape(T=8, d=64, E=4, k=2, F=32, shared=True, fp8=True)
    L = _layer(shape, seed=26)
    L["q_gate_up"][:, shape.F:, :] = 0          # routed outputs 0
    r = oracle.forward_tokens(oracle.OracleLayer(L))
    dec = lambda q, s: (q.view(torch.float8_e4m3fn).to(torch.float64) *  # noqa: E731
                        s.to(torch.float64)[:, None]).numpy()
    gu = dec(L["q_shared_gate_up"], L["s_shared_gate_up"])
    dn = dec(L["q_shared_down"], L["s_shared_down"])
    want = _np_expert(_f64(L["x"]), gu[None], dn[None], 0, shape.F)
    assert np.allclose(r["out_f64"], want, rtol=1e-9, atol=1e-12)


def test_moe_layer_parameter_count_with_the_shared_expert_matches_the_page(golden):
    shp = tensor_shapes("decode")
    per_expert = math.prod(shp["w_gate_up"][1:]) + math.prod(shp["w_down"][1:])
    L = _layer(LayerShape(T=1, d=256, E=2, k=1, F=128, shared=True), seed=0)
    assert L["w_shared_gate_up"].shape[1:] == L["w_gate_up"].shape[2:]  # same SwiGLU shape
    layer = math.prod(shp["w_gate"]) + (shp["w_gate_up"][0] + 1) * per_expert
    assert round(layer / 1e9, 2) * 1e9 == golden["moe_layer_params"]["printed"]
    assert round(per_expert / 1e6, 2) * 1e6 == golden["moe_layer_params"]["shared_expert_params_printed"]
    frac = per_expert / ((shp["w_gate_up"][0] + 1) * per_expert)
    assert round(100 * frac, 2) == golden["shared_expert_fraction"]["printed_percent"]


# ------------------------------------------------------------------ route_norm:
# the router scores RMSNorm(x) (weight g, eps inside the root); the experts take x

def _np_rmsnorm(x64, g, eps):
    return x64 / np.sqrt((x64 * x64).mean(axis=1, keepdims=True) + eps) * g[None, :]


def test_route_norm_scores_the_rmsnorm_of_the_token():
    shape = LayerShape(T=20, d=64, E=10, k=3, F=32, route_norm=True)
    L = _layer(shape, seed=41)
    g = L["route_norm_weight"].numpy().astype(np.float64)
    r = oracle.route(_bits(L["x"]), _bits(L["w_gate"]), 3, 2.826, want_scores=True,
                     norm_w=L["route_norm_weight"].numpy(), norm_eps=1e-6)
    want = _np_rmsnorm(_f64(L["x"]), g, 1e-6) @ _f64(L["w_gate"]).T
    assert np.allclose(r["logits"], want, rtol=1e-12, atol=1e-14)
    s = 1.0 / (1.0 + np.exp(-want))
    for t in range(20):
        assert list(r["idx"][t]) == sorted(range(10), key=lambda e: (-s[t, e], e))[:3]


def test_route_norm_makes_the_routing_independent_of_the_token_scale():
    shape = LayerShape(T=30, d=64, E=12, k=4, F=32, route_norm=True)
    L = _layer(shape, seed=42)
    nw = L["route_norm_weight"].numpy()
    x1, x4 = _bits(L["x"]), _bits(L["x"] * 4)       # x4 = 4 x exactly (bf16)
    a = oracle.route(x1, _bits(L["w_gate"]), 4, 2.826, norm_w=nw)
    b = oracle.route(x4, _bits(L["w_gate"]), 4, 2.826, norm_w=nw)
    assert np.array_equal(a["idx"], b["idx"])
    assert np.allclose(a["w"], b["w"], rtol=1e-5)
    c = oracle.route(x1, _bits(L["w_gate"]), 4, 2.826)
    d = oracle.route(x4, _bits(L["w_gate"]), 4, 2.826)
    assert not np.allclose(c["w"], d["w"], rtol=1e-3)   # without route_norm it is not


def test_route_norm_epsilon_sits_inside_the_root():
    """Tokens of size ~2^-12 (mean square ~6e-8, below eps = 1e-6): only
    x / sqrt(mean(x^2) + eps) reproduces the oracle's logits."""
    shape = LayerShape(T=8, d=64, E=6, k=2, F=32, route_norm=True)
    L = _layer(shape, seed=43)
    xs = (L["x"].float() * 2.0 ** -12).to(torch.bfloat16)
    g = L["route_norm_weight"].numpy().astype(np.float64)
    r = oracle.route(_bits(xs), _bits(L["w_gate"]), 2, 2.826, want_scores=True,
                     norm_w=L["route_norm_weight"].numpy(), norm_eps=1e-6)
    want = _np_rmsnorm(_f64(xs), g, 1e-6) @ _f64(L["w_gate"]).T
    assert np.allclose(r["logits"], want, rtol=1e-12, atol=1e-16)


def test_zero_route_norm_weight_gives_equal_scores():
    L = _layer(LayerShape(T=5, d=64, E=8, k=3, F=32, route_norm=True), seed=44)
    r = oracle.route(_bits(L["x"]), _bits(L["w_gate"]), 3, 2.826,
                     norm_w=np.zeros(64, np.float32))
    assert np.all(r["idx"] == np.arange(3)[None, :])
    assert np.allclose(r["w"], 2.826 / 3, rtol=1e-15)


def test_route_norm_leaves_the_experts_on_the_token():
    """k = E: out = sum_e w_e(RMSNorm(x)) * expert_e(x) -- the weights come from
    the normalised token, the expert outputs from the token itself."""
    shape = LayerShape(T=6, d=64, E=4, k=4, F=32, route_norm=True)
    L = _layer(shape, seed=45)
    r = oracle.forward_tokens(oracle.OracleLayer(L))
    x64, wgu, wd = _f64(L["x"]), _f64(L["w_gate_up"]), _f64(L["w_down"])
    g = L["route_norm_weight"].numpy().astype(np.float64)
    s = 1.0 / (1.0 + np.exp(-(_np_rmsnorm(x64, g, 1e-6) @ _f64(L["w_gate"]).T)))
    w = 2.826 * s / s.sum(axis=1, keepdims=True)
    want = sum(w[:, e:e + 1] * _np_expert(x64, wgu, wd, e, shape.F) for e in range(4))
    assert np.allclose(r["out_f64"], want, rtol=1e-9, atol=1e-12)


# ------------------------------------------------------------------ the second routing and
# precision variant: sqrt(softplus) scores, FP4 (E2M1 + E8M0 block-32) routed experts

# OCP Microscaling (MX) formats v1.0: E2M1 magnitudes of codes 0..7 (bit 3 = sign)
SPEC_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _np_decode_fp4(packed, scales):
    """Independent numpy decode: [..., rows, cols/2] nibbles + [..., rows, cols/32]
    E8M0 bytes -> float64 [..., rows, cols]."""
    lo, hi = packed & 0xF, packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(*packed.shape[:-1], packed.shape[-1] * 2)
    mag = np.asarray(SPEC_E2M1)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    sc = np.ldexp(1.0, scales.astype(np.int64) - 127)
    return mag * np.repeat(sc, 32, axis=-1)


def test_e2m1_decode_matches_the_spec_table():
    got = oracle.double_from_e2m1(np.arange(16, dtype=np.uint8))
    want = SPEC_E2M1 + [-v for v in SPEC_E2M1]
    assert [float(v) for v in got] == want


def test_e8m0_decode_is_a_power_of_two():
    got = oracle.double_from_e8m0(np.array([127, 128, 120, 0, 254, 255], np.uint8))
    assert list(got[:5]) == [1.0, 2.0, 2.0 ** -7, 2.0 ** -127, 2.0 ** 127]
    assert math.isnan(got[5])


def test_fp4_encoding_rounds_to_the_grid_within_half_a_step():
    from synthetic.moe_inputs import encode_e2m1_blocks

    w = (torch.randn((3, 64, 96), generator=torch.Generator().manual_seed(3)) * 0.02).to(
        torch.bfloat16)
    q, s = encode_e2m1_blocks(w)
    dec = _np_decode_fp4(q.numpy(), s.numpy())
    ref = _f64(w)
    scale = np.repeat(np.ldexp(1.0, s.numpy().astype(np.int64) - 127), 32, axis=-1)
    # the grid step at magnitude m (in scale units): 0.5 below 2, 1 below 4, 2 above
    m = np.abs(ref) / scale
    step = np.where(m < 2, 0.5, np.where(m < 4, 1.0, 2.0))
    assert np.all(np.abs(dec - ref) <= 0.5 * step * scale + 1e-12)
    assert np.all(np.abs(ref).reshape(3, 64, 3, 32).max(-1) <= 6 * scale[..., ::32] + 1e-12)


def test_fp4_expert_is_the_textbook_mlp_on_decoded_weights():
    shape = LayerShape(T=6, d=64, E=3, k=1, F=64, fp4=True)
    L = _layer(shape, seed=61)
    O = oracle.OracleLayer(L)
    gu = _np_decode_fp4(O.wgu4, O.sgu8)
    dn = _np_decode_fp4(O.wd4, O.sd8)
    experts = np.array([0, 1, 2, 2, 1, 0], np.int32)
    y = oracle.expert_rows_fp4(O.x, experts, O.wgu4, O.sgu8, O.wd4, O.sd8)
    x64 = _f64(L["x"])
    for r, e in enumerate(experts):
        want = _np_expert(x64[r:r + 1], gu, dn, e, shape.F)[0]
        assert np.allclose(y[r], want, rtol=1e-9, atol=1e-12)


def test_sqrt_softplus_scores_and_weights():
    shape = LayerShape(T=25, d=64, E=16, k=6, F=32, scale=1.5, score_fn="sqrtsoftplus")
    L = _layer(shape, seed=62)
    r = oracle.route(_bits(L["x"]), _bits(L["w_gate"]), 6, 1.5, want_scores=True,
                     score_fn="sqrtsoftplus")
    z = _np_logits(L)
    s = np.sqrt(np.log1p(np.exp(z)))
    assert np.allclose(r["scores"], s, rtol=1e-12)
    for t in range(25):
        want = sorted(range(16), key=lambda e: (-s[t, e], e))[:6]
        assert list(r["idx"][t]) == want
        assert list(r["idx"][t]) == sorted(range(16), key=lambda e: (-z[t, e], e))[:6]
        assert np.allclose(r["w"][t], 1.5 * s[t, want] / s[t, want].sum(), rtol=1e-12)
    x, wg = _unit_router([0.0, -1.0])
    r1 = oracle.route(x, wg, 1, 1.5, want_scores=True, score_fn="sqrtsoftplus")
    assert math.isclose(r1["scores"][0, 0], math.sqrt(math.log(2.0)), rel_tol=1e-15)
    assert r1["idx"][0, 0] == 0 and r1["w"][0, 0] == 1.5


def test_fp4_layer_routes_like_its_router_and_sums_its_experts():
    shape = LayerShape(T=8, d=64, E=6, k=2, F=64, scale=1.5, fp4=True, score_fn="sqrtsoftplus")
    L = _layer(shape, seed=63)
    O = oracle.OracleLayer(L)
    r = oracle.forward_tokens(O)
    rr = oracle.route(O.x, O.wg, 2, 1.5, score_fn="sqrtsoftplus")
    assert np.array_equal(r["idx"], rr["idx"]) and np.array_equal(r["w"], rr["w"])
    y = oracle.expert_rows_fp4(np.repeat(O.x, 2, axis=0), r["idx"].reshape(-1), O.wgu4, O.sgu8,
                               O.wd4, O.sd8).reshape(8, 2, 64)
    assert np.allclose(r["out_f64"], (r["w"][:, :, None] * y).sum(axis=1), rtol=1e-12, atol=1e-15)


def test_sqrt_softplus_layer_with_k_equal_E_is_the_dense_weighted_sum():
    shape = LayerShape(T=10, d=64, E=4, k=4, F=32, scale=1.5, score_fn="sqrtsoftplus")
    L = _layer(shape, seed=64)
    r = oracle.forward_tokens(oracle.OracleLayer(L))
    x64, wgu, wd = _f64(L["x"]), _f64(L["w_gate_up"]), _f64(L["w_down"])
    s = np.sqrt(np.log1p(np.exp(_np_logits(L))))
    w = 1.5 * s / s.sum(axis=1, keepdims=True)
    want = sum(w[:, e:e + 1] * _np_expert(x64, wgu, wd, e, shape.F) for e in range(4))
    assert np.allclose(r["out_f64"], want, rtol=1e-9, atol=1e-12)
