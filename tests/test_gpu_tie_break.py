"""Exact ties on the GPU: both routers against the fp64 oracle, index ORDER
bit-exact on every token, no near-tie exemption.

The routing flow of "Tencent Hy3-295B 架构深度拆解" §4.1 takes the top-8 of the
sigmoid scores; equal scores go to the lower expert index, and the selection
is listed in descending score order. These inputs make scores exactly equal
on both sides (equal logits: zero tokens, constant biases, duplicated router
rows), so the oracle's gap at the k-th place is 0 and the general parity
tests would exempt them. Here nothing is exempt: the GPU's [T, k] index array
must equal the oracle's element by element, and the weights agree to a few
fp32 ulps (the oracle renormalises in fp64).

Both router kernels run: T = 64 takes the K-split CUDA-core router, T = 256
the tensor-core router (tcgen05 logits; a 128-token tile split over 8 CTAs,
8 lanes per token's selection, each scanning 24 experts, their lists merged),
at the Hy3 router shape d = 4096, E = 192, k = 8. The cross-lane case puts
the tied experts in different lanes' ranges (and, at T = 2048, the 4-way
split's 48-expert ranges), so the merges must keep the lower index.
"""

import numpy as np
import pytest
import torch

import oracle
from sparse_moe_transformer_gemm_b200 import build as moe_build
from sparse_moe_transformer_gemm_b200 import moe
from synthetic import CONFIGS, make_layer

pytestmark = pytest.mark.gpu

D, E, K, SCALE = 4096, 192, 8, 2.826
W_RTOL_TIE = 2e-6   # fp32 sigmoid, sum and division against fp64: a few ulps
SIX = [5, 40, 77, 130, 160, 191]        # experts lifted by distinct logit biases
TIED = [100, 101, 102, 103]             # experts with identical router rows
LIFT4 = [5, 40, 77, 131]                # four experts lifted by distinct biases
CROSS = [20, 30, 50, 70, 120, 170]      # identical rows in different selection lanes


@pytest.fixture(scope="module", autouse=True)
def _built():
    moe_build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _router_weights():
    """W_gate of the Hy3 decode draw (seed 0) with rows 101..103 set equal to row 100."""
    wg = make_layer(CONFIGS["decode"], seed=0, device="cuda", with_experts=False)["w_gate"]
    wg = wg.clone()
    wg[TIED[1:]] = wg[TIED[0]].clone()
    return wg


def _router_weights_cross():
    """The same draw with the rows of CROSS set equal to row CROSS[0]."""
    wg = make_layer(CONFIGS["decode"], seed=0, device="cuda", with_experts=False)["w_gate"]
    wg = wg.clone()
    wg[CROSS[1:]] = wg[CROSS[0]].clone()
    return wg


def _tokens(T, kind):
    g = torch.Generator(device="cuda")
    g.manual_seed(T)
    if kind == "zero":
        return torch.zeros((T, D), dtype=torch.bfloat16, device="cuda")
    # every fourth token a zero row, the rest N(0, 0.01^2): logits within ~0.05
    x = (0.01 * torch.randn((T, D), generator=g, device="cuda")).to(torch.bfloat16)
    x[::4] = 0
    return x


def _case(name, T):
    """(x, w_gate, gate_bias, score_bias) of one tie case."""
    wg = _router_weights()
    gb = sb = None
    if name == "all_zero":
        x = _tokens(T, "zero")
    elif name == "constant_gate_bias":
        x = _tokens(T, "zero")
        gb = torch.full((E,), 0.3, dtype=torch.float32, device="cuda")
    elif name == "duplicated_rows":
        # six experts lifted by 3.0, 2.8, ..., 2.0 and the four identical rows by
        # 1.0: two of the four tied experts take places 7 and 8 on every token
        x = _tokens(T, "mixed")
        gb = torch.zeros(E, dtype=torch.float32, device="cuda")
        gb[SIX] = torch.tensor([3.0, 2.8, 2.6, 2.4, 2.2, 2.0], device="cuda")
        gb[TIED] = 1.0
    elif name == "saturated":
        # logits 45 (expert 9) and 40 (expert 3): both sigmoids are 1.0 in fp32
        # and fp64; the exact scores still put 9 first, then the logit-0 experts
        x = _tokens(T, "zero")
        gb = torch.zeros(E, dtype=torch.float32, device="cuda")
        gb[9], gb[3] = 45.0, 40.0
    elif name == "constant_score_bias":
        x = _tokens(T, "zero")
        sb = torch.full((E,), 0.05, dtype=torch.float32, device="cuda")
    elif name == "cross_lane_ties":
        # four experts lifted by 3.0 .. 2.4 and the six identical rows by 1.0:
        # the four tied experts with the lowest indices take places 5..8
        x = _tokens(T, "mixed")
        wg = _router_weights_cross()
        gb = torch.zeros(E, dtype=torch.float32, device="cuda")
        gb[LIFT4] = torch.tensor([3.0, 2.8, 2.6, 2.4], device="cuda")
        gb[CROSS] = 1.0
    elif name == "duplicated_rows_score_bias":
        x, wg, gb, _ = _case("duplicated_rows", T)
        # small per-expert score biases (0 .. 0.004), equal on the tied four
        sb = 0.001 * (torch.arange(E, device="cuda") % 5).to(torch.float32)
        sb[TIED] = 0.002
    else:
        raise KeyError(name)
    return x, wg, gb, sb


def _expected_structure(name, idx):
    """What the oracle's own selection must look like, so that the case really
    puts ties at the k-th place."""
    if name in ("all_zero", "constant_gate_bias", "constant_score_bias"):
        assert np.all(idx == np.arange(K)), name
    elif name == "duplicated_rows":
        assert np.all(idx == np.array(SIX + TIED[:2])), name
    elif name == "saturated":
        assert np.all(idx == np.array([9, 3, 0, 1, 2, 4, 5, 6])), name
    elif name == "cross_lane_ties":
        assert np.all(idx == np.array(LIFT4 + CROSS[:4])), name


CASES = ["all_zero", "constant_gate_bias", "duplicated_rows", "saturated",
         "constant_score_bias", "duplicated_rows_score_bias", "cross_lane_ties"]


@pytest.mark.parametrize("name,T", [(n, T) for n in CASES for T in (64, 256)] +
                         [("cross_lane_ties", 2048)])
def test_exact_ties_take_the_lower_index_in_score_order(name, T):
    x, wg, gb, sb = _case(name, T)
    cfg = moe.config(T, D, E, K, 1536, SCALE)
    ws = moe.workspace(cfg)
    idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, K), -1.0, dtype=torch.float32, device="cuda")
    moe.moe_route2(cfg, x, wg, gb, sb, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()

    ref = oracle.route(oracle.bf16_bits(x), oracle.bf16_bits(wg), K, SCALE,
                       None if gb is None else gb.cpu().numpy(),
                       score_bias=None if sb is None else sb.cpu().numpy())
    _expected_structure(name, ref["idx"])
    assert np.any(ref["gap"] == 0.0), "the case has no exact tie at the k-th place"
    bad = np.nonzero(np.any(gi != ref["idx"], axis=1))[0]
    assert bad.size == 0, (f"{bad.size} tokens differ in index order, first {bad[:4].tolist()}: "
                           f"gpu {gi[bad[0]].tolist()} oracle {ref['idx'][bad[0]].tolist()}")
    np.testing.assert_allclose(gw, ref["w"], rtol=W_RTOL_TIE, atol=0)
    if name in ("all_zero", "constant_gate_bias", "constant_score_bias"):
        np.testing.assert_allclose(gw, SCALE / K, rtol=W_RTOL_TIE)   # 0.35325
    print(name, T, "tokens with a zero gap:", int((ref["gap"] == 0).sum()))
