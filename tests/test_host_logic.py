"""Host-side logic that needs no GPU: the synthetic generator's draw order,
the binding's argument assembly, the workspace sizing and the benchmark's
work accounting."""

import dataclasses

import pytest
import torch

from sparse_moe_transformer_gemm_b200 import build as moe_build
from sparse_moe_transformer_gemm_b200 import moe, work
from synthetic import CONFIGS, LayerShape, make_layer
from synthetic.moe_inputs import encode_e2m1_blocks

BASE = LayerShape(T=12, d=128, E=6, k=2, F=128)


def test_generator_is_deterministic_per_seed():
    a, b, c = make_layer(BASE, seed=3), make_layer(BASE, seed=3), make_layer(BASE, seed=4)
    for key in ("x", "w_gate", "w_gate_up", "w_down"):
        assert torch.equal(a[key], b[key]), key
        assert not torch.equal(a[key], c[key]), key


def test_optional_draws_come_last_and_leave_earlier_tensors_alone():
    plain = make_layer(BASE, seed=5)
    full = make_layer(dataclasses.replace(BASE, shared=True, score_bias_std=0.05,
                                          route_norm=True), seed=5)
    for key in ("x", "w_gate", "w_gate_up", "w_down"):
        assert torch.equal(plain[key], full[key]), key
    assert full["w_shared_gate_up"].shape == (2 * BASE.F, BASE.d)
    assert full["w_shared_down"].shape == (BASE.d, BASE.F)
    assert full["score_bias"].shape == (BASE.E,) and full["score_bias"].dtype == torch.float32
    assert full["route_norm_weight"].shape == (BASE.d,)
    assert plain["score_bias"] is None and plain["route_norm_weight"] is None


def test_router_only_draw_matches_the_full_draw():
    r = make_layer(CONFIGS["tiny"], seed=2, with_experts=False)
    f = make_layer(CONFIGS["tiny"], seed=2)
    assert torch.equal(r["x"], f["x"]) and torch.equal(r["w_gate"], f["w_gate"])


def test_layer_args_append_the_shared_expert_as_expert_E():
    sh = dataclasses.replace(BASE, shared=True)
    L = make_layer(sh, seed=1)
    gu, s_gu, dn, s_dn = moe.layer_args(L)
    assert gu.shape == (BASE.E + 1, 2 * BASE.F, BASE.d) and s_gu is None
    assert torch.equal(gu[:BASE.E], L["w_gate_up"]) and torch.equal(gu[BASE.E], L["w_shared_gate_up"])
    assert torch.equal(dn[BASE.E], L["w_shared_down"]) and s_dn is None
    f8 = make_layer(dataclasses.replace(sh, fp8=True), seed=1)
    q_gu, s_gu, q_dn, s_dn = moe.layer_args(f8)
    assert q_gu.shape[0] == s_gu.shape[0] == q_dn.shape[0] == s_dn.shape[0] == BASE.E + 1
    assert torch.equal(s_gu[BASE.E], f8["s_shared_gate_up"])


def test_config_flags():
    c = moe.config(64, 4096, 192, 8, 1536, fp8=True, path="stream")
    assert c.flags == moe.MOE_FLAG_FP8_WEIGHTS | moe.MOE_FLAG_STREAM_PATH
    c = moe.config(64, 4096, 192, 8, 1536, packed=True, shared=True, path="gemm")
    assert c.flags == (moe.MOE_FLAG_PACKED_WEIGHTS | moe.MOE_FLAG_SHARED_EXPERT |
                       moe.MOE_FLAG_GEMM_PATH)
    with pytest.raises(ValueError):
        moe.config(64, 4096, 192, 8, 1536, path="fast")
    assert moe.config_of(dataclasses.replace(CONFIGS["decode"], shared=True)).flags == \
        moe.MOE_FLAG_SHARED_EXPERT
    assert moe.config_of(CONFIGS["fp4_decode"]).flags == moe.MOE_FLAG_FP4_WEIGHTS


def test_fp4_layer_args_are_the_codes_and_block_scales():
    sh = dataclasses.replace(BASE, fp4=True)
    L = make_layer(sh, seed=2)
    q_gu, s_gu, q_dn, s_dn = moe.layer_args(L)
    assert q_gu.dtype == s_gu.dtype == torch.uint8
    assert q_gu.shape == (sh.E, 2 * sh.F, sh.d // 2) and s_gu.shape == (sh.E, 2 * sh.F, sh.d // 32)
    assert q_dn.shape == (sh.E, sh.d, sh.F // 2) and s_dn.shape == (sh.E, sh.d, sh.F // 32)
    # one expert at a time is the same encoding as the whole tensor at once
    q_all, s_all = encode_e2m1_blocks(L["w_gate_up"])
    assert torch.equal(q_all, q_gu) and torch.equal(s_all, s_gu)


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def test_workspace_grows_with_the_batch_and_the_shared_slot(lib):
    sizes = [moe.moe_workspace_size(moe.config(T, 4096, 192, 8, 1536)) for T in (1, 64, 4096)]
    assert sizes[0] < sizes[1] < sizes[2]
    R = 4096 * 8
    assert sizes[2] >= R * 4096 * 2 * 2 + R * 1536 * 2          # x_perm + y + h at prefill
    assert moe.moe_workspace_size(moe.config(64, 4096, 192, 8, 1536, shared=True)) >= \
        64 * 9 * (4096 * 2 * 2 + 1536 * 2)


def test_work_accounting_matches_the_page_figures():
    # 3 d F parameters per expert, 6 d F FLOPs per token per expert (Hy3 pages)
    assert work.expert_bytes(4096, 1536) == 3 * 4096 * 1536 * 2
    assert work.expert_bytes(4096, 1536, fp8=True) == 3 * 4096 * 1536 + (2 * 1536 + 4096) * 4
    # FP4: half a byte per weight and one E8M0 byte per 32 weights of a row
    assert work.expert_bytes(4096, 1536, fp4=True) == 3 * 4096 * 1536 // 2 + 3 * 4096 * 1536 // 32
    gw = work.gate_up_work(64, 384, 150, 4096, 1536, fp4=True)
    assert gw["bytes"] == 150 * (3072 * 4096 // 2 + 3072 * 128) + 64 * 4096 * 2
    # the grouped rows beyond the T tokens and the h write are implementation traffic
    assert gw["implementation_bytes"] == (384 - 64) * 4096 * 2 + 384 * 1536 * 2
    dw = work.down_work(384, 150, 4096, 1536)
    assert dw["bytes"] == 150 * 4096 * 1536 * 2
    assert dw["implementation_bytes"] == 384 * (1536 + 4096) * 2
    # the two steps' algorithmic bytes add up to the layer's, less the router and out
    lw = work.layer_work(64, 4096, 192, 6, 1536, touched=150, fp4=True)
    assert gw["bytes"] + work.down_work(384, 150, 4096, 1536, fp4=True)["bytes"] == \
        lw["bytes"] - 192 * 4096 * 2 - 64 * 4096 * 2
    lw = work.layer_work(64, 4096, 192, 8, 1536, touched=175)
    assert lw["flops"] == 2 * 64 * 4096 * 192 + 6 * 64 * 8 * 4096 * 1536
    assert lw["bytes"] >= 175 * work.expert_bytes(4096, 1536)


def test_gemm_tile_models_partition_each_experts_rows():
    """The token-tile models the GPU tests use to pick tokens that cover every
    tile: per expert the tiles are contiguous, start at row 0, end at n_e, and
    respect their maximum; all but an expert's last tile hold a multiple of 32
    rows (gemm_tiles); FP8 down's sub-tiles hold at most 192 rows and, below
    128 rows per expert on average, are gate_up's 192-row tiles."""
    import numpy as np
    import parity

    rng = np.random.default_rng(0)
    for _ in range(50):
        E = int(rng.integers(1, 40))
        counts = rng.integers(0, 1200, size=E)
        counts[rng.random(E) < 0.2] = 0
        for nmax in (64, 192, 256, 384):
            tiles = list(parity.gemm_tiles(counts, nmax))
            for e in range(E):
                mine = [(s, n) for ee, s, n in tiles if ee == e]
                assert sum(n for _, n in mine) == counts[e]
                pos = 0
                for j, (s, n) in enumerate(mine):
                    assert s == pos and 0 < n <= nmax
                    if j < len(mine) - 1:
                        assert n % 32 == 0
                    pos += n
        k = 8
        for T in (int(counts.sum()) // k, 16 * E):  # both sides of T*k = 128 E
            down = list(parity.fp8_down_tiles(counts, T, k, E))
            if T * k < 128 * E:
                assert down == list(parity.gemm_tiles(counts, parity.FP8_NMAX))
            for e in range(E):
                mine = [(s, n) for ee, s, n in down if ee == e]
                assert sum(n for _, n in mine) == counts[e]
                assert all(0 < n <= parity.FP8_SUB for _, n in mine)
                assert [s for s, _ in mine] == sorted(s for s, _ in mine)
