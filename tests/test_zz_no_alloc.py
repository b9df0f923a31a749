"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers of the library cannot call cudaMalloc or keep a workspace (a host
framework that hands plugins no device memory, a latency-critical loop where
an allocation may synchronise the device). moe_route_noalloc serves them: its
scratch is a fixed device array inside the library. These tests call it
through the C ABI and check it against moe_route (the workspace entry point)
on two calls in a row, so that the second call sees the array as the first
one left it, and against the oracle on a tiny layer. The file is collected
last and passes alone or after the rest.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from sparse_moe_transformer_gemm_b200 import build as moe_build
from sparse_moe_transformer_gemm_b200 import moe
from synthetic import CONFIGS, LayerShape, make_layer

pytestmark = pytest.mark.gpu

W_RTOL = 2e-5    # the routing-weight tolerance of the parity tests
NEAR_TIE = 1e-5  # tokens whose k-th/(k+1)-th oracle score gap is below this may differ


def _route_ws(cfg, layer):
    T, k = cfg.T, cfg.k
    ws = moe.workspace(cfg)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, layer["x"], layer["w_gate"], layer.get("gate_bias"), idx, w, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


def _route_noalloc(cfg, layer):
    T, k = cfg.T, cfg.k
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    rc = moe.lib().moe_route_noalloc(ctypes.byref(cfg), ptr(layer["x"]), ptr(layer["w_gate"]),
                                     ptr(layer.get("gate_bias")), ptr(idx), ptr(w),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == moe.MOE_OK, moe.moe_status_string(rc)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("shape", [
    CONFIGS["decode"],
    CONFIGS["tiny"],
    LayerShape(T=100, d=256, E=32, k=12, F=128),   # k > 8: the CUDA-core router at any T
], ids=["decode", "tiny", "k12"])
def test_noalloc_route_is_moe_route_bitwise_on_two_calls(shape):
    """Where moe_route runs the CUDA-core router (T <= 128, or k > 8) both calls
    run the same kernel with the same K split: identical bits, twice in a row
    (the second call finds the array as the first one left it)."""
    moe_build.build()
    layer = make_layer(shape, seed=7, device="cuda", with_experts=False)
    cfg = moe.config_of(shape)
    want_idx, want_w = _route_ws(cfg, layer)
    for _ in range(2):
        idx, w = _route_noalloc(cfg, layer)
        assert np.array_equal(idx, want_idx)
        assert np.array_equal(w.view(np.uint32), want_w.view(np.uint32))


def test_noalloc_route_at_the_largest_batch_agrees_with_moe_route_on_two_calls():
    """T = 2728 at E = 192 with the skewed logit bias: the largest batch whose
    logits fit the array. moe_route runs the tensor-core router here (another
    fp32 summation order), so the two agree in expert order on every token
    whose k-th/(k+1)-th oracle score gap is at least 1e-5, and in weight to
    2e-5 relative."""
    moe_build.build()
    shape = LayerShape(T=2728, d=4096, E=192, k=8, F=1536, zipf_bias=True)
    layer = make_layer(shape, seed=7, device="cuda", with_experts=False)
    cfg = moe.config_of(shape)
    want_idx, want_w = _route_ws(cfg, layer)
    gap = oracle.route(oracle.bf16_bits(layer["x"]), oracle.bf16_bits(layer["w_gate"]), shape.k,
                       shape.scale, layer["gate_bias"].cpu().numpy())["gap"]
    firm = np.nonzero(gap >= NEAR_TIE)[0]
    for _ in range(2):
        idx, w = _route_noalloc(cfg, layer)
        assert np.array_equal(idx[firm], want_idx[firm])
        np.testing.assert_allclose(w[firm], want_w[firm], rtol=W_RTOL, atol=0)


def test_noalloc_route_matches_the_oracle_on_a_tiny_layer():
    moe_build.build()
    shape = CONFIGS["tiny"]
    layer = make_layer(shape, seed=9, device="cuda", with_experts=False)
    ref = oracle.route(oracle.bf16_bits(layer["x"]), oracle.bf16_bits(layer["w_gate"]), shape.k,
                       shape.scale)
    idx, w = _route_noalloc(moe.config_of(shape), layer)
    firm = np.nonzero(ref["gap"] >= NEAR_TIE)[0]
    assert firm.size > 0.9 * shape.T
    assert np.array_equal(idx[firm], ref["idx"][firm])
    np.testing.assert_allclose(w[firm], ref["w"][firm], rtol=W_RTOL, atol=0)


@pytest.mark.parametrize("with_bias", [False, True])
def test_noalloc_route_rejects_batches_beyond_its_scratch(with_bias):
    """T = 2729 at E = 192 needs 4*2729*192 bytes of logits plus 1536 bytes of
    counters: more than the array holds (T = 2728 fits, above)."""
    moe_build.build()
    shape = LayerShape(T=2729, d=4096, E=192, k=8, F=1536)
    assert 4 * 2729 * 192 + 1536 > moe.MOE_NOALLOC_SCRATCH_BYTES >= 4 * 2728 * 192 + 1536
    cfg = moe.config_of(shape)
    x = torch.zeros((shape.T, shape.d), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros((shape.E, shape.d), dtype=torch.bfloat16, device="cuda")
    gb = torch.zeros(shape.E, dtype=torch.float32, device="cuda") if with_bias else None
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as err:
        moe.moe_route_noalloc(cfg, x, wg, gb, idx, w)
    assert err.value.code == moe.MOE_ERR_UNSUPPORTED_SHAPE
