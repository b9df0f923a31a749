"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers of the library cannot call cudaMalloc or keep a workspace (a host
framework that hands plugins no device memory, a latency-critical loop where
an allocation may synchronise the device). moe_route_noalloc serves them: its
scratch is a fixed device array inside the library. These tests call it
through the C ABI and check it against moe_route (the workspace entry point)
on two calls in a row, so that the second call sees the array as the first
one left it. The file is collected last and passes alone or after the rest.
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
    LayerShape(T=2728, d=4096, E=192, k=8, F=1536, zipf_bias=True),  # the largest batch that fits
    CONFIGS["tiny"],
], ids=["decode", "largest_T_for_E192", "tiny"])
def test_noalloc_route_matches_moe_route_on_two_calls(shape):
    moe_build.build()
    layer = make_layer(shape, seed=7, device="cuda", with_experts=False)
    cfg = moe.config_of(shape)
    want_idx, want_w = _route_ws(cfg, layer)
    gb = layer.get("gate_bias")
    gap = oracle.route(oracle.bf16_bits(layer["x"]), oracle.bf16_bits(layer["w_gate"]), shape.k,
                       shape.scale, None if gb is None else gb.cpu().numpy())["gap"]
    firm = gap >= NEAR_TIE
    for _ in range(2):
        idx, w = _route_noalloc(cfg, layer)
        for t in np.nonzero(firm)[0]:
            assert set(idx[t]) == set(want_idx[t]), t
            ref = dict(zip(want_idx[t].tolist(), want_w[t].tolist()))
            for j, e in enumerate(idx[t].tolist()):
                assert abs(w[t, j] - ref[e]) <= W_RTOL * abs(ref[e]), (t, e)


def test_noalloc_route_rejects_batches_beyond_its_scratch():
    moe_build.build()
    shape = LayerShape(T=2729, d=4096, E=192, k=8, F=1536)
    cfg = moe.config_of(shape)
    x = torch.zeros((shape.T, shape.d), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros((shape.E, shape.d), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as err:
        moe.moe_route_noalloc(cfg, x, wg, None, idx, w)
    assert err.value.code == moe.MOE_ERR_UNSUPPORTED_SHAPE
