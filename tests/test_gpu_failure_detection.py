"""Failure detection on the device, without faulting, trapping or hanging the
GPU: a bounded wait on a barrier that nothing completes gives up after its
limit, records MOE_ERR_TIMEOUT in the workspace status word, and the context
stays usable (a layer call afterwards is correct and leaves the status ok)."""

import time

import pytest
import torch

from sparse_moe_transformer_gemm_b200 import build as moe_build
from sparse_moe_transformer_gemm_b200 import moe
from synthetic import CONFIGS, make_layer

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_reports_timeout_and_the_context_survives():
    moe_build.build()
    cfg = moe.config_of(CONFIGS["tiny"])
    ws = moe.workspace(cfg)
    assert moe.moe_read_status(ws) == moe.MOE_OK
    t0 = time.time()
    moe.moe_selftest_bounded_wait(ws, 50_000_000)          # 50 ms
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert moe.moe_read_status(ws) == moe.MOE_ERR_TIMEOUT
    assert moe.moe_read_status(ws) == moe.MOE_OK            # reading resets the word
    layer = make_layer(CONFIGS["tiny"], seed=0, device="cuda")
    out = torch.empty((64, 256), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(cfg, layer["x"], layer["w_gate"], None, *moe.layer_args(layer), out, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == moe.MOE_OK
    assert torch.isfinite(out.float()).all()


def test_selftest_rejects_bad_limits():
    moe_build.build()
    ws = moe.workspace(moe.config_of(CONFIGS["tiny"]))
    for bad in (0, 10_000_000_001):
        with pytest.raises(moe.MoeError):
            moe.moe_selftest_bounded_wait(ws, bad)
