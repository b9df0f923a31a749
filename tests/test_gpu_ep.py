"""Expert parallelism through the C ABI on one GPU ("DeepSeek V4-Flash 架构 QA"
Q4.7 and Q4.10): P ranks run in lockstep in one process (no kernel of one
rank waits on another's; the exchanges are slices), each with the C-ABI ops of
sparse_moe_transformer_gemm_b200.ep. Every rank's output must equal, bitwise,
moe_forward on that rank's tokens with all experts on one GPU -- and that one
is checked against the oracle by the parity tests.
"""

import dataclasses
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import parity
from sparse_moe_transformer_gemm_b200 import build as moe_build
from sparse_moe_transformer_gemm_b200 import ep, moe
from synthetic import CONFIGS, LayerShape, make_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    moe_build.build()
    oracle.build()
    assert torch.cuda.is_available()


def _ep_vs_forward(shape, P, seed, bias_first_rank=False):
    L = make_layer(shape, seed=seed, device="cuda")
    if bias_first_rank:
        # every token routes to experts of rank 0: the others receive no rows
        b = torch.zeros(shape.E, dtype=torch.float32, device="cuda")
        b[: shape.E // P] = 30.0
        L["gate_bias"] = b
    cfg = moe.config_of(shape)
    part = ep.Partition(shape.E, P)
    wgu, sgu, wd, sd = moe.layer_args(L)
    ops = [ep.ep_layer_ops(cfg, part, r, L["w_gate"], L["gate_bias"], wgu, sgu, wd, sd)
           for r in range(P)]
    xs = list(torch.chunk(L["x"], P))
    outs = ep.ep_forward_lockstep(ops, part, xs)
    torch.cuda.synchronize()
    for r in range(P):
        Tr = xs[r].shape[0]
        c = moe.config_of(dataclasses.replace(shape, T=Tr))
        ws = moe.workspace(c)
        want = torch.empty((Tr, shape.d), dtype=torch.bfloat16, device="cuda")
        moe.moe_forward(c, xs[r].contiguous(), L["w_gate"], L["gate_bias"], wgu, sgu, wd, sd,
                        want, ws)
        torch.cuda.synchronize()
        assert moe.moe_read_status(ws) == moe.MOE_OK
        assert torch.equal(outs[r], want), f"rank {r} of {P}"
    return L, outs


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_ep_on_the_hy3_decode_shape_equals_moe_forward_per_rank(P):
    """T = 64 tokens per rank, 192 experts over P ranks (24 each at P = 8)."""
    shape = dataclasses.replace(CONFIGS["decode"], T=64 * P)
    _ep_vs_forward(shape, P, seed=40 + P)


@pytest.mark.parametrize("name,shape", [
    ("pair_ragged", LayerShape(T=333, d=768, E=24, k=6, F=256, zipf_bias=True)),
    ("single_sm", LayerShape(T=300, d=512, E=32, k=8, F=384)),
    ("fp8", LayerShape(T=333, d=768, E=24, k=6, F=512, fp8=True)),
])
def test_ep_small_shapes_equal_moe_forward_and_the_oracle(name, shape):
    L, outs = _ep_vs_forward(shape, 4 if shape.E % 4 == 0 else 2, seed=7)
    # and the gathered outputs against the oracle on every token
    out = torch.cat(outs)
    res = parity.check_forward(L, out, None, parity.gpu_route(L))
    print(name, res)


def test_ep_with_ranks_that_receive_nothing():
    shape = LayerShape(T=128, d=512, E=16, k=4, F=256)
    _ep_vs_forward(shape, 4, seed=3, bias_first_rank=True)


@pytest.mark.parametrize("n_src,e_local", [(1, 1), (3, 24), (8, 24), (5, 256), (32, 256)])
def test_row_experts_kernel_expands_the_counts(n_src, e_local):
    g = torch.Generator().manual_seed(n_src * 1000 + e_local)
    counts = torch.randint(0, 40, (n_src, e_local), generator=g, dtype=torch.int32)
    counts[0, 0] = 0
    counts[-1, -1] = 0
    n = int(counts.sum())
    want = np.repeat(np.tile(np.arange(e_local), n_src), counts.numpy().reshape(-1))
    ids = torch.full((n + 5,), 7, dtype=torch.int32, device="cuda")
    moe.moe_ep_row_experts(counts.cuda(), n_src, e_local, ids)
    torch.cuda.synchronize()
    got = ids.cpu().numpy()
    assert np.array_equal(got[:n], want)
    assert np.all(got[n:] == -1)


def test_pipelined_driver_on_one_nccl_rank_equals_moe_forward_per_chunk():
    """ep_forward_pipelined through a one-rank NCCL group: 192 tokens in three
    chunks of 64 (the Hy3 decode shape per chunk), each chunk's output bitwise
    moe_forward's on those tokens."""
    import torch.distributed as dist

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        shape = dataclasses.replace(CONFIGS["decode"], T=192)
        L = make_layer(shape, seed=11, device="cuda")
        cfg = moe.config_of(shape)
        part = ep.Partition(shape.E, 1)
        wgu, sgu, wd, sd = moe.layer_args(L)
        ops = ep.ep_layer_ops(cfg, part, 0, L["w_gate"], L["gate_bias"], wgu, sgu, wd, sd)
        y = ep.ep_forward_pipelined(ops, part, L["x"], chunks=3)
        torch.cuda.synchronize()
        for c in range(3):
            xc = L["x"][64 * c:64 * (c + 1)].contiguous()
            cc = moe.config_of(dataclasses.replace(shape, T=64))
            ws = moe.workspace(cc)
            want = torch.empty((64, shape.d), dtype=torch.bfloat16, device="cuda")
            moe.moe_forward(cc, xc, L["w_gate"], L["gate_bias"], wgu, sgu, wd, sd, want, ws)
            torch.cuda.synchronize()
            assert moe.moe_read_status(ws) == moe.MOE_OK
            assert torch.equal(y[64 * c:64 * (c + 1)], want), f"chunk {c}"
    finally:
        dist.destroy_process_group()
