"""Expert parallelism ("DeepSeek V4-Flash 架构 QA" Q4.7 and Q4.10) on CPU
ranks: the dispatch / exchange / combine logic of
sparse_moe_transformer_gemm_b200.ep, with the fp64 oracle doing each rank's
compute (tests/ep_oracle_ops.py).

* P ranks in one process (the lockstep driver) give every rank bitwise the
  output of one rank holding all experts, for P = 2 and 4, including a rank
  that receives no rows;
* two gloo processes (the torch.distributed driver, all_to_all_single) give
  the same bits as the lockstep driver, and so does the pipelined driver on
  1, 3 or 30 chunks of each rank's tokens (30 > tokens: empty chunks);
* the single-rank result matches the oracle's own forward within the layer's
  output tolerance (the EP path stores the expert outputs as bf16, as the GPU
  path does; the oracle keeps them in fp64).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import parity
from ep_oracle_ops import OracleOps
from sparse_moe_transformer_gemm_b200 import ep
from synthetic import LayerShape, make_layer

SHAPE = LayerShape(T=48, d=256, E=16, k=4, F=128)


def _layer(bias_rank0=False):
    L = make_layer(SHAPE, seed=21)
    if bias_rank0:
        # every token picks 4 of experts 0..7: with P = 2, rank 1 receives nothing
        b = torch.zeros(SHAPE.E)
        b[:8] = 30.0
        L["gate_bias"] = b
    return L


def _ops(L, part, rank):
    return OracleOps(part, rank, L["w_gate"], L.get("gate_bias"), L["w_gate_up"], L["w_down"],
                     SHAPE.k, SHAPE.scale)


def _shards(x, P):
    return list(torch.chunk(x, P))


def test_partition_splits_experts_evenly():
    part = ep.Partition(E=192, P=8)
    assert part.E_local == 24 and part.experts_of(3) == range(72, 96)
    assert part.owner(95) == 3 and part.owner(96) == 4
    with pytest.raises(ValueError):
        ep.Partition(E=192, P=7)


@pytest.mark.parametrize("P", [2, 4])
@pytest.mark.parametrize("bias_rank0", [False, True])
def test_lockstep_ranks_equal_one_rank_bitwise(P, bias_rank0):
    L = _layer(bias_rank0)
    one = ep.Partition(SHAPE.E, 1)
    part = ep.Partition(SHAPE.E, P)
    xs = _shards(L["x"], P)
    outs = ep.ep_forward_lockstep([_ops(L, part, r) for r in range(P)], part, xs)
    for r in range(P):
        want = ep.ep_forward_lockstep([_ops(L, one, 0)], one, [xs[r]])[0]
        assert torch.equal(outs[r].view(torch.int16), want.view(torch.int16)), r


def test_one_rank_matches_the_oracle_forward():
    L = _layer()
    one = ep.Partition(SHAPE.E, 1)
    out = ep.ep_forward_lockstep([_ops(L, one, 0)], one, [L["x"]])[0]
    ref = oracle.forward_tokens(oracle.OracleLayer(L))
    rel, mx = parity.compare_out(oracle.bf16_bits(out), ref["out_bf16"])
    assert rel <= parity.REL_L2 and mx <= parity.MAX_ABS, (rel, mx)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, bias_rank0, out, chunks=0):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = _layer(bias_rank0)
        part = ep.Partition(SHAPE.E, world)
        x = _shards(L["x"], world)[rank]
        if chunks:
            y = ep.ep_forward_pipelined(_ops(L, part, rank), part, x, chunks=chunks)
        else:
            y = ep.ep_forward(_ops(L, part, rank), part, x)
        out[rank] = oracle.bf16_bits(y)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bias_rank0", [False, True])
def test_two_gloo_ranks_equal_the_lockstep_driver(bias_rank0):
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, bias_rank0, out), nprocs=world, join=True)
        res = dict(out)
    L = _layer(bias_rank0)
    part = ep.Partition(SHAPE.E, world)
    want = ep.ep_forward_lockstep([_ops(L, part, r) for r in range(world)], part,
                                  _shards(L["x"], world))
    for r in range(world):
        assert np.array_equal(res[r], oracle.bf16_bits(want[r])), r


def test_chunk_bounds_cover_the_tokens_in_order():
    assert ep.chunk_bounds(10, 3) == [0, 4, 7, 10]
    assert ep.chunk_bounds(2, 3) == [0, 1, 2, 2]
    assert ep.chunk_bounds(0, 2) == [0, 0, 0]
    with pytest.raises(ValueError):
        ep.chunk_bounds(5, 0)


@pytest.mark.parametrize("chunks", [1, 3, 30])
def test_two_gloo_ranks_pipelined_equal_the_lockstep_driver(chunks):
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, True, out, chunks), nprocs=world, join=True)
        res = dict(out)
    L = _layer(True)
    part = ep.Partition(SHAPE.E, world)
    want = ep.ep_forward_lockstep([_ops(L, part, r) for r in range(world)], part,
                                  _shards(L["x"], world))
    for r in range(world):
        assert np.array_equal(res[r], oracle.bf16_bits(want[r])), r
