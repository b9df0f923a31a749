"""The expert-parallel phases' compute done by the fp64 oracle, on CPU
tensors, for the multi-rank tests without a GPU (test infrastructure).

Each op mirrors one C-ABI call of sparse_moe_transformer_gemm_b200.ep.CudaOps:
route (oracle.route), group (oracle.permute plus the row gather it defines),
row_experts (the local expert of each received row, from the counts),
local_experts (oracle.expert_rows on the rank's expert slice, outputs rounded
to bf16 as the GPU path stores y) and combine (oracle.combine, fp64 sum, one
bf16 rounding).
"""

from __future__ import annotations

import numpy as np
import torch

import oracle


def _bits(t: torch.Tensor) -> np.ndarray:
    return oracle.bf16_bits(t)


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


class OracleOps:
    def __init__(self, part, rank, w_gate, gate_bias, w_gate_up, w_down, k, scale):
        self.part, self.rank, self.k, self.scale = part, rank, k, scale
        self.wg = _bits(w_gate)
        self.gb = None if gate_bias is None else gate_bias.numpy().astype(np.float32)
        sl = slice(rank * part.E_local, (rank + 1) * part.E_local)
        self.wgu = _bits(w_gate_up[sl])
        self.wd = _bits(w_down[sl])

    def route(self, x):
        r = oracle.route(_bits(x), self.wg, self.k, self.scale, self.gb)
        return torch.from_numpy(r["idx"]), torch.from_numpy(r["w"])

    def group(self, idx, x):
        T, k = idx.shape
        g = oracle.permute(idx.numpy(), self.part.E)
        row_of = g["row_of"]
        token_of_row = np.empty(T * k, dtype=np.int64)
        token_of_row[row_of] = np.arange(T * k) // k
        return (torch.from_numpy(g["counts"]), torch.from_numpy(row_of),
                x[torch.from_numpy(token_of_row)])

    def row_experts(self, recv_counts_pe, n_rows):
        c = recv_counts_pe.numpy()
        ids = np.tile(np.arange(self.part.E_local), c.shape[0])
        out = np.repeat(ids, c.reshape(-1)).astype(np.int32)
        assert out.size == n_rows
        return torch.from_numpy(out)

    def local_experts(self, rows, expert_of_row):
        y = oracle.expert_rows(_bits(rows), expert_of_row.numpy(), self.wgu, self.wd)
        return _bf16(oracle.bf16_from_double(y))

    def combine(self, y_back, row_of, w, T):
        y = oracle.double_from_bf16(_bits(y_back))[row_of.numpy()].reshape(T, self.k, -1)
        return _bf16(oracle.combine(y, w.numpy()))
