"""Expert parallelism of the routed-MoE layer over P ranks.

"DeepSeek V4-Flash 架构 QA" (cctoctofx.netlify.app) Q4.7 describes the MoE's
expert-parallel strategy: the experts are split over the GPUs, every token is
sent to the GPUs that hold the experts it selected, and their outputs come
back for the weighted sum -- two all-to-all exchanges per layer, whose
traffic Q4.10 counts (T*k*d activations each way). Here:

  rank r holds the E_local = E/P experts [r*E_local, (r+1)*E_local) and its
  own batch of tokens (every rank keeps the whole router weight).
  1. dispatch: route the rank's tokens (moe_route3) and group their
     token-slots by expert (moe_permute). A rank's experts are consecutive,
     so the grouped rows already form one block per destination rank.
  2. exchange the per-(destination, expert) row counts, then the rows.
  3. experts: the local expert of every received row (moe_ep_row_experts),
     the rows regrouped by expert (moe_permute with k = 1), the SwiGLU grouped
     GEMMs on the rank's expert weights (moe_experts), and the outputs put
     back in arrival order (moe_combine with k = 1 and weight 1: an exact
     copy of each bf16 row).
  4. exchange the outputs back: each source receives its rows' outputs in
     the order it sent them, which is its own grouped order.
  5. combine: the fp32 weighted sum with the source's row_of and routing
     weights (moe_combine), as in the single-GPU layer.

Every output row of the grouped GEMMs depends only on its token row and its
expert's weights, and the combine sums the same k rows in the same slot
order, so a rank's result is bitwise what moe_forward gives for its tokens
with all E experts on one GPU.

Three drivers run the same phases: ``ep_forward`` exchanges through
torch.distributed (all_to_all_single; NCCL on GPUs, any backend that has it
on CPU tensors); ``ep_forward_pipelined`` does the same on C chunks of the
rank's tokens with the row exchanges in flight while the experts of an
earlier chunk run (Q4.10's point that the all-to-all time should hide
behind the expert compute); ``ep_forward_lockstep`` runs all P ranks in one
process and exchanges by slicing (no kernel of one rank waits on another's,
so the ranks can share one device). The compute is an ``ops`` object:
``CudaOps`` calls the library's C ABI; the phases never compute on the host.
"""

from __future__ import annotations

import dataclasses
from typing import List

import torch

from . import moe


@dataclasses.dataclass(frozen=True)
class Partition:
    """E experts over P ranks, E_local consecutive experts each."""

    E: int
    P: int

    def __post_init__(self):
        if self.P < 1 or self.E % self.P != 0:
            raise ValueError(f"{self.E} experts do not split evenly over {self.P} ranks")

    @property
    def E_local(self) -> int:
        return self.E // self.P

    def experts_of(self, rank: int) -> range:
        return range(rank * self.E_local, (rank + 1) * self.E_local)

    def owner(self, e: int) -> int:
        return e // self.E_local


@dataclasses.dataclass
class Dispatched:
    """A rank's state between dispatch and combine."""

    idx: torch.Tensor        # [T, k] int32 routing
    w: torch.Tensor          # [T, k] routing weights
    row_of: torch.Tensor     # [T*k] grouped row of each token-slot
    x_perm: torch.Tensor     # [T*k, d] grouped token rows (the send buffer)
    counts_pe: torch.Tensor  # [P, E_local] rows per (destination, expert), on the host
    T: int

    @property
    def send_splits(self) -> List[int]:
        return self.counts_pe.sum(dim=1).tolist()


def dispatch(ops, part: Partition, x: torch.Tensor) -> Dispatched:
    """Phase 1: route and group the rank's tokens; the send blocks per destination.
    No tokens: empty blocks (no call into ops)."""
    T = x.shape[0]
    if T == 0:
        k = ops.k
        return Dispatched(torch.empty((0, k), dtype=torch.int32, device=x.device),
                          torch.empty((0, k), dtype=torch.float32, device=x.device),
                          torch.empty(0, dtype=torch.int32, device=x.device), x[:0],
                          torch.zeros((part.P, part.E_local), dtype=torch.int64), 0)
    idx, w = ops.route(x)
    counts, row_of, x_perm = ops.group(idx, x)
    counts_pe = counts.to("cpu", torch.int64).view(part.P, part.E_local)
    return Dispatched(idx, w, row_of, x_perm, counts_pe, T)


def run_experts(ops, part: Partition, rows: torch.Tensor,
                recv_counts_pe: torch.Tensor) -> torch.Tensor:
    """Phase 3: the received rows ([n, d], source by source, each grouped by
    local expert, recv_counts_pe [P, E_local] on the host) through the rank's
    experts; outputs in arrival order."""
    if rows.shape[0] == 0:
        return rows.clone()
    expert_of_row = ops.row_experts(recv_counts_pe, rows.shape[0])
    return ops.local_experts(rows, expert_of_row)


def combine(ops, state: Dispatched, y_back: torch.Tensor) -> torch.Tensor:
    """Phase 5: the fp32 weighted combine of the returned rows."""
    if state.T == 0:
        return y_back[:0]
    return ops.combine(y_back, state.row_of, state.w, state.T)


# ---------------------------------------------------------------- drivers


def _a2a_rows(dist, group, send: torch.Tensor, send_splits, recv_splits) -> torch.Tensor:
    """all_to_all_single of [n, d] rows with per-rank splits (bf16 rows travel
    as int32 pairs -- d is even -- which every backend carries)."""
    out = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype,
                      device=send.device)
    s = send.contiguous()
    if send.dtype == torch.bfloat16:
        s, o = s.view(torch.int32), out.view(torch.int32)
    else:
        o = out
    dist.all_to_all_single(o, s, recv_splits, send_splits, group=group)
    return out


def ep_forward(ops, part: Partition, x: torch.Tensor, group=None) -> torch.Tensor:
    """The expert-parallel layer on this rank (torch.distributed process group
    of P ranks, rank r holding part.experts_of(r)). Every rank takes the same
    collective steps in the same order, with empty blocks where it has none."""
    import torch.distributed as dist

    if dist.get_world_size(group) != part.P:
        raise ValueError("the process group does not have P ranks")
    st = dispatch(ops, part, x)
    dev = st.x_perm.device
    send_c = st.counts_pe.to(device=dev, dtype=torch.int64).contiguous()
    recv_c = torch.empty_like(send_c)
    dist.all_to_all_single(recv_c, send_c, group=group)  # row p goes to rank p
    recv_counts_pe = recv_c.to("cpu")
    recv_splits = recv_counts_pe.sum(dim=1).tolist()
    rows = _a2a_rows(dist, group, st.x_perm, st.send_splits, recv_splits)
    y = run_experts(ops, part, rows, recv_counts_pe)
    y_back = _a2a_rows(dist, group, y, recv_splits, st.send_splits)
    return combine(ops, st, y_back)


def _a2a_rows_async(dist, group, send: torch.Tensor, send_splits, recv_splits):
    """_a2a_rows started asynchronously: (output, work handle)."""
    out = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype,
                      device=send.device)
    s = send.contiguous()
    if send.dtype == torch.bfloat16:
        s, o = s.view(torch.int32), out.view(torch.int32)
    else:
        o = out
    work = dist.all_to_all_single(o, s, recv_splits, send_splits, group=group, async_op=True)
    return out, (work, s)  # the send buffer stays referenced until the wait


def chunk_bounds(T: int, chunks: int) -> List[int]:
    """Token offsets of C near-equal contiguous chunks (empty ones when T < C)."""
    if chunks < 1:
        raise ValueError("chunks must be >= 1")
    q, r = divmod(T, chunks)
    b = [0]
    for c in range(chunks):
        b.append(b[-1] + q + (1 if c < r else 0))
    return b


def ep_forward_pipelined(ops, part: Partition, x: torch.Tensor, chunks: int = 2,
                         group=None) -> torch.Tensor:
    """ep_forward on `chunks` contiguous chunks of the rank's tokens, pipelined:
    every chunk is dispatched and its rows sent first (the row exchanges in
    flight together); then each chunk's experts run as soon as its rows have
    arrived, and its outputs start back while the next chunk's experts run;
    the combines come last. Every rank takes the same collective steps in the
    same order (chunks number the same on every rank; empty chunks exchange
    empty blocks). A token's output depends only on its own rows, so the
    result equals ep_forward on each chunk by itself."""
    import torch.distributed as dist

    if dist.get_world_size(group) != part.P:
        raise ValueError("the process group does not have P ranks")
    b = chunk_bounds(x.shape[0], chunks)
    sts, rows, recv = [], [], []
    for c in range(chunks):
        st = dispatch(ops, part, x[b[c]:b[c + 1]])
        dev = st.x_perm.device
        send_c = st.counts_pe.to(device=dev, dtype=torch.int64).contiguous()
        recv_c = torch.empty_like(send_c)
        dist.all_to_all_single(recv_c, send_c, group=group)  # row p goes to rank p
        recv_counts_pe = recv_c.to("cpu")
        sts.append(st)
        recv.append(recv_counts_pe)
        rows.append(_a2a_rows_async(dist, group, st.x_perm, st.send_splits,
                                    recv_counts_pe.sum(dim=1).tolist()))
    backs = []
    for c in range(chunks):
        r, (work, _) = rows[c]
        work.wait()
        y = run_experts(ops, part, r, recv[c])
        backs.append(_a2a_rows_async(dist, group, y, recv[c].sum(dim=1).tolist(),
                                     sts[c].send_splits))
    outs = []
    for c in range(chunks):
        y_back, (work, _) = backs[c]
        work.wait()
        outs.append(combine(ops, sts[c], y_back))
    return torch.cat(outs) if outs else x.new_empty((0, x.shape[1]))


def ep_forward_lockstep(ops_per_rank, part: Partition, xs) -> List[torch.Tensor]:
    """All P ranks in one process (rank r: ops_per_rank[r], tokens xs[r]); the
    exchanges are done by slicing the send buffers."""
    P = part.P
    sts = [dispatch(ops_per_rank[r], part, xs[r]) for r in range(P)]
    blocks = []  # blocks[r][p]: rows rank r sends to rank p
    for st in sts:
        off = [0]
        for n in st.send_splits:
            off.append(off[-1] + n)
        blocks.append([st.x_perm[off[p]:off[p + 1]] for p in range(P)])
    ys = []
    for p in range(P):
        recv_counts_pe = torch.stack([sts[r].counts_pe[p] for r in range(P)])
        rows = torch.cat([blocks[r][p] for r in range(P)])
        ys.append((run_experts(ops_per_rank[p], part, rows, recv_counts_pe),
                   recv_counts_pe.sum(dim=1).tolist()))
    outs = []
    for r in range(P):
        back = []
        for p in range(P):
            y, splits = ys[p]
            start = sum(splits[:r])
            back.append(y[start:start + splits[r]])
        outs.append(combine(ops_per_rank[r], sts[r], torch.cat(back)))
    return outs


# ---------------------------------------------------------------- CUDA ops


class CudaOps:
    """The phases' compute through the library's C ABI, for one rank.

    cfg: the layer's moe_config with all E experts (T is taken from each call);
    w_gate [E, d] and gate_bias (nullable [E]) the full router; w_gate_up /
    w_down (and s_gate_up / s_down for FP8) the rank's E_local experts.
    """

    def __init__(self, cfg, part: Partition, w_gate, gate_bias, w_gate_up, s_gate_up, w_down,
                 s_down, route_options=None, stream=None):
        if cfg.flags & moe.MOE_FLAG_SHARED_EXPERT:
            raise ValueError("expert parallelism here covers the routed experts only")
        self.cfg, self.part = cfg, part
        self.w_gate, self.gate_bias = w_gate, gate_bias
        self.w_gate_up, self.s_gate_up = w_gate_up, s_gate_up
        self.w_down, self.s_down = w_down, s_down
        self.ropt = route_options
        self.stream = stream
        self.dev = w_gate.device
        self.k = cfg.k

    def _cfg(self, T: int, E: int, k: int):
        return moe.MoeConfig(T, self.cfg.d, E, k, self.cfg.d_ff, self.cfg.scale, self.cfg.flags)

    def route(self, x):
        T, k = x.shape[0], self.cfg.k
        c = self._cfg(T, self.part.E, k)
        self._ws = moe.workspace(c, device=self.dev, stream=self.stream)
        idx = torch.empty((T, k), dtype=torch.int32, device=self.dev)
        w = torch.empty((T, k), dtype=torch.float32, device=self.dev)
        moe.moe_route3(c, x, self.w_gate, self.gate_bias, self.ropt, idx, w, self._ws,
                       self.stream)
        return idx, w

    def group(self, idx, x):
        T, k = idx.shape
        c = self._cfg(T, self.part.E, k)
        counts = torch.empty(self.part.E, dtype=torch.int32, device=self.dev)
        offsets = torch.empty(self.part.E + 1, dtype=torch.int32, device=self.dev)
        row_of = torch.empty(T * k, dtype=torch.int32, device=self.dev)
        x_perm = torch.empty((T * k, self.cfg.d), dtype=torch.bfloat16, device=self.dev)
        moe.moe_permute(c, idx, x, counts, offsets, row_of, x_perm, self._ws, self.stream)
        return counts, row_of, x_perm

    def row_experts(self, recv_counts_pe, n_rows: int):
        counts = recv_counts_pe.to(device=self.dev, dtype=torch.int32).contiguous()
        ids = torch.empty(n_rows, dtype=torch.int32, device=self.dev)
        moe.moe_ep_row_experts(counts, counts.shape[0], counts.shape[1], ids, self.stream)
        return ids

    def local_experts(self, rows, expert_of_row):
        n, El = rows.shape[0], self.part.E_local
        c = self._cfg(n, El, 1)
        ws = moe.workspace(c, device=self.dev, stream=self.stream)
        counts = torch.empty(El, dtype=torch.int32, device=self.dev)
        offsets = torch.empty(El + 1, dtype=torch.int32, device=self.dev)
        row_of = torch.empty(n, dtype=torch.int32, device=self.dev)
        x_perm = torch.empty_like(rows)
        y = torch.empty_like(rows)
        moe.moe_permute(c, expert_of_row.view(n, 1), rows, counts, offsets, row_of, x_perm, ws,
                        self.stream)
        moe.moe_experts(c, x_perm, offsets, self.w_gate_up, self.s_gate_up, self.w_down,
                        self.s_down, y, ws, self.stream)
        ones = torch.ones(n, dtype=torch.float32, device=self.dev)
        back = torch.empty_like(rows)
        moe.moe_combine(c, y, row_of, ones, back, ws, self.stream)  # exact copy per row
        return back

    def combine(self, y_back, row_of, w, T: int):
        c = self._cfg(T, self.part.E, self.cfg.k)
        out = torch.empty((T, self.cfg.d), dtype=torch.bfloat16, device=self.dev)
        moe.moe_combine(c, y_back, row_of, w, out, self._ws, self.stream)
        return out


def local_expert_weights(part: Partition, rank: int, w_gate_up, w_down, s_gate_up=None,
                         s_down=None):
    """The slices of the experts' weights (and FP8 scales) that rank holds."""
    sl = slice(rank * part.E_local, (rank + 1) * part.E_local)
    pick = (lambda t: None if t is None else t[sl])  # noqa: E731
    return pick(w_gate_up), pick(s_gate_up), pick(w_down), pick(s_down)


def ep_layer_ops(cfg, part: Partition, rank: int, w_gate, gate_bias, w_gate_up, s_gate_up,
                 w_down, s_down, route_options=None, stream=None) -> CudaOps:
    """CudaOps for rank ``rank`` from the full layer's tensors (the rank keeps
    views of its experts' slices)."""
    gu, sgu, dn, sdn = local_expert_weights(part, rank, w_gate_up, w_down, s_gate_up, s_down)
    return CudaOps(cfg, part, w_gate, gate_bias, gu, sgu, dn, sdn, route_options, stream)


__all__ = ["Partition", "Dispatched", "dispatch", "run_experts", "combine", "ep_forward",
           "ep_forward_pipelined", "chunk_bounds", "ep_forward_lockstep", "CudaOps",
           "local_expert_weights", "ep_layer_ops"]
