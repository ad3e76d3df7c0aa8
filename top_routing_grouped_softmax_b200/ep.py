"""Expert parallelism for the MoE block forward: experts sharded over ranks,
token rows dispatched to their experts' owners by an all-to-all and returned
by a second one.

The pages name this scheme without fixing its layout: data parallelism plus
expert parallelism with an all-to-all between them ("MoE acceleration
engine", section 4.3), and a hierarchical all-to-all for dispatch and
combine (the Hunyuan-Large overview, section 5.1).  Reading used here, one
process per GPU:

* Rank r of W owns the contiguous expert block [r * E / W, (r + 1) * E / W)
  (E % W == 0) and holds the weights of those experts only.  Every rank
  keeps the whole router.
* Each rank routes and groups its own tokens over all E experts with the
  library's kernels (moe_route, moe_permute).  Because groups are laid out in
  expert order and owners hold contiguous expert blocks, the rows bound for
  rank q are one contiguous slice of the grouped rows.
* The per-expert counts go first (an all-to-all of W x E/W integers), so
  every rank knows how many rows each source sends for each of its experts;
  then the grouped rows (bf16) and their routing weights (fp32) go by an
  all-to-all with those split sizes.
* The received rows arrive source-major (all of source 0's rows for local
  experts 0, 1, ..., then source 1's, ...).  A row gather (moe_gather_rows)
  regroups them expert-major, the local grouped GEMMs (moe_expert_ffn) run on
  the local experts, a second gather restores the source-major order and the
  reverse all-to-all sends each y row back to the rank whose token it is.
* Each rank sums its tokens' k rows (moe_combine) exactly as on one GPU.

The transfers use torch.distributed all_to_all_single (NCCL between GPUs);
no TMA load in the library uses cluster multicast, and remote rows are read
only after they landed in local memory.  The per-step host work is the
split sizes (a device-to-host copy of W x E/W counts) and the two row
permutations built from them.

``plan_dispatch`` and ``ExpertParallelMoE`` take their stage functions and
process group as arguments, so the host logic runs unchanged over gloo on
the CPU in the tests, with CPU stand-ins for the kernels there.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.distributed as dist


def owner_block(E: int, world: int, rank: int) -> tuple[int, int]:
    """The experts [e0, e1) rank `rank` owns."""
    if E % world != 0:
        raise ValueError(f"E = {E} must be a multiple of the number of ranks {world}")
    n = E // world
    return rank * n, (rank + 1) * n


@dataclass
class DispatchPlan:
    """Layouts of the rows one rank receives.

    recv_counts[s][e]: rows source s sends for local expert e.
    regroup[i]: the received (source-major) row that grouped (expert-major)
    row i takes.  ungroup[j]: the grouped row that received row j came to,
    i.e. its inverse.  offsets: the expert-major group starts (E_local + 1).
    """

    recv_counts: np.ndarray
    regroup: np.ndarray
    ungroup: np.ndarray
    offsets: np.ndarray


def plan_dispatch(recv_counts: np.ndarray) -> DispatchPlan:
    """Row permutations between the source-major received order and the
    expert-major grouped order, from the per-(source, local expert) counts."""
    c = np.asarray(recv_counts, dtype=np.int64)
    W, El = c.shape
    # start of block (s, e) in the received, source-major order
    src_start = np.concatenate([[0], np.cumsum(c.reshape(-1))])[:-1].reshape(W, El)
    # start of block (e, s) in the grouped, expert-major order
    grp = c.T.reshape(-1)
    grp_start = np.concatenate([[0], np.cumsum(grp)])[:-1].reshape(El, W)
    n = int(c.sum())
    regroup = np.empty(n, dtype=np.int32)
    for e in range(El):
        for s in range(W):
            m = int(c[s, e])
            g0 = int(grp_start[e, s])
            r0 = int(src_start[s, e])
            regroup[g0:g0 + m] = np.arange(r0, r0 + m, dtype=np.int32)
    ungroup = np.empty(n, dtype=np.int32)
    ungroup[regroup] = np.arange(n, dtype=np.int32)
    offsets = np.concatenate([[0], np.cumsum(c.sum(axis=0))]).astype(np.int32)
    return DispatchPlan(c, regroup, ungroup, offsets)


class CudaStages:
    """The library's kernels as the stages of the expert-parallel forward."""

    y_dtype = torch.float16  # the grouped GEMM's y rows

    def __init__(self):
        import top_routing_grouped_softmax_b200 as moe
        self.moe = moe

    def route(self, x, w_router, k, bias):
        return self.moe.route(x, w_router, k, bias=bias)

    def permute(self, x, ids, w, E):
        return self.moe.permute(x, ids, w, E)

    def gather_rows(self, src, idx):
        return self.moe.gather_rows(src, idx)

    def expert_ffn(self, x_rows, w_rows, offsets, w_gate, w_up, w_down):
        return self.moe.expert_ffn(x_rows, w_rows, offsets, w_gate, w_up, w_down)[1]

    def combine(self, y, inv, T, k):
        return self.moe.combine(y, inv, T, k)


def _exchange(t: torch.Tensor, out_rows: int, out_split, in_split, group) -> torch.Tensor:
    """all_to_all_single of whole rows.  Rows of 16-bit values (bf16, fp16;
    an even count per row) travel as int32 pairs, a type every backend
    moves."""
    t = t.contiguous()
    packed = t.element_size() == 2
    row = 1
    for n in t.shape[1:]:
        row *= int(n)
    # an explicit row width: a rank may send no rows at all
    view = t.view(t.shape[0], row).view(torch.int32) if packed else t
    out = torch.empty((out_rows,) + tuple(view.shape[1:]), dtype=view.dtype, device=view.device)
    dist.all_to_all_single(out, view, output_split_sizes=out_split, input_split_sizes=in_split, group=group)
    return out.view(t.dtype).view((out_rows,) + tuple(t.shape[1:])) if packed else out


class ExpertParallelMoE:
    """One rank's share of an expert-parallel MoE block forward.

    w_router [d, E] and bias [E] (optional) are whole; w_gate_local /
    w_up_local [E/W, d, f] and w_down_local [E/W, f, d] are the weights of
    this rank's expert block.  forward(x) takes this rank's tokens x [T_r, d]
    and returns their out [T_r, d] fp32 -- the rows the one-GPU forward gives
    for the same tokens.
    """

    def __init__(self, w_router, w_gate_local, w_up_local, w_down_local, k, bias=None, group=None, stages=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E = int(w_router.shape[1])
        self.E_local = int(w_gate_local.shape[0])
        e0, e1 = owner_block(self.E, self.world, self.rank)
        if e1 - e0 != self.E_local:
            raise ValueError(f"rank {self.rank} owns experts [{e0}, {e1}) but got {self.E_local} expert weights")
        self.k = int(k)
        self.w_router, self.bias = w_router, bias
        self.w_gate, self.w_up, self.w_down = w_gate_local, w_up_local, w_down_local
        self.stages = stages if stages is not None else CudaStages()
        self.last_plan = None

    def forward(self, x):
        st, W, El = self.stages, self.world, self.E_local
        T = int(x.shape[0])
        dev = x.device
        ids, w = st.route(x, self.w_router, self.k, self.bias)
        pm = st.permute(x, ids, w, self.E)
        # 1. counts: send_counts[q][e] = rows of this rank for rank q's local expert e
        send_counts = pm["counts"].to(torch.int64).view(W, El).contiguous()
        recv_counts = torch.empty_like(send_counts)
        dist.all_to_all_single(recv_counts, send_counts, group=self.group)
        send_counts_h = send_counts.cpu().numpy()
        recv_counts_h = recv_counts.cpu().numpy()
        send_split = send_counts_h.sum(axis=1).tolist()
        recv_split = recv_counts_h.sum(axis=1).tolist()
        n_recv = int(sum(recv_split))
        # 2. dispatch: this rank's grouped rows are in expert order, so rank q's
        #    rows are one contiguous slice
        x_recv = _exchange(pm["x_perm"], n_recv, recv_split, send_split, self.group)
        w_recv = _exchange(pm["w_perm"], n_recv, recv_split, send_split, self.group)
        plan = plan_dispatch(recv_counts_h)
        self.last_plan = plan
        regroup = torch.from_numpy(plan.regroup).to(dev)
        ungroup = torch.from_numpy(plan.ungroup).to(dev)
        offsets = torch.from_numpy(plan.offsets).to(dev)
        # 3. local experts over the expert-major regrouped rows
        if n_recv > 0:
            x_grp = st.gather_rows(x_recv, regroup)
            w_grp = st.gather_rows(w_recv, regroup)
            y_grp = st.expert_ffn(x_grp, w_grp, offsets, self.w_gate, self.w_up, self.w_down)
            y_recv = st.gather_rows(y_grp, ungroup)
        else:
            # no rows for this rank's experts: an empty block of the stages' y type
            y_recv = torch.empty(0, x.shape[1], dtype=getattr(st, "y_dtype", torch.float16), device=dev)
        # 4. return: the reverse exchange puts every y row back at its grouped
        #    position on the rank that owns the token
        y_back = _exchange(y_recv, T * self.k, send_split, recv_split, self.group)
        return st.combine(y_back, pm["inv"], T, self.k)


__all__ = ["owner_block", "plan_dispatch", "DispatchPlan", "CudaStages", "ExpertParallelMoE"]
