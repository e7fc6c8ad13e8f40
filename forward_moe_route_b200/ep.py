"""Expert parallelism for the DeepSeekMoE layer: routed experts split over
ranks, rows exchanged by all-to-all, redundant copies of hot experts.

"DeepSeek Technical Report: MoE Architecture", §3.8 (expert parallelism: each
GPU holds a contiguous share of the routed experts; tokens are dispatched to
the GPUs holding their experts and the results combined back, with FP8
dispatch and BF16 combine in §3.6's low-precision communication list) and
§3.11 (inference deployment: redundant experts, extra copies of the most
loaded experts placed on other GPUs so that each copy serves part of the
expert's tokens).

Layout of one rank's step (world W, this rank r, T_r own tokens):
  1. moe_route + moe_permute (maps only) on the rank's own tokens: the rows
     of the pairs expert by expert (global routed-expert order), offsets[N+1].
  2. plan (this module, host integers): every routed expert j has holders
     (its home rank, then its redundant copies); the rank's rows of j are cut
     into one contiguous chunk per holder.  The send buffer lists, for each
     destination rank q in order, the chunks of q's local expert slots in
     slot order.
  3. exchange: per-(destination, slot) row counts by all-to-all, then the rows
     (bf16) and their gate weights by one uneven all-to-all each.
  4. moe_expert_ffn on the received rows: one group per (source rank, local
     slot), output in the received order, gate weight applied.
  5. exchange back with the splits reversed; moe_combine_rows adds the
     residual, the rank's own shared-expert outputs and the K returned rows of
     each token, in the order of the single-GPU combine.

Only the plan and the collectives live here; every other step runs in the
library's CUDA kernels (moe_route, moe_permute, moe_dispatch_rows,
moe_expert_ffn, moe_combine_rows).  The phases (ep_dispatch, ep_compute,
ep_combine) are separate functions so that the exchange between them can be
any transport; ep_forward chains them over torch.distributed.  The plan needs
the rank's per-expert row counts on the host, so a step reads N integers back
from the device before the exchange.

Exchange over peer memory (PeerExchange, ep_forward_peer): instead of a
collective, the dispatch kernel stores each row straight into the receive
buffer of the rank holding its expert, and the down projection of the
expert GEMMs stores each output row straight into the return buffer of the
rank that sent it (other processes' buffers mapped through CUDA IPC).  The
ranks only all-gather their send matrices and order the phases with
barriers.

E4M3 layers (§3.6: FP8 dispatch, BF16 combine): the rows travel as 1x128
E4M3 codes with their fp32 scales and the expert outputs come back in bf16,
on either exchange.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------- placement
@dataclass(frozen=True)
class Placement:
    """Which rank holds which routed expert.

    home(j) = j // (N / W) (contiguous ranges, as in §3.8).  replicas[j] lists
    the extra ranks holding a redundant copy of expert j (§3.11).  Rank r's
    local slots are its home experts in index order, then its redundant
    copies in expert order; slot s of rank r runs expert slots[r][s]."""
    n_routed: int
    world: int
    replicas: Dict[int, tuple] = field(default_factory=dict)

    def __post_init__(self):
        if self.world < 1 or self.n_routed % self.world:
            raise ValueError("the routed experts must split evenly over the ranks")
        for j, ranks in self.replicas.items():
            if not 0 <= j < self.n_routed:
                raise ValueError(f"replica of unknown expert {j}")
            if len(set(ranks)) != len(ranks) or self.home(j) in ranks or \
                    any(not 0 <= q < self.world for q in ranks):
                raise ValueError(f"bad replica ranks {ranks} for expert {j}")

    @property
    def per_rank(self) -> int:
        return self.n_routed // self.world

    def home(self, j: int) -> int:
        return j // self.per_rank

    def holders(self, j: int) -> List[int]:
        return [self.home(j)] + list(self.replicas.get(j, ()))

    def slots(self, r: int) -> List[int]:
        own = list(range(r * self.per_rank, (r + 1) * self.per_rank))
        return own + [j for j in sorted(self.replicas) if r in self.replicas[j]]

    @property
    def max_slots(self) -> int:
        return max(len(self.slots(r)) for r in range(self.world))


def choose_replicas(loads: Sequence[int], world: int, n_redundant: int) -> Dict[int, tuple]:
    """Redundant copies for the n_redundant most loaded experts.

    loads[j] = rows of expert j over all ranks.  Greedy: take the experts by
    load (descending, ties to the lower index); each gets one copy on the rank
    whose projected load is lowest (ties to the lower rank), not its home;
    the expert's load is then shared equally between its holders."""
    loads = np.asarray(loads, np.int64)
    N = len(loads)
    per = N // world
    rank_load = np.zeros(world)
    for j in range(N):
        rank_load[j // per] += loads[j]
    order = sorted(range(N), key=lambda j: (-int(loads[j]), j))
    out: Dict[int, tuple] = {}
    for j in order[:n_redundant]:
        if loads[j] == 0:
            break
        home = j // per
        cand = [q for q in range(world) if q != home]
        if not cand:
            break
        q = min(cand, key=lambda q: (rank_load[q], q))
        half = loads[j] / 2.0
        rank_load[home] -= half
        rank_load[q] += half
        out[j] = (q,)
    return out


def chunk_bounds(rows: int, n: int) -> List[int]:
    """Cut `rows` consecutive rows into n contiguous chunks: chunk c is
    [b[c], b[c+1]) with b[c] = floor(c * rows / n)."""
    return [(c * rows) // n for c in range(n + 1)]


# ----------------------------------------------------------------------------- one rank's plan
@dataclass
class DispatchPlan:
    """What rank r sends where, and how its returned rows map back.

    send_perm[i]       x_perm row placed at send-buffer row i
    send_splits[q]     rows sent to rank q
    send_counts[q, s]  rows sent to rank q for q's local slot s
    row_of[p]          send-buffer row holding pair p = t*K + k (the rows come
                       back in the same order)"""
    send_perm: np.ndarray
    send_splits: List[int]
    send_counts: np.ndarray
    row_of: np.ndarray


def dispatch_plan(pl: Placement, counts: Sequence[int], offsets: Sequence[int],
                  slot_of: Sequence[int]) -> DispatchPlan:
    """The plan of one rank from its own routing (counts [N], offsets [N+1] and
    slot_of [T*K] as moe_permute writes them)."""
    counts = np.asarray(counts, np.int64)
    offsets = np.asarray(offsets, np.int64)
    slot_of = np.asarray(slot_of, np.int64)
    N, W = pl.n_routed, pl.world
    if counts.shape != (N,) or offsets.shape != (N + 1,):
        raise ValueError("counts / offsets do not match the placement's expert count")
    if not np.array_equal(np.diff(offsets), counts) or offsets[0] != 0:
        raise ValueError("offsets are not the exclusive scan of counts")
    # chunk c of expert j goes to holder c
    chunk_of = {}
    for j in range(N):
        h = pl.holders(j)
        b = chunk_bounds(int(counts[j]), len(h))
        for c, q in enumerate(h):
            chunk_of[(j, q)] = (int(offsets[j]) + b[c], int(offsets[j]) + b[c + 1])
    S = pl.max_slots
    send_counts = np.zeros((W, S), np.int64)
    pieces, splits = [], []
    for q in range(W):
        tot = 0
        for s, j in enumerate(pl.slots(q)):
            a, b = chunk_of[(j, q)]
            pieces.append(np.arange(a, b, dtype=np.int64))
            send_counts[q, s] = b - a
            tot += b - a
        splits.append(tot)
    send_perm = np.concatenate(pieces) if pieces else np.zeros(0, np.int64)
    if len(send_perm) != int(offsets[-1]) or \
            not np.array_equal(np.sort(send_perm), np.arange(int(offsets[-1]))):
        raise AssertionError("the plan does not send every row exactly once")
    inv = np.empty(len(send_perm), np.int64)
    inv[send_perm] = np.arange(len(send_perm))
    row_of = inv[slot_of] if len(slot_of) else np.zeros(0, np.int64)
    return DispatchPlan(send_perm, splits, send_counts, row_of)


@dataclass
class ReceivePlan:
    """Rows rank r receives: from source s, for local slot l, in (s, l) order.

    groups[i] = (row0, rows, slot, out0) for the expert FFN over the received
    rows (the output keeps the received order, so out0 = row0)."""
    recv_splits: List[int]
    groups: np.ndarray
    slot_rows: np.ndarray      # rows of each local slot over all sources


def receive_plan(pl: Placement, rank: int, recv_counts: np.ndarray) -> ReceivePlan:
    """recv_counts[s, l] = rows source s sent for this rank's local slot l."""
    recv_counts = np.asarray(recv_counts, np.int64)
    n_slots = len(pl.slots(rank))
    groups, splits, run = [], [], 0
    for s in range(pl.world):
        tot = 0
        for l in range(n_slots):
            c = int(recv_counts[s, l])
            if c:
                groups.append((run, c, l, run))
            run += c
            tot += c
        splits.append(tot)
    g = np.array(groups, np.int64).reshape(-1, 4)
    return ReceivePlan(splits, g, recv_counts[:, :n_slots].sum(axis=0))


# ----------------------------------------------------------------------------- exchange
class Transport:
    """All-to-all of rows between ranks.  The default is torch.distributed
    (NCCL for device tensors, gloo for host tensors)."""

    def all_to_all(self, send, send_splits: List[int], recv_splits: List[int]):
        import torch
        import torch.distributed as dist
        out = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype,
                          device=send.device)
        dist.all_to_all_single(out, send.contiguous(), output_split_sizes=list(recv_splits),
                               input_split_sizes=list(send_splits))
        return out

    def counts(self, send_counts: np.ndarray) -> np.ndarray:
        """send_counts [W, S] -> recv_counts [W, S] (row q of the result came from rank q)."""
        import torch
        import torch.distributed as dist
        backend = dist.get_backend()
        dev = "cuda" if backend == "nccl" else "cpu"
        t = torch.as_tensor(np.ascontiguousarray(send_counts), dtype=torch.int64, device=dev)
        out = torch.empty_like(t)
        dist.all_to_all_single(out, t)
        return out.cpu().numpy()


# ----------------------------------------------------------------------------- GPU step
def is_fp8(desc) -> bool:
    """E4M3 layer: rows travel as 1x128-quantised codes with their fp32 scales
    (§3.6: FP8 dispatch), and come back as bf16 (BF16 combine)."""
    from . import DT_E4M3
    return desc.w_dtype == DT_E4M3

@dataclass
class RankStep:
    """One rank's state between the phases of an expert-parallel forward."""
    rank: int
    plan: DispatchPlan
    x_send: object = None
    w_send: object = None
    recv: Optional[ReceivePlan] = None
    y_recv: object = None
    topk_w: object = None
    s_send: object = None       # E4M3 layers: the 1x128 scales of the send rows


def ep_dispatch(desc, pl: Placement, rank: int, x, w_router, bias, ws=None,
                build_send: bool = True) -> RankStep:
    """Phase 1 on the rank's GPU: routing, the permutation maps, the plan and
    the send buffer (rows grouped by destination rank, with gate weights).
    With build_send=False the send buffer is skipped (the peer-memory exchange
    writes the rows straight into the receiving ranks' buffers)."""
    import torch

    from . import moe_dispatch_rows, moe_permute, moe_route, workspace
    T, K, N, d = desc.T, desc.top_k, desc.n_routed, desc.d
    dev = x.device
    ws = workspace(desc) if ws is None else ws
    i32 = dict(dtype=torch.int32, device=dev)
    idx = torch.empty(max(T, 1), K, **i32)
    w = torch.empty(max(T, 1), K, dtype=torch.float32, device=dev)
    counts = torch.empty(N, **i32)
    moe_route(desc, x, w_router, bias, idx, w, counts, ws)
    offsets = torch.empty(N + 1, **i32)
    perm_src = torch.empty(max(T * K, 1), **i32)
    slot_of = torch.empty(max(T * K, 1), **i32)
    moe_permute(desc, x, idx, counts, offsets, perm_src, slot_of, None, None, ws)   # maps only
    plan = dispatch_plan(pl, counts.cpu().numpy(), offsets.cpu().numpy(),
                         slot_of[:T * K].cpu().numpy())
    if not build_send:
        st = RankStep(rank, plan)
        st.topk_w = w
        return st
    row_of = torch.as_tensor(plan.row_of, dtype=torch.int32, device=dev)
    w_send = torch.empty(T * K, dtype=torch.float32, device=dev)
    if is_fp8(desc):
        from . import moe_dispatch_rows_fp8
        x_send = torch.empty(T * K, d, dtype=torch.uint8, device=dev)
        s_send = torch.empty(T * K, d // 128, dtype=torch.float32, device=dev)
        moe_dispatch_rows_fp8(desc, x, w, row_of, x_send, s_send, w_send)
        st = RankStep(rank, plan, x_send, w_send)
        st.s_send = s_send
        return st
    x_send = torch.empty(T * K, d, dtype=x.dtype, device=dev)
    moe_dispatch_rows(desc, x, w, row_of, x_send, w_send)
    return RankStep(rank, plan, x_send, w_send)


def ep_compute(desc, pl: Placement, st: RankStep, recv_counts: np.ndarray, x_recv, w_recv,
               w_gu_local, w_down_local, s_recv=None, w_gu_scale=None, w_down_scale=None):
    """Phase 2 on the rank's GPU: the experts it holds on the rows it received
    (one group per source rank and local slot), gate weights applied.  E4M3
    layers take the received codes with their scales (s_recv) and the local
    weights' block scales, and return bf16 rows."""
    import torch

    from . import moe_expert_ffn, moe_expert_ffn_fp8, moe_expert_ffn_workspace_size
    st.recv = receive_plan(pl, st.rank, recv_counts)
    n_recv = int(sum(st.recv.recv_splits))
    dev = x_recv.device
    fp8 = is_fp8(desc)
    y = torch.empty(n_recv, desc.d, dtype=torch.bfloat16 if fp8 else x_recv.dtype, device=dev)
    if n_recv and len(st.recv.groups):
        g = st.recv.groups.copy()
        g[:, 2] += desc.n_shared            # local weight index of slot l
        groups = torch.as_tensor(g, dtype=torch.int32, device=dev)
        fws = torch.empty(moe_expert_ffn_workspace_size(desc, len(g), n_recv),
                          dtype=torch.uint8, device=dev)
        if fp8:
            moe_expert_ffn_fp8(desc, w_gu_local.shape[0], groups, n_recv, n_recv, x_recv, s_recv,
                               w_recv, w_gu_local, w_gu_scale, w_down_local, w_down_scale, fws,
                               y_rows=y)
        else:
            moe_expert_ffn(desc, w_gu_local.shape[0], groups, x_recv, w_recv, w_gu_local,
                           w_down_local, y, fws)
    st.y_recv = y
    return y


def ep_combine(desc, st: RankStep, x, x_residual, y_back, w_gu_local, w_down_local,
               w_gu_scale=None, w_down_scale=None):
    """Phase 3 on the rank's GPU: its shared experts on its own tokens and the
    combine of the returned rows, in the single-GPU combine's order (bf16 for
    E4M3 layers, whose shared experts read the tokens quantised per 1x128)."""
    import torch

    from . import (moe_combine_rows, moe_expert_ffn, moe_expert_ffn_fp8,
                   moe_expert_ffn_workspace_size, moe_quantize_rows_fp8)
    T, d, Ks = desc.T, desc.d, desc.n_shared
    dev = x.device
    y_shared = None
    if Ks and T:
        sg = torch.as_tensor([[0, T, s, s * T] for s in range(Ks)], dtype=torch.int32, device=dev)
        y_shared = torch.empty(Ks * T, d, dtype=x.dtype, device=dev)
        sws = torch.empty(moe_expert_ffn_workspace_size(desc, Ks, Ks * T), dtype=torch.uint8,
                          device=dev)
        if is_fp8(desc):
            xq = torch.empty(T, d, dtype=torch.uint8, device=dev)
            xs = torch.empty(T, d // 128, dtype=torch.float32, device=dev)
            moe_quantize_rows_fp8(desc, x, xq, xs)
            moe_expert_ffn_fp8(desc, w_gu_local.shape[0], sg, T, Ks * T, xq, xs, None,
                               w_gu_local, w_gu_scale, w_down_local, w_down_scale, sws,
                               y_rows=y_shared)
        else:
            moe_expert_ffn(desc, w_gu_local.shape[0], sg, x, None, w_gu_local, w_down_local,
                           y_shared, sws)
    h = torch.empty(max(T, 1), d, dtype=x.dtype, device=dev)
    row_of = torch.as_tensor(st.plan.row_of, dtype=torch.int32, device=dev)
    y_rows = y_back if len(y_back) else torch.zeros(1, d, dtype=x.dtype, device=dev)
    moe_combine_rows(desc, x if x_residual is None else x_residual, y_shared, y_rows, row_of, h)
    return h[:T]


def ep_forward(desc, pl: Placement, rank: int, x, x_residual, w_router, bias, w_gu_local,
               w_down_local, transport: Optional[Transport] = None, ws=None, w_gu_scale=None,
               w_down_scale=None):
    """One expert-parallel layer forward of this rank's tokens (all ranks call
    it together).  w_gu_local / w_down_local hold the rank's experts: the Ks
    shared experts first, then local slot s at index Ks + s (pl.slots(rank));
    for E4M3 layers also their 128x128 block scales.  Returns h [T, d] and the
    number of rows this rank's experts processed."""
    transport = transport or Transport()
    st = ep_dispatch(desc, pl, rank, x, w_router, bias, ws)
    recv_counts = transport.counts(st.plan.send_counts)
    recv_splits = [int(v) for v in recv_counts[:, :len(pl.slots(rank))].sum(axis=1)]
    x_recv = transport.all_to_all(st.x_send, st.plan.send_splits, recv_splits)
    w_recv = transport.all_to_all(st.w_send, st.plan.send_splits, recv_splits)
    s_recv = transport.all_to_all(st.s_send, st.plan.send_splits, recv_splits) \
        if st.s_send is not None else None
    y = ep_compute(desc, pl, st, recv_counts, x_recv, w_recv, w_gu_local, w_down_local, s_recv,
                   w_gu_scale, w_down_scale)
    y_back = transport.all_to_all(y, recv_splits, st.plan.send_splits)
    h = ep_combine(desc, st, x, x_residual, y_back, w_gu_local, w_down_local, w_gu_scale,
                   w_down_scale)
    return h, len(y)


def local_weights(pl: Placement, rank: int, n_shared: int, *full):
    """The rank's expert tensors (shared experts, then its local slots) taken
    from full [Ks+N, ...] tensors (weights, and for E4M3 layers their block
    scales): the placement a deployment would load."""
    import torch
    ids = list(range(n_shared)) + [n_shared + j for j in pl.slots(rank)]
    sel = torch.as_tensor(ids, device=full[0].device)
    return tuple(t.index_select(0, sel).contiguous() for t in full)


# ----------------------------------------------------------------------------- peer-memory exchange
def peer_offsets(M: np.ndarray, rank: int):
    """Where this rank's send-order rows land, from the send matrix of all
    ranks (M[s, q, l] = rows rank s sends to rank q for q's local slot l):
    start[q] .. start[q+1] are the rows it sends to rank q (its send order is
    destination-major), placed from row base[q] of q's receive buffer, after
    the rows of every lower-numbered source (the order an all-to-all would
    concatenate them in)."""
    M = np.asarray(M, np.int64)
    W = M.shape[0]
    per_dest = M[rank].sum(axis=1)                       # rows to each rank
    start = np.concatenate([[0], np.cumsum(per_dest)]).astype(np.int64)
    base = M[:rank].sum(axis=(0, 2)) if rank else np.zeros(W, np.int64)
    return [int(v) for v in start], [int(v) for v in base]


def peer_return_rows(M: np.ndarray, rank: int, recv: ReceivePlan):
    """For each received group (source s, slot l, row0, rows): the row of the
    source's send order its outputs return to.  The source sent its rows for
    this rank from send-order row start_s[rank] on, in slot order, which is
    the order they arrived in."""
    M = np.asarray(M, np.int64)
    W = M.shape[0]
    recv_start = np.concatenate([[0], np.cumsum(M[:, rank, :].sum(axis=1))])
    out = []
    for row0, rows, slot, _ in recv.groups:
        # the source whose block [recv_start[s], recv_start[s+1]) holds row0
        s = int(np.searchsorted(recv_start, row0, side="right") - 1)
        start_s = int(M[s, :rank].sum())
        out.append((s, start_s + int(row0 - recv_start[s])))
    return out


class PeerExchange:
    """The buffers of one rank for the peer-memory exchange, and the device
    addresses of every rank's buffers in this process.

    recv_x [capacity, d] / recv_w [capacity] receive the rows other ranks
    dispatch to this rank's experts; ret_y [T*K, d] receives the expert
    outputs of this rank's own rows, in its send order.  Ranks in other
    processes are reached through CUDA IPC (open_peers); ranks emulated in one
    process share their local addresses (link)."""

    def __init__(self, desc, pl: Placement, rank: int, capacity: int, device, dtype):
        """dtype: the layer's activation type (bf16 / fp32); an E4M3 layer's
        rows arrive as uint8 codes with fp32 1x128 scales (recv_s) and return
        as bf16."""
        import torch
        self.desc, self.pl, self.rank, self.capacity = desc, pl, rank, int(capacity)
        d, TK, cap = desc.d, max(desc.T * desc.top_k, 1), max(self.capacity, 1)
        fp8 = is_fp8(desc)
        self.recv_x = torch.empty(cap, d, dtype=torch.uint8 if fp8 else dtype, device=device)
        self.recv_s = torch.empty(cap, d // 128, dtype=torch.float32, device=device) if fp8 \
            else None
        self.recv_w = torch.empty(cap, dtype=torch.float32, device=device)
        self.ret_y = torch.empty(TK, d, dtype=torch.bfloat16 if fp8 else dtype, device=device)
        W = pl.world
        self.x_addr = [0] * W
        self.w_addr = [0] * W
        self.s_addr = [0] * W
        self.ret_addr = [0] * W
        self.x_addr[rank] = self.recv_x.data_ptr()
        self.w_addr[rank] = self.recv_w.data_ptr()
        self.s_addr[rank] = self.recv_s.data_ptr() if fp8 else 0
        self.ret_addr[rank] = self.ret_y.data_ptr()
        self._opened: List[int] = []

    def _buffers(self):
        return [self.recv_x, self.recv_w, self.ret_y] + \
            ([self.recv_s] if self.recv_s is not None else [])

    @staticmethod
    def link(exchanges: Sequence["PeerExchange"]) -> None:
        """Ranks emulated in one process: every rank sees the others' buffers."""
        for ex in exchanges:
            for other in exchanges:
                q = other.rank
                ex.x_addr[q] = other.recv_x.data_ptr()
                ex.w_addr[q] = other.recv_w.data_ptr()
                ex.ret_addr[q] = other.ret_y.data_ptr()
                ex.s_addr[q] = other.recv_s.data_ptr() if other.recv_s is not None else 0

    def open_peers(self, group=None) -> None:
        """Ranks in separate processes: exchange CUDA IPC handles over the
        process group and map every other rank's buffers."""
        import torch.distributed as dist

        from . import moe_ipc_get_handle, moe_ipc_open
        mine = tuple(moe_ipc_get_handle(b) for b in self._buffers())
        allh = [None] * self.pl.world
        dist.all_gather_object(allh, mine, group=group)
        bases = {}        # an allocation is mapped once, however many buffers it holds
        for q, handles in enumerate(allh):
            if q == self.rank:
                continue
            addrs = []
            for h, off in handles:
                if h not in bases:
                    bases[h] = moe_ipc_open(h)
                    self._opened.append(bases[h])
                addrs.append(bases[h] + off)
            self.x_addr[q], self.w_addr[q], self.ret_addr[q] = addrs[:3]
            if len(addrs) > 3:
                self.s_addr[q] = addrs[3]

    def close(self) -> None:
        from . import moe_ipc_close
        for a in self._opened:
            moe_ipc_close(a)
        self._opened = []


def peer_dispatch(desc, ex: PeerExchange, st: RankStep, x, M: np.ndarray) -> None:
    """Dispatch phase: the rank's rows and gate weights go straight into the
    holders' receive buffers (one kernel, peer stores)."""
    import torch

    from . import moe_dispatch_rows_to
    T, K = desc.T, desc.top_k
    if not T:
        return
    start, base = peer_offsets(M, st.rank)
    for q in range(ex.pl.world):      # every rank's buffer holds ex.capacity rows
        if base[q] + start[q + 1] - start[q] > ex.capacity:
            raise ValueError(f"rank {q}'s receive buffer is too small")
    row_of = torch.as_tensor(st.plan.row_of, dtype=torch.int32, device=x.device)
    moe_dispatch_rows_to(desc, x, st.topk_w, row_of, T * K, ex.x_addr, ex.w_addr, start, base,
                         s_addr=ex.s_addr if is_fp8(desc) else None)


def peer_compute(desc, ex: PeerExchange, st: RankStep, M: np.ndarray, w_gu_local,
                 w_down_local, w_gu_scale=None, w_down_scale=None) -> int:
    """Expert phase: the rank's experts on the rows it received; the down
    projection stores each output row straight into its source rank's return
    buffer (bf16 for E4M3 layers).  Returns the number of rows processed."""
    import torch

    from . import moe_expert_ffn_fp8, moe_expert_ffn_to, moe_expert_ffn_workspace_size
    M = np.asarray(M, np.int64)
    r = st.rank
    st.recv = receive_plan(ex.pl, r, M[:, r, :])
    n_recv = int(sum(st.recv.recv_splits))
    if n_recv > ex.capacity:
        raise ValueError("receive buffer too small")
    if not n_recv or not len(st.recv.groups):
        return 0
    esz = ex.ret_y.element_size()
    back = peer_return_rows(M, r, st.recv)
    addrs = [ex.ret_addr[s] + row * desc.d * esz for s, row in back]
    dev = ex.recv_x.device
    g = st.recv.groups.copy()
    g[:, 2] += desc.n_shared
    groups = torch.as_tensor(g, dtype=torch.int32, device=dev)
    group_out = torch.as_tensor(np.array(addrs, np.uint64).view(np.int64), device=dev)
    fws = torch.empty(moe_expert_ffn_workspace_size(desc, len(g), n_recv), dtype=torch.uint8,
                      device=dev)
    if is_fp8(desc):
        moe_expert_ffn_fp8(desc, w_gu_local.shape[0], groups, n_recv, n_recv, ex.recv_x,
                           ex.recv_s, ex.recv_w, w_gu_local, w_gu_scale, w_down_local,
                           w_down_scale, fws, group_out=group_out)
    else:
        moe_expert_ffn_to(desc, w_gu_local.shape[0], groups, n_recv, n_recv, ex.recv_x,
                          ex.recv_w, w_gu_local, w_down_local, group_out, fws)
    return n_recv


def peer_combine(desc, ex: PeerExchange, st: RankStep, x, x_residual, w_gu_local, w_down_local,
                 w_gu_scale=None, w_down_scale=None):
    """Combine phase: the returned rows are in the rank's send order already."""
    T, K = desc.T, desc.top_k
    return ep_combine(desc, st, x, x_residual, ex.ret_y[:max(T * K, 1)], w_gu_local,
                      w_down_local, w_gu_scale, w_down_scale)


def ep_forward_peer(desc, pl: Placement, rank: int, x, x_residual, w_router, bias, w_gu_local,
                    w_down_local, ex: PeerExchange, group=None, ws=None, w_gu_scale=None,
                    w_down_scale=None):
    """One expert-parallel layer forward over peer memory (all ranks call it
    together, each in its own process with ex.open_peers() done): the send
    matrix by all-gather, then dispatch, expert and combine phases separated
    by a device synchronise and a barrier over the ranks."""
    import torch
    import torch.distributed as dist
    st = ep_dispatch(desc, pl, rank, x, w_router, bias, ws, build_send=False)
    mine = np.ascontiguousarray(st.plan.send_counts)
    allm = [None] * pl.world
    dist.all_gather_object(allm, mine, group=group)
    M = np.stack(allm)
    peer_dispatch(desc, ex, st, x, M)
    torch.cuda.synchronize()
    dist.barrier(group=group)
    n = peer_compute(desc, ex, st, M, w_gu_local, w_down_local, w_gu_scale, w_down_scale)
    torch.cuda.synchronize()
    dist.barrier(group=group)
    return peer_combine(desc, ex, st, x, x_residual, w_gu_local, w_down_local, w_gu_scale,
                        w_down_scale), n
