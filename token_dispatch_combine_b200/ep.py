"""Expert parallelism over several ranks: torch-facing wrappers of the moe_ep_*
calls (argument marshalling only) and the per-rank buffers of one layer.

"EP: Partition Experts and Route Tokens", "Send tokens to experts and return
their results": each rank routes its own tokens and sends each token vector to
the rank holding its selected expert; results return to the source rank and
token, which forms the weighted sum ("Return multiple expert results to the
same token"; input delivery is shared when two of a token's experts sit on
the same rank).  "Expert Parallelism (EP)", "Limitations" 3-4: rank d holds
experts [d*E/R, (d+1)*E/R).

The step of one rank (``MoEEPRank``):
  plan      route its tokens, plan one send row per (token, destination);
  counts    every rank learns every source's send counts (the caller's
            collective: ``torch.distributed.all_gather`` or, on one GPU,
            a stack) -> ``set_counts``;
  pack      write its rows into the destinations' receive buffers (peer
            memory) or into a local buffer for a staged all-to-all;
  experts   count-sort the received rows by local expert, run the gathering
            gate/up and the down projection over its local experts, and sum
            each received row's weighted expert outputs (one partial per row);
  return    each source's partials go back to its return buffer;
  finish    each token's partials summed: its output.
``ep_round_trip_one_gpu`` runs R ranks on one GPU, the exchange through
device memory (each rank's pack writes straight into the other ranks'
receive buffers, as peer stores would).  ``ep_share_buffers`` +
``ep_round_trip_ranks`` run it with one process per rank: every rank's
receive and return buffers are mapped into every other rank's process (CUDA
IPC, one node), so the pack kernel stores rows straight into the peers'
memory and the partials return by peer copies; the counts go through
``torch.distributed`` and host barriers separate the phases, so no kernel
ever waits on another rank's kernel.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _native
from ._native import check
from .api import (_dtype, _ptr, _stream, moe_combine, moe_dispatch_workspace_bytes, moe_ffn_down,
                  moe_ffn_gate_up_gather, moe_route)

_I32 = torch.int32


def moe_ep_plan_workspace_bytes(T: int, R: int) -> int:
    return int(_native.lib().moe_ep_plan_workspace_bytes(int(T), int(R)))


def ep_rows_max(T: int, k: int, R: int) -> int:
    """Largest number of send rows a source of T tokens can have."""
    return T * min(k, R)


class EpPlan:
    """Device buffers of one source rank's send plan (moe_ep_plan)."""

    def __init__(self, T, k, E, R, device):
        n = max(1, ep_rows_max(T, k, R))
        kw = dict(dtype=_I32, device=device)
        self.T, self.k, self.E, self.R = T, k, E, R
        self.send_counts = torch.zeros(R, **kw)
        self.send_offsets = torch.zeros(R + 1, **kw)
        self.slot_send_row = torch.empty(max(1, T * k), **kw)
        self.ret_row = torch.empty(max(1, T * k), **kw)
        self.row_token = torch.empty(n, **kw)
        self.row_ids = torch.empty((n, k), **kw)
        self.row_w = torch.empty((n, k), dtype=torch.float32, device=device)
        self.workspace = torch.empty(max(16, moe_ep_plan_workspace_bytes(T, R)), dtype=torch.uint8, device=device)


def moe_ep_plan(topk_ids, topk_w, E: int, R: int, plan: EpPlan | None = None, stream=None) -> EpPlan:
    """One send row per (token, destination rank holding any of its experts), ordered by
    destination then token, with the token's local expert ids and weights there."""
    T, k = topk_ids.shape
    if plan is None:
        plan = EpPlan(T, k, E, R, topk_ids.device)
    check(_native.lib().moe_ep_plan(
        _ptr(topk_ids, "topk_ids", _I32), _ptr(topk_w, "topk_w", torch.float32), T, k, int(E), int(R),
        _ptr(plan.send_counts, "send_counts", _I32), _ptr(plan.send_offsets, "send_offsets", _I32),
        _ptr(plan.slot_send_row, "slot_send_row", _I32), _ptr(plan.ret_row, "ret_row", _I32),
        _ptr(plan.row_token, "row_token", _I32), _ptr(plan.row_ids, "row_ids", _I32),
        _ptr(plan.row_w, "row_w", torch.float32), _ptr(plan.workspace, "workspace", torch.uint8),
        plan.workspace.numel(), _stream(stream)), "moe_ep_plan")
    return plan


def moe_ep_plan_host(topk_ids: np.ndarray, topk_w: np.ndarray, E: int, R: int) -> dict:
    """The send plan on the host (numpy in and out, no device work); same layout as moe_ep_plan.
    Keys: send_counts, send_offsets, slot_send_row, ret_row, row_token, row_ids, row_w (the
    row arrays cut to the send rows)."""
    ids = np.ascontiguousarray(topk_ids, np.int32)
    w = np.ascontiguousarray(topk_w, np.float32)
    T, k = ids.shape
    n = max(1, ep_rows_max(T, k, R))
    out = dict(send_counts=np.zeros(R, np.int32), send_offsets=np.zeros(R + 1, np.int32),
               slot_send_row=np.empty(max(1, T * k), np.int32), ret_row=np.empty(max(1, T * k), np.int32),
               row_token=np.empty(n, np.int32), row_ids=np.empty((n, k), np.int32), row_w=np.empty((n, k), np.float32))
    check(_native.lib().moe_ep_plan_host(ids.ctypes.data, w.ctypes.data, T, k, int(E), int(R),
                                         *(out[key].ctypes.data for key in ("send_counts", "send_offsets",
                                                                            "slot_send_row", "ret_row", "row_token",
                                                                            "row_ids", "row_w"))),
          "moe_ep_plan_host")
    rows = int(out["send_offsets"][-1])
    for key in ("row_token", "row_ids", "row_w"):
        out[key] = out[key][:rows]
    for key in ("slot_send_row", "ret_row"):
        out[key] = out[key][:T * k]
    return out


def moe_ep_exchange_offsets(counts, rank: int):
    """From every source's send counts ([R, R], row s = source s) for `rank`: (dst_base [R],
    recv_base [R + 1], ret_base [R]) as numpy int32 (see moe_ep_exchange_offsets)."""
    c = np.ascontiguousarray(np.asarray(counts), np.int32)
    R = c.shape[0]
    if c.shape != (R, R):
        raise ValueError("counts must be [R, R]")
    dst_base = np.empty(R, np.int32)
    recv_base = np.empty(R + 1, np.int32)
    ret_base = np.empty(R, np.int32)
    check(_native.lib().moe_ep_exchange_offsets(c.ctypes.data, R, int(rank), dst_base.ctypes.data,
                                                recv_base.ctypes.data, ret_base.ctypes.data),
          "moe_ep_exchange_offsets")
    return dst_base, recv_base, ret_base


def moe_ep_pack(x, plan: EpPlan, dst_base, dst_x, dst_ids, dst_w, stream=None):
    """Write every send row of destination d (x row, local ids, weights) to dst_x[d] / dst_ids[d]
    / dst_w[d] at row dst_base[d] + (row - send_offsets[d]).  dst_* are lists of R device tensors
    (another rank's receive buffers, or slices of a local staging buffer); dst_base a device
    int32 tensor [R]."""
    T, H = x.shape
    R, k = plan.R, plan.k
    if not (len(dst_x) == len(dst_ids) == len(dst_w) == R):
        raise ValueError("one destination buffer set per rank")
    px = (ctypes.c_void_p * R)(*[_ptr(t, f"dst_x[{d}]", x.dtype) for d, t in enumerate(dst_x)])
    pi = (ctypes.c_void_p * R)(*[_ptr(t, f"dst_ids[{d}]", _I32) for d, t in enumerate(dst_ids)])
    pw = (ctypes.c_void_p * R)(*[_ptr(t, f"dst_w[{d}]", torch.float32) for d, t in enumerate(dst_w)])
    cap = np.array([t.shape[0] for t in dst_x], np.int32)
    for d in range(R):
        if dst_ids[d].shape[0] < cap[d] or dst_w[d].shape[0] < cap[d]:
            raise ValueError(f"dst_ids[{d}] / dst_w[{d}] hold fewer rows than dst_x[{d}]")
    check(_native.lib().moe_ep_pack(
        _ptr(x, "x"), _dtype(x), T, H, k, R, _ptr(plan.send_offsets, "send_offsets", _I32),
        _ptr(dst_base, "dst_base", _I32), _ptr(plan.row_token, "row_token", _I32), _ptr(plan.row_ids, "row_ids", _I32),
        _ptr(plan.row_w, "row_w", torch.float32), px, pi, pw, cap.ctypes.data, _stream(stream)), "moe_ep_pack")


def moe_ep_recv_index(recv_ids, EL: int, expert_counts, expert_offsets, slot_to_row, row_to_slot, workspace,
                      stream=None):
    """Counting sort of received rows ([T_recv, k] local ids, -1 = padding) by local expert."""
    T_recv, k = recv_ids.shape
    check(_native.lib().moe_ep_recv_index(
        _ptr(recv_ids, "recv_ids", _I32), T_recv, k, int(EL), _ptr(expert_counts, "expert_counts", _I32),
        _ptr(expert_offsets, "expert_offsets", _I32), _ptr(slot_to_row, "slot_to_row", _I32),
        _ptr(row_to_slot, "row_to_slot", _I32), _ptr(workspace, "workspace", torch.uint8), workspace.numel(),
        _stream(stream)), "moe_ep_recv_index")


def moe_enable_peer_access(peer_device: int) -> None:
    """Let kernels on the current device load and store memory of device ``peer_device``
    (no-op for the current device itself or when already enabled)."""
    check(_native.lib().moe_enable_peer_access(int(peer_device)), "moe_enable_peer_access")


class MoEEPRank:
    """One rank of an expert-parallel MoE layer over R ranks: its T tokens, its E/R local
    experts, and every buffer of its step (allocated here, once).  ``recv_capacity`` bounds
    the rows it can receive (default R * T: one row per token of every source at most)."""

    def __init__(self, rank, R, T, H, I, E, k, dtype, device="cuda", recv_capacity=None):
        if E % R:
            raise ValueError("R must divide E")
        self.rank, self.R, self.T, self.H, self.I, self.E, self.k = rank, R, T, H, I, E, k
        self.EL = E // R
        self.dtype = dtype
        self.device = torch.device(device)
        dev = self.device
        cap = R * T if recv_capacity is None else int(recv_capacity)
        self.cap = cap
        self.topk_ids = torch.empty((T, k), dtype=_I32, device=dev)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.plan = EpPlan(T, k, E, R, dev)
        self.dst_base = torch.zeros(R, dtype=_I32, device=dev)
        self.recv_base = np.zeros(R + 1, np.int32)
        self.ret_base = np.zeros(R, np.int32)
        self.counts = None  # [R, R] host: every source's send counts
        self.x_recv = torch.empty((max(1, cap), H), dtype=dtype, device=dev)
        self.recv_ids = torch.full((max(1, cap), k), -1, dtype=_I32, device=dev)
        self.recv_w = torch.zeros((max(1, cap), k), dtype=torch.float32, device=dev)
        self.expert_counts = torch.empty(self.EL, dtype=_I32, device=dev)
        self.expert_offsets = torch.empty(self.EL + 1, dtype=_I32, device=dev)
        self.slot_to_row = torch.empty(max(1, cap * k), dtype=_I32, device=dev)
        self.row_to_slot = torch.empty(max(1, cap * k), dtype=_I32, device=dev)
        self.recv_ws = torch.zeros(max(16, moe_dispatch_workspace_bytes(cap, k, self.EL, 1)), dtype=torch.uint8,
                                   device=dev)
        self.h = torch.empty((max(1, cap * k), I), dtype=dtype, device=dev)
        self.y_gemm = torch.empty((max(1, cap * k), H), dtype=dtype, device=dev)
        self.y_recv = torch.empty((max(1, cap), H), dtype=dtype, device=dev)
        self.y_ret = torch.zeros((max(1, ep_rows_max(T, k, R)), H), dtype=dtype, device=dev)
        self.ones = torch.ones((T, k), dtype=torch.float32, device=dev)
        self.y = torch.empty((T, H), dtype=dtype, device=dev)

    @property
    def n_recv(self) -> int:
        return int(self.recv_base[-1])

    def route_and_plan(self, logits, stream=None):
        moe_route(logits, self.k, self.topk_ids, self.topk_w, stream)
        moe_ep_plan(self.topk_ids, self.topk_w, self.E, self.R, self.plan, stream)

    def set_counts(self, counts):
        """Every source's send counts ([R, R] host array, row s = source s's plan.send_counts)."""
        self.counts = np.ascontiguousarray(np.asarray(counts), np.int32)
        dst_base, self.recv_base, self.ret_base = moe_ep_exchange_offsets(self.counts, self.rank)
        if self.n_recv > self.cap:
            raise RuntimeError(f"rank {self.rank} would receive {self.n_recv} rows, capacity {self.cap}")
        self.dst_base.copy_(torch.from_numpy(dst_base), non_blocking=False)

    def pack_to(self, x, ranks, stream=None):
        """Write this rank's send rows straight into the destination ranks' receive buffers."""
        moe_ep_pack(x, self.plan, self.dst_base, [r.x_recv for r in ranks], [r.recv_ids for r in ranks],
                    [r.recv_w for r in ranks], stream)

    def experts(self, w_gate, w_up, w_down, stream=None):
        """Local experts over the received rows: partials y_recv[:n_recv].  w_* are the E/R local
        experts' weights ([EL, H, I] / [EL, I, H]; e.g. slices of the full [E, ...] tensors)."""
        n = self.n_recv
        if n == 0:
            return self.y_recv[:0]
        k = self.k
        moe_ep_recv_index(self.recv_ids[:n], self.EL, self.expert_counts, self.expert_offsets,
                          self.slot_to_row[:n * k], self.row_to_slot[:n * k], self.recv_ws, stream)
        moe_ffn_gate_up_gather(self.x_recv[:n], self.row_to_slot[:n * k], k, w_gate, w_up, self.expert_offsets,
                               self.h[:n * k], stream)
        moe_ffn_down(self.h[:n * k], w_down, self.expert_offsets, self.y_gemm[:n * k], stream)
        return moe_combine(self.y_gemm[:n * k], self.recv_w[:n], self.slot_to_row[:n * k], self.y_recv[:n], stream)

    def return_to(self, ranks, stream=None):
        """Copy each source's partials back into its return buffer (peer copies across GPUs)."""
        with torch.cuda.stream(stream) if stream is not None else _nullctx():
            for s, src in enumerate(ranks):
                lo, hi = int(self.recv_base[s]), int(self.recv_base[s + 1])
                if hi > lo:
                    at = int(self.ret_base[s])
                    src.y_ret[at:at + hi - lo].copy_(self.y_recv[lo:hi], non_blocking=True)

    def finish(self, stream=None):
        """Each token's output: the sum of its partials (one per destination holding its experts)."""
        return moe_combine(self.y_ret, self.ones, self.plan.ret_row[:self.T * self.k], self.y, stream)


class _nullctx:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def ep_round_trip_one_gpu(ranks, xs, logits, w_gate, w_up, w_down, stream=None):
    """The expert-parallel step of R ranks on one GPU: every rank's plan, the counts exchange
    (a host copy of the R send-count vectors), each rank's pack straight into the others'
    receive buffers, each rank's local experts, the partials' return and each rank's sum.
    w_* are the full [E, ...] weight tensors (rank d uses experts [d*E/R, (d+1)*E/R)).
    Returns the R outputs."""
    R = len(ranks)
    for r, x, lg in zip(ranks, xs, logits):
        r.route_and_plan(lg, stream)
    counts = torch.stack([r.plan.send_counts for r in ranks]).cpu().numpy()
    for r in ranks:
        r.set_counts(counts)
    for r, x in zip(ranks, xs):
        r.pack_to(x, ranks, stream)
    for d, r in enumerate(ranks):
        lo, hi = d * r.EL, (d + 1) * r.EL
        r.experts(w_gate[lo:hi], w_up[lo:hi], w_down[lo:hi], stream)
    for r in ranks:
        r.return_to(ranks, stream)
    return [r.finish(stream) for r in ranks[:R]]


class EpPeer:
    """Another rank's receive buffers (x_recv, recv_ids, recv_w) and return buffer (y_ret) as
    mapped into this process: what ``MoEEPRank.pack_to`` and ``return_to`` write into."""

    def __init__(self, rank, x_recv, recv_ids, recv_w, y_ret):
        self.rank = rank
        self.x_recv, self.recv_ids, self.recv_w, self.y_ret = x_recv, recv_ids, recv_w, y_ret


def ep_share_buffers(me: MoEEPRank, group=None) -> list:
    """Every rank's buffers as seen from this process (one process per rank, all on one node):
    this rank's own ``MoEEPRank`` at its index, an ``EpPeer`` for each other rank.  The buffers'
    CUDA IPC handles (torch's tensor sharing) travel through ``all_gather_object`` on ``group``;
    opening one maps the owner's memory (with peer access when it lives on another GPU).  The
    owners must keep their ``MoEEPRank`` alive while any peer holds the mapping."""
    import io
    import pickle
    from multiprocessing.reduction import ForkingPickler

    import torch.distributed as dist
    import torch.multiprocessing  # noqa: F401  (registers the CUDA tensor reductions)

    def handles_for_one_peer():  # torch counts each pickled handle as one receiver
        buf = io.BytesIO()
        ForkingPickler(buf, pickle.HIGHEST_PROTOCOL).dump((me.x_recv, me.recv_ids, me.recv_w, me.y_ret))
        return buf.getvalue()

    mine = [b"" if d == me.rank else handles_for_one_peer() for d in range(me.R)]
    every = [None] * me.R
    dist.all_gather_object(every, mine, group=group)  # every[s][d]: source s's handles for rank d
    peers = [me if s == me.rank else EpPeer(s, *pickle.loads(every[s][me.rank])) for s in range(me.R)]
    with torch.cuda.device(me.device):
        for p in peers:  # the pack kernel stores into peers' buffers that may live on other GPUs
            if p.x_recv.device != me.device:
                moe_enable_peer_access(p.x_recv.device.index)
    return peers


def ep_round_trip_ranks(me: MoEEPRank, peers: list, x, logits, w_gate, w_up, w_down, group=None):
    """One step of the expert-parallel layer for this process's rank, the other ranks running the
    same call in their processes.  ``peers`` from ``ep_share_buffers``; w_* this rank's E/R local
    experts ([EL, H, I] / [EL, I, H]).  Phases (each ends with this rank's kernels done and a
    barrier of all ranks, so a rank writes into a peer's buffer only once the peer has finished
    with it): plan and counts exchange; pack into the destinations' receive buffers; local
    experts and return of the partials into the sources' return buffers; then the sum of each
    token's partials, which is returned."""
    import torch.distributed as dist

    def fence():
        torch.cuda.synchronize(me.device)
        dist.barrier(group=group)

    me.route_and_plan(logits)
    counts = [None] * me.R
    dist.all_gather_object(counts, me.plan.send_counts.cpu().numpy().astype(np.int32), group=group)
    me.set_counts(np.stack(counts))
    fence()  # every receive buffer is free (its owner finished the previous step with it)
    me.pack_to(x, peers)
    fence()  # every row has landed
    me.experts(w_gate, w_up, w_down)
    me.return_to(peers)
    fence()  # every partial has returned
    return me.finish()

