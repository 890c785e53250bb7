"""Torch-facing wrappers of the C ABI: same names as the C calls, argument
marshalling only (device pointers, sizes, the current CUDA stream).

PyTorch supplies device memory and streams; every step of the round trip
runs in libmoe_b200.so.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch

from . import _native
from ._native import FFN_GATE_UP, MOE_BF16, MOE_F32, check

_DT = {torch.float32: MOE_F32, torch.bfloat16: MOE_BF16}


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None, name: str, dtype=None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"activations/weights must be float32 or bfloat16, got {t.dtype}")
    return _DT[t.dtype]


def moe_route(logits: torch.Tensor, k: int, topk_ids: torch.Tensor | None = None, topk_w: torch.Tensor | None = None,
              stream=None):
    """Top-k expert ids [T,k] int32 and softmax-over-top-k weights [T,k] float32."""
    T, E = logits.shape
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    check(_native.lib().moe_route(_ptr(logits, "logits", torch.float32), T, E, k, _ptr(topk_ids, "topk_ids", torch.int32),
                                  _ptr(topk_w, "topk_w", torch.float32), _stream(stream)), "moe_route")
    return topk_ids, topk_w


def moe_router_topk(x: torch.Tensor, w_router: torch.Tensor, k: int, bias: torch.Tensor | None = None,
                    topk_ids: torch.Tensor | None = None, topk_w: torch.Tensor | None = None,
                    logits: torch.Tensor | None = None, want_logits: bool = False, stream=None):
    """Router affinities x @ w_router.T (+ bias) on tensor cores, then the top-k
    selection and softmax weights of ``moe_route`` on them, in one kernel.

    x [T,H] bf16, w_router [E,H] bf16, bias [E] float32 or None.  Returns
    (topk_ids [T,k] int32, topk_w [T,k] float32) and, when ``want_logits`` or
    ``logits`` is given, the [T,E] float32 affinities as a third value."""
    T, H = x.shape
    E = w_router.shape[0]
    dev = x.device
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    if logits is None and want_logits:
        logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    check(_native.lib().moe_router_topk(
        _ptr(x, "x", torch.bfloat16), _ptr(w_router, "w_router", torch.bfloat16), _ptr(bias, "bias", torch.float32),
        T, H, E, k, _ptr(logits, "logits", torch.float32), _ptr(topk_ids, "topk_ids", torch.int32),
        _ptr(topk_w, "topk_w", torch.float32), _stream(stream)), "moe_router_topk")
    return (topk_ids, topk_w, logits) if logits is not None else (topk_ids, topk_w)


def moe_dispatch_workspace_bytes(T: int, k: int, E: int, R: int) -> int:
    return int(_native.lib().moe_dispatch_workspace_bytes(T, k, E, R))


@dataclass
class DispatchOut:
    x_disp: torch.Tensor | None  # None: index-only dispatch (the gate/up projection gathers from x)
    expert_counts: torch.Tensor
    expert_offsets: torch.Tensor
    rank_counts: torch.Tensor
    rank_offsets: torch.Tensor
    slot_to_row: torch.Tensor
    row_to_slot: torch.Tensor
    src_expert_counts: torch.Tensor | None

    @staticmethod
    def empty(T, H, k, E, R, dtype, device, src_counts=True, rows=True) -> "DispatchOut":
        S = T * k
        i32 = dict(dtype=torch.int32, device=device)
        return DispatchOut(
            x_disp=torch.empty((S, H), dtype=dtype, device=device) if rows else None,
            expert_counts=torch.empty(E, **i32), expert_offsets=torch.empty(E + 1, **i32),
            rank_counts=torch.empty(R, **i32), rank_offsets=torch.empty(R + 1, **i32),
            slot_to_row=torch.empty(S, **i32), row_to_slot=torch.empty(S, **i32),
            src_expert_counts=torch.empty((R, E), **i32) if src_counts else None)


def moe_route_count_workspace_bytes(T: int, k: int, E: int, R: int) -> int:
    return int(_native.lib().moe_route_count_workspace_bytes(T, k, E, R))


def new_dispatch_workspace(T: int, k: int, E: int, R: int, device) -> torch.Tensor:
    """Zero-filled workspace large enough for moe_dispatch and for the counted pair
    (moe_route_count + moe_dispatch_counted)."""
    n = max(moe_dispatch_workspace_bytes(T, k, E, R), moe_route_count_workspace_bytes(T, k, E, R))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_dispatch(x: torch.Tensor | None, topk_ids: torch.Tensor, E: int, R: int, out: DispatchOut,
                 workspace: torch.Tensor, stream=None, H: int | None = None, dtype=None,
                 _entry: str = "moe_dispatch") -> DispatchOut:
    """Dispatch; with x None and out.x_disp None it is index-only (counts,
    offsets and permutation; no rows move), and H / dtype name the row shape."""
    if x is not None:
        T, H = x.shape
        dtype = x.dtype
    else:
        T = topk_ids.shape[0]
        if H is None or dtype is None:
            raise ValueError("index-only dispatch needs H and dtype")
    k = topk_ids.shape[1]
    i32 = torch.int32
    check(getattr(_native.lib(), _entry)(
        _ptr(x, "x"), _DT[dtype] if dtype in _DT else _dtype(x), T, H, _ptr(topk_ids, "topk_ids", i32), k, E, R,
        _ptr(out.x_disp, "x_disp", dtype),
        _ptr(out.expert_counts, "expert_counts", i32), _ptr(out.expert_offsets, "expert_offsets", i32),
        _ptr(out.rank_counts, "rank_counts", i32), _ptr(out.rank_offsets, "rank_offsets", i32),
        _ptr(out.slot_to_row, "slot_to_row", i32), _ptr(out.row_to_slot, "row_to_slot", i32),
        _ptr(out.src_expert_counts, "src_expert_counts", i32), _ptr(workspace, "workspace", torch.uint8),
        workspace.numel(), _stream(stream)), _entry)
    return out


def moe_route_count(logits: torch.Tensor, k: int, R: int, workspace: torch.Tensor, topk_ids=None, topk_w=None,
                    stream=None):
    """moe_route plus the dispatch's counting into `workspace` (a moe_dispatch workspace for
    these T, k, E, R): moe_dispatch_counted on the same ids and workspace then skips its counting."""
    T, E = logits.shape
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    check(_native.lib().moe_route_count(_ptr(logits, "logits", torch.float32), T, E, k, int(R),
                                        _ptr(topk_ids, "topk_ids", torch.int32), _ptr(topk_w, "topk_w", torch.float32),
                                        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream)),
          "moe_route_count")
    return topk_ids, topk_w


def moe_dispatch_counted(x: torch.Tensor | None, topk_ids: torch.Tensor, E: int, R: int, out: DispatchOut,
                         workspace: torch.Tensor, stream=None, H: int | None = None, dtype=None) -> DispatchOut:
    """moe_dispatch for the ids moe_route_count last wrote with this workspace (same arguments)."""
    return moe_dispatch(x, topk_ids, E, R, out, workspace, stream, H, dtype, _entry="moe_dispatch_counted")


def moe_ffn_gate_up(x_disp, w_gate, w_up, expert_offsets, h, stream=None):
    S, H = x_disp.shape
    E, _, I = w_gate.shape
    check(_native.lib().moe_ffn_gate_up(
        _ptr(x_disp, "x_disp"), _dtype(x_disp), _ptr(w_gate, "w_gate", x_disp.dtype), _ptr(w_up, "w_up", x_disp.dtype),
        _ptr(expert_offsets, "expert_offsets", torch.int32), E, H, I, S, _ptr(h, "h", x_disp.dtype),
        _stream(stream)), "moe_ffn_gate_up")
    return h


def moe_ffn_down(h, w_down, expert_offsets, y_disp, stream=None):
    S, I = h.shape
    E, _, H = w_down.shape
    check(_native.lib().moe_ffn_down(
        _ptr(h, "h"), _dtype(h), _ptr(w_down, "w_down", h.dtype), _ptr(expert_offsets, "expert_offsets", torch.int32),
        E, H, I, S, _ptr(y_disp, "y_disp", h.dtype), _stream(stream)), "moe_ffn_down")
    return y_disp


def moe_ffn_down_combine(h, w_down, expert_offsets, row_to_slot, topk_w, y_acc, stream=None):
    """y_acc[t] += sum_j w[t, j] * (h Wd)[row of slot t*k+j]: the down projection with the combine
    in its epilogue (float32 atomics; y_disp is not formed).  y_acc [T, H] float32, zero on the
    first call (moe_combine_finalize leaves it zero)."""
    S, I = h.shape
    E, _, H = w_down.shape
    T, k = topk_w.shape
    check(_native.lib().moe_ffn_down_combine(
        _ptr(h, "h"), _dtype(h), _ptr(w_down, "w_down", h.dtype), _ptr(expert_offsets, "expert_offsets", torch.int32),
        E, H, I, S, _ptr(row_to_slot, "row_to_slot", torch.int32), _ptr(topk_w, "topk_w", torch.float32), T, k,
        _ptr(y_acc, "y_acc", torch.float32), _stream(stream)), "moe_ffn_down_combine")
    return y_acc


def moe_combine_finalize(y_acc, y, stream=None):
    """y = y_acc rounded to y's dtype (bf16); y_acc zeroed for the next moe_ffn_down_combine."""
    T, H = y.shape
    check(_native.lib().moe_combine_finalize(_ptr(y_acc, "y_acc", torch.float32), _dtype(y), T, H, _ptr(y, "y"),
                                             _stream(stream)), "moe_combine_finalize")
    return y


def moe_ffn_gate_up_gather(x, row_to_slot, k, w_gate, w_up, expert_offsets, h, stream=None):
    """h = SiLU(x[row_to_slot // k] Wg_e) * (x[row_to_slot // k] Wu_e): the gate/up
    projection reading its rows straight from x (no x_disp)."""
    T, H = x.shape
    S = row_to_slot.shape[0]
    E, _, I = w_gate.shape
    dt = x.dtype
    check(_native.lib().moe_ffn_gate_up_gather(
        _ptr(x, "x"), _dtype(x), T, _ptr(row_to_slot, "row_to_slot", torch.int32), int(k), _ptr(w_gate, "w_gate", dt),
        _ptr(w_up, "w_up", dt), _ptr(expert_offsets, "expert_offsets", torch.int32), E, H, I, S, _ptr(h, "h", dt),
        _stream(stream)), "moe_ffn_gate_up_gather")
    return h


def moe_expert_ffn_gather(x, row_to_slot, k, w_gate, w_up, w_down, expert_offsets, h, y_disp, stream=None):
    T, H = x.shape
    S = row_to_slot.shape[0]
    E, _, I = w_gate.shape
    dt = x.dtype
    check(_native.lib().moe_expert_ffn_gather(
        _ptr(x, "x"), _dtype(x), T, _ptr(row_to_slot, "row_to_slot", torch.int32), int(k), _ptr(w_gate, "w_gate", dt),
        _ptr(w_up, "w_up", dt), _ptr(w_down, "w_down", dt), _ptr(expert_offsets, "expert_offsets", torch.int32),
        E, H, I, S, _ptr(h, "h", dt), _ptr(y_disp, "y_disp", dt), _stream(stream)), "moe_expert_ffn_gather")
    return y_disp


def moe_expert_ffn(x_disp, w_gate, w_up, w_down, expert_offsets, h, y_disp, stream=None):
    S, H = x_disp.shape
    E, _, I = w_gate.shape
    dt = x_disp.dtype
    check(_native.lib().moe_expert_ffn(
        _ptr(x_disp, "x_disp"), _dtype(x_disp), _ptr(w_gate, "w_gate", dt), _ptr(w_up, "w_up", dt),
        _ptr(w_down, "w_down", dt), _ptr(expert_offsets, "expert_offsets", torch.int32), E, H, I, S,
        _ptr(h, "h", dt), _ptr(y_disp, "y_disp", dt), _stream(stream)), "moe_expert_ffn")
    return y_disp


def moe_combine(y_disp, topk_w, slot_to_row, y, stream=None):
    T, H = y.shape
    k = topk_w.shape[1]
    check(_native.lib().moe_combine(
        _ptr(y_disp, "y_disp", y.dtype), _dtype(y), _ptr(topk_w, "topk_w", torch.float32),
        _ptr(slot_to_row, "slot_to_row", torch.int32), T, k, H, _ptr(y, "y"), _stream(stream)), "moe_combine")
    return y


def moe_combine_rank_partials(y_disp, topk_w, topk_ids, slot_to_row, E: int, R: int, y_part=None, stream=None):
    """Masking form of expert parallelism: y_part[r, t] = the w-weighted sum of token t's expert
    outputs whose expert rank r owns (experts [r*E/R, (r+1)*E/R)), zero where it owns none.
    Returns y_part [R, T, H] (allocated if not given)."""
    T, k = topk_w.shape
    H = y_disp.shape[1]
    if y_part is None:
        y_part = torch.empty((R, T, H), dtype=y_disp.dtype, device=y_disp.device)
    check(_native.lib().moe_combine_rank_partials(
        _ptr(y_disp, "y_disp"), _dtype(y_disp), _ptr(topk_w, "topk_w", torch.float32),
        _ptr(topk_ids, "topk_ids", torch.int32), _ptr(slot_to_row, "slot_to_row", torch.int32), T, k, H, int(E),
        int(R), _ptr(y_part, "y_part", y_disp.dtype), _stream(stream)), "moe_combine_rank_partials")
    return y_part


def moe_reduce_rank_partials(y_part, y=None, stream=None):
    """y[t] = sum over ranks r (in order) of y_part[r, t]: the reduce-scatter / all-reduce of the
    masking form, on one GPU."""
    R, T, H = y_part.shape
    if y is None:
        y = torch.empty((T, H), dtype=y_part.dtype, device=y_part.device)
    check(_native.lib().moe_reduce_rank_partials(_ptr(y_part, "y_part"), _dtype(y_part), T, H, R,
                                                 _ptr(y, "y", y_part.dtype), _stream(stream)),
          "moe_reduce_rank_partials")
    return y


def moe_set_ffn_tiling(mode: int) -> None:
    """Tile shape of the bf16 expert FFN for the whole process:
    FFN_TILING_AUTO (0), FFN_TILING_SINGLE (1, 128-row tiles on one SM) or
    FFN_TILING_PAIR (2, 256-row tiles on a 2-SM cluster)."""
    check(_native.lib().moe_set_ffn_tiling(int(mode)), "moe_set_ffn_tiling")


def moe_get_ffn_tiling() -> int:
    return _native.lib().moe_get_ffn_tiling()


def moe_ffn_tiling_for(E: int, S: int, projection: int = FFN_GATE_UP) -> int:
    """The tile shape (SINGLE or PAIR) a bf16 call of one projection
    (FFN_GATE_UP or FFN_DOWN) with E experts and S rows would use now."""
    return _native.lib().moe_ffn_tiling_for(int(E), int(S), int(projection))


def moe_get_error(stream=None) -> tuple[int, int]:
    """Synchronise the stream; return (status, error-word bits) and clear the word."""
    bits = ctypes.c_uint32(0)
    st = _native.lib().moe_get_error(_stream(stream), ctypes.byref(bits))
    return st, bits.value


class MoERoundTrip:
    """Buffers and the four calls of one MoE layer round trip on one GPU.

    Route -> dispatch -> grouped SwiGLU FFN -> combine, all on `stream`.
    Device memory for every intermediate is allocated once here (through
    torch); ``forward`` enqueues five kernels (route, dispatch, gate/up, down,
    combine) and allocates nothing.

    gather=True fuses the row scatter into the gate/up projection: dispatch
    is index-only and moe_ffn_gate_up_gather reads each row from x, so the
    [S, H] x_disp buffer is neither allocated nor written (same results, bit
    for bit).  gather="auto" (the default) fuses where that is measured to be
    faster: bf16 layers with fewer than GATHER_MAX_ROWS_PER_EXPERT rows per
    expert, whose FFN streams weights from HBM, so the x_disp round trip is
    extra HBM traffic.  With more rows per expert the FFN is tensor-bound and
    the gathering producer costs more than the dispatch it saves.
    """

    GATHER_MAX_ROWS_PER_EXPERT = 384

    @classmethod
    def gathers_by_default(cls, T, k, E, dtype) -> bool:
        """gather="auto": bf16 layers with fewer than GATHER_MAX_ROWS_PER_EXPERT rows per expert."""
        return dtype == torch.bfloat16 and T * k < cls.GATHER_MAX_ROWS_PER_EXPERT * E

    def __init__(self, T, H, I, E, k, R, dtype, device="cuda", src_counts=True, gather="auto", rank_partials=False,
                 route_counts=True, combine_in_down=False):
        self.T, self.H, self.I, self.E, self.k, self.R = T, H, I, E, k, R
        self.dtype = dtype
        self.device = torch.device(device)
        if gather == "auto":
            gather = self.gathers_by_default(T, k, E, dtype)
        self.gather = bool(gather)
        # route() also does the dispatch's counting (moe_route_count) and dispatch() reads it
        # (moe_dispatch_counted); False: moe_route and moe_dispatch
        self.route_counts = bool(route_counts)
        self._x = None
        S = T * k
        self.topk_ids = torch.empty((T, k), dtype=torch.int32, device=self.device)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=self.device)
        self.disp = DispatchOut.empty(T, H, k, E, R, dtype, self.device, src_counts, rows=not self.gather)
        self.workspace = new_dispatch_workspace(T, k, E, R, self.device)
        self.h = torch.empty((S, I), dtype=dtype, device=self.device)
        self.y_disp = torch.empty((S, H), dtype=dtype, device=self.device)
        self.y = torch.empty((T, H), dtype=dtype, device=self.device)
        # the masking form's per-rank partial outputs (combine_masked), [R, T, H]
        self.y_part = torch.empty((R, T, H), dtype=dtype, device=self.device) if rank_partials else None
        # combine_in_down: the down projection adds w * output into a float32 [T, H] accumulator
        # (moe_ffn_down_combine) and a finalize kernel rounds it into y; y_disp is not used (bf16)
        self.combine_in_down = bool(combine_in_down) and dtype == torch.bfloat16
        self.y_acc = torch.zeros((T, H), dtype=torch.float32, device=self.device) if self.combine_in_down else None

    def route(self, logits, stream=None):
        if self.route_counts:
            return moe_route_count(logits, self.k, self.R, self.workspace, self.topk_ids, self.topk_w, stream)
        return moe_route(logits, self.k, self.topk_ids, self.topk_w, stream)

    def dispatch(self, x, stream=None):
        fn = moe_dispatch_counted if self.route_counts else moe_dispatch
        if self.gather:  # the rows stay in x; gate_up reads them there
            self._x = x
            return fn(None, self.topk_ids, self.E, self.R, self.disp, self.workspace, stream, H=self.H,
                      dtype=self.dtype)
        return fn(x, self.topk_ids, self.E, self.R, self.disp, self.workspace, stream)

    def gate_up(self, w_gate, w_up, stream=None):
        if self.gather:
            if self._x is None:
                raise RuntimeError("gate_up of a gathering round trip needs dispatch(x) first")
            return moe_ffn_gate_up_gather(self._x, self.disp.row_to_slot, self.k, w_gate, w_up,
                                          self.disp.expert_offsets, self.h, stream)
        return moe_ffn_gate_up(self.disp.x_disp, w_gate, w_up, self.disp.expert_offsets, self.h, stream)

    def down(self, w_down, stream=None):
        if self.combine_in_down:
            return moe_ffn_down_combine(self.h, w_down, self.disp.expert_offsets, self.disp.row_to_slot, self.topk_w,
                                        self.y_acc, stream)
        return moe_ffn_down(self.h, w_down, self.disp.expert_offsets, self.y_disp, stream)

    def combine(self, stream=None, y=None):
        if self.combine_in_down:
            return moe_combine_finalize(self.y_acc, self.y if y is None else y, stream)
        return moe_combine(self.y_disp, self.topk_w, self.disp.slot_to_row, self.y if y is None else y, stream)

    def combine_masked(self, stream=None, y=None):
        """The masking form's return path in place of combine: per-rank partial outputs
        (self.y_part, [R, T, H]) and their rank-ordered sum.  Needs rank_partials=True."""
        if self.y_part is None:
            raise RuntimeError("combine_masked needs MoERoundTrip(..., rank_partials=True)")
        moe_combine_rank_partials(self.y_disp, self.topk_w, self.topk_ids, self.disp.slot_to_row, self.E, self.R,
                                  self.y_part, stream)
        return moe_reduce_rank_partials(self.y_part, self.y if y is None else y, stream)

    def forward(self, x, logits, w_gate, w_up, w_down, stream=None, y=None):
        self.route(logits, stream)
        self.dispatch(x, stream)
        self.gate_up(w_gate, w_up, stream)
        self.down(w_down, stream)
        return self.combine(stream, y)

    def forward_masked(self, x, logits, w_gate, w_up, w_down, stream=None, y=None):
        """forward with the masking form's return path (combine_masked): six kernels."""
        self.route(logits, stream)
        self.dispatch(x, stream)
        self.gate_up(w_gate, w_up, stream)
        self.down(w_down, stream)
        return self.combine_masked(stream, y)

    KERNELS_PER_FORWARD = 5  # route, dispatch, gate/up, down, combine

    def capture(self, x, logits, w_gate, w_up, w_down, y=None, stream=None):
        """Record ``forward`` on these fixed buffers into a CUDA graph.

        Returns a ``torch.cuda.CUDAGraph``; ``graph.replay()`` reruns the whole
        round trip on whatever ``x`` and ``logits`` then hold, with one launch
        from the host.  Call ``forward`` once before capturing (the library sets
        kernel attributes on first use, which must not happen during capture).
        """
        g = torch.cuda.CUDAGraph()
        s = stream if stream is not None else torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.graph(g, stream=s):
            self.forward(x, logits, w_gate, w_up, w_down, stream=s, y=y)
        torch.cuda.current_stream(self.device).wait_stream(s)
        return g


@dataclass
class EplbPlan:
    """Placement of P = R * slots physical experts (replicas of the E logical ones)
    from moe_eplb_plan; host arrays plus device copies of the remap tables."""
    E: int
    R: int
    slots: int
    phys_to_logical: np.ndarray   # [P] int32
    replica_offsets: np.ndarray   # [E + 1] int32
    replicas: np.ndarray          # [P] int32
    replica_offsets_dev: torch.Tensor
    replicas_dev: torch.Tensor

    @property
    def P(self) -> int:
        return self.R * self.slots

    def replica_counts(self) -> np.ndarray:
        return np.diff(self.replica_offsets)


def moe_eplb_plan(load, R: int, slots_per_rank: int, device="cuda") -> EplbPlan:
    """Plan replicas and their placement on R ranks of slots_per_rank physical experts from
    per-expert loads (numpy or torch, any integer dtype; e.g. expert_counts of earlier steps)."""
    if isinstance(load, torch.Tensor):
        load = load.detach().cpu().numpy()
    load = np.ascontiguousarray(np.asarray(load, dtype=np.int64))
    E = int(load.shape[0])
    P = int(R) * int(slots_per_rank)
    p2l = np.empty(max(P, 0), np.int32)
    off = np.empty(E + 1, np.int32)
    reps = np.empty(max(P, 0), np.int32)
    check(_native.lib().moe_eplb_plan(load.ctypes.data, E, int(R), int(slots_per_rank), p2l.ctypes.data,
                                      off.ctypes.data, reps.ctypes.data), "moe_eplb_plan")
    return EplbPlan(E, int(R), int(slots_per_rank), p2l, off, reps,
                    torch.from_numpy(off).to(device), torch.from_numpy(reps).to(device))


def moe_eplb_remap(topk_ids: torch.Tensor, plan: EplbPlan, out: torch.Tensor | None = None, stream=None):
    """Logical expert ids [T, k] -> physical replica ids (round robin over token index)."""
    T, k = topk_ids.shape
    if out is None:
        out = torch.empty_like(topk_ids)
    i32 = torch.int32
    check(_native.lib().moe_eplb_remap(
        _ptr(topk_ids, "topk_ids", i32), T, k, plan.E, _ptr(plan.replica_offsets_dev, "replica_offsets", i32),
        _ptr(plan.replicas_dev, "replicas", i32), plan.P, _ptr(out, "phys_ids", i32), _stream(stream)),
        "moe_eplb_remap")
    return out


def moe_eplb_replicate(w: torch.Tensor, plan: EplbPlan, out: torch.Tensor | None = None, stream=None):
    """Weights of the physical experts: out[p] = w[plan.phys_to_logical[p]] (w is [E, ...])."""
    if w.shape[0] != plan.E:
        raise ValueError(f"w has {w.shape[0]} experts, the plan {plan.E}")
    if out is None:
        out = torch.empty((plan.P, *w.shape[1:]), dtype=w.dtype, device=w.device)
    _ptr(w, "w")
    _ptr(out, "out", w.dtype)
    expert_bytes = w[0].numel() * w.element_size()
    check(_native.lib().moe_eplb_replicate(w.data_ptr(), expert_bytes, plan.E, plan.phys_to_logical.ctypes.data,
                                           plan.P, out.data_ptr(), _stream(stream)), "moe_eplb_replicate")
    return out


class MoEBalancedRoundTrip:
    """The round trip over replicated experts: route on the E logical experts, remap each
    slot to a physical replica (moe_eplb_remap), then dispatch, FFN and combine over the
    P = R * slots_per_rank physical experts, rank r holding physical experts
    [r * slots_per_rank, (r + 1) * slots_per_rank).  Outputs equal MoERoundTrip's bit for
    bit (a replica has its expert's weights); the per-rank row counts follow the plan.
    ``set_plan`` installs a plan and copies the weights of its physical experts."""

    def __init__(self, T, H, I, E, k, R, slots_per_rank, dtype, device="cuda", gather="auto"):
        self.E, self.k, self.R, self.slots = E, k, R, slots_per_rank
        self.P = R * slots_per_rank
        # ids are remapped between routing and dispatch: the dispatch counts them itself
        self.rt = MoERoundTrip(T, H, I, self.P, k, R, dtype, device=device, gather=gather, route_counts=False)
        self.logical_ids = torch.empty((T, k), dtype=torch.int32, device=self.rt.device)
        self.plan = None
        self.w = None

    def set_plan(self, plan: EplbPlan, w_gate, w_up, w_down, stream=None):
        if plan.E != self.E or plan.R != self.R or plan.slots != self.slots:
            raise ValueError("plan sizes differ from the round trip's")
        if self.w is None:
            self.w = [torch.empty((self.P, *w.shape[1:]), dtype=w.dtype, device=w.device)
                      for w in (w_gate, w_up, w_down)]
        for dst, w in zip(self.w, (w_gate, w_up, w_down)):
            moe_eplb_replicate(w, plan, out=dst, stream=stream)
        self.plan = plan

    def route(self, logits, stream=None):
        moe_route(logits, self.k, self.logical_ids, self.rt.topk_w, stream)
        return moe_eplb_remap(self.logical_ids, self.plan, out=self.rt.topk_ids, stream=stream)

    def forward(self, x, logits, stream=None, y=None):
        if self.plan is None:
            raise RuntimeError("set_plan first")
        self.route(logits, stream)
        self.rt.dispatch(x, stream)
        self.rt.gate_up(self.w[0], self.w[1], stream)
        self.rt.down(self.w[2], stream)
        return self.rt.combine(stream, y)

    KERNELS_PER_FORWARD = 6  # route, remap, dispatch, gate/up, down, combine


class MoEHostPipeline:
    """Round trips over a sequence of host-resident batches.

    Each batch's inputs (x, logits) start in pinned host memory and its output
    y ends there.  Three CUDA streams overlap the host->device copy of batch
    i+1 and the device->host copy of batch i-1 with the compute of batch i;
    device inputs and outputs are double-buffered, and events order every
    reuse of a buffer after the work that last touched it.  With ``graphs``
    (the default) the round trip of each buffer set is a captured CUDA graph,
    replayed once per batch.
    """

    def __init__(self, rt: MoERoundTrip, w_gate, w_up, w_down, compute_stream=None, graphs=True):
        self.rt = rt
        self.w = (w_gate, w_up, w_down)
        dev = rt.device
        self.comp = compute_stream if compute_stream is not None else torch.cuda.current_stream(dev)
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.x_dev = [torch.zeros((rt.T, rt.H), dtype=rt.dtype, device=dev) for _ in range(2)]
        self.l_dev = [torch.zeros((rt.T, rt.E), dtype=torch.float32, device=dev) for _ in range(2)]
        self.y_dev = [torch.empty((rt.T, rt.H), dtype=rt.dtype, device=dev) for _ in range(2)]
        ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
        self.in_ready, self.in_free, self.out_ready, self.out_free = ev(), ev(), ev(), ev()
        self._used = [False, False]
        self.graphs = None
        if graphs:
            # one CUDA graph per buffer set: a step then costs the host one launch instead of the
            # round trip's calls (first use of each kernel happens here, outside the capture)
            rt.forward(self.x_dev[0], self.l_dev[0], *self.w, stream=self.comp, y=self.y_dev[0])
            self.comp.synchronize()
            self.graphs = [rt.capture(self.x_dev[b], self.l_dev[b], *self.w, y=self.y_dev[b]) for b in range(2)]
            torch.cuda.synchronize(dev)

    @staticmethod
    def _as_dev_dtype(host: torch.Tensor, dev: torch.Tensor) -> torch.Tensor:
        # bfloat16 data may be held on the host as raw int16 bit patterns
        return host.view(dev.dtype) if host.dtype != dev.dtype and host.element_size() == dev.element_size() else host

    def run(self, batches):
        """batches: iterable of (x_host, logits_host, y_host), pinned CPU tensors.
        Enqueues everything and returns; y_host is valid after the d2h stream syncs."""
        for i, (xh, lh, yh) in enumerate(batches):
            b = i & 1
            if self._used[b]:
                self.h2d.wait_event(self.in_free[b])   # compute of batch i-2 is done with x/l buffers
            with torch.cuda.stream(self.h2d):
                self.x_dev[b].copy_(self._as_dev_dtype(xh, self.x_dev[b]), non_blocking=True)
                self.l_dev[b].copy_(lh, non_blocking=True)
                self.in_ready[b].record(self.h2d)
            self.comp.wait_event(self.in_ready[b])
            if self._used[b]:
                self.comp.wait_event(self.out_free[b])  # y of batch i-2 has been copied out
            if self.graphs is not None:
                with torch.cuda.stream(self.comp):
                    self.graphs[b].replay()
            else:
                self.rt.forward(self.x_dev[b], self.l_dev[b], *self.w, stream=self.comp, y=self.y_dev[b])
            self.in_free[b].record(self.comp)
            self.out_ready[b].record(self.comp)
            self.d2h.wait_event(self.out_ready[b])
            with torch.cuda.stream(self.d2h):
                yh.copy_(self.y_dev[b].view(yh.dtype) if yh.dtype != self.y_dev[b].dtype else self.y_dev[b],
                         non_blocking=True)
                self.out_free[b].record(self.d2h)
            self._used[b] = True
        return self.d2h
