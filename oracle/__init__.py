"""CPU oracle for the MoE token round trip (route, dispatch, SwiGLU FFN, combine).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference leg of ``bench.py``.  The product library
(``token_dispatch_combine_b200``) never imports it, and the two share no code.

The arithmetic lives in ``moe_oracle.c`` (plain C, float64); this module only
builds it with gcc and marshals numpy arrays.  Each C function cites the page
passage it follows.  Every function is pinned by ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc -O2, OpenMP, strict IEEE)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _configure(lib):
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.oracle_route.argtypes = [vp, i32, i32, i32, vp, vp]
    lib.oracle_route.restype = i32
    lib.oracle_src_rank.argtypes = [i32, i32, i32]
    lib.oracle_src_rank.restype = i32
    lib.oracle_dispatch_index.argtypes = [vp, i32, i32, i32, i32] + [vp] * 7
    lib.oracle_dispatch_index.restype = i32
    lib.oracle_dispatch_rows.argtypes = [vp, sz, i32, i32, vp, vp]
    lib.oracle_ffn_rows.argtypes = [vp, i32, vp, i32, vp, vp, vp, i32, i32, i32, vp, vp]
    lib.oracle_combine.argtypes = [vp, vp, vp, i32, i32, i32, vp]
    lib.oracle_router_logits.argtypes = [vp, i32, vp, i32, vp, i32, i32, i32, vp]
    lib.oracle_router_logits.restype = i32
    lib.oracle_eplb_plan.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    lib.oracle_eplb_plan.restype = i32
    lib.oracle_eplb_remap.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    lib.oracle_rank_partials.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]
    lib.oracle_rank_partials.restype = i32
    lib.oracle_reduce_ranks.argtypes = [vp, i32, i32, i32, vp]
    lib.oracle_ep_plan.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.oracle_ep_plan.restype = i32
    return lib


def _get():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _configure(ctypes.CDLL(build()))
    return _lib


@contextlib.contextmanager
def _substitute_library(path: str):
    """Run the wrappers against another build of the oracle source (used by the
    mutation tests, which plant a mistake in a copy and expect a pin to fail)."""
    global _lib
    _get()
    saved = _lib
    _lib = _configure(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def route(logits: np.ndarray, k: int):
    """Top-k ids [T,k] int32 (logit desc, lower id on ties) and softmax weights [T,k] float32."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    if _get().oracle_route(logits.ctypes.data, T, E, k, ids.ctypes.data, w.ctypes.data) != 0:
        raise ValueError("oracle_route: bad sizes")
    return ids, w


def router_logits(x: np.ndarray, w_router: np.ndarray, bias=None) -> np.ndarray:
    """Affinities [T,E] float32 = round_f32(x @ w_router.T + bias) in float64.

    ``x`` [T,H] and ``w_router`` [E,H] are float32 or bf16 bits (uint16);
    ``bias`` [E] (any float type) or None."""
    x = np.ascontiguousarray(x)
    w = np.ascontiguousarray(w_router)
    T, H = x.shape
    E = w.shape[0]
    if w.shape[1] != H:
        raise ValueError("w_router must be [E, H]")
    b = None if bias is None else _c(bias, np.float64)
    out = np.empty((T, E), np.float32)
    if _get().oracle_router_logits(x.ctypes.data, _dt(x), w.ctypes.data, _dt(w),
                                   None if b is None else b.ctypes.data, T, H, E, out.ctypes.data) != 0:
        raise ValueError("oracle_router_logits: bad sizes")
    return out


def src_rank(t: int, T: int, R: int) -> int:
    return _get().oracle_src_rank(t, T, R)


def dispatch_index(ids: np.ndarray, E: int, R: int) -> dict:
    """Counts, offsets and the stable slot<->row permutation (see moe_oracle.c)."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    S = T * k
    out = dict(
        expert_counts=np.empty(E, np.int32), expert_offsets=np.empty(E + 1, np.int32),
        rank_counts=np.empty(R, np.int32), rank_offsets=np.empty(R + 1, np.int32),
        slot_to_row=np.empty(S, np.int32), row_to_slot=np.empty(S, np.int32),
        src_expert_counts=np.empty((R, E), np.int32),
    )
    dropped = _get().oracle_dispatch_index(
        ids.ctypes.data, T, k, E, R, *(out[n].ctypes.data for n in (
            "expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row",
            "row_to_slot", "src_expert_counts")))
    if dropped < 0:
        raise ValueError("oracle_dispatch_index: bad sizes")
    out["dropped"] = dropped
    return out


def dispatch_rows(x: np.ndarray, k: int, slot_to_row: np.ndarray, n_rows: int | None = None) -> np.ndarray:
    """x_disp[slot_to_row[s]] = x[s // k]; rows never written stay zero."""
    x = np.ascontiguousarray(x)
    T = x.shape[0]
    n_rows = T * k if n_rows is None else n_rows
    xd = np.zeros((n_rows,) + x.shape[1:], dtype=x.dtype)
    s2r = _c(slot_to_row, np.int32)
    _get().oracle_dispatch_rows(x.ctypes.data, x[0].nbytes if T else 0, T, k, s2r.ctypes.data, xd.ctypes.data)
    return xd


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bfloat16 bits (uint16), got {a.dtype}")


def ffn_rows(x_rows: np.ndarray, row_expert: np.ndarray, w_gate, w_up, w_down, H: int, I: int,
             want_act: bool = False):
    """SwiGLU expert MLP of each row in float64.

    ``w_gate``/``w_up``/``w_down`` map expert id -> that expert's matrix
    ([H,I], [H,I], [I,H]; float32 or bf16 bits).  They may be full [E,...]
    arrays or dicts holding only the experts that ``row_expert`` uses.
    Returns y [n,H] (and the activations [n,I] when ``want_act``).
    """
    x_rows = np.ascontiguousarray(x_rows)
    n = x_rows.shape[0]
    rexp = _c(row_expert, np.int32)
    if isinstance(w_gate, np.ndarray):
        E = w_gate.shape[0]
        g = {e: w_gate[e] for e in range(E)}
        u = {e: w_up[e] for e in range(E)}
        d = {e: w_down[e] for e in range(E)}
    else:
        g, u, d = w_gate, w_up, w_down
    E = (max(g.keys()) + 1) if g else 1
    keep = []

    def ptrs(m):
        arr = (ctypes.c_void_p * E)()
        for e, a in m.items():
            a = np.ascontiguousarray(a)
            keep.append(a)
            arr[e] = a.ctypes.data
        return arr

    pg, pu, pd = ptrs(g), ptrs(u), ptrs(d)
    wdt = _dt(next(iter(g.values()))) if g else F32
    for e in set(rexp.tolist()):
        if e not in g:
            raise KeyError(f"weights of expert {e} not supplied")
    y = np.empty((n, H), np.float64)
    a = np.empty((n, I), np.float64) if want_act else None
    if n:
        _get().oracle_ffn_rows(x_rows.ctypes.data, _dt(x_rows), rexp.ctypes.data, n, pg, pu, pd, wdt, H, I,
                               a.ctypes.data if want_act else None, y.ctypes.data)
    return (y, a) if want_act else y


def combine(y_disp: np.ndarray, topk_w: np.ndarray, slot_to_row: np.ndarray) -> np.ndarray:
    """y[t] = sum_j w[t,j] * y_disp[slot_to_row[t*k+j]] in float64."""
    y_disp = _c(y_disp, np.float64)
    topk_w = _c(topk_w, np.float32)
    s2r = _c(slot_to_row, np.int32)
    T, k = topk_w.shape
    H = y_disp.shape[1]
    y = np.empty((T, H), np.float64)
    _get().oracle_combine(y_disp.ctypes.data, topk_w.ctypes.data, s2r.ctypes.data, T, k, H, y.ctypes.data)
    return y


def rank_partials(y_disp: np.ndarray, topk_w: np.ndarray, topk_ids: np.ndarray, slot_to_row: np.ndarray, E: int,
                  R: int) -> np.ndarray:
    """Masking form: part[r][t] = sum of w[t,j] * y_disp[slot_to_row[t*k+j]] over the choices j of
    token t whose expert sits on rank r (experts [r*E/R, (r+1)*E/R)); [R, T, H] float64."""
    y_disp = _c(y_disp, np.float64)
    topk_w = _c(topk_w, np.float32)
    ids = _c(topk_ids, np.int32)
    s2r = _c(slot_to_row, np.int32)
    T, k = topk_w.shape
    H = y_disp.shape[1]
    part = np.empty((R, T, H), np.float64)
    if _get().oracle_rank_partials(y_disp.ctypes.data, topk_w.ctypes.data, ids.ctypes.data, s2r.ctypes.data, T, k,
                                   H, E, R, part.ctypes.data) != 0:
        raise ValueError("oracle_rank_partials: bad sizes")
    return part


def reduce_ranks(part: np.ndarray) -> np.ndarray:
    """y[t] = sum over ranks r (ascending) of part[r][t], float64."""
    part = _c(part, np.float64)
    R, T, H = part.shape
    y = np.empty((T, H), np.float64)
    _get().oracle_reduce_ranks(part.ctypes.data, T, H, R, y.ctypes.data)
    return y


def ep_plan(topk_ids: np.ndarray, topk_w: np.ndarray, E: int, R: int) -> dict:
    """Send plan of one source rank in the expert-parallel exchange (oracle_ep_plan): one row per
    (token, destination rank) holding any of its experts, ordered by destination then token, with
    the token's local expert ids and weights on that rank.  Keys: send_counts [R], send_offsets
    [R+1], slot_send_row [T*k], row_token [n], row_ids [n, k], row_w [n, k] (n = send rows)."""
    ids = _c(topk_ids, np.int32)
    w = _c(topk_w, np.float32)
    T, k = ids.shape
    cnt = np.empty(R, np.int32)
    off = np.empty(R + 1, np.int32)
    ssr = np.empty(T * k, np.int32)
    cap = max(1, T * k)
    tok = np.empty(cap, np.int32)
    rid = np.empty((cap, k), np.int32)
    rw = np.empty((cap, k), np.float32)
    n = _get().oracle_ep_plan(ids.ctypes.data, w.ctypes.data, T, k, E, R, cnt.ctypes.data, off.ctypes.data,
                              ssr.ctypes.data, tok.ctypes.data, rid.ctypes.data, rw.ctypes.data)
    if n < 0:
        raise ValueError("oracle_ep_plan: bad sizes")
    return dict(send_counts=cnt, send_offsets=off, slot_send_row=ssr, row_token=tok[:n].copy(),
                row_ids=rid[:n].copy(), row_w=rw[:n].copy())


def ep_round_trip(xs, logits_list, k: int, E: int, R: int, w_gate, w_up, w_down) -> dict:
    """The expert-parallel round trip over R source ranks on the CPU: each rank routes its own
    tokens and plans its sends (ep_plan); destination d receives the rows of sources 0..R-1 in
    turn (each source's rows for d in its send order), runs each row through its local experts
    and sums their weighted outputs (one partial per received row); the partials return to
    their source rows, and each token's output is the sum of its partials over destinations
    in ascending order.  Returns per-rank lists: plans, received rows / ids / weights / source,
    partials and outputs y (float64)."""
    EL = E // R
    H = xs[0].shape[1]
    I = w_gate.shape[-1] if isinstance(w_gate, np.ndarray) else next(iter(w_gate.values())).shape[-1]
    routes = [route(lg, k) for lg in logits_list]
    plans = [ep_plan(ids, w, E, R) for ids, w in routes]
    recv_x, recv_ids, recv_w, recv_src, partial = [], [], [], [], []
    for d in range(R):
        xr, ir, wr, sr = [], [], [], []
        for s in range(R):
            p = plans[s]
            lo, hi = p["send_offsets"][d], p["send_offsets"][d + 1]
            xr.append(xs[s][p["row_token"][lo:hi]])
            ir.append(p["row_ids"][lo:hi])
            wr.append(p["row_w"][lo:hi])
            sr.append(np.full(hi - lo, s, np.int32))
        xr = np.concatenate(xr) if xr else np.zeros((0, H), xs[0].dtype)
        ir, wr, sr = np.concatenate(ir), np.concatenate(wr), np.concatenate(sr)
        part = np.zeros((len(xr), H))
        for i in range(ir.shape[1]):  # choice i of every received row that has one
            sel = np.nonzero(ir[:, i] >= 0)[0]
            if len(sel):
                u = ffn_rows(xr[sel], ir[sel, i] + d * EL, w_gate, w_up, w_down, H, I)
                part[sel] += wr[sel, i].astype(np.float64)[:, None] * u
        recv_x.append(xr)
        recv_ids.append(ir)
        recv_w.append(wr)
        recv_src.append(sr)
        partial.append(part)
    ys = []
    for s in range(R):
        p = plans[s]
        T = xs[s].shape[0]
        ret = np.zeros((p["send_offsets"][R], H))
        for d in range(R):  # rows of source s at destination d come back in send order
            at = sum(plans[q]["send_counts"][d] for q in range(s))
            n = p["send_counts"][d]
            ret[p["send_offsets"][d]:p["send_offsets"][d] + n] = partial[d][at:at + n]
        y = np.zeros((T, H))
        ids = routes[s][0]
        for t in range(T):
            for d in range(R):
                rows = [p["slot_send_row"][t * k + j] for j in range(k)
                        if 0 <= ids[t, j] < E and ids[t, j] // EL == d]
                if rows:
                    y[t] += ret[rows[0]]
        ys.append(y)
    return dict(routes=routes, plans=plans, recv_x=recv_x, recv_ids=recv_ids, recv_w=recv_w, recv_src=recv_src,
                partial=partial, y=ys)


def round_trip(x: np.ndarray, logits: np.ndarray, k: int, E: int, R: int, w_gate, w_up, w_down):
    """The whole layer on the CPU: route -> dispatch -> FFN -> combine.  Returns a dict of every stage."""
    H = x.shape[1]
    I = w_gate.shape[-1] if isinstance(w_gate, np.ndarray) else next(iter(w_gate.values())).shape[-1]
    ids, w = route(logits, k)
    idx = dispatch_index(ids, E, R)
    x_disp = dispatch_rows(x, k, idx["slot_to_row"])
    S = ids.size
    row_expert = np.repeat(np.arange(E, dtype=np.int32), idx["expert_counts"])
    n = int(idx["expert_offsets"][-1])
    y_disp, act = ffn_rows(x_disp[:n], row_expert, w_gate, w_up, w_down, H, I, want_act=True)
    if n < S:
        y_disp = np.concatenate([y_disp, np.zeros((S - n, H))])
    y = combine(y_disp, w, idx["slot_to_row"])
    return dict(ids=ids, w=w, x_disp=x_disp, act=act, y_disp=y_disp, y=y, **idx)


def eplb_plan(load, R: int, slots: int) -> dict:
    """Expert placement with replicas from per-expert loads (oracle_eplb_plan):
    phys_to_logical [R*slots], replica_offsets [E+1], replicas [R*slots], and
    the per-rank sum of replica shares the plan expects (rank_load [R])."""
    load = _c(np.asarray(load), np.int64)
    E = load.shape[0]
    P = R * slots
    p2l = np.full(P, -1, np.int32)
    off = np.zeros(E + 1, np.int32)
    reps = np.full(P, -1, np.int32)
    st = _get().oracle_eplb_plan(load.ctypes.data, E, R, slots, p2l.ctypes.data, off.ctypes.data, reps.ctypes.data)
    if st != 0:
        raise ValueError("eplb_plan: need E, R, slots >= 1 and R * slots >= E")
    n = np.diff(off)
    rank_load = np.zeros(R, np.int64)
    for e in range(E):
        for j in range(n[e]):
            share = load[e] // n[e] + (1 if j < load[e] % n[e] else 0)
            rank_load[reps[off[e] + j] // slots] += share
    return {"phys_to_logical": p2l, "replica_offsets": off, "replicas": reps, "rank_load": rank_load}


def eplb_remap(ids: np.ndarray, E: int, replica_offsets: np.ndarray, replicas: np.ndarray) -> np.ndarray:
    """Logical expert ids [T, k] -> physical replica ids (oracle_eplb_remap)."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    out = np.empty_like(ids)
    _get().oracle_eplb_remap(ids.ctypes.data, T, k, E, _c(replica_offsets, np.int32).ctypes.data,
                             _c(replicas, np.int32).ctypes.data, out.ctypes.data)
    return out
