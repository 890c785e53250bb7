"""The expert-parallel exchange's host functions (moe_ep_plan_host,
moe_ep_exchange_offsets) against the oracle, and the whole exchange protocol
between ranks driven through torch.distributed with gloo on CPU (world sizes
2 and 4).

In the gloo test each process is one rank: it routes its own tokens (the
oracle's route: input preparation), plans its sends with the library's host
plan, learns every source's send counts by all_gather, takes its offsets from
the library, and moves its rows and their (local expert id, weight) lists with
all_to_all_single in the order the plan gives.  The receiver's expert outputs
come from the oracle's FFN (no GPU here); its per-row partials return by a
second all_to_all_single, and the source sums them through the plan's ret_row.
Received buffers and outputs are compared with the oracle's exchange
(oracle.ep_round_trip) and with the one-GPU round trip (oracle.round_trip)."""
import datetime
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
from token_dispatch_combine_b200 import _native, moe_ep_exchange_offsets, moe_ep_plan_host

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _routing(T, E, k, seed, hot=0.0, R=1):
    rng = np.random.default_rng(seed)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[:, :E // R] += hot
    return oracle.route(lg, k)


@pytest.mark.parametrize("T,E,k,R,hot", [(300, 16, 4, 4, 0.0), (257, 32, 8, 8, 1.0), (64, 8, 1, 2, 0.0),
                                         (1000, 256, 8, 32, 0.5), (50, 6, 6, 3, 0.0), (40, 4, 2, 1, 0.0),
                                         (0, 8, 2, 2, 0.0), (2500, 64, 8, 64, 0.0), (500, 8, 4, 4, 0.0)])
def test_host_plan_matches_oracle(T, E, k, R, hot):
    ids, w = _routing(T, E, k, T + E, hot, R)
    got = moe_ep_plan_host(ids, w, E, R)
    ref = oracle.ep_plan(ids, w, E, R)
    for key in ("send_counts", "send_offsets", "slot_send_row", "row_token", "row_ids"):
        assert np.array_equal(got[key], ref[key]), key
    assert np.array_equal(got["row_w"], ref["row_w"])  # copies of the weights, bit for bit
    # ret_row: the slot's row for its first choice on that destination, -1 for later ones
    EL = E // R
    want = np.full(T * k, -1, np.int32)
    for t in range(T):
        seen = set()
        for j in range(k):
            d = int(ids[t, j]) // EL
            if d not in seen:
                seen.add(d)
                want[t * k + j] = ref["slot_send_row"][t * k + j]
    assert np.array_equal(got["ret_row"], want)


def test_host_plan_drops_bad_ids():
    ids, w = _routing(20, 8, 2, 3)
    ids[3, 1] = 8
    ids[7, 0] = -2
    with pytest.raises(_native.MoeError) as e:
        moe_ep_plan_host(ids, w, 8, 4)
    assert e.value.status == _native.MOE_ERR_DEVICE
    ref = oracle.ep_plan(ids, w, 8, 4)
    assert ref["slot_send_row"][3 * 2 + 1] == -1 and ref["slot_send_row"][7 * 2] == -1


def test_exchange_offsets_hand_example():
    # 3 ranks; counts[s][d] = rows source s sends to destination d
    counts = np.array([[2, 0, 5],
                       [1, 3, 0],
                       [4, 1, 1]], np.int32)
    dst_base, recv_base, ret_base = moe_ep_exchange_offsets(counts, 1)
    assert dst_base.tolist() == [2, 0, 5]        # rank 1's rows land after rank 0's at each destination
    assert recv_base.tolist() == [0, 0, 3, 4]    # rank 1 receives 0 from s0, 3 from s1, 1 from s2
    assert ret_base.tolist() == [2, 1, 4]        # its partials go after each source's rows for rank 0
    dst_base, recv_base, ret_base = moe_ep_exchange_offsets(counts, 0)
    assert dst_base.tolist() == [0, 0, 0] and recv_base.tolist() == [0, 2, 3, 7] and ret_base.tolist() == [0, 0, 0]


@pytest.mark.parametrize("kw,needle", [(dict(R=65), b"[1, 64]"), (dict(rank=3), b"rank"), (dict(neg=True), b">= 0")])
def test_exchange_offsets_rejects(kw, needle):
    R = kw.get("R", 3)
    c = np.ones((R, R), np.int32)
    if kw.get("neg"):
        c[1, 2] = -1
    out = [np.empty(R + 1, np.int32) for _ in range(3)]
    st = _native.lib().moe_ep_exchange_offsets(c.ctypes.data, R, kw.get("rank", 0), *(o.ctypes.data for o in out))
    assert st == _native.MOE_ERR_INVALID_ARG
    assert needle in _native.lib().moe_last_error_message()


# --------------------------------------------------------------------------- gloo ranks
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(world):
    """Layer of the gloo test: per-rank token counts, shapes, seeded inputs (the same in every process)."""
    sizes = [37, 0, 53, 21][:world] if world == 4 else [41, 29]
    H, I, k = 16, 24, 3
    E = 4 * world
    rng = np.random.default_rng(100 + world)
    xs = [rng.standard_normal((T, H)).astype(np.float32) for T in sizes]
    lg = [rng.standard_normal((T, E)).astype(np.float32) for T in sizes]
    for a in lg:
        a[:, :4] += 1.0  # rank 0's experts popular: shared deliveries there
    wg = (rng.standard_normal((E, H, I)) / math.sqrt(H)).astype(np.float32)
    wu = (rng.standard_normal((E, H, I)) / math.sqrt(H)).astype(np.float32)
    wd = (rng.standard_normal((E, I, H)) / math.sqrt(I)).astype(np.float32)
    return sizes, H, I, E, k, xs, lg, wg, wu, wd


def _ep_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle as orc
    from token_dispatch_combine_b200 import moe_ep_exchange_offsets as offsets
    from token_dispatch_combine_b200 import moe_ep_plan_host as plan_host
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sizes, H, I, E, k, xs, lg, wg, wu, wd = _case(world)
        R, EL = world, E // world
        x = xs[rank]
        ids, w = orc.route(lg[rank], k)
        p = plan_host(ids, w, E, R)
        # counts exchange: every rank learns every source's send counts
        mine = torch.from_numpy(p["send_counts"].astype(np.int64))
        gathered = [torch.empty(R, dtype=torch.int64) for _ in range(R)]
        dist.all_gather(gathered, mine)
        counts = torch.stack(gathered).numpy().astype(np.int32)
        dst_base, recv_base, ret_base = offsets(counts, rank)
        n_recv = int(recv_base[-1])
        # rows (and their local ids / weights) in send order, one block per destination
        send_x = torch.from_numpy(x[p["row_token"]] if len(p["row_token"]) else np.zeros((0, H), np.float32))
        send_meta = torch.from_numpy(np.concatenate([p["row_ids"].astype(np.float32), p["row_w"]], axis=1)
                                     if len(p["row_token"]) else np.zeros((0, 2 * k), np.float32))
        splits_out = p["send_counts"].tolist()
        splits_in = counts[:, rank].tolist()
        recv_x = torch.empty((n_recv, H))
        recv_meta = torch.empty((n_recv, 2 * k))
        dist.all_to_all_single(recv_x, send_x, splits_in, splits_out)
        dist.all_to_all_single(recv_meta, send_meta, splits_in, splits_out)
        rx = recv_x.numpy()
        rid = recv_meta[:, :k].numpy().astype(np.int32)
        rw = recv_meta[:, k:].numpy()
        # the destination's experts (oracle FFN: no GPU here) and its per-row partials
        part = np.zeros((n_recv, H))
        for i in range(k):
            sel = np.nonzero(rid[:, i] >= 0)[0]
            if len(sel):
                u = orc.ffn_rows(rx[sel], rid[sel, i] + rank * EL, wg, wu, wd, H, I)
                part[sel] += rw[sel, i].astype(np.float64)[:, None] * u
        # partials return to their sources, landing in send order
        back = torch.empty((int(p["send_offsets"][-1]), H), dtype=torch.float64)
        dist.all_to_all_single(back, torch.from_numpy(part), splits_out, splits_in)
        y = np.zeros((x.shape[0], H))
        rr = p["ret_row"].reshape(-1, k) if x.shape[0] else np.zeros((0, k), np.int32)
        for t in range(x.shape[0]):
            for j in range(k):
                if rr[t, j] >= 0:
                    y[t] += back.numpy()[rr[t, j]]
        q.put((rank, dict(recv_x=rx, recv_ids=rid, recv_w=rw, n_recv=n_recv, y=y, ret_base=ret_base.tolist(),
                          dst_base=dst_base.tolist())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_exchange_protocol_over_gloo_ranks(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    sizes, H, I, E, k, xs, lg, wg, wu, wd = _case(world)
    ep = oracle.ep_round_trip(xs, lg, k, E, world, wg, wu, wd)
    one = oracle.round_trip(np.concatenate(xs), np.concatenate(lg), k, E, world, wg, wu, wd)
    start = np.concatenate([[0], np.cumsum(sizes)])
    for r in range(world):
        got = res[r]
        assert np.array_equal(got["recv_x"], ep["recv_x"][r]), r
        assert np.array_equal(got["recv_ids"], ep["recv_ids"][r]), r
        assert np.array_equal(got["recv_w"], ep["recv_w"][r]), r
        np.testing.assert_allclose(got["y"], ep["y"][r], rtol=0, atol=1e-12)
        np.testing.assert_allclose(got["y"], one["y"][start[r]:start[r + 1]], rtol=0, atol=1e-10)
