"""ep_round_trip_ranks' protocol between rank processes, on the CPU: gloo ranks
(world sizes 2 and 4) drive stand-in ranks that record what they are asked to
do.  Checks that every rank receives every source's send counts in rank
order, and that the phases are separated across ALL ranks: no rank packs into
a peer before every rank has set its counts, no rank runs its experts before
every rank has packed, and no rank sums its partials before every rank has
returned them (counters shared between the processes)."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PHASES = ("set_counts", "pack_to", "experts", "return_to")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _Plan:
    def __init__(self, counts):
        self.send_counts = torch.tensor(counts, dtype=torch.int32)


class _StandInRank:
    """The attributes and methods of MoEEPRank that ep_round_trip_ranks uses, recording calls."""

    def __init__(self, rank, R, done, errors):
        self.rank, self.R = rank, R
        self.device = torch.device("cpu")
        self.plan = _Plan([(rank + 1) * 10 + d for d in range(R)])  # distinct per (source, destination)
        self.done, self.errors = done, errors
        self.counts = None
        self.log = []

    def _enter(self, phase):
        i = PHASES.index(phase)
        if i > 0 and self.done[i - 1].value != self.R:  # every rank must have finished the previous phase
            with self.errors.get_lock():
                self.errors.value += 1
        self.log.append(phase)

    def _leave(self, phase):
        with self.done[PHASES.index(phase)].get_lock():
            self.done[PHASES.index(phase)].value += 1

    def route_and_plan(self, logits):
        self.log.append("route_and_plan")

    def set_counts(self, counts):
        self._enter("set_counts")
        self.counts = np.asarray(counts)
        self._leave("set_counts")

    def pack_to(self, x, peers):
        self._enter("pack_to")
        assert [p.rank for p in peers] == list(range(self.R))
        self._leave("pack_to")

    def experts(self, w_gate, w_up, w_down):
        self._enter("experts")
        self._leave("experts")

    def return_to(self, peers):
        self.log.append("return_to")  # (same phase as experts: no barrier between them)
        self._leave("return_to")

    def finish(self):
        if self.done[PHASES.index("return_to")].value != self.R:
            with self.errors.get_lock():
                self.errors.value += 1
        self.log.append("finish")
        return self.rank


def _worker(rank, R, port, done, errors, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from token_dispatch_combine_b200 import ep
    torch.cuda.synchronize = lambda *a, **k: None  # stand-in ranks launch no device work
    dist.init_process_group("gloo", rank=rank, world_size=R, timeout=datetime.timedelta(seconds=60))
    try:
        me = _StandInRank(rank, R, done, errors)
        peers = [me if d == rank else ep.EpPeer(d, None, None, None, None) for d in range(R)]
        out = ep.ep_round_trip_ranks(me, peers, None, None, None, None, None)
        q.put((rank, me.log, me.counts, out))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("R", [2, 4])
def test_round_trip_ranks_protocol_over_gloo(R):
    ctx = mp.get_context("spawn")
    done = [ctx.Value("i", 0) for _ in PHASES]
    errors = ctx.Value("i", 0)
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, R, port, done, errors, q)) for r in range(R)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(R):
            r, log, counts, out = q.get(timeout=120)
            res[r] = (log, counts, out)
        for p in procs:
            p.join(60)
    finally:
        for p in procs:
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0] * R
    assert errors.value == 0  # a phase started before every rank had finished the one before
    want = np.array([[(s + 1) * 10 + d for d in range(R)] for s in range(R)])
    for r in range(R):
        log, counts, out = res[r]
        assert log == ["route_and_plan", "set_counts", "pack_to", "experts", "return_to", "finish"]
        assert np.array_equal(counts, want)  # row s = source s's send counts
        assert out == r
