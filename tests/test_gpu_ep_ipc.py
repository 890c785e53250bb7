"""Expert-parallel exchange with one process per rank: every rank's receive and
return buffers mapped into the other ranks' processes through CUDA IPC
(ep_share_buffers), the pack kernel storing rows straight into the peers'
memory and the partials returning by peer copies, the counts through
torch.distributed (gloo) and host barriers between the phases
(ep_round_trip_ranks).

Here every process runs on the one GPU the test has; no kernel waits on
another process's kernel (the barriers are on the host, after each rank's
kernels have finished), so the ranks need not run at the same time.

Checks, for two consecutive steps on the same buffers: each rank's received
rows and local ids and its output equal, bit for bit, those of the same ranks
emulated in one process (ep_round_trip_one_gpu), and the outputs match the
oracle's exchange within the layer's normwise bound (per tensor and per row)."""
import datetime
import gc
import os
import queue
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth
from tests.gpu_layer import TOL, DeviceLayer, dev_to_np, row_errors

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STEPS = 2


def _workload(name, sizes):
    if name == "e256":  # DeepSeek-R1-like routing: 256 experts, top-8, 8 ranks of 32 experts
        return synth.Workload("ep_ipc_e256", T=sum(sizes), H=128, I=128, E=256, k=8, R=len(sizes), dtype="bf16",
                              seed=47, bias="normal0.5")
    return synth.Workload("ep_ipc", T=sum(sizes), H=256, I=384, E=16, k=4, R=len(sizes), dtype="bf16", seed=46,
                          bias="zipf1.2")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _require_shared_gpu():
    """Several processes on one GPU need the default compute mode."""
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            mode = pynvml.nvmlDeviceGetComputeMode(pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device()))
        finally:
            pynvml.nvmlShutdown()
    except Exception:  # no NVML: let the processes try
        return
    if mode != pynvml.NVML_COMPUTEMODE_DEFAULT:
        pytest.skip(f"GPU compute mode {mode}: one process per GPU only")


def _rank_worker(rank, name, sizes, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from tests.gpu_layer import DeviceLayer as Layer
    from tests.gpu_layer import dev_to_np as to_np
    from token_dispatch_combine_b200 import MoEEPRank, ep_round_trip_ranks, ep_share_buffers, moe_get_error
    R = len(sizes)
    dist.init_process_group("gloo", rank=rank, world_size=R, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        wl = _workload(name, sizes)
        layer = Layer(wl)
        start = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
        x = layer.x_dev[start[rank]:start[rank + 1]].contiguous()
        lg = layer.logits_dev[start[rank]:start[rank + 1]].contiguous()
        me = MoEEPRank(rank, R, sizes[rank], wl.H, wl.I, wl.E, wl.k, x.dtype, recv_capacity=sum(sizes))
        peers = ep_share_buffers(me)
        lo, hi = rank * me.EL, (rank + 1) * me.EL
        ys = []
        for _ in range(STEPS):
            y = ep_round_trip_ranks(me, peers, x, lg, layer.w_gate[lo:hi], layer.w_up[lo:hi], layer.w_down[lo:hi])
            ys.append(to_np(y))
        n = me.n_recv
        q.put((rank, dict(y=ys, n=n, x_recv=to_np(me.x_recv[:n]), recv_ids=to_np(me.recv_ids[:n]),
                          err=moe_get_error())))
        del peers  # drop the mappings of the other ranks' buffers before their owners free them
        gc.collect()
        torch.cuda.synchronize()
        dist.barrier()
        del me
        torch.cuda.ipc_collect()
    finally:
        dist.destroy_process_group()


def _run_ranks(name, sizes):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_worker, args=(r, name, sizes, port, q)) for r in range(len(sizes))]
    for p in procs:
        p.start()
    res = {}
    try:
        deadline = 600
        while len(res) < len(sizes) and deadline > 0:
            try:
                r, out = q.get(timeout=5)
                res[r] = out
            except queue.Empty:
                deadline -= 5
                if any(p.exitcode not in (None, 0) for p in procs):
                    break
        for p in procs:
            p.join(120)
    finally:
        for p in procs:
            if p.is_alive():
                p.kill()
    codes = [p.exitcode for p in procs]
    assert codes == [0] * len(sizes) and len(res) == len(sizes), (codes, sorted(res))
    return res


@pytest.mark.parametrize("name,sizes", [("e16", (120, 77)), ("e16", (200, 0, 150, 300)),
                                        ("e256", (96, 96, 31, 1, 64, 0, 12, 100))])
def test_ranks_as_processes_exchange_through_ipc(name, sizes):
    _require_shared_gpu()
    from token_dispatch_combine_b200 import MoEEPRank, ep_round_trip_one_gpu, moe_get_error
    res = _run_ranks(name, sizes)
    R = len(sizes)
    wl = _workload(name, sizes)
    layer = DeviceLayer(wl)
    start = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
    xs = [layer.x_dev[start[r]:start[r + 1]].contiguous() for r in range(R)]
    lg = [layer.logits_dev[start[r]:start[r + 1]].contiguous() for r in range(R)]
    ranks = [MoEEPRank(r, R, sizes[r], wl.H, wl.I, wl.E, wl.k, layer.x_dev.dtype, recv_capacity=sum(sizes))
             for r in range(R)]
    ys = ep_round_trip_one_gpu(ranks, xs, lg, layer.w_gate, layer.w_up, layer.w_down)
    assert moe_get_error() == (0, 0)
    g, u, d = layer.host_weights(range(wl.E))
    ep = oracle.ep_round_trip([layer.x[start[r]:start[r + 1]] for r in range(R)],
                              [layer.logits[start[r]:start[r + 1]] for r in range(R)], wl.k, wl.E, R, g, u, d)
    for r in range(R):
        got = res[r]
        assert got["err"] == (0, 0), r
        n = ranks[r].n_recv
        assert got["n"] == n
        assert np.array_equal(got["x_recv"], dev_to_np(ranks[r].x_recv[:n])), r
        assert np.array_equal(got["recv_ids"], dev_to_np(ranks[r].recv_ids[:n])), r
        y_one = dev_to_np(ys[r])
        for step in range(STEPS):
            assert np.array_equal(got["y"][step], y_one), (r, step)
        if sizes[r]:
            whole, worst, _ = row_errors(got["y"][0], ep["y"][r])
            assert whole <= TOL["bf16"] and worst <= TOL["bf16"], (r, whole, worst)


def test_enable_peer_access_on_one_gpu():
    from token_dispatch_combine_b200 import _native, moe_enable_peer_access
    moe_enable_peer_access(torch.cuda.current_device())  # the device itself: nothing to enable
    assert _native.lib().moe_enable_peer_access(torch.cuda.device_count()) == _native.MOE_ERR_INVALID_ARG
