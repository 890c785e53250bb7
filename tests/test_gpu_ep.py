"""Expert-parallel exchange on the GPU: R ranks' kernels on one GPU (each rank's
buffers of its own, the exchange through device memory), against the oracle.

- moe_ep_plan (device) equals the oracle's plan and the library's host plan,
  element for element, bad ids included.
- The round trip of R ranks (ep_round_trip_one_gpu): every destination's
  received rows and local expert ids equal the oracle's exchange bit for bit,
  their weights within the routing tolerance (1e-6); every rank's output matches the oracle's exchange and the
  one-GPU round trip of the concatenated tokens within the layer's normwise
  bound (per tensor and per row).
- The GPT-OSS layer spread over 8 ranks of 512 tokens, in full.
- A destination buffer too small: its extra rows are skipped and flagged."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_layer import TOL, DeviceLayer, dev_to_np, row_errors

pytestmark = pytest.mark.gpu


def _routing(T, E, k, seed, hot=0.0, R=1):
    rng = np.random.default_rng(seed)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[:, :E // R] += hot
    return oracle.route(lg, k)


@pytest.mark.parametrize("T,E,k,R,hot", [(3000, 32, 4, 8, 0.0), (2500, 256, 8, 32, 0.7), (64, 8, 1, 2, 0.0),
                                         (5000, 64, 8, 64, 0.0), (1, 4, 2, 2, 0.0), (2048, 16, 6, 4, 2.0)])
def test_device_plan_matches_oracle(T, E, k, R, hot):
    from token_dispatch_combine_b200 import moe_ep_plan, moe_ep_plan_host, moe_get_error
    ids, w = _routing(T, E, k, T * 3 + E, hot, R)
    plan = moe_ep_plan(torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), E, R)
    assert moe_get_error() == (0, 0)
    ref = oracle.ep_plan(ids, w, E, R)
    host = moe_ep_plan_host(ids, w, E, R)
    n = int(ref["send_offsets"][-1])
    got = {key: dev_to_np(getattr(plan, key)) for key in ("send_counts", "send_offsets", "slot_send_row", "ret_row",
                                                          "row_token", "row_ids", "row_w")}
    for key in ("send_counts", "send_offsets", "slot_send_row"):
        assert np.array_equal(got[key][:len(ref[key])], ref[key]), key
    for key in ("row_token", "row_ids", "row_w"):
        assert np.array_equal(got[key][:n], ref[key]), key
    assert np.array_equal(got["ret_row"][:T * k], host["ret_row"])


def test_device_plan_flags_bad_ids():
    from token_dispatch_combine_b200 import _native, moe_ep_plan, moe_get_error
    ids, w = _routing(500, 16, 4, 9, R=4)
    ids[10, 2] = 16
    ids[77, 0] = -5
    plan = moe_ep_plan(torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), 16, 4)
    st, bits = moe_get_error()
    assert st == _native.MOE_ERR_DEVICE and bits & _native.ERR_BAD_ID
    ref = oracle.ep_plan(ids, w, 16, 4)
    n = int(ref["send_offsets"][-1])
    assert np.array_equal(dev_to_np(plan.slot_send_row)[:500 * 4], ref["slot_send_row"])
    assert np.array_equal(dev_to_np(plan.row_ids)[:n], ref["row_ids"])


def _ranks(sizes, wl, dtype):
    from token_dispatch_combine_b200 import MoEEPRank
    R = len(sizes)
    return [MoEEPRank(r, R, sizes[r], wl.H, wl.I, wl.E, wl.k, dtype, recv_capacity=sum(sizes)) for r in range(R)]


def _split(layer, sizes):
    start = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
    xs = [layer.x_dev[start[r]:start[r + 1]].contiguous() for r in range(len(sizes))]
    lg = [layer.logits_dev[start[r]:start[r + 1]].contiguous() for r in range(len(sizes))]
    return start, xs, lg


@pytest.mark.parametrize("name,sizes", [
    ("bf16", (200, 0, 150, 300)),
    ("f32", (60, 41)),
    ("bf16_e256", (96, 96, 31, 1, 64, 0, 12, 100)),
    ("bf16_el2", (100, 50, 0, 80)),  # 2 experts per rank, top-4: rows carry at most 2 of 4 id columns
])
def test_round_trip_of_ranks_on_one_gpu(name, sizes):
    from token_dispatch_combine_b200 import ep_round_trip_one_gpu, moe_get_error
    W = synth.Workload
    T = sum(sizes)
    R = len(sizes)
    wl = {"bf16": W("ep_bf16", T=T, H=256, I=384, E=16, k=4, R=R, dtype="bf16", seed=41, bias="zipf1.2"),
          "f32": W("ep_f32", T=T, H=96, I=160, E=8, k=3, R=R, dtype="f32", seed=42),
          "bf16_e256": W("ep_e256", T=T, H=128, I=128, E=256, k=8, R=R, dtype="bf16", seed=43, bias="normal0.5"),
          "bf16_el2": W("ep_el2", T=T, H=128, I=192, E=8, k=4, R=R, dtype="bf16", seed=44)}[name]
    layer = DeviceLayer(wl)
    start, xs, lg = _split(layer, sizes)
    ranks = _ranks(sizes, wl, layer.x_dev.dtype)
    ys = ep_round_trip_one_gpu(ranks, xs, lg, layer.w_gate, layer.w_up, layer.w_down)
    assert moe_get_error() == (0, 0)
    g, u, d = layer.host_weights(range(wl.E))
    xh = [layer.x[start[r]:start[r + 1]] for r in range(R)]
    lh = [layer.logits[start[r]:start[r + 1]] for r in range(R)]
    ep = oracle.ep_round_trip(xh, lh, wl.k, wl.E, R, g, u, d)
    one = oracle.round_trip(layer.x, layer.logits, wl.k, wl.E, R, g, u, d)
    tol = TOL[wl.dtype]
    for r, rank in enumerate(ranks):
        n = rank.n_recv
        assert n == len(ep["recv_x"][r])
        assert np.array_equal(dev_to_np(rank.x_recv[:n]), ep["recv_x"][r]), r
        assert np.array_equal(dev_to_np(rank.recv_ids[:n]), ep["recv_ids"][r]), r
        # the weights are the GPU router's softmax: within 1e-6 of the oracle's (ids are exact)
        np.testing.assert_allclose(dev_to_np(rank.recv_w[:n]), ep["recv_w"][r], rtol=0, atol=1e-6)
        if sizes[r] == 0:
            continue
        y = dev_to_np(ys[r])
        whole, worst, _ = row_errors(y, ep["y"][r])
        assert whole <= tol and worst <= tol, (r, whole, worst)
        whole, worst, _ = row_errors(y, one["y"][start[r]:start[r + 1]])
        assert whole <= tol and worst <= tol, (r, whole, worst)


def test_gptoss_layer_over_eight_ranks():
    """The GPT-OSS layer (4096 tokens, E = 32, top-4) as 8 ranks of 512 tokens with 4 experts
    each; every token's output against the oracle's one-GPU round trip, in full."""
    from token_dispatch_combine_b200 import ep_round_trip_one_gpu, moe_get_error
    wl = synth.WORKLOADS["gptoss_uniform"]
    layer = DeviceLayer(wl)
    sizes = [wl.T // 8] * 8
    start, xs, lg = _split(layer, sizes)
    ranks = _ranks(sizes, wl, torch.bfloat16)
    ys = ep_round_trip_one_gpu(ranks, xs, lg, layer.w_gate, layer.w_up, layer.w_down)
    assert moe_get_error() == (0, 0)
    y = torch.cat(ys).contiguous()
    from tests.test_gpu_parity import _EXPECTED, _expected
    ids, w = oracle.route(layer.logits, wl.k)
    ref = oracle.dispatch_index(ids, wl.E, wl.R)
    exp = _EXPECTED.get("gptoss_uniform") or _expected("gptoss_uniform", layer, w, ref)
    whole, worst, at = row_errors(dev_to_np(y), exp["y"])
    print(f"EP over 8 ranks: normwise {whole:.3e}, worst row {worst:.3e} (token {at})")
    assert whole <= TOL["bf16"] and worst <= TOL["bf16"]
    # shared delivery: rows sent = distinct (token, destination) pairs, fewer than the slots
    sent = sum(int(r.plan.send_offsets[-1]) for r in ranks)
    pairs = len({(t, int(e) // 4) for t in range(wl.T) for e in ids[t]})
    assert sent == pairs < wl.S


def test_pack_flags_rows_beyond_capacity():
    from token_dispatch_combine_b200 import _native, moe_ep_pack, moe_ep_plan, moe_get_error
    T, E, k, R, H = 300, 8, 2, 2, 64
    ids, w = _routing(T, E, k, 5, R=R)
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    plan = moe_ep_plan(torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), E, R)
    ref = oracle.ep_plan(ids, w, E, R)
    cap = int(ref["send_counts"][1]) - 7  # destination 1's buffer 7 rows short
    dst_x = [torch.zeros(int(ref["send_counts"][0]), H, dtype=torch.bfloat16, device="cuda"),
             torch.zeros(cap, H, dtype=torch.bfloat16, device="cuda")]
    dst_i = [torch.full((t.shape[0], k), -9, dtype=torch.int32, device="cuda") for t in dst_x]
    dst_w = [torch.zeros((t.shape[0], k), device="cuda") for t in dst_x]
    base = torch.zeros(R, dtype=torch.int32, device="cuda")  # each destination's buffer starts at its row 0
    moe_ep_pack(x, plan, base, dst_x, dst_i, dst_w)
    st, bits = moe_get_error()
    assert st == _native.MOE_ERR_DEVICE and bits & _native.ERR_BAD_ROW
    # rows within capacity arrived: destination 0 in full, destination 1 up to its capacity
    xh = dev_to_np(x)
    for d, n in ((0, int(ref["send_counts"][0])), (1, cap)):
        lo = int(ref["send_offsets"][d])
        assert np.array_equal(dev_to_np(dst_x[d]), xh[ref["row_token"][lo:lo + n]]), d
        assert np.array_equal(dev_to_np(dst_i[d]), ref["row_ids"][lo:lo + n]), d
    # a single staging buffer for every destination: base = the send offsets, rows in send order
    n_all = int(ref["send_offsets"][-1])
    stage = torch.zeros(n_all, H, dtype=torch.bfloat16, device="cuda")
    st_i = torch.zeros((n_all, k), dtype=torch.int32, device="cuda")
    st_w = torch.zeros((n_all, k), device="cuda")
    moe_ep_pack(x, plan, plan.send_offsets[:R].contiguous(), [stage] * R, [st_i] * R, [st_w] * R)
    assert moe_get_error() == (0, 0)
    assert np.array_equal(dev_to_np(stage), xh[ref["row_token"]])
    assert np.array_equal(dev_to_np(st_w), ref["row_w"])
