"""Dispatch fused into the gate/up projection (moe_ffn_gate_up_gather).

The gathering kernels read each dispatched row's A operand straight from x
(token row_to_slot[r] / k) instead of from x_disp, and dispatch runs
index-only.  They form the same products in the same order, so the check is
exact: index-only dispatch gives the same counts, offsets and permutation
as the full dispatch, and h, y_disp and y equal the unfused round trip's bit
for bit, under both tile shapes.  The fused round trip is also checked
against the CPU oracle directly."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_layer import TOL, DeviceLayer, dev_to_np, expert_of_rows, rel_err

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = {
    "toy_fp32": synth.WORKLOADS["toy_fp32"],
    "f32_top4": W("f32_top4", T=100, H=96, I=160, E=8, k=4, R=2, dtype="f32", seed=15),
    "bf16_multi_tile": W("bf16_multi_tile", T=512, H=256, I=384, E=8, k=2, R=4, dtype="bf16", seed=11,
                         bias="zipf1.2"),
    # K tails (H = 200), odd T, k = 3
    "bf16_ragged": W("bf16_ragged", T=333, H=200, I=200, E=6, k=3, R=3, dtype="bf16", seed=12, bias="normal0.5"),
    "bf16_one_token": W("bf16_one_token", T=1, H=64, I=64, E=4, k=1, R=2, dtype="bf16", seed=14),
    "bf16_top8_e256": W("bf16_top8_e256", T=96, H=128, I=128, E=256, k=8, R=32, dtype="bf16", seed=16),
    # the largest expert count: 1024-expert tile prefix in shared memory (gathered by default)
    "bf16_e1024": W("bf16_e1024", T=2048, H=128, I=192, E=1024, k=8, R=8, dtype="bf16", seed=21),
    # ~512 rows per expert: full pair tiles, M=128 pair tails and single M=64 tails
    "bf16_pair_sized": W("bf16_pair_sized", T=2048, H=256, I=256, E=8, k=2, R=2, dtype="bf16", seed=22),
}
INDEX_OUTPUTS = ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row", "row_to_slot",
                 "src_expert_counts")


def run_pair(layer):
    """The unfused and the fused round trip on the same layer."""
    from token_dispatch_combine_b200 import MoERoundTrip, moe_get_error
    wl = layer.wl
    out = []
    for gather in (False, True):
        rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, layer.x_dev.dtype, gather=gather)
        rt.forward(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down)
        st, bits = moe_get_error()
        assert st == 0 and bits == 0, (gather, st, bits)
        out.append(rt)
    return out


def assert_same_round_trip(ref, rt):
    assert rt.disp.x_disp is None
    for name in INDEX_OUTPUTS:
        assert torch.equal(getattr(rt.disp, name), getattr(ref.disp, name)), name
    n = int(ref.disp.expert_offsets[-1])
    assert torch.equal(rt.h[:n], ref.h[:n])
    assert torch.equal(rt.y_disp[:n], ref.y_disp[:n])
    assert torch.equal(rt.y, ref.y)
    return n


@pytest.mark.parametrize("ffn_tiling", ["single", "pair"], indirect=True)
@pytest.mark.parametrize("name", sorted(CASES))
def test_gather_matches_unfused_and_oracle(name, ffn_tiling):
    wl = CASES[name]
    layer = DeviceLayer(wl)
    ref, rt = run_pair(layer)
    n = assert_same_round_trip(ref, rt)
    # the fused round trip against the oracle, element by element
    ids, w = oracle.route(layer.logits, wl.k)
    idx = oracle.dispatch_index(ids, wl.E, wl.R)
    for name_ in INDEX_OUTPUTS:
        assert (dev_to_np(getattr(rt.disp, name_)) == idx[name_]).all(), name_
    x_disp = oracle.dispatch_rows(layer.x, wl.k, idx["slot_to_row"])
    row_expert = expert_of_rows(idx["expert_offsets"], np.arange(n))
    g, u, d = layer.host_weights(range(wl.E))
    y_rows, a_rows = oracle.ffn_rows(x_disp[:n], row_expert, g, u, d, wl.H, wl.I, want_act=True)
    tol = TOL[wl.dtype]
    assert rel_err(dev_to_np(rt.h)[:n], a_rows) <= tol
    assert rel_err(dev_to_np(rt.y), oracle.combine(y_rows, w, idx["slot_to_row"])) <= tol


@pytest.mark.parametrize("name", ["gptoss_uniform", "gptoss_zipf", "dsr1_decode"])
def test_gather_full_size_bit_identical(name):
    """Full-size layers, the tile shape auto picks: fused and unfused agree bit for bit."""
    layer = DeviceLayer(synth.WORKLOADS[name])
    ref, rt = run_pair(layer)
    assert_same_round_trip(ref, rt)


@pytest.mark.parametrize("ffn_tiling", ["single", "pair"], indirect=True)
@pytest.mark.parametrize("name", ["bf16_multi_tile", "f32_top4"])
def test_gather_bad_slot_is_flagged(name, ffn_tiling):
    """A row_to_slot entry outside [0, T*k) is flagged (bit 4) and read as token 0; nothing faults."""
    from token_dispatch_combine_b200 import moe_ffn_gate_up_gather, moe_get_error
    from token_dispatch_combine_b200._native import ERR_BAD_ROW, MOE_ERR_DEVICE
    wl = CASES[name]
    layer = DeviceLayer(wl)
    ref, rt = run_pair(layer)
    n = int(ref.disp.expert_offsets[-1])
    for bad in (-5, -1, wl.T * wl.k + 3):  # -1 included: it must not pass for "no row"
        rts = rt.disp.row_to_slot.clone()
        rts[0] = bad
        rts[1] = wl.T * wl.k + 3
        h = torch.zeros_like(rt.h)
        moe_ffn_gate_up_gather(layer.x_dev, rts, wl.k, layer.w_gate, layer.w_up, rt.disp.expert_offsets, h)
        st, bits = moe_get_error()
        assert st == MOE_ERR_DEVICE and bits & ERR_BAD_ROW, bad
        assert torch.equal(h[2:n], ref.h[2:n])  # every other row is unaffected
    assert moe_get_error() == (0, 0)  # the word was cleared


def test_gather_graph_replay_matches_forward():
    from token_dispatch_combine_b200 import MoERoundTrip
    wl = CASES["bf16_pair_sized"]
    layer = DeviceLayer(wl)
    rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, torch.bfloat16, gather=True)
    rt.forward(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down)
    y0 = rt.y.clone()
    rt.y.zero_()
    g = rt.capture(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(rt.y, y0)
    del g
