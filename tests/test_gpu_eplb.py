"""Expert placement with replicas on the GPU.

moe_eplb_remap is integer work: equal to the oracle's remap element for
element.  The round trip over the physical experts of a plan must give the
same outputs as the plain round trip bit for bit (a replica has its expert's
weights and every row's arithmetic is unchanged), and its per-rank row counts
must be the oracle's dispatch of the remapped ids."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_layer import DeviceLayer, dev_to_np

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = {
    # (layer, slots per rank)
    "bf16_zipf": (W("bf16_zipf", T=512, H=256, I=256, E=16, k=2, R=4, dtype="bf16", seed=31, bias="zipf1.2"), 5),
    "bf16_top8": (W("bf16_top8", T=200, H=128, I=192, E=64, k=8, R=8, dtype="bf16", seed=32, bias="normal0.5"), 10),
    "f32_zipf": (W("f32_zipf", T=100, H=96, I=160, E=8, k=2, R=2, dtype="f32", seed=33, bias="zipf1.2"), 6),
    "bf16_pairs": (W("bf16_pairs", T=2048, H=256, I=256, E=8, k=2, R=2, dtype="bf16", seed=34, bias="zipf1.2"), 5),
}


def plain_and_balanced(layer, slots, load=None):
    from token_dispatch_combine_b200 import MoEBalancedRoundTrip, MoERoundTrip, moe_eplb_plan, moe_get_error
    wl = layer.wl
    dt = layer.x_dev.dtype
    plain = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, dt)
    y0 = plain.forward(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down).clone()
    if load is None:
        load = dev_to_np(plain.disp.expert_counts)
    plan = moe_eplb_plan(load, wl.R, slots)
    bal = MoEBalancedRoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, slots, dt)
    bal.set_plan(plan, layer.w_gate, layer.w_up, layer.w_down)
    y1 = bal.forward(layer.x_dev, layer.logits_dev)
    st, bits = moe_get_error()
    assert st == 0 and bits == 0, (st, bits)
    return plain, y0, bal, y1, plan, load


@pytest.mark.parametrize("name", sorted(CASES))
def test_balanced_round_trip_equals_plain_and_oracle_counts(name):
    wl, slots = CASES[name]
    layer = DeviceLayer(wl)
    plain, y0, bal, y1, plan, load = plain_and_balanced(layer, slots)
    assert torch.equal(y1, y0)
    # the remap and the physical dispatch against the oracle
    ids, _ = oracle.route(layer.logits, wl.k)
    ref_plan = oracle.eplb_plan(load, wl.R, slots)
    assert plan.replicas.tolist() == ref_plan["replicas"].tolist()
    phys = oracle.eplb_remap(ids, wl.E, ref_plan["replica_offsets"], ref_plan["replicas"])
    assert (dev_to_np(bal.rt.topk_ids) == phys).all()
    idx = oracle.dispatch_index(phys, bal.P, wl.R)
    for key in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row", "row_to_slot"):
        assert (dev_to_np(getattr(bal.rt.disp, key)) == idx[key]).all(), key
    # balance: the busiest rank carries no more rows than under the static layout
    assert dev_to_np(bal.rt.disp.rank_counts).max() <= dev_to_np(plain.disp.rank_counts).max()


def test_balanced_full_size_zipf_layer():
    """GPT-OSS-shaped layer with Zipf routing, planned on its own expert counts with one spare slot per
    rank: same output bit for bit, and the busiest rank falls from several times the mean to near it."""
    wl = synth.WORKLOADS["gptoss_zipf"]
    layer = DeviceLayer(wl)
    plain, y0, bal, y1, plan, load = plain_and_balanced(layer, 5)
    assert torch.equal(y1, y0)
    before = dev_to_np(plain.disp.rank_counts)
    after = dev_to_np(bal.rt.disp.rank_counts)
    assert before.max() / before.mean() > 3.0
    assert after.max() / after.mean() < 1.15
    assert after.sum() == before.sum() == wl.S


def test_remap_matches_oracle_and_flags_bad_ids():
    from token_dispatch_combine_b200 import moe_eplb_plan, moe_eplb_remap, moe_get_error
    from token_dispatch_combine_b200._native import ERR_BAD_ID, MOE_ERR_DEVICE
    rng = np.random.default_rng(5)
    E, R, slots, T, k = 24, 4, 9, 1000, 6
    plan = moe_eplb_plan(rng.integers(0, 900, E), R, slots)
    ids = rng.integers(0, E, (T, k)).astype(np.int32)
    out = moe_eplb_remap(torch.from_numpy(ids).cuda(), plan)
    ref = oracle.eplb_remap(ids, E, plan.replica_offsets, plan.replicas)
    assert moe_get_error() == (0, 0)
    assert (dev_to_np(out) == ref).all()
    ids[3, 2], ids[500, 0], ids[999, 5] = -1, E, 1 << 30
    out = moe_eplb_remap(torch.from_numpy(ids).cuda(), plan)
    st, bits = moe_get_error()
    assert st == MOE_ERR_DEVICE and bits & ERR_BAD_ID
    assert (dev_to_np(out) == oracle.eplb_remap(ids, E, plan.replica_offsets, plan.replicas)).all()
    assert dev_to_np(out)[3, 2] == -1


def test_remap_with_inconsistent_tables_is_flagged_not_faulting():
    from token_dispatch_combine_b200 import EplbPlan, moe_eplb_remap, moe_get_error
    from token_dispatch_combine_b200._native import ERR_BAD_OFFSETS, MOE_ERR_DEVICE
    E, P = 4, 6
    off = np.array([0, 2, 2, 9, 6], np.int32)       # expert 1 empty, expert 2 runs past P
    reps = np.array([0, 1, 2, 3, 4, 77], np.int32)  # 77 is no physical id
    plan = EplbPlan(E, 2, 3, np.zeros(P, np.int32), off, reps, torch.from_numpy(off).cuda(),
                    torch.from_numpy(reps).cuda())
    ids = torch.tensor([[0], [1], [2], [3], [0], [3]], dtype=torch.int32, device="cuda")
    out = dev_to_np(moe_eplb_remap(ids, plan)).ravel().tolist()
    st, bits = moe_get_error()
    assert st == MOE_ERR_DEVICE and bits & ERR_BAD_OFFSETS
    # expert 0: replicas 0, 1 by t mod 2; expert 3: offsets 9..6 are invalid
    assert out == [0, -1, -1, -1, 0, -1]
