"""moe_route_count + moe_dispatch_counted (the dispatch's counting done by the
routing kernel) against moe_route + moe_dispatch and the oracle.

Ids and weights must equal moe_route's bit for bit (and the oracle's ids,
weights within 1e-6); counts, offsets, the permutation and the dispatched
rows must equal the oracle's exactly.  Shapes cover a count table small
enough for the barrier-free dispatch and a large one (E = 1024), chunks whose
boundary splits a token's slots (k = 3), one token, and index-only dispatch;
a second counted dispatch on the same counting gives the same result; counts
that belong to other ids are flagged and never move a row out of its
expert's segment."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_layer import dev_to_np

pytestmark = pytest.mark.gpu

KEYS = ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row", "row_to_slot",
        "src_expert_counts")


def _logits(T, E, seed, hot=None):
    rng = np.random.default_rng(seed)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    if hot is not None:
        lg[:, hot] += 1.5
    lg[::11, :4] = 0.25  # exact ties between experts 0..3 on some tokens
    return lg


@pytest.mark.parametrize("T,E,k,R,H,index_only", [
    (4096, 32, 4, 8, 2880, False),    # GPT-OSS shape: 32 x 32 count table, no grid barrier
    (128, 256, 8, 32, 256, False),    # decode shape: 8192-entry table (the small-table limit)
    (2048, 1024, 8, 32, 128, False),  # large table: one grid barrier
    (1000, 6, 3, 1, 64, False),       # chunk boundaries split tokens' slots
    (1, 4, 2, 2, 64, False),
    (8192, 256, 8, 32, 64, True),     # DeepSeek-R1 prefill routing, index only
    (777, 64, 4, 8, 96, True),
])
def test_counted_pair_matches_plain_pair_and_oracle(T, E, k, R, H, index_only):
    import token_dispatch_combine_b200 as m
    lg_np = _logits(T, E, T + E, hot=1 % E)
    lg = torch.from_numpy(lg_np).cuda()
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    ws = m.new_dispatch_workspace(T, k, E, R, "cuda")
    ids, w = m.moe_route_count(lg, k, R, ws)
    ids_ref, w_ref = m.moe_route(lg, k)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids_ref) and torch.equal(w.view(torch.int32), w_ref.view(torch.int32))
    o_ids, o_w = oracle.route(lg_np, k)
    assert (dev_to_np(ids) == o_ids).all()
    np.testing.assert_allclose(dev_to_np(w), o_w, rtol=0, atol=1e-6)
    out = m.DispatchOut.empty(T, H, k, E, R, torch.bfloat16, "cuda", rows=not index_only)
    ref = oracle.dispatch_index(o_ids, E, R)
    for _ in range(2):  # the counting is kept: a second counted dispatch gives the same result
        m.moe_dispatch_counted(None if index_only else x, ids, E, R, out, ws, H=H, dtype=torch.bfloat16)
        assert m.moe_get_error() == (0, 0)
        for key in KEYS:
            assert (dev_to_np(getattr(out, key)) == ref[key]).all(), key
        if not index_only:
            assert (dev_to_np(out.x_disp) == oracle.dispatch_rows(dev_to_np(x), k, ref["slot_to_row"])).all()


def test_round_trip_default_uses_the_counted_pair_and_matches_the_plain_one():
    """MoERoundTrip routes with counting by default; its outputs equal the plain pair's bit for bit."""
    import token_dispatch_combine_b200 as m
    T, H, I, E, k, R = 512, 256, 384, 16, 4, 4
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    lg = torch.from_numpy(_logits(T, E, 3)).cuda()
    wg = (torch.randn(E, H, I, device="cuda") / 16).to(torch.bfloat16)
    wu = (torch.randn(E, H, I, device="cuda") / 16).to(torch.bfloat16)
    wd = (torch.randn(E, I, H, device="cuda") / 20).to(torch.bfloat16)
    a = m.MoERoundTrip(T, H, I, E, k, R, torch.bfloat16, gather=False)
    b = m.MoERoundTrip(T, H, I, E, k, R, torch.bfloat16, gather=False, route_counts=False)
    assert a.route_counts and not b.route_counts
    ya = a.forward(x, lg, wg, wu, wd)
    yb = b.forward(x, lg, wg, wu, wd)
    assert m.moe_get_error() == (0, 0)
    assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))
    assert torch.equal(a.disp.slot_to_row, b.disp.slot_to_row)


def test_counts_of_other_ids_are_flagged_and_stay_in_segment():
    """Misuse: the counting belongs to one routing, the ids given to the dispatch to another.
    No row may leave its expert's segment; the inconsistency is flagged (bit 2)."""
    import token_dispatch_combine_b200 as m
    from token_dispatch_combine_b200 import _native
    T, E, k, R, H = 600, 16, 2, 4, 64
    ws = m.new_dispatch_workspace(T, k, E, R, "cuda")
    lg_a = torch.from_numpy(_logits(T, E, 1, hot=3)).cuda()
    lg_b = torch.from_numpy(_logits(T, E, 2, hot=9)).cuda()
    m.moe_route_count(lg_a, k, R, ws)
    ids_b, _ = m.moe_route(lg_b, k)
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    out = m.DispatchOut.empty(T, H, k, E, R, torch.bfloat16, "cuda")
    out.slot_to_row.fill_(-7)
    m.moe_dispatch_counted(x, ids_b, E, R, out, ws)
    st, bits = m.moe_get_error()
    assert st == _native.MOE_ERR_DEVICE and bits & _native.ERR_BAD_OFFSETS
    s2r = dev_to_np(out.slot_to_row)
    off = dev_to_np(out.expert_offsets)
    ib = dev_to_np(ids_b).ravel()
    placed = s2r >= 0
    assert ((s2r[placed] >= off[ib[placed]]) & (s2r[placed] < off[ib[placed] + 1])).all()
    # the next consistent pair on the same workspace is exact again
    ids, _ = m.moe_route_count(lg_b, k, R, ws)
    m.moe_dispatch_counted(x, ids, E, R, out, ws)
    assert m.moe_get_error() == (0, 0)
    ref = oracle.dispatch_index(dev_to_np(ids), E, R)
    for key in KEYS:
        assert (dev_to_np(getattr(out, key)) == ref[key]).all(), key
