"""GPU edge cases: worked example of the pages, ties, empty inputs, bad data
that must be flagged (never faulted on), and the bounded-wait self-test."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_layer import dev_to_np

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _api():
    import token_dispatch_combine_b200 as m
    return m


def test_worked_example_on_gpu():
    m = _api()
    g = json.load(open(os.path.join(GOLDEN, "ep_worked_example.json")))
    ex = g["expected"]
    logits = torch.tensor(g["logits"], dtype=torch.float32, device="cuda")
    H = 8
    x = torch.arange(g["T"] * H, dtype=torch.float32, device="cuda").reshape(g["T"], H)
    rt = m.MoERoundTrip(g["T"], H, 8, g["E"], 1, g["R"], torch.float32)
    rt.route(logits)
    rt.dispatch(x)
    torch.cuda.synchronize()
    assert dev_to_np(rt.topk_ids).tolist() == ex["topk_ids"]
    assert dev_to_np(rt.topk_w).tolist() == ex["topk_w"]
    for key in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_to_slot", "slot_to_row",
                "src_expert_counts"):
        assert dev_to_np(getattr(rt.disp, key)).tolist() == ex[key], key
    # E2's rows are A2 then B2; results return in A1, A2, B1, B2 order (identity experts)
    assert (dev_to_np(rt.disp.x_disp)[2:4] == dev_to_np(x)[[1, 3]]).all()
    y = torch.empty_like(x)
    m.moe_combine(rt.disp.x_disp, rt.topk_w, rt.disp.slot_to_row, y)
    assert (dev_to_np(y) == dev_to_np(x)).all()


def test_route_ties_and_signed_zero_match_oracle():
    m = _api()
    rng = np.random.default_rng(3)
    logits = np.round(rng.standard_normal((500, 64)) * 2).astype(np.float32)  # many exact ties
    logits[::7] = 0.0
    logits[1::7] = -0.0
    logits[2::7, ::3] = -0.0
    ids_ref, w_ref = oracle.route(logits, 8)
    ids, w = m.moe_route(torch.from_numpy(logits).cuda(), 8)
    assert (dev_to_np(ids) == ids_ref).all()
    np.testing.assert_allclose(dev_to_np(w), w_ref, rtol=0, atol=1e-6)


@pytest.mark.parametrize("E", [1, 3, 32, 33, 100, 256, 1024])
def test_route_expert_counts(E):
    m = _api()
    rng = np.random.default_rng(E)
    k = min(E, 8)
    logits = rng.standard_normal((77, E)).astype(np.float32)
    ids_ref, w_ref = oracle.route(logits, k)
    ids, w = m.moe_route(torch.from_numpy(logits).cuda(), k)
    assert (dev_to_np(ids) == ids_ref).all()
    np.testing.assert_allclose(dev_to_np(w), w_ref, rtol=0, atol=1e-6)


def test_zero_tokens_is_a_no_op_that_zeroes_counts():
    m = _api()
    rt = m.MoERoundTrip(0, 64, 64, 8, 2, 4, torch.bfloat16)
    rt.disp.expert_counts.fill_(7)
    rt.route(torch.empty((0, 8), dtype=torch.float32, device="cuda"))
    rt.dispatch(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert dev_to_np(rt.disp.expert_counts).tolist() == [0] * 8
    assert dev_to_np(rt.disp.expert_offsets).tolist() == [0] * 9


def test_bad_expert_ids_are_dropped_and_flagged():
    m = _api()
    T, H, E, k, R = 50, 32, 8, 2, 2
    rng = np.random.default_rng(9)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    ids[3, 1] = 8
    ids[10, 0] = -5
    ids[49, 1] = 1 << 30
    x = torch.randn(T, H, device="cuda")
    out = m.DispatchOut.empty(T, H, k, E, R, torch.float32, "cuda")
    ws = m.new_dispatch_workspace(T, k, E, R, "cuda")
    m.moe_dispatch(x, torch.from_numpy(ids).cuda(), E, R, out, ws)
    st, bits = m.moe_get_error()
    assert st == 4 and bits & 1
    ref = oracle.dispatch_index(ids, E, R)
    assert ref["dropped"] == 3
    for key in ("expert_counts", "expert_offsets", "slot_to_row", "row_to_slot", "src_expert_counts"):
        assert (dev_to_np(getattr(out, key)) == ref[key]).all(), key
    assert m.moe_get_error() == (0, 0)  # cleared


def test_combine_skips_out_of_range_rows():
    m = _api()
    T, H, k = 10, 16, 2
    y_disp = torch.randn(T * k, H, device="cuda")
    w = torch.full((T, k), 0.5, device="cuda")
    s2r = torch.arange(T * k, dtype=torch.int32, device="cuda")
    s2r[5] = 10**6
    y = torch.empty(T, H, device="cuda")
    m.moe_combine(y_disp, w, s2r, y)
    st, bits = m.moe_get_error()
    assert st == 4 and bits & 4
    yn, ydn = dev_to_np(y), dev_to_np(y_disp)
    np.testing.assert_allclose(yn[2], 0.5 * ydn[4], rtol=1e-6)  # slot 5 (token 2, j=1) skipped
    np.testing.assert_allclose(yn[3], 0.5 * ydn[6] + 0.5 * ydn[7], rtol=1e-6)


@pytest.mark.parametrize("dtype,ffn_tiling", [(torch.float32, "auto"), (torch.bfloat16, "single"),
                                              (torch.bfloat16, "pair")], indirect=["ffn_tiling"])
def test_ffn_clamps_inconsistent_offsets(dtype, ffn_tiling):
    m = _api()
    E, H, I, S = 4, 64, 64, 40
    x = torch.randn(S, H, device="cuda").to(dtype)
    wg = torch.randn(E, H, I, device="cuda").to(dtype)
    wd = torch.randn(E, I, H, device="cuda").to(dtype)
    off = torch.tensor([0, 30, 10, 50, 999], dtype=torch.int32, device="cuda")  # decreasing and past S
    h = torch.zeros(S, I, device="cuda", dtype=dtype)
    y = torch.zeros(S, H, device="cuda", dtype=dtype)
    m.moe_expert_ffn(x, wg, wg, wd, off, h, y)
    st, bits = m.moe_get_error()
    assert st == 4 and bits & 2
    assert torch.isfinite(y.float()).all()


def test_invalid_arguments_raise_without_launch():
    m = _api()
    logits = torch.randn(4, 8, device="cuda")
    with pytest.raises(m.MoeError):
        m.moe_route(logits, 9)
    with pytest.raises(m.MoeError):
        m.moe_dispatch(torch.randn(4, 6, device="cuda"), torch.zeros(4, 1, dtype=torch.int32, device="cuda"), 8, 2,
                       m.DispatchOut.empty(4, 6, 1, 8, 2, torch.float32, "cuda"),
                       m.new_dispatch_workspace(4, 1, 8, 2, "cuda"))


def test_bounded_wait_times_out_and_context_survives():
    m = _api()
    from token_dispatch_combine_b200 import _native
    stream = torch.cuda.current_stream().cuda_stream
    assert _native.lib().moe_selftest_wait_timeout(20000, stream) == 0  # 20 ms
    st, bits = m.moe_get_error()
    assert st == _native.MOE_ERR_TIMEOUT and bits & _native.ERR_TIMEOUT
    # the context is still usable
    ids, w = m.moe_route(torch.randn(16, 8, device="cuda"), 2)
    torch.cuda.synchronize()
    assert (dev_to_np(w).sum(1) > 0.999).all()


@pytest.mark.parametrize("T,E,k,R", [(2048, 1024, 8, 32),   # count table too big to stage in shared memory
                                     (100, 64, 8, 8),        # T not a multiple of R
                                     (5000, 16, 1, 16)])
def test_dispatch_index_against_oracle(T, E, k, R):
    m = _api()
    rng = np.random.default_rng(T + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[:, 1] += 1.5  # a hot expert
    ids, _ = oracle.route(logits, k)
    x = torch.randn(T, 64, device="cuda", dtype=torch.bfloat16)
    out = m.DispatchOut.empty(T, 64, k, E, R, torch.bfloat16, "cuda")
    ws = m.new_dispatch_workspace(T, k, E, R, "cuda")
    for _ in range(2):  # the workspace must be reusable
        m.moe_dispatch(x, torch.from_numpy(ids).cuda(), E, R, out, ws)
        assert m.moe_get_error() == (0, 0)
        ref = oracle.dispatch_index(ids, E, R)
        for key in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row", "row_to_slot",
                    "src_expert_counts"):
            assert (dev_to_np(getattr(out, key)) == ref[key]).all(), key
        xd = oracle.dispatch_rows(dev_to_np(x), k, ref["slot_to_row"])
        assert (dev_to_np(out.x_disp) == xd).all()


@pytest.mark.parametrize("T,E,k,R,index_only", [(512, 8, 2, 4, False),     # one grid barrier (count table in smem)
                                                (2048, 1024, 8, 32, False),  # two grid barriers
                                                (777, 64, 4, 8, True)])     # index-only dispatch
def test_dispatch_recovers_from_grid_barrier_timeout(T, E, k, R, index_only):
    """A dispatch whose grid barrier times out reports MOE_ERR_TIMEOUT, and the next
    moe_dispatch on the same workspace is complete and exact: the kernel's last CTA
    to finish zeroes the barrier's counters on every exit path."""
    m = _api()
    from token_dispatch_combine_b200 import _native
    lib = _native.lib()
    rng = np.random.default_rng(T + k)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ids, _ = oracle.route(logits, k)
    ids_dev = torch.from_numpy(ids).cuda()
    H = 64
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    out = m.DispatchOut.empty(T, H, k, E, R, torch.bfloat16, "cuda", rows=not index_only)
    ws = m.new_dispatch_workspace(T, k, E, R, "cuda")
    xp = None if index_only else x.data_ptr()
    xdp = None if index_only else out.x_disp.data_ptr()
    args = [xp, _native.MOE_BF16, T, H, ids_dev.data_ptr(), k, E, R, xdp, out.expert_counts.data_ptr(),
            out.expert_offsets.data_ptr(), out.rank_counts.data_ptr(), out.rank_offsets.data_ptr(),
            out.slot_to_row.data_ptr(), out.row_to_slot.data_ptr(), out.src_expert_counts.data_ptr(),
            ws.data_ptr(), ws.numel()]
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.moe_selftest_dispatch_timeout(*args, 20, stream) == 0  # 20 us per barrier wait
    st, bits = m.moe_get_error()
    assert st == _native.MOE_ERR_TIMEOUT and bits & _native.ERR_TIMEOUT
    ctrl = ws[:256].view(torch.int32).cpu()
    assert int(ctrl[16]) == 0 and int(ctrl[48]) == 0  # arrival count (byte 64), exit count (byte 192)
    for _ in range(2):
        m.moe_dispatch(None if index_only else x, ids_dev, E, R, out, ws, H=H, dtype=torch.bfloat16)
        assert m.moe_get_error() == (0, 0)
        ref = oracle.dispatch_index(ids, E, R)
        for key in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row", "row_to_slot",
                    "src_expert_counts"):
            assert (dev_to_np(getattr(out, key)) == ref[key]).all(), key
        if not index_only:
            assert (dev_to_np(out.x_disp) == oracle.dispatch_rows(dev_to_np(x), k, ref["slot_to_row"])).all()
