"""The masking form of expert parallelism on the GPU (moe_combine_rank_partials,
moe_reduce_rank_partials) against the oracle's rank_partials / reduce_ranks.

"Expert Parallelism (EP)", Collective Patterns / Prefill (CTE kernel) and Why a
Single All-Reduce/Reduce-Scatter Works: rank r's partial output holds only its
own experts' weighted outputs (zeros for tokens routed elsewhere), and the sum
over ranks is the full output.  Each rank's plane is compared with the
oracle's within the layer's normwise bound (per plane and per row); a row the
oracle leaves exactly zero must be exactly zero; the reduction is compared
with the oracle's reduction and with the plain combine's tolerance."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_layer import TOL, DeviceLayer, dev_to_np, oracle_ffn_rows_by_expert, rel_err, row_errors, widen
from tests.test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu


def _run_masked(layer):
    from token_dispatch_combine_b200 import MoERoundTrip, moe_get_error
    wl = layer.wl
    rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, layer.x_dev.dtype, rank_partials=True)
    rt.forward_masked(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down)
    assert moe_get_error() == (0, 0)
    return rt


def _check_planes(rt, wl, ids, w, ref, y_disp_ref):
    tol = TOL[wl.dtype]
    part_ref = oracle.rank_partials(y_disp_ref, w, ids, ref["slot_to_row"], wl.E, wl.R)
    part = dev_to_np(rt.y_part)
    for r in range(wl.R):
        got = part[r]
        zero_rows = ~part_ref[r].any(axis=1)
        g = widen(got) if got.dtype == np.uint16 else got
        assert not g[zero_rows].any(), f"rank {r}: a token routed to none of its experts got a nonzero partial"
        nz = ~zero_rows
        if nz.any():
            whole, worst, at = row_errors(got[nz], part_ref[r][nz])
            assert whole <= tol and worst <= tol, (r, whole, worst, at)
    y_ref = oracle.reduce_ranks(part_ref)
    assert rel_err(dev_to_np(rt.y), y_ref) <= tol
    whole, worst, _ = row_errors(dev_to_np(rt.y), y_ref)
    assert worst <= tol, worst


@pytest.mark.parametrize("name", ["toy_fp32", "bf16_multi_tile", "bf16_ragged", "f32_top4", "bf16_top8_e256",
                                  "bf16_one_token"])
def test_rank_partials_small_layer(name):
    wl = SMALL[name]
    layer = DeviceLayer(wl)
    rt = _run_masked(layer)
    ids, w = oracle.route(layer.logits, wl.k)
    ref = oracle.dispatch_index(ids, wl.E, wl.R)
    n = int(ref["expert_offsets"][-1])
    _, y_disp_ref = oracle_ffn_rows_by_expert(layer, np.arange(n), ref["row_to_slot"], ref["expert_offsets"])
    _check_planes(rt, wl, ids, w, ref, y_disp_ref)


def test_rank_partials_full_gptoss_layer():
    """The GPT-OSS layer (R = 8 planes of [4096, 2880]) in full."""
    wl = synth.WORKLOADS["gptoss_uniform"]
    layer = DeviceLayer(wl)
    rt = _run_masked(layer)
    ids, w = oracle.route(layer.logits, wl.k)
    ref = oracle.dispatch_index(ids, wl.E, wl.R)
    n = int(ref["expert_offsets"][-1])
    from tests.test_gpu_parity import _EXPECTED
    exp = _EXPECTED.get("gptoss_uniform")  # shared with the parity test when both run in one process
    if exp is not None and len(exp["rows"]) == n:
        y_disp_ref = exp["y_disp"]
    else:
        _, y_disp_ref = oracle_ffn_rows_by_expert(layer, np.arange(n), ref["row_to_slot"], ref["expert_offsets"])
    _check_planes(rt, wl, ids, w, ref, y_disp_ref)


def test_rank_partials_sum_equals_plain_combine_with_identity_experts():
    """With y_disp := x_disp (identity experts) and float32 rows, the reduced partials equal the
    plain combine's output within float32 rounding of a few terms."""
    from token_dispatch_combine_b200 import (MoERoundTrip, moe_combine, moe_combine_rank_partials,
                                             moe_reduce_rank_partials)
    wl = synth.Workload("ident_masked", T=300, H=64, I=64, E=16, k=4, R=4, dtype="f32", seed=31)
    layer = DeviceLayer(wl)
    rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, torch.float32, gather=False)
    rt.route(layer.logits_dev)
    rt.dispatch(layer.x_dev)
    y = torch.empty_like(layer.x_dev)
    moe_combine(rt.disp.x_disp, rt.topk_w, rt.disp.slot_to_row, y)
    part = moe_combine_rank_partials(rt.disp.x_disp, rt.topk_w, rt.topk_ids, rt.disp.slot_to_row, wl.E, wl.R)
    y2 = moe_reduce_rank_partials(part)
    torch.cuda.synchronize()
    np.testing.assert_allclose(dev_to_np(y2), dev_to_np(y), rtol=0, atol=4e-6 * np.abs(layer.x).max())
    np.testing.assert_allclose(dev_to_np(y2), layer.x, rtol=0, atol=4e-6 * np.abs(layer.x).max())


def test_rank_partials_flag_and_skip_a_bad_row():
    from token_dispatch_combine_b200 import _native, moe_combine_rank_partials, moe_get_error
    T, H, E, k, R = 64, 64, 8, 2, 4
    rng = np.random.default_rng(2)
    ids, w = oracle.route(rng.standard_normal((T, E)).astype(np.float32), k)
    idx = oracle.dispatch_index(ids, E, R)
    y_disp = rng.standard_normal((T * k, H)).astype(np.float32)
    s2r = idx["slot_to_row"].copy()
    s2r[0] = T * k + 5  # token 0's first choice points past the buffer
    part = moe_combine_rank_partials(torch.from_numpy(y_disp).cuda(), torch.from_numpy(w).cuda(),
                                     torch.from_numpy(ids).cuda(), torch.from_numpy(s2r).cuda(), E, R)
    st, bits = moe_get_error()
    assert st == _native.MOE_ERR_DEVICE and bits & _native.ERR_BAD_ROW
    s2r_ref = s2r.copy()
    s2r_ref[0] = -1
    ref = oracle.rank_partials(y_disp, w, ids, s2r_ref, E, R)
    np.testing.assert_allclose(dev_to_np(part), ref, rtol=0, atol=1e-5)
