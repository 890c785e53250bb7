"""The down projection with the combine in its epilogue (moe_ffn_down_combine +
moe_combine_finalize) against the oracle and the unfused round trip.

The float32 atomic additions make the summation order of each output vary,
so results are compared within the layer's normwise bound (per tensor and
per row), not bit for bit: against the oracle's y, and against the unfused
round trip's y.  Two calls in a row check that the finalize leaves the
accumulator at zero; a slot outside [0, T*k) is skipped and flagged."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_layer import TOL, DeviceLayer, dev_to_np, oracle_ffn_rows_by_expert, row_errors
from tests.test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu


def _oracle_y(layer):
    wl = layer.wl
    ids, w = oracle.route(layer.logits, wl.k)
    ref = oracle.dispatch_index(ids, wl.E, wl.R)
    n = int(ref["expert_offsets"][-1])
    _, y_disp = oracle_ffn_rows_by_expert(layer, np.arange(n), ref["row_to_slot"], ref["expert_offsets"])
    return oracle.combine(y_disp, w, ref["slot_to_row"])


@pytest.mark.parametrize("name", ["bf16_multi_tile", "bf16_ragged_n", "bf16_top8_e256", "bf16_e1024", "dsr1_decode"])
def test_down_combine_matches_oracle_and_unfused(name):
    from token_dispatch_combine_b200 import MoERoundTrip, moe_get_error
    wl = SMALL.get(name) or synth.WORKLOADS[name]
    layer = DeviceLayer(wl)
    fused = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, torch.bfloat16, combine_in_down=True)
    plain = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, torch.bfloat16)
    assert fused.combine_in_down
    y_plain = plain.forward(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down).clone()
    y_ref = _oracle_y(layer)
    tol = TOL["bf16"]
    for call in range(2):  # the finalize re-zeroes the accumulator for the next call
        y = fused.forward(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down)
        assert moe_get_error() == (0, 0)
        whole, worst, at = row_errors(dev_to_np(y), y_ref)
        print(f"{name} call {call}: vs oracle normwise {whole:.3e}, worst row {worst:.3e} (token {at})")
        assert whole <= tol and worst <= tol
        whole, worst, _ = row_errors(dev_to_np(y), widen_np(dev_to_np(y_plain)))
        assert whole <= tol and worst <= tol
    assert not fused.y_acc.any()


def widen_np(a):
    from tests.gpu_layer import widen
    return widen(a)


def test_down_combine_flags_a_bad_slot():
    from token_dispatch_combine_b200 import (MoERoundTrip, _native, moe_combine_finalize, moe_ffn_down_combine,
                                             moe_get_error)
    wl = SMALL["bf16_multi_tile"]
    layer = DeviceLayer(wl)
    rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, torch.bfloat16, gather=False)
    rt.forward(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down)
    assert moe_get_error() == (0, 0)
    r2s = rt.disp.row_to_slot.clone()
    r2s[5] = wl.T * wl.k + 3
    acc = torch.zeros((wl.T, wl.H), dtype=torch.float32, device="cuda")
    moe_ffn_down_combine(rt.h, layer.w_down, rt.disp.expert_offsets, r2s, rt.topk_w, acc)
    y = torch.empty_like(rt.y)
    moe_combine_finalize(acc, y)
    st, bits = moe_get_error()
    assert st == _native.MOE_ERR_DEVICE and bits & _native.ERR_BAD_ROW
    # every token but the one whose slot was broken gets the plain combine's output
    bad_tok = int(rt.disp.row_to_slot[5]) // wl.k
    keep = np.ones(wl.T, bool)
    keep[bad_tok] = False
    whole, worst, _ = row_errors(dev_to_np(y)[keep], widen_np(dev_to_np(rt.y))[keep])
    assert whole <= TOL["bf16"] and worst <= TOL["bf16"]
