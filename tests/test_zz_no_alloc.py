"""moe_dispatch_noalloc -- dispatch for callers that cannot allocate device
memory (no workspace argument; the scratch is a fixed array inside the
library).  Called through the C ABI and compared with moe_dispatch, which gets
a caller-allocated workspace, on two calls in a row with different routings:
every output must be identical (dispatch outputs are integers and copied
rows, compared bit for bit).

This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _routing(T, E, k, seed, hot=None):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if hot is not None:
        logits[:, hot] += 2.0
    return np.argsort(-logits, axis=1, kind="stable")[:, :k].astype(np.int32)


def _call(lib_fn, x, ids, E, R, ws=None):
    from token_dispatch_combine_b200 import _native
    from token_dispatch_combine_b200.api import DispatchOut
    T, H = x.shape
    k = ids.shape[1]
    out = DispatchOut.empty(T, H, k, E, R, x.dtype, x.device)
    for t in (out.x_disp, out.expert_counts, out.slot_to_row, out.row_to_slot, out.src_expert_counts):
        t.fill_(-7) if t.dtype == torch.int32 else t.zero_()
    dt = _native.MOE_BF16 if x.dtype == torch.bfloat16 else _native.MOE_F32
    args = [x.data_ptr(), dt, T, H, ids.data_ptr(), k, E, R, out.x_disp.data_ptr(), out.expert_counts.data_ptr(),
            out.expert_offsets.data_ptr(), out.rank_counts.data_ptr(), out.rank_offsets.data_ptr(),
            out.slot_to_row.data_ptr(), out.row_to_slot.data_ptr(), out.src_expert_counts.data_ptr()]
    stream = torch.cuda.current_stream().cuda_stream
    if ws is None:
        st = lib_fn(*args, stream)
    else:
        st = lib_fn(*args, ws.data_ptr(), ws.numel(), stream)
    assert st == 0, _native.lib().moe_last_error_message()
    return out


@pytest.mark.parametrize("T,H,E,k,R,dtype", [(4096, 2880, 32, 4, 8, torch.bfloat16),
                                             (1000, 256, 256, 8, 32, torch.bfloat16),
                                             (333, 96, 6, 3, 3, torch.float32)])
def test_noalloc_dispatch_matches_workspace_dispatch_twice(T, H, E, k, R, dtype):
    from token_dispatch_combine_b200 import _native, new_dispatch_workspace
    lib = _native.lib()
    for call, seed in enumerate((T, T + 1)):  # two calls in a row, different routing
        x = torch.randn(T, H, device="cuda").to(dtype)
        ids = torch.from_numpy(_routing(T, E, k, seed, hot=call)).cuda()
        ws = new_dispatch_workspace(T, k, E, R, "cuda")
        ref = _call(lib.moe_dispatch, x, ids, E, R, ws)
        got = _call(lib.moe_dispatch_noalloc, x, ids, E, R)
        st = ctypes.c_uint32(0)
        assert lib.moe_get_error(torch.cuda.current_stream().cuda_stream, ctypes.byref(st)) == 0
        for name in ("x_disp", "expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row",
                     "row_to_slot", "src_expert_counts"):
            a, b = getattr(ref, name), getattr(got, name)
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b), (call, name)


def test_noalloc_dispatch_rejects_sizes_beyond_its_scratch():
    from token_dispatch_combine_b200 import _native
    lib = _native.lib()
    T, k, E, R = 1 << 19, 8, 256, 32  # needs far more than the built-in scratch
    assert lib.moe_dispatch_workspace_bytes(T, k, E, R) > (2 << 20)
    fake = 0x1000
    st = lib.moe_dispatch_noalloc(fake, 1, T, 64, fake, k, E, R, *([fake] * 7), None, None)
    assert st == _native.MOE_ERR_INVALID_ARG
    assert b"built-in" in lib.moe_last_error_message()
