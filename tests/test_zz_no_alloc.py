"""moe_dispatch_noalloc -- dispatch for callers that cannot allocate device
memory (no workspace argument; the scratch is a fixed array inside the
library).  Called through the C ABI and compared with moe_dispatch, which gets
a caller-allocated workspace: every output must be identical (dispatch outputs
are integers and copied rows, compared bit for bit).

Cases: the first call in the process allocates no device memory; two calls in
a row with different routings; a shape whose scratch need is exactly the
built-in size, then a smaller shape (what the large call left behind must not
matter); sizes one token past the limit are rejected on the host.

This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

SCRATCH = 2 << 20  # MOE_DISPATCH_NOALLOC_SCRATCH_BYTES
# DeepSeek-R1 routing shape whose dispatch scratch is exactly SCRATCH bytes
LIMIT_T, LIMIT_K, LIMIT_E, LIMIT_R = 32728, 8, 256, 32


def _routing(T, E, k, seed, hot=None):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if hot is not None:
        logits[:, hot] += 2.0
    return np.argsort(-logits, axis=1, kind="stable")[:, :k].astype(np.int32)


def _outputs(x, k, E, R):
    from token_dispatch_combine_b200.api import DispatchOut
    T, H = x.shape
    out = DispatchOut.empty(T, H, k, E, R, x.dtype, x.device)
    for t in (out.x_disp, out.expert_counts, out.slot_to_row, out.row_to_slot, out.src_expert_counts):
        t.fill_(-7) if t.dtype == torch.int32 else t.zero_()
    return out


def _call(lib_fn, x, ids, E, R, ws=None, out=None):
    from token_dispatch_combine_b200 import _native
    T, H = x.shape
    k = ids.shape[1]
    out = _outputs(x, k, E, R) if out is None else out
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


def _assert_same(ref, got, tag):
    from token_dispatch_combine_b200 import _native
    st = ctypes.c_uint32(0)
    assert _native.lib().moe_get_error(torch.cuda.current_stream().cuda_stream, ctypes.byref(st)) == 0
    for name in ("x_disp", "expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row",
                 "row_to_slot", "src_expert_counts"):
        a, b = getattr(ref, name), getattr(got, name)
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b), (tag, name)


def test_first_noalloc_call_allocates_no_device_memory():
    """The promise of the entry point: no device memory is taken.  The library's module and the
    dispatch kernel are loaded first (by a workspace dispatch of the same shape), so the first
    no-alloc call in the process finds nothing left to load; free device memory must not move."""
    from token_dispatch_combine_b200 import _native, new_dispatch_workspace
    lib = _native.lib()
    T, H, E, k, R = 2048, 512, 64, 4, 8
    x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
    ids = torch.from_numpy(_routing(T, E, k, 5)).cuda()
    ws = new_dispatch_workspace(T, k, E, R, "cuda")
    ref = _call(lib.moe_dispatch, x, ids, E, R, ws)
    out = _outputs(x, k, E, R)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    got = _call(lib.moe_dispatch_noalloc, x, ids, E, R, out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device memory fell by {free0 - free1} bytes"
    _assert_same(ref, got, "first")


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
        _assert_same(ref, got, call)


def test_noalloc_at_the_scratch_limit_then_a_smaller_shape():
    """A call that fills the built-in scratch exactly, then a small call: the leftovers of the
    large call (its count tables and ranks) must not leak into the small one."""
    from token_dispatch_combine_b200 import _native, new_dispatch_workspace
    lib = _native.lib()
    assert lib.moe_dispatch_workspace_bytes(LIMIT_T, LIMIT_K, LIMIT_E, LIMIT_R) == SCRATCH
    shapes = [(LIMIT_T, 64, LIMIT_E, LIMIT_K, LIMIT_R, 7), (300, 128, 16, 2, 4, 8), (LIMIT_T, 64, LIMIT_E, LIMIT_K,
                                                                                     LIMIT_R, 9)]
    for T, H, E, k, R, seed in shapes:
        x = torch.randn(T, H, device="cuda").to(torch.bfloat16)
        ids = torch.from_numpy(_routing(T, E, k, seed, hot=seed % E)).cuda()
        ws = new_dispatch_workspace(T, k, E, R, "cuda")
        ref = _call(lib.moe_dispatch, x, ids, E, R, ws)
        got = _call(lib.moe_dispatch_noalloc, x, ids, E, R)
        _assert_same(ref, got, (T, E))


@pytest.mark.parametrize("T,k,E,R", [(LIMIT_T + 1, LIMIT_K, LIMIT_E, LIMIT_R), (1 << 19, 8, 256, 32)])
def test_noalloc_dispatch_rejects_sizes_beyond_its_scratch(T, k, E, R):
    """Every pointer is NULL: should the size check ever let such a call through, the argument
    checks still reject it on the host (with a different message), and nothing is launched."""
    from token_dispatch_combine_b200 import _native
    lib = _native.lib()
    assert lib.moe_dispatch_workspace_bytes(T, k, E, R) > SCRATCH
    st = lib.moe_dispatch_noalloc(None, 1, T, 64, None, k, E, R, *([None] * 8), None)
    assert st == _native.MOE_ERR_INVALID_ARG
    assert b"built-in" in lib.moe_last_error_message()
