"""The C-ABI library builds, loads without a GPU, exports every function that
include/moe_b200.h declares, and rejects bad arguments on the host before any
CUDA call (these calls return before touching the device)."""
import ctypes
import os
import re

import pytest

from token_dispatch_combine_b200 import _native

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe_b200.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(moe_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_round_trip_calls():
    names = declared_functions()
    for required in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_get_error",
                     "moe_dispatch_workspace_bytes"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = _native.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(_native.EXPORTS) <= set(declared_functions())
    # and the binding configures every declared call (argument and result types)
    assert set(declared_functions()) <= set(_native.EXPORTS)
    for name in declared_functions():
        assert getattr(lib, name).restype is not None, name


def test_version_and_status_strings():
    lib = _native.lib()
    assert lib.moe_abi_version() >= 1
    assert lib.moe_status_string(0) == b"ok"
    assert lib.moe_status_string(_native.MOE_ERR_TIMEOUT) == b"device wait timed out"


def test_workspace_query_is_host_only():
    lib = _native.lib()
    n = lib.moe_dispatch_workspace_bytes(4096, 4, 32, 8)
    # control word + two [chunks, E] tables + one int per slot
    assert n >= 256 + 4 * 4096 * 4
    assert lib.moe_dispatch_workspace_bytes(-1, 4, 32, 8) == 0


def test_counted_pair_workspace_query_is_host_only():
    """The counted pair counts in chunks of at most 128 slots (moe_dispatch: 512), so its
    workspace holds at least as many chunk counts; both queries reject bad sizes with 0."""
    lib = _native.lib()
    for T, k, E, R in [(4096, 4, 32, 8), (128, 8, 256, 32), (8192, 8, 256, 32), (1, 1, 4, 2), (1000, 3, 6, 1)]:
        plain = lib.moe_dispatch_workspace_bytes(T, k, E, R)
        counted = lib.moe_route_count_workspace_bytes(T, k, E, R)
        assert counted >= plain > 0
    # GPT-OSS shape: 8 ranks x 2048 slots, 512-slot chunks -> 32 chunks; 128-slot chunks -> 128
    assert lib.moe_dispatch_workspace_bytes(4096, 4, 32, 8) == 256 + 4 * (2 * 32 * 32 + 16384 + 32)
    assert lib.moe_route_count_workspace_bytes(4096, 4, 32, 8) == 256 + 4 * (2 * 128 * 32 + 16384 + 32)
    assert lib.moe_route_count_workspace_bytes(-1, 4, 32, 8) == 0


FAKE = 0x1000  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("T,E,k", [(-1, 4, 1), (4, 0, 1), (4, 4, 0), (4, 4, 5), (4, 2000, 1), (4, 16, 9)])
def test_route_rejects_bad_sizes(T, E, k):
    st = _native.lib().moe_route(FAKE, T, E, k, FAKE, FAKE, None)
    assert st == _native.MOE_ERR_INVALID_ARG


def test_route_rejects_misaligned_pointer():
    lib = _native.lib()
    assert lib.moe_route(FAKE + 2, 4, 8, 2, FAKE, FAKE, None) == _native.MOE_ERR_INVALID_ARG
    assert b"logits" in lib.moe_last_error_message()


def _dispatch(**kw):
    a = dict(x=FAKE, dtype=1, T=8, H=64, ids=FAKE, k=2, E=8, R=2, ws_bytes=1 << 20, x_disp=FAKE)
    a.update(kw)
    return _native.lib().moe_dispatch(a["x"], a["dtype"], a["T"], a["H"], a["ids"], a["k"], a["E"], a["R"],
                                      a["x_disp"], FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, a["ws_bytes"], None)


@pytest.mark.parametrize("kw,needle", [
    (dict(E=9, R=2), b"divide E"),                 # experts must split evenly over ranks
    (dict(H=60), b"multiple of 16"),               # 120-byte rows break 16-byte vectors
    (dict(dtype=7), b"dtype"),
    (dict(k=3, E=2, R=1), b"k must"),
    (dict(ws_bytes=16), b"workspace_bytes"),
    (dict(x=FAKE + 8), b"x is not"),
    (dict(x=None), b"both"),                       # index-only dispatch needs x and x_disp both NULL
    (dict(x_disp=None), b"both"),
])
def test_dispatch_rejects(kw, needle):
    assert _dispatch(**kw) == _native.MOE_ERR_INVALID_ARG
    assert needle in _native.lib().moe_last_error_message()


def test_noalloc_dispatch_rejects_bad_arguments_before_any_device_work():
    """Sizes within the built-in scratch but a bad argument: rejected on the host by the same
    checks as moe_dispatch (no CUDA call is made, so this runs without a GPU)."""
    lib = _native.lib()
    args = [FAKE, 1, 8, 64, FAKE, 2, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None]
    bad = list(args)
    bad[7] = 3  # R does not divide E
    assert lib.moe_dispatch_noalloc(*bad, None) == _native.MOE_ERR_INVALID_ARG
    assert b"divide E" in lib.moe_last_error_message()
    bad = list(args)
    bad[13] = None  # slot_to_row
    assert lib.moe_dispatch_noalloc(*bad, None) == _native.MOE_ERR_INVALID_ARG
    assert b"slot_to_row" in lib.moe_last_error_message()


def test_ep_recv_index_accepts_more_columns_than_local_experts():
    """A received row holds at most min(k, E/R) local ids padded to k columns: k > E/R is valid
    (rejected here only for the missing workspace size, i.e. after the k / EL checks)."""
    lib = _native.lib()
    st = lib.moe_ep_recv_index(FAKE, 10, 8, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None)
    assert st == _native.MOE_ERR_INVALID_ARG
    assert b"workspace_bytes" in lib.moe_last_error_message()
    assert lib.moe_ep_recv_index(FAKE, 10, 9, 4, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert b"k must" in lib.moe_last_error_message()


@pytest.mark.parametrize("limit_us,T,needle", [(0, 8, b"limit_us"), (2000000, 8, b"limit_us"), (20, 0, b"T must"),
                                               (20, -3, b"T must")])
def test_dispatch_timeout_selftest_rejects(limit_us, T, needle):
    lib = _native.lib()
    st = lib.moe_selftest_dispatch_timeout(FAKE, 1, T, 64, FAKE, 2, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                           None, FAKE, 1 << 20, limit_us, None)
    assert st == _native.MOE_ERR_INVALID_ARG
    assert needle in lib.moe_last_error_message()


def test_route_count_rejects_a_workspace_sized_for_moe_dispatch():
    lib = _native.lib()
    T, k, E, R = 4096, 4, 32, 8
    small = lib.moe_dispatch_workspace_bytes(T, k, E, R)
    assert lib.moe_route_count(FAKE, T, E, k, R, FAKE, FAKE, FAKE, small, None) == _native.MOE_ERR_INVALID_ARG
    assert b"moe_route_count_workspace_bytes" in lib.moe_last_error_message()
    st = lib.moe_dispatch_counted(FAKE, 1, T, 64, FAKE, k, E, R, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                  small, None)
    assert st == _native.MOE_ERR_INVALID_ARG
    assert b"moe_route_count_workspace_bytes" in lib.moe_last_error_message()


@pytest.mark.parametrize("kw,needle", [
    (dict(k=9), b"k must"),
    (dict(S=17), b"S must be <= T * k"),
    (dict(rts=FAKE + 2), b"row_to_slot"),
    (dict(x=FAKE + 8), b"x is not"),
    (dict(H=68), b"multiples of 16"),
    (dict(T=-1), b"T must"),
])
def test_gate_up_gather_rejects(kw, needle):
    a = dict(x=FAKE, dtype=1, T=8, rts=FAKE, k=2, E=4, H=64, I=64, S=16)
    a.update(kw)
    lib = _native.lib()
    st = lib.moe_ffn_gate_up_gather(a["x"], a["dtype"], a["T"], a["rts"], a["k"], FAKE, FAKE, FAKE, a["E"], a["H"],
                                    a["I"], a["S"], FAKE, None)
    assert st == _native.MOE_ERR_INVALID_ARG
    assert needle in lib.moe_last_error_message()
    st = lib.moe_expert_ffn_gather(a["x"], a["dtype"], a["T"], a["rts"], a["k"], FAKE, FAKE, FAKE, FAKE, a["E"],
                                   a["H"], a["I"], a["S"], FAKE, FAKE, None)
    assert st == _native.MOE_ERR_INVALID_ARG


def test_gate_up_gather_zero_rows_is_a_no_op():
    # S = 0: validated, then nothing to launch (no device needed)
    assert _native.lib().moe_ffn_gate_up_gather(FAKE, 1, 0, None, 2, None, None, FAKE, 4, 64, 64, 0, None, None) == 0


def test_ffn_and_combine_reject():
    lib = _native.lib()
    # bf16 needs H, I multiples of 8 (16-byte rows for TMA)
    assert lib.moe_expert_ffn(FAKE, 1, FAKE, FAKE, FAKE, FAKE, 4, 68, 64, 16, FAKE, FAKE, None) == 1
    assert lib.moe_ffn_gate_up(FAKE, 1, FAKE, FAKE, FAKE, 0, 64, 64, 16, FAKE, None) == 1
    assert lib.moe_ffn_down(FAKE, 1, FAKE, None, 4, 64, 64, 16, FAKE, None) == 1
    assert lib.moe_combine(FAKE, 1, FAKE, FAKE, 4, 9, 64, FAKE, None) == 1
    assert lib.moe_combine(FAKE, 0, FAKE, FAKE, 4, 2, 6, FAKE, None) == 1


def test_python_wrapper_raises_moe_error():
    with pytest.raises(_native.MoeError):
        _native.check(_native.lib().moe_route(FAKE, 4, 4, 9, FAKE, FAKE, None), "moe_route")


def test_ffn_tiling_setting_is_host_only():
    """The tiling mode is host state: set, read back, resolved by rows per expert."""
    import token_dispatch_combine_b200 as moe
    lib = _native.lib()
    assert moe.moe_get_ffn_tiling() == moe.FFN_TILING_AUTO
    try:
        # auto: pair tiles from 448 (gate/up) / 384 (down) rows per expert on
        GU, DN = moe.FFN_GATE_UP, moe.FFN_DOWN
        assert moe.moe_ffn_tiling_for(32, 16384) == moe.FFN_TILING_PAIR  # gate/up by default
        assert moe.moe_ffn_tiling_for(32, 16384, DN) == moe.FFN_TILING_PAIR
        assert moe.moe_ffn_tiling_for(32, 448 * 32, GU) == moe.FFN_TILING_PAIR
        assert moe.moe_ffn_tiling_for(32, 448 * 32 - 1, GU) == moe.FFN_TILING_SINGLE
        assert moe.moe_ffn_tiling_for(32, 384 * 32, DN) == moe.FFN_TILING_PAIR
        assert moe.moe_ffn_tiling_for(32, 384 * 32 - 1, DN) == moe.FFN_TILING_SINGLE
        assert moe.moe_ffn_tiling_for(32, 400 * 32, GU) == moe.FFN_TILING_SINGLE
        assert moe.moe_ffn_tiling_for(32, 400 * 32, DN) == moe.FFN_TILING_PAIR
        assert moe.moe_ffn_tiling_for(256, 65536, GU) == moe.FFN_TILING_SINGLE
        assert moe.moe_ffn_tiling_for(256, 65536, DN) == moe.FFN_TILING_SINGLE
        assert moe.moe_ffn_tiling_for(0, 10) == -1
        assert moe.moe_ffn_tiling_for(32, 10, 2) == -1
        for mode in (moe.FFN_TILING_SINGLE, moe.FFN_TILING_PAIR):
            moe.moe_set_ffn_tiling(mode)
            assert moe.moe_get_ffn_tiling() == mode
            for proj in (GU, DN):
                assert moe.moe_ffn_tiling_for(256, 1, proj) == mode
                assert moe.moe_ffn_tiling_for(1, 1 << 20, proj) == mode
        assert lib.moe_set_ffn_tiling(3) == _native.MOE_ERR_INVALID_ARG
        assert lib.moe_set_ffn_tiling(-1) == _native.MOE_ERR_INVALID_ARG
        assert moe.moe_get_ffn_tiling() == moe.FFN_TILING_PAIR  # unchanged by the rejected calls
        with pytest.raises(moe.MoeError):
            moe.moe_set_ffn_tiling(7)
    finally:
        moe.moe_set_ffn_tiling(moe.FFN_TILING_AUTO)


def test_library_override_variable_is_honoured(tmp_path):
    """MOE_B200_LIBRARY names a prebuilt copy of the library to load instead of the in-tree build."""
    import shutil
    import subprocess
    import sys
    copy = tmp_path / "libmoe_copy.so"
    shutil.copy(_native._build.build(), copy)
    code = ("import token_dispatch_combine_b200 as m; "
            "print(m._native.library_path()); print(m._native.lib().moe_abi_version())")
    env = dict(os.environ, MOE_B200_LIBRARY=str(copy))
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, check=True,
                         cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__)))).stdout.split()
    assert out[0] == str(copy) and int(out[1]) >= 1


@pytest.mark.parametrize("kw,needle", [
    (dict(E=257), b"E must be <= 256"),
    (dict(H=60), b"multiple of 8"),
    (dict(H=0), b"multiple of 8"),
    (dict(k=9), b"k must"),
    (dict(k=5, E=4), b"k must"),
    (dict(T=-1), b"T must"),
    (dict(x=FAKE + 8), b"x is not"),
    (dict(bias=FAKE + 2), b"bias is not"),
])
def test_router_topk_rejects(kw, needle):
    a = dict(x=FAKE, w=FAKE, bias=None, T=8, H=64, E=32, k=4, logits=None)
    a.update(kw)
    st = _native.lib().moe_router_topk(a["x"], a["w"], a["bias"], a["T"], a["H"], a["E"], a["k"], a["logits"],
                                       FAKE, FAKE, None)
    assert st == _native.MOE_ERR_INVALID_ARG
    assert needle in _native.lib().moe_last_error_message()


def test_router_topk_zero_tokens_is_a_host_no_op():
    # T = 0 returns before any pointer is read or any launch
    assert _native.lib().moe_router_topk(None, None, None, 0, 64, 32, 4, None, None, None, None) == 0


def test_round_trip_gathers_where_the_ffn_streams_weights():
    """MoERoundTrip(gather="auto") fuses the row scatter into the gate/up projection only for bf16
    layers with fewer than 384 rows per expert (host rule, no device needed)."""
    import torch
    from token_dispatch_combine_b200 import MoERoundTrip
    rule = MoERoundTrip.gathers_by_default
    bf16, f32 = torch.bfloat16, torch.float32
    assert not rule(4096, 4, 32, bf16)        # GPT-OSS layer, 512 rows per expert: tensor-bound
    assert rule(8192, 8, 256, bf16)           # DeepSeek-R1 prefill, 256 rows per expert
    assert rule(128, 8, 256, bf16)            # decode
    assert rule(383 * 32 // 4, 4, 32, bf16)   # just under 384 rows per expert
    assert not rule(384 * 32 // 4, 4, 32, bf16)
    assert not rule(128, 8, 256, f32)         # float32 layers keep the row-moving dispatch


def test_enable_peer_access_rejects_a_negative_device():
    assert _native.lib().moe_enable_peer_access(-1) == _native.MOE_ERR_INVALID_ARG
    assert b"peer_device" in _native.lib().moe_last_error_message()
