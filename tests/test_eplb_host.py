"""moe_eplb_plan (a host function of the C ABI) against the oracle: the plan is an
exact integer function of the loads, so it must agree element for element."""
import numpy as np
import pytest

import oracle
from token_dispatch_combine_b200 import _native


def lib_plan(load, R, slots):
    from token_dispatch_combine_b200 import moe_eplb_plan
    return moe_eplb_plan(load, R, slots, device="cpu")


CASES = [(8, 2, 5), (32, 8, 5), (32, 8, 4), (256, 32, 9), (256, 32, 8), (20, 4, 6), (7, 3, 3), (1, 1, 1),
         (1, 4, 3), (1024, 8, 160)]


@pytest.mark.parametrize("E,R,slots", CASES)
@pytest.mark.parametrize("law", ["zipf", "uniform", "ties", "zeros", "one_hot"])
def test_plan_matches_oracle(E, R, slots, law):
    rng = np.random.default_rng(E * 131 + R * 7 + slots)
    if law == "zipf":
        load = (rng.zipf(1.2, E) * 13) % 100000
    elif law == "uniform":
        load = rng.integers(0, 5000, E)
    elif law == "ties":
        load = rng.integers(0, 4, E) * 100  # many equal loads and equal shares
    elif law == "zeros":
        load = np.zeros(E, np.int64)
    else:
        load = np.zeros(E, np.int64)
        load[rng.integers(0, E)] = 12345
    load = load.astype(np.int64)
    got = lib_plan(load, R, slots)
    ref = oracle.eplb_plan(load, R, slots)
    assert got.phys_to_logical.tolist() == ref["phys_to_logical"].tolist()
    assert got.replica_offsets.tolist() == ref["replica_offsets"].tolist()
    assert got.replicas.tolist() == ref["replicas"].tolist()


def test_plan_balances_the_zipf_layer():
    """GPT-OSS-shaped Zipf routing (rank 0 ~5x the mean under the static layout): with one
    spare slot per rank the planned rank loads come within a few percent of the mean."""
    E, R = 32, 8
    p = np.arange(1, E + 1, dtype=np.float64) ** -1.2
    load = np.round(16384 * p / p.sum()).astype(np.int64)
    static = load.reshape(R, -1).sum(1)
    ref = oracle.eplb_plan(load, R, 5)
    assert static.max() / static.mean() > 3.0
    assert ref["rank_load"].max() / ref["rank_load"].mean() < 1.1
    got = lib_plan(load, R, 5)
    assert got.phys_to_logical.tolist() == ref["phys_to_logical"].tolist()


@pytest.mark.parametrize("kw,needle", [
    (dict(R=0), b">= 1"),
    (dict(slots=0), b">= 1"),
    (dict(R=1, slots=3), b">= E"),          # 3 slots for 8 experts
    (dict(R=1 << 11, slots=1 << 10), b"2^20"),
    (dict(neg=True), b"[0, 2^40)"),
])
def test_plan_rejects(kw, needle):
    lib = _native.lib()
    E = 8
    load = np.ones(E, np.int64)
    if kw.get("neg"):
        load[3] = -1
    R, slots = kw.get("R", 2), kw.get("slots", 5)
    out = np.zeros(max(1, R * slots) if R * slots <= (1 << 20) else 1, np.int32)
    off = np.zeros(E + 1, np.int32)
    st = lib.moe_eplb_plan(load.ctypes.data, E, R, slots, out.ctypes.data, off.ctypes.data, out.ctypes.data)
    assert st == _native.MOE_ERR_INVALID_ARG
    assert needle in lib.moe_last_error_message()


def test_remap_and_replicate_reject_on_the_host():
    lib = _native.lib()
    FAKE = 1 << 20
    assert lib.moe_eplb_remap(FAKE, 4, 9, 8, FAKE, FAKE, 10, FAKE, None) == _native.MOE_ERR_INVALID_ARG  # k = 9
    assert lib.moe_eplb_remap(FAKE, 4, 2, 8, FAKE, FAKE, 7, FAKE, None) == _native.MOE_ERR_INVALID_ARG  # P < E
    assert lib.moe_eplb_remap(FAKE + 2, 4, 2, 8, FAKE, FAKE, 10, FAKE, None) == _native.MOE_ERR_INVALID_ARG
    assert lib.moe_eplb_remap(None, 0, 2, 8, None, None, 10, None, None) == _native.MOE_OK  # T = 0
    p2l = np.array([0, 1, 8], np.int32)  # 8 is no expert of E = 8
    assert lib.moe_eplb_replicate(FAKE, 64, 8, p2l.ctypes.data, 3, FAKE * 4, None) == _native.MOE_ERR_INVALID_ARG
    assert b"[0, E)" in lib.moe_last_error_message()
    p2l = np.array([0, 1, 2], np.int32)
    assert lib.moe_eplb_replicate(FAKE, 64, 8, p2l.ctypes.data, 3, FAKE + 64, None) == _native.MOE_ERR_INVALID_ARG
    assert b"overlap" in lib.moe_last_error_message()


def test_plan_with_loads_near_the_limit_matches_oracle():
    """Loads up to 2^40 - 1 with up to thousands of replicas: load * n stays below 2^63 in both
    implementations and they still agree exactly; 2^40 itself is rejected."""
    rng = np.random.default_rng(7)
    E, R, slots = 64, 16, 200  # 3200 slots: experts get up to hundreds of replicas
    load = rng.integers(0, 1 << 40, E, dtype=np.int64)
    load[5] = (1 << 40) - 1
    load[9] = 0
    got = lib_plan(load, R, slots)
    ref = oracle.eplb_plan(load, R, slots)
    assert got.replicas.tolist() == ref["replicas"].tolist()
    assert got.phys_to_logical.tolist() == ref["phys_to_logical"].tolist()
    load[3] = 1 << 40
    with pytest.raises(Exception):
        lib_plan(load, R, slots)


@pytest.mark.parametrize("seed", range(20))
def test_plan_random_sizes_match_oracle(seed):
    rng = np.random.default_rng(1000 + seed)
    R = int(rng.integers(1, 9))
    E = int(rng.integers(1, 65))
    slots = int(rng.integers(-(-E // R), -(-E // R) + 4))  # ceil(E / R) .. + 3 spare slots per rank
    load = rng.integers(0, 10 ** int(rng.integers(1, 7)), E).astype(np.int64)
    got = lib_plan(load, R, slots)
    ref = oracle.eplb_plan(load, R, slots)
    assert got.phys_to_logical.tolist() == ref["phys_to_logical"].tolist()
    assert got.replica_offsets.tolist() == ref["replica_offsets"].tolist()
    assert got.replicas.tolist() == ref["replicas"].tolist()
