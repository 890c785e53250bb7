"""The seeded input generator: published SplitMix64 outputs, slice
addressability, distribution sanity and the workload recipes."""
import numpy as np

import synth

GAMMA = 0x9E3779B97F4A7C15
# First outputs of SplitMix64 seeded with state 0 (Vigna's reference generator).
SPLITMIX64_SEED0 = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC]


def test_mixer_is_splitmix64():
    # bits(seed=0, stream=0, i) = mix(key + i) with key = mix(0) = first SplitMix64 output;
    # the n-th SplitMix64 output is mix((n-1) * GAMMA), reached with i = (n-1)*GAMMA - key.
    key = SPLITMIX64_SEED0[0]
    for n, want in enumerate(SPLITMIX64_SEED0):
        first = (n * GAMMA - key) % 2**64
        assert int(synth.raw_bits(0, 0, first, 1)[0]) == want


def test_slices_are_addressable():
    full = synth.normal_f32(7, 3, (1000,))
    part = synth.normal_f32(7, 3, (300,), first=500)
    assert (full[500:800] == part).all()
    fb = synth.normal_bf16(7, 3, (1000,))
    assert (fb[123:456] == synth.normal_bf16(7, 3, (333,), first=123)).all()


def test_bf16_is_round_to_nearest_even_of_f32():
    f = synth.normal_f32(9, 4, (100000,), std=3.0)
    b = synth.normal_bf16(9, 4, (100000,), std=3.0)
    wide = synth.bf16_bits_to_f32(b).astype(np.float64)
    err = np.abs(wide - f.astype(np.float64))
    ulp = np.spacing(np.abs(wide).astype(np.float32)).astype(np.float64) * 2**16
    assert (err <= ulp / 2 + 1e-30).all()


def test_normal_moments_and_streams_differ():
    z = synth.normal_f32(1, 1, (1 << 20,)).astype(np.float64)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1.0) < 5e-3
    assert abs((z[0::2] * z[1::2]).mean()) < 5e-3  # the two Box-Muller halves are uncorrelated
    assert not (synth.normal_f32(1, 2, (16,)) == synth.normal_f32(1, 1, (16,))).any()


def test_workload_recipes():
    w = synth.WORKLOADS["toy_fp32"]
    assert (w.T, w.H, w.I, w.E, w.k, w.R, w.dtype) == (64, 128, 256, 4, 1, 2, "f32")
    assert w.S == 64
    g = synth.WORKLOADS["gptoss_uniform"]
    assert (g.T, g.H, g.I, g.E, g.k, g.R) == (4096, 2880, 3072, 32, 4, 8)
    d = synth.WORKLOADS["dsr1_prefill"]
    assert (d.T, d.H, d.I, d.E, d.k, d.R) == (8192, 7168, 2048, 256, 8, 32)
    small = g.replace(T=64, H=64, I=128)
    wg = small.w_gate()
    assert wg.shape == (32, 64, 128) and wg.dtype == np.uint16
    assert (small.w_gate(5, 7) == wg[5:7]).all()
    z = synth.WORKLOADS["gptoss_zipf"].router_bias()
    assert (np.diff(z) < 0).all()  # expert 0 is the most popular
    lg = small.logits()
    assert lg.shape == (64, 32) and lg.dtype == np.float32
