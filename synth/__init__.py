"""Seeded synthetic inputs for the MoE token round trip.

This module is the one source of inputs that both sides read: the CUDA path
(through the C-ABI library) and the CPU oracle.  It holds none of the MoE
method's arithmetic -- no top-k, no counts, no permutation, no expert MLP, no
combine.  Its only computation beyond random draws is the router affinity
matrix ``logits = x @ W_router + bias`` (float64, rounded once to float32),
which is input preparation: the round trip's first call, ``moe_route``,
starts from these logits ("Expert Parallelism (EP)", Collective Patterns,
Prefill step 1: the router matmul happens before dispatch).

Random numbers come from a counter-based generator defined in
``synth_gen.c`` (SplitMix64 + Box-Muller): every element is a pure function of
(seed, stream, flat index), so any slice -- e.g. one expert's weights -- can be
regenerated on its own.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_gen.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

# stream ids, one per tensor kind
STREAM_X = 1
STREAM_ROUTER = 2
STREAM_BIAS = 3
STREAM_GATE = 4
STREAM_UP = 5
STREAM_DOWN = 6


def build(force: bool = False) -> str:
    """Compile synth_gen.c into libsynth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _get():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, dbl, vp = ctypes.c_uint64, ctypes.c_double, ctypes.c_void_p
            lib.synth_normal_f32.argtypes = [u64, u64, u64, u64, dbl, vp]
            lib.synth_normal_bf16.argtypes = [u64, u64, u64, u64, dbl, vp]
            lib.synth_bits.argtypes = [u64, u64, u64, u64, vp]
            _lib = lib
    return _lib


def normal_f32(seed: int, stream: int, shape, std: float = 1.0, first: int = 0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _get().synth_normal_f32(seed, stream, first, out.size, std, out.ctypes.data)
    return out


def normal_bf16(seed: int, stream: int, shape, std: float = 1.0, first: int = 0) -> np.ndarray:
    """bfloat16 values as their raw uint16 bit patterns."""
    out = np.empty(shape, dtype=np.uint16)
    _get().synth_normal_bf16(seed, stream, first, out.size, std, out.ctypes.data)
    return out


def raw_bits(seed: int, stream: int, first: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _get().synth_bits(seed, stream, first, n, out.ctypes.data)
    return out


def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (u16.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, dtype and value recipe of one synthetic MoE layer."""

    name: str
    T: int  # tokens
    H: int  # hidden size
    I: int  # expert SwiGLU intermediate size
    E: int  # experts
    k: int  # experts per token
    R: int  # logical EP ranks (experts [r*E/R, (r+1)*E/R) live on rank r)
    dtype: str  # "f32" or "bf16" for activations and expert weights
    seed: int
    bias: str = "none"  # "none" | "zipf1.2" | "normal0.5"

    @property
    def S(self) -> int:
        return self.T * self.k

    def _gen(self, stream, shape, std, first=0):
        if self.dtype == "bf16":
            return normal_bf16(self.seed, stream, shape, std, first)
        return normal_f32(self.seed, stream, shape, std, first)

    # --- activations and router -------------------------------------------
    def x(self) -> np.ndarray:
        """Token activations [T, H], N(0, 1) (uint16 bf16 bits or float32)."""
        return self._gen(STREAM_X, (self.T, self.H), 1.0)

    def x_f32(self) -> np.ndarray:
        x = self.x()
        return bf16_bits_to_f32(x) if self.dtype == "bf16" else x

    def router_weight(self) -> np.ndarray:
        """Router weight [H, E] float32, N(0, 1/H)."""
        return normal_f32(self.seed, STREAM_ROUTER, (self.H, self.E), 1.0 / math.sqrt(self.H))

    def router_bias(self) -> np.ndarray:
        """Per-expert logit bias [E] (float64) for the skewed-routing workloads."""
        if self.bias == "none":
            return np.zeros(self.E, dtype=np.float64)
        if self.bias == "zipf1.2":
            # popularity p_e proportional to (e+1)^-1.2; bias = ln p_e
            p = np.arange(1, self.E + 1, dtype=np.float64) ** -1.2
            return np.log(p / p.sum())
        if self.bias == "normal0.5":
            return normal_f32(self.seed, STREAM_BIAS, (self.E,), 0.5).astype(np.float64)
        raise ValueError(self.bias)

    def logits(self, x_f32: np.ndarray | None = None) -> np.ndarray:
        """Router affinities [T, E] float32 = round_f32(x @ W_router + bias), in float64."""
        if x_f32 is None:
            x_f32 = self.x_f32()
        acc = x_f32.astype(np.float64) @ self.router_weight().astype(np.float64)
        acc += self.router_bias()[None, :]
        return acc.astype(np.float32)

    # --- expert weights ------------------------------------------------------
    def w_gate(self, e0: int = 0, e1: int | None = None) -> np.ndarray:
        """Experts [e0, e1) of the gate weight [E, H, I], N(0, 1/H)."""
        e1 = self.E if e1 is None else e1
        n = self.H * self.I
        return self._gen(STREAM_GATE, (e1 - e0, self.H, self.I), 1.0 / math.sqrt(self.H), e0 * n)

    def w_up(self, e0: int = 0, e1: int | None = None) -> np.ndarray:
        e1 = self.E if e1 is None else e1
        n = self.H * self.I
        return self._gen(STREAM_UP, (e1 - e0, self.H, self.I), 1.0 / math.sqrt(self.H), e0 * n)

    def w_down(self, e0: int = 0, e1: int | None = None) -> np.ndarray:
        """Experts [e0, e1) of the down weight [E, I, H], N(0, 1/I)."""
        e1 = self.E if e1 is None else e1
        n = self.I * self.H
        return self._gen(STREAM_DOWN, (e1 - e0, self.I, self.H), 1.0 / math.sqrt(self.I), e0 * n)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five synthetic layers: a toy fp32 layer, a GPT-OSS-20B-shaped layer with
# balanced and with Zipf-skewed routing, and DeepSeek-R1-shaped prefill and
# decode layers.
WORKLOADS = {
    "toy_fp32": Workload("toy_fp32", T=64, H=128, I=256, E=4, k=1, R=2, dtype="f32", seed=0),
    "gptoss_uniform": Workload("gptoss_uniform", T=4096, H=2880, I=3072, E=32, k=4, R=8, dtype="bf16", seed=1),
    "gptoss_zipf": Workload("gptoss_zipf", T=4096, H=2880, I=3072, E=32, k=4, R=8, dtype="bf16", seed=2,
                            bias="zipf1.2"),
    "dsr1_prefill": Workload("dsr1_prefill", T=8192, H=7168, I=2048, E=256, k=8, R=32, dtype="bf16", seed=3,
                             bias="normal0.5"),
    "dsr1_decode": Workload("dsr1_decode", T=128, H=7168, I=2048, E=256, k=8, R=32, dtype="bf16", seed=4),
}

# Profiling cases (not benchmark layers): the DeepSeek-R1 prefill layer's shapes with 32 experts,
# so that a multi-pass profiler capture holds a few GB (256 rows per expert on average, the same
# routing bias and seed).
PROFILE_WORKLOADS = {
    "dsr1_prefill_slice": Workload("dsr1_prefill_slice", T=1024, H=7168, I=2048, E=32, k=8, R=8, dtype="bf16",
                                   seed=3, bias="normal0.5"),
}
