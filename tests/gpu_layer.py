"""Helpers for the GPU parity tests: build a synthetic layer on the device,
run the round trip through the C ABI, and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

TOL = {"f32": 1e-4, "bf16": 2e-2}  # normwise: max|gpu - oracle| / max|oracle|


def np_to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:  # bfloat16 bit patterns
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def dev_to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def widen(a: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(widen(gpu) if gpu.dtype == np.uint16 else gpu).max())
    g = widen(gpu) if gpu.dtype == np.uint16 else gpu.astype(np.float64)
    return float(np.abs(g - ref).max() / scale)


def torch_dtype(wl: synth.Workload):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


class DeviceLayer:
    """One synthetic layer: host inputs, device inputs, device weights."""

    def __init__(self, wl: synth.Workload, device="cuda", logits: np.ndarray | None = None):
        self.wl = wl
        self.x = wl.x()
        self.logits = wl.logits(widen(self.x).astype(np.float32) if wl.dtype == "bf16" else self.x) \
            if logits is None else logits.astype(np.float32)
        self.x_dev = np_to_dev(self.x, device)
        self.logits_dev = np_to_dev(self.logits, device)
        dt = torch_dtype(wl)
        E, H, I = wl.E, wl.H, wl.I
        self.w_gate = torch.empty((E, H, I), dtype=dt, device=device)
        self.w_up = torch.empty((E, H, I), dtype=dt, device=device)
        self.w_down = torch.empty((E, I, H), dtype=dt, device=device)
        step = max(1, (64 << 20) // max(1, H * I))  # generate ~64M elements at a time
        for e0 in range(0, E, step):
            e1 = min(E, e0 + step)
            self.w_gate[e0:e1].copy_(np_to_dev(wl.w_gate(e0, e1), device))
            self.w_up[e0:e1].copy_(np_to_dev(wl.w_up(e0, e1), device))
            self.w_down[e0:e1].copy_(np_to_dev(wl.w_down(e0, e1), device))

    def host_weights(self, experts) -> tuple[dict, dict, dict]:
        """Oracle-side copies of the given experts' weights, regenerated on the host."""
        wl = self.wl
        g, u, d = {}, {}, {}
        for e in sorted(set(int(x) for x in experts)):
            g[e] = wl.w_gate(e, e + 1)[0]
            u[e] = wl.w_up(e, e + 1)[0]
            d[e] = wl.w_down(e, e + 1)[0]
        return g, u, d


def expert_of_rows(offsets: np.ndarray, rows: np.ndarray) -> np.ndarray:
    return (np.searchsorted(offsets, rows, side="right") - 1).astype(np.int32)
