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


def row_errors(gpu: np.ndarray, ref: np.ndarray) -> tuple[float, float, int]:
    """(normwise error of the whole tensor, worst per-row normwise error, that row's index):
    the per-row figure scales each row by its own largest reference value, so one wrong tile
    cannot hide under the tensor-wide maximum."""
    ref = np.asarray(ref, np.float64)
    g = widen(gpu) if gpu.dtype == np.uint16 else gpu.astype(np.float64)
    diff = np.abs(g - ref)
    whole = float(diff.max() / max(np.abs(ref).max(), 1e-300)) if ref.size else 0.0
    if not ref.size:
        return whole, 0.0, -1
    per_row = diff.max(axis=1) / np.maximum(np.abs(ref).max(axis=1), 1e-300)
    worst = int(np.argmax(per_row))
    return whole, float(per_row[worst]), worst


def oracle_ffn_rows_by_expert(layer: "DeviceLayer", rows: np.ndarray, row_to_slot: np.ndarray,
                              expert_offsets: np.ndarray, host_bytes: int = 2 << 30):
    """The oracle's SwiGLU outputs (h, y_disp) of the given dispatched rows, in float64.

    Each row's input is its token's row of x (the oracle's dispatch: x_disp[r] = x[row_to_slot[r] / k]);
    the experts' weights are regenerated on the host a few experts at a time (at most
    ``host_bytes`` of weights at once), so the largest layers fit."""
    wl = layer.wl
    rows = np.asarray(rows, np.int64)
    experts = expert_of_rows(expert_offsets, rows)
    x_rows = layer.x[row_to_slot[rows] // wl.k]
    h = np.empty((len(rows), wl.I), np.float64)
    y = np.empty((len(rows), wl.H), np.float64)
    per_expert = 3 * wl.H * wl.I * (2 if wl.dtype == "bf16" else 4)
    step = max(1, host_bytes // per_expert)
    uniq = np.unique(experts)
    for i in range(0, len(uniq), step):
        es = uniq[i:i + step]
        sel = np.isin(experts, es)
        g, u, d = layer.host_weights(es)
        y[sel], h[sel] = oracle.ffn_rows(x_rows[sel], experts[sel], g, u, d, wl.H, wl.I, want_act=True)
    return h, y
