"""GPU round trip (through the C ABI) against the CPU oracle.

The small layers run the row-moving dispatch (x_disp is checked against the
oracle's); the full-size layers, the host-pipeline and the graph tests run
the round trip's default choice between that and the dispatch fused into
the gate/up projection (checked on its own in test_gpu_gather.py).

Integer outputs (ids, counts, offsets, permutation, dispatched rows) must be
bit-exact; combination weights within 1e-6; float outputs within the
normwise bound max|gpu - oracle| / max|oracle| <= 1e-4 (float32 layers) or
2e-2 (bf16 layers, float32 accumulation).

Every layer is checked element by element: routing and dispatch in full
everywhere; h, y_disp and y in full on the small layers, the GPT-OSS layers
and DeepSeek-R1 decode.  On DeepSeek-R1 prefill (5.8 TFLOP of FFN, beyond
what the oracle finishes in minutes) h and y_disp are compared on a seeded
sample of 1024 tokens (all their k rows) plus every expert's first and last
row and both rows at every 128-row tile boundary, and y on those 1024 tokens.
Beside the normwise bound of each tensor, every row must meet the same bound
scaled by its own largest value."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_layer import (TOL, DeviceLayer, dev_to_np, expert_of_rows, oracle_ffn_rows_by_expert, rel_err,
                             row_errors, widen)

pytestmark = pytest.mark.gpu

W = synth.Workload
SMALL = {
    "toy_fp32": synth.WORKLOADS["toy_fp32"],
    # several 128-row tiles per hot expert, zero-row experts (Zipf skew)
    "bf16_multi_tile": W("bf16_multi_tile", T=512, H=256, I=384, E=8, k=2, R=4, dtype="bf16", seed=11,
                         bias="zipf1.2"),
    # K tails (H = 200 = 3*64 + 8), h column tail (I = 200), odd T
    "bf16_ragged": W("bf16_ragged", T=333, H=200, I=200, E=6, k=3, R=3, dtype="bf16", seed=12, bias="normal0.5"),
    # down-projection N tail (H = 320 -> 192-wide tiles), I = 136, k = 4 over 16 experts
    "bf16_ragged_n": W("bf16_ragged_n", T=257, H=320, I=136, E=16, k=4, R=4, dtype="bf16", seed=13),
    "bf16_one_token": W("bf16_one_token", T=1, H=64, I=64, E=4, k=1, R=2, dtype="bf16", seed=14),
    "f32_top4": W("f32_top4", T=100, H=96, I=160, E=8, k=4, R=2, dtype="f32", seed=15),
    "bf16_top8_e256": W("bf16_top8_e256", T=96, H=128, I=128, E=256, k=8, R=32, dtype="bf16", seed=16),
    # the largest expert count the calls accept, top-8: large dispatch count table
    # (second grid barrier), 1024-expert tile prefix in the GEMMs' shared memory
    "bf16_e1024": W("bf16_e1024", T=2048, H=128, I=192, E=1024, k=8, R=8, dtype="bf16", seed=21),
}


def run_gpu(layer: DeviceLayer, rt=None):
    from token_dispatch_combine_b200 import MoERoundTrip, moe_get_error
    wl = layer.wl
    if rt is None:
        rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, layer.x_dev.dtype, gather=False)
    rt.forward(layer.x_dev, layer.logits_dev, layer.w_gate, layer.w_up, layer.w_down)
    st, bits = moe_get_error()
    assert st == 0 and bits == 0, (st, bits)
    return rt


def check_routing_and_dispatch(layer: DeviceLayer, rt):
    wl = layer.wl
    ids, w = oracle.route(layer.logits, wl.k)
    assert (dev_to_np(rt.topk_ids) == ids).all()
    np.testing.assert_allclose(dev_to_np(rt.topk_w), w, rtol=0, atol=1e-6)
    ref = oracle.dispatch_index(ids, wl.E, wl.R)
    for name in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "slot_to_row", "row_to_slot",
                 "src_expert_counts"):
        got = dev_to_np(getattr(rt.disp, name))
        assert (got == ref[name]).all(), name
    x_disp = None
    if rt.disp.x_disp is not None:  # (index-only dispatch when the gate/up projection gathers)
        x_disp = oracle.dispatch_rows(layer.x, wl.k, ref["slot_to_row"])
        assert (dev_to_np(rt.disp.x_disp) == x_disp).all()
    return ids, w, ref, x_disp


@pytest.mark.parametrize("ffn_tiling", ["single", "pair"], indirect=True)
@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_layer_full_parity(name, ffn_tiling):
    wl = SMALL[name]
    layer = DeviceLayer(wl)
    rt = run_gpu(layer)
    ids, w, ref, x_disp = check_routing_and_dispatch(layer, rt)
    if x_disp is None:
        x_disp = oracle.dispatch_rows(layer.x, wl.k, ref["slot_to_row"])
    n = int(ref["expert_offsets"][-1])
    row_expert = expert_of_rows(ref["expert_offsets"], np.arange(n))
    g, u, d = layer.host_weights(range(wl.E))
    y_ref, a_ref = oracle.ffn_rows(x_disp[:n], row_expert, g, u, d, wl.H, wl.I, want_act=True)
    tol = TOL[wl.dtype]
    assert rel_err(dev_to_np(rt.h)[:n], a_ref) <= tol
    assert rel_err(dev_to_np(rt.y_disp)[:n], y_ref) <= tol
    y = oracle.combine(y_ref, w, ref["slot_to_row"])
    assert rel_err(dev_to_np(rt.y), y) <= tol


# Layers whose FFN is compared on a seeded token sample (and the sample size); all others in full.
SAMPLED_TOKENS = {"dsr1_prefill": 1024}
TILE_ROWS = 128
_EXPECTED = {}  # layer name -> the oracle's rows / tokens and their outputs (shared by both tilings)


def _boundary_rows(offsets: np.ndarray) -> np.ndarray:
    """Every expert's first and last row and both rows at each 128-row tile boundary inside it."""
    rows = []
    for e in range(len(offsets) - 1):
        o0, o1 = int(offsets[e]), int(offsets[e + 1])
        if o1 > o0:
            rows += [o0, o1 - 1]
            for b in range(o0 + TILE_ROWS, o1, TILE_ROWS):
                rows += [b - 1, b]
    return np.asarray(rows, np.int64)


def _expected(name: str, layer: DeviceLayer, w: np.ndarray, ref: dict) -> dict:
    """The oracle's h and y_disp on the rows compared, and y on the tokens compared."""
    if name in _EXPECTED:
        return _EXPECTED[name]
    wl = layer.wl
    n = int(ref["expert_offsets"][-1])
    s2r = ref["slot_to_row"].reshape(wl.T, wl.k)
    if name in SAMPLED_TOKENS:
        rng = np.random.default_rng(wl.seed)
        tokens = np.sort(rng.choice(wl.T, size=SAMPLED_TOKENS[name], replace=False))
        tok_rows = s2r[tokens].ravel()
        rows = np.unique(np.concatenate([tok_rows[tok_rows >= 0], _boundary_rows(ref["expert_offsets"])]))
    else:
        tokens = np.arange(wl.T)
        rows = np.arange(n, dtype=np.int64)
    h, y_disp = oracle_ffn_rows_by_expert(layer, rows, ref["row_to_slot"], ref["expert_offsets"])
    pos = np.full(wl.S, -1, np.int32)  # dispatched row -> its index among the rows compared
    pos[rows] = np.arange(len(rows), dtype=np.int32)
    sub = s2r[tokens]
    y = oracle.combine(y_disp, w[tokens], np.where(sub >= 0, pos[np.maximum(sub, 0)], -1).ravel())
    _EXPECTED[name] = dict(rows=rows, tokens=tokens, h=h, y_disp=y_disp, y=y)
    return _EXPECTED[name]


def _check_rows(what: str, gpu: np.ndarray, ref: np.ndarray, index: np.ndarray, tol: float):
    whole, worst, at = row_errors(gpu, ref)
    print(f"{what}: {len(index)} rows, normwise {whole:.3e}, worst row {worst:.3e} (row {int(index[at])})")
    assert whole <= tol, (what, whole)
    assert worst <= tol, (what, "row", int(index[at]), worst)


@pytest.mark.parametrize("name", ["gptoss_uniform", "gptoss_zipf", "dsr1_decode", "dsr1_prefill"])
def test_full_size_layer(name):
    check_full_size_layer(name)


@pytest.mark.parametrize("ffn_tiling,name", [("single", "gptoss_zipf"), ("pair", "dsr1_decode"),
                                              ("pair", "dsr1_prefill")], indirect=["ffn_tiling"])
def test_full_size_layer_other_tiling(name, ffn_tiling):
    """The full-size layers again with the tile shape that auto does not pick for them."""
    check_full_size_layer(name)


def check_full_size_layer(name):
    """The layer in the form bench.py times (MoERoundTrip's default dispatch: rows through
    x_disp, or gathered by the gate/up projection where that is faster), against the oracle
    element by element."""
    from token_dispatch_combine_b200 import MoERoundTrip
    wl = synth.WORKLOADS[name]
    layer = DeviceLayer(wl)
    rt = run_gpu(layer, MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, layer.x_dev.dtype))
    ids, w, ref, _ = check_routing_and_dispatch(layer, rt)
    exp = _expected(name, layer, w, ref)
    tol = TOL[wl.dtype]
    rows_dev = torch.from_numpy(exp["rows"]).cuda()
    _check_rows("h", dev_to_np(rt.h[rows_dev]), exp["h"], exp["rows"], tol)
    _check_rows("y_disp", dev_to_np(rt.y_disp[rows_dev]), exp["y_disp"], exp["rows"], tol)
    _check_rows("y", dev_to_np(rt.y[torch.from_numpy(exp["tokens"]).cuda()]), exp["y"], exp["tokens"], tol)
    assert torch.isfinite(rt.y.float()).all()  # every token's output, compared or not


def test_single_and_pair_tiles_agree_bit_for_bit():
    """Both tile shapes form the same products in the same K order: h and y_disp
    are identical, including at expert boundaries, half tiles and N tails."""
    from token_dispatch_combine_b200 import MoERoundTrip, moe_set_ffn_tiling
    for wl in (SMALL["bf16_multi_tile"], SMALL["bf16_ragged_n"], synth.WORKLOADS["gptoss_zipf"]):
        layer = DeviceLayer(wl)
        outs = []
        try:
            for mode in (1, 2):
                moe_set_ffn_tiling(mode)
                rt = run_gpu(layer, MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, layer.x_dev.dtype,
                                                 gather=False))
                outs.append([t.view(torch.int16).clone() for t in (rt.h, rt.y_disp, rt.y)])
        finally:
            moe_set_ffn_tiling(0)
        for a, b in zip(*outs):
            assert torch.equal(a, b), wl.name
        del layer, outs
        torch.cuda.empty_cache()


def test_repeated_calls_are_identical():
    wl = SMALL["bf16_multi_tile"]
    layer = DeviceLayer(wl)
    rt = run_gpu(layer)
    first = [dev_to_np(t).copy() for t in (rt.disp.x_disp, rt.h, rt.y_disp, rt.y)]
    run_gpu(layer, rt)  # workspace reused: the control word must have been reset
    for a, t in zip(first, (rt.disp.x_disp, rt.h, rt.y_disp, rt.y)):
        assert (a == dev_to_np(t)).all()


@pytest.mark.parametrize("ffn_tiling", ["single", "pair"], indirect=True)
def test_all_tokens_to_one_expert(ffn_tiling):
    wl = W("one_hot", T=300, H=128, I=128, E=8, k=1, R=2, dtype="bf16", seed=17)
    logits = np.zeros((wl.T, wl.E), np.float32)
    logits[:, 5] = 1.0
    layer = DeviceLayer(wl, logits=logits)
    rt = run_gpu(layer)
    _, _, ref, _ = check_routing_and_dispatch(layer, rt)
    assert ref["expert_counts"].tolist() == [0, 0, 0, 0, 0, 300, 0, 0]
    x = widen(layer.x)
    # y = FFN_5(x) for every token; compare with the oracle row by row
    g, u, d = layer.host_weights([5])
    y_ref = oracle.ffn_rows(layer.x, np.full(wl.T, 5, np.int32), g, u, d, wl.H, wl.I)
    assert rel_err(dev_to_np(rt.y), y_ref) <= TOL["bf16"]
    assert np.isfinite(x).all()


def test_identity_experts_combine_reproduces_input():
    """combine(dispatch(x)) with y_disp := x_disp and weights summing to one gives x back."""
    from token_dispatch_combine_b200 import MoERoundTrip, moe_combine
    wl = W("ident", T=200, H=64, I=64, E=8, k=4, R=4, dtype="f32", seed=18)
    layer = DeviceLayer(wl)
    rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, torch.float32, gather=False)
    rt.route(layer.logits_dev)
    rt.dispatch(layer.x_dev)
    y = torch.empty_like(layer.x_dev)
    moe_combine(rt.disp.x_disp, rt.topk_w, rt.disp.slot_to_row, y)
    np.testing.assert_allclose(dev_to_np(y), layer.x, rtol=0, atol=1e-6 * np.abs(layer.x).max())


@pytest.mark.parametrize("graphs", [True, False])
def test_host_pipeline_matches_forward(graphs):
    """MoEHostPipeline (overlapped upload/compute/download; each batch a CUDA graph replay,
    or eager calls) gives, per batch, exactly what a plain forward of that batch gives."""
    from token_dispatch_combine_b200 import MoEHostPipeline, MoERoundTrip
    wl = W("pipe", T=300, H=256, I=384, E=8, k=2, R=4, dtype="bf16", seed=19)
    layer = DeviceLayer(wl)
    rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, torch.bfloat16)
    batches, want = [], []
    for b in range(5):
        x = torch.randn(wl.T, wl.H, device="cuda").to(torch.bfloat16)
        lg = torch.randn(wl.T, wl.E, device="cuda")
        want.append(rt.forward(x, lg, layer.w_gate, layer.w_up, layer.w_down).clone())
        batches.append((x.view(torch.int16).cpu().pin_memory(), lg.cpu().pin_memory(),
                        torch.empty(wl.T, wl.H, dtype=torch.int16).pin_memory()))
    torch.cuda.synchronize()
    pipe = MoEHostPipeline(rt, layer.w_gate, layer.w_up, layer.w_down, graphs=graphs)
    pipe.run(batches).synchronize()
    torch.cuda.synchronize()
    for (_, _, yh), y in zip(batches, want):
        assert torch.equal(yh, y.view(torch.int16).cpu())


@pytest.mark.parametrize("dtype,ffn_tiling", [("bf16", "single"), ("bf16", "pair"), ("f32", "auto")],
                         indirect=["ffn_tiling"])
def test_graph_replay_matches_forward(dtype, ffn_tiling):
    """The whole round trip captured in a CUDA graph gives the eager result, and a
    replay after new inputs are written gives that new batch's result."""
    from token_dispatch_combine_b200 import MoERoundTrip
    wl = W("graph", T=200, H=256, I=256, E=8, k=2, R=4, dtype=dtype, seed=20)
    layer = DeviceLayer(wl)
    dt = layer.x_dev.dtype
    rt = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, dt)
    x = layer.x_dev.clone()
    lg = layer.logits_dev.clone()
    want1 = rt.forward(x, lg, layer.w_gate, layer.w_up, layer.w_down).clone()
    g = rt.capture(x, lg, layer.w_gate, layer.w_up, layer.w_down)
    rt.y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(rt.y, want1)
    x2 = torch.randn_like(x.float()).to(dt)
    lg2 = torch.randn_like(lg)
    want2 = MoERoundTrip(wl.T, wl.H, wl.I, wl.E, wl.k, wl.R, dt).forward(x2, lg2, layer.w_gate, layer.w_up,
                                                                          layer.w_down).clone()
    x.copy_(x2)
    lg.copy_(lg2)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(rt.y, want2)
