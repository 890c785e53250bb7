"""Pins for the CPU oracle: worked examples from the pages, closed forms,
library routines and a dense brute-force MoE -- nothing here re-calls the
oracle to produce its own expected values."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# Worked example: "EP: Partition Experts and Route Tokens", "Send tokens to
# experts and return their results" (Top-1, weight one, A1->E0, A2->E2,
# B1->E1, B2->E2, E0/E1 on GPU 0, E2/E3 on GPU 1).
# ---------------------------------------------------------------------------
def test_worked_example_route_and_dispatch():
    g = _load("ep_worked_example.json")
    ex = g["expected"]
    logits = np.array(g["logits"], np.float32)
    ids, w = oracle.route(logits, g["k"])
    assert ids.tolist() == ex["topk_ids"]
    assert w.tolist() == ex["topk_w"]  # exactly one: Top-1 weight fixed to one
    idx = oracle.dispatch_index(ids, g["E"], g["R"])
    for key in ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "row_to_slot",
                "slot_to_row", "src_expert_counts"):
        assert idx[key].tolist() == ex[key], key
    tokens = g["tokens"]
    EL = g["E"] // g["R"]
    crossing = [tokens[t] for t in range(g["T"])
                if oracle.src_rank(t, g["T"], g["R"]) != ids[t, 0] // EL]
    assert crossing == ex["cross_rank_tokens"]
    e2 = idx["row_to_slot"][idx["expert_offsets"][2]:idx["expert_offsets"][3]]
    assert [tokens[s] for s in e2] == ex["expert2_rows_in_order"]


def test_worked_example_results_return_in_original_order():
    g = _load("ep_worked_example.json")
    ids, w = oracle.route(np.array(g["logits"], np.float32), 1)
    idx = oracle.dispatch_index(ids, g["E"], g["R"])
    # Each dispatched row's "expert output" is a marker naming (expert, token);
    # combine must put it back at the token's own position.
    T, H = g["T"], 2
    y_disp = np.zeros((T, H))
    for row in range(T):
        s = idx["row_to_slot"][row]
        y_disp[row] = [ids[s, 0], s]
    y = oracle.combine(y_disp, w, idx["slot_to_row"])
    assert y.tolist() == [[0, 0], [2, 1], [1, 2], [2, 3]]  # A1<-E0, A2<-E2, B1<-E1, B2<-E2


def test_top2_weights_and_combine():
    g = _load("top2_combine.json")
    ids, w = oracle.route(np.array(g["logits"], np.float32), g["k"])
    assert ids.tolist() == g["expected"]["topk_ids"]
    np.testing.assert_allclose(w, g["expected"]["topk_w"], atol=g["expected"]["weight_tol"], rtol=0)
    idx = oracle.dispatch_index(ids, g["E"], 2)
    y_disp = np.zeros((2, 4))
    y_disp[idx["slot_to_row"][0]] = g["u0"]
    y_disp[idx["slot_to_row"][1]] = g["u2"]
    y = oracle.combine(y_disp, w, idx["slot_to_row"])
    np.testing.assert_allclose(y[0], g["y"], atol=1e-6, rtol=0)


def test_imbalance_example():
    g = _load("imbalance.json")
    logits = np.zeros((g["T"], g["E"]), np.float32)
    logits[np.arange(g["T"]), g["choice"]] = 1.0
    ids, _ = oracle.route(logits, 1)
    idx = oracle.dispatch_index(ids, g["E"], g["R"])
    assert idx["expert_counts"].tolist() == g["expected"]["expert_counts"]
    assert idx["rank_counts"].tolist() == g["expected"]["rank_counts"]


def test_masked_sum_ep8():
    g = _load("masked_sum_ep8.json")
    E, R, k = g["E"], g["R"], g["k"]
    logits = np.full((1, E), -30.0, np.float32)
    logits[0, g["experts"]] = np.log(g["affinities"])
    ids, w = oracle.route(logits, k)
    assert ids.tolist() == g["expected"]["topk_ids"]
    np.testing.assert_allclose(w[0], g["affinities"], atol=1e-7, rtol=0)
    idx = oracle.dispatch_index(ids, E, R)
    assert idx["rank_counts"].tolist() == g["expected"]["rank_counts"]
    EL = E // R
    assert sorted({int(e) // EL for e in ids[0]}) == g["expected"]["contributing_ranks"]
    # Per-rank partial outputs (masked to the rank's experts) add up to the full output.
    rng = np.random.default_rng(0)
    y_disp = rng.standard_normal((k, 5))
    full = oracle.combine(y_disp, w, idx["slot_to_row"])
    parts = []
    for r in range(R):
        wr = np.where((ids // EL) == r, w, 0.0).astype(np.float32)
        parts.append(oracle.combine(y_disp, wr, idx["slot_to_row"]))
        if r not in g["expected"]["contributing_ranks"]:
            assert not parts[-1].any()
    np.testing.assert_allclose(sum(parts), full, rtol=0, atol=1e-12)
    # The masking form's own functions: a contributing rank holds exactly its expert's output
    # times its affinity, every other rank exactly zero, and the reduction gives the output.
    part = oracle.rank_partials(y_disp, w, ids, idx["slot_to_row"], E, R)
    rows = idx["slot_to_row"]
    for j, e in enumerate(ids[0]):
        r = int(e) // EL
        np.testing.assert_array_equal(part[r, 0], float(w[0, j]) * y_disp[rows[j]])
    for r in range(R):
        if r not in g["expected"]["contributing_ranks"]:
            assert not part[r].any()
    np.testing.assert_allclose(oracle.reduce_ranks(part), full, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Route: tie rule, signed zero, and agreement with a library sort.
# ---------------------------------------------------------------------------
def test_route_ties_lower_id_first_and_signed_zero():
    logits = np.array([[1.0, 3.0, 3.0, -1.0],
                       [0.0, -0.0, 0.0, -0.0],
                       [-0.0, 0.0, -5.0, 2.0]], np.float32)
    ids, w = oracle.route(logits, 3)
    assert ids.tolist() == [[1, 2, 0], [0, 1, 2], [3, 0, 1]]
    np.testing.assert_allclose(w[1], [1 / 3] * 3, atol=1e-7)


def test_route_k1_weight_is_exactly_one():
    rng = np.random.default_rng(1)
    _, w = oracle.route(rng.standard_normal((50, 7)).astype(np.float32), 1)
    assert (w == 1.0).all()


@pytest.mark.parametrize("T,E,k", [(1, 4, 4), (37, 8, 2), (64, 32, 4), (16, 256, 8), (5, 3, 1)])
def test_route_matches_lexsort(T, E, k):
    rng = np.random.default_rng(T * 1000 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[:, : E // 2] = np.round(logits[:, : E // 2])  # plenty of ties
    ids, w = oracle.route(logits, k)
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))  # key: logit desc, then id asc
        assert ids[t].tolist() == order[:k].tolist()
        sel = logits[t, order[:k]].astype(np.float64)
        ref = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()  # softmax of the selected logits
        np.testing.assert_allclose(w[t], ref, rtol=0, atol=2e-7)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)


# ---------------------------------------------------------------------------
# Dispatch index: invariants and the stable-sort special case.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,E,k,R", [(1, 4, 1, 2), (64, 4, 1, 2), (127, 8, 2, 4), (300, 32, 4, 8),
                                     (200, 256, 8, 32), (33, 5, 3, 5)])
def test_dispatch_index_invariants(T, E, k, R):
    rng = np.random.default_rng(T + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[:, 0] += 3.0  # one hot expert
    ids, _ = oracle.route(logits, k)
    d = oracle.dispatch_index(ids, E, R)
    S = T * k
    s2r, r2s = d["slot_to_row"], d["row_to_slot"]
    assert sorted(s2r.tolist()) == list(range(S))  # bijection onto [0, S)
    assert (r2s[s2r] == np.arange(S)).all()  # inverse
    assert d["expert_counts"].sum() == S
    assert d["expert_counts"].tolist() == np.bincount(ids.ravel(), minlength=E).tolist()
    assert d["expert_offsets"].tolist() == [0] + np.cumsum(d["expert_counts"]).tolist()
    EL = E // R
    assert d["rank_counts"].tolist() == d["expert_counts"].reshape(R, EL).sum(1).tolist()
    assert d["rank_offsets"].tolist() == d["expert_offsets"][::EL].tolist()
    # the stable sort of the flat ids by expert is the row order
    assert r2s.tolist() == np.argsort(ids.ravel(), kind="stable").tolist()
    for e in range(E):
        seg = r2s[d["expert_offsets"][e]:d["expert_offsets"][e + 1]]
        assert (ids.ravel()[seg] == e).all()
        assert (np.diff(seg // k) > 0).all()  # strictly increasing token index
    src = (np.arange(T) * R) // T
    want = np.zeros((R, E), np.int64)
    np.add.at(want, (np.repeat(src, k), ids.ravel()), 1)
    assert (d["src_expert_counts"] == want).all()
    assert (d["src_expert_counts"].sum(0) == d["expert_counts"]).all()


def test_src_rank_matches_toy_layer_statement():
    # toy layer: tokens 0..31 'from rank 0', 32..63 'from rank 1'
    assert [oracle.src_rank(t, 64, 2) for t in range(64)] == [0] * 32 + [1] * 32


def test_dispatch_index_drops_out_of_range_ids():
    ids = np.array([[0, 5], [1, -1], [3, 2]], np.int32)
    d = oracle.dispatch_index(ids, 4, 2)
    assert d["dropped"] == 2
    assert d["expert_counts"].tolist() == [1, 1, 1, 1]
    assert d["slot_to_row"].tolist() == [0, -1, 1, -1, 3, 2]
    assert d["row_to_slot"].tolist() == [0, 2, 5, 4, -1, -1]


def test_dispatch_rows_is_gather_by_inverse_permutation():
    rng = np.random.default_rng(3)
    T, k, E, H = 40, 3, 6, 24
    ids, _ = oracle.route(rng.standard_normal((T, E)).astype(np.float32), k)
    d = oracle.dispatch_index(ids, E, 3)
    x = rng.integers(0, 65535, (T, H), dtype=np.uint16)
    xd = oracle.dispatch_rows(x, k, d["slot_to_row"])
    order = np.argsort(ids.ravel(), kind="stable")
    assert (xd == x[order // k]).all()


# ---------------------------------------------------------------------------
# FFN: closed forms of SwiGLU and a dense brute-force MoE.
# ---------------------------------------------------------------------------
def _one(v):
    return np.array(v, np.float32).reshape(1, 1, 1)


def test_swiglu_closed_forms():
    x = np.ones((1, 1), np.float32)
    # y = Wd * SiLU(Wg x) * (Wu x); SiLU(1) = 1 / (1 + e^-1)
    y = oracle.ffn_rows(x, np.zeros(1, np.int32), _one(1.0), _one(2.0), _one(3.0), 1, 1)
    assert y[0, 0] == pytest.approx(4.386351471780029, abs=1e-14)  # 6 / (1 + e^-1)
    # swapping gate and up changes the answer: SiLU(2) * 1 = 2 / (1 + e^-2)
    y = oracle.ffn_rows(x, np.zeros(1, np.int32), _one(2.0), _one(1.0), _one(1.0), 1, 1)
    assert y[0, 0] == pytest.approx(1.7615941559557650, abs=1e-14)
    # SiLU(0) = 0; SiLU(z) -> z for large z; SiLU(z) -> 0 for very negative z
    y = oracle.ffn_rows(x, np.zeros(1, np.int32), _one(0.0), _one(5.0), _one(1.0), 1, 1)
    assert y[0, 0] == 0.0
    y = oracle.ffn_rows(x, np.zeros(1, np.int32), _one(40.0), _one(1.0), _one(1.0), 1, 1)
    assert y[0, 0] == pytest.approx(40.0, rel=1e-15)
    y = oracle.ffn_rows(x, np.zeros(1, np.int32), _one(-40.0), _one(1.0), _one(1.0), 1, 1)
    assert abs(y[0, 0]) < 1e-15


def _dense_moe(x, logits, k, wg, wu, wd):
    """Every expert on every token, masked by the top-k choice (float64 numpy)."""
    T, E = logits.shape
    y = np.zeros((T, x.shape[1]))
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))[:k]
        sel = logits[t, order].astype(np.float64)
        p = np.exp(sel - sel.max())
        p /= p.sum()
        mask_w = np.zeros(E)
        mask_w[order] = p
        for e in range(E):
            g = x[t] @ wg[e]
            u = x[t] @ wu[e]
            out = (g / (1.0 + np.exp(-g)) * u) @ wd[e]
            y[t] += mask_w[e] * out  # zero for unselected experts
    return y


@pytest.mark.parametrize("T,H,I,E,k,R", [(9, 8, 12, 4, 1, 2), (16, 32, 64, 8, 2, 4), (13, 24, 40, 6, 3, 3),
                                         (7, 16, 8, 8, 8, 2)])
def test_round_trip_equals_dense_masked_moe(T, H, I, E, k, R):
    rng = np.random.default_rng(T * H + I)
    x = rng.standard_normal((T, H)).astype(np.float32)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wg = (rng.standard_normal((E, H, I)) / math.sqrt(H)).astype(np.float32)
    wu = (rng.standard_normal((E, H, I)) / math.sqrt(H)).astype(np.float32)
    wd = (rng.standard_normal((E, I, H)) / math.sqrt(I)).astype(np.float32)
    out = oracle.round_trip(x, logits, k, E, R, wg, wu, wd)
    ref = _dense_moe(x.astype(np.float64), logits, k, wg.astype(np.float64), wu.astype(np.float64),
                     wd.astype(np.float64))
    np.testing.assert_allclose(out["y"], ref, rtol=1e-5, atol=1e-6)  # weights are float32-rounded
    # per-rank partial sums (masked to each rank's experts) add up to y
    EL = E // R
    parts = sum(oracle.combine(out["y_disp"], np.where(out["ids"] // EL == r, out["w"], 0).astype(np.float32),
                               out["slot_to_row"]) for r in range(R))
    np.testing.assert_allclose(parts, out["y"], rtol=0, atol=1e-12)


def _dense_moe_rank(x, logits, k, wg, wu, wd, r, EL):
    """Rank r's output in the masking form, by brute force: every token through every expert
    of rank r, each masked by the token's top-k softmax weight for that expert (float64)."""
    T, E = logits.shape
    y = np.zeros((T, x.shape[1]))
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))[:k]
        sel = logits[t, order].astype(np.float64)
        p = np.exp(sel - sel.max())
        p /= p.sum()
        mask_w = np.zeros(E)
        mask_w[order] = p
        for e in range(r * EL, (r + 1) * EL):
            g = x[t] @ wg[e]
            u = x[t] @ wu[e]
            y[t] += mask_w[e] * ((g / (1.0 + np.exp(-g)) * u) @ wd[e])
    return y


@pytest.mark.parametrize("T,H,I,E,k,R", [(12, 8, 12, 4, 2, 2), (9, 16, 24, 8, 3, 4), (7, 8, 16, 6, 6, 3)])
def test_rank_partials_equal_dense_masked_moe_per_rank(T, H, I, E, k, R):
    """Each rank's partial output of the masking form equals that rank's experts run densely
    over all tokens with the top-k mask, and the rank-ordered reduction equals the round trip."""
    rng = np.random.default_rng(T * 7 + H + E)
    x = rng.standard_normal((T, H)).astype(np.float32)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wg = (rng.standard_normal((E, H, I)) / math.sqrt(H)).astype(np.float32)
    wu = (rng.standard_normal((E, H, I)) / math.sqrt(H)).astype(np.float32)
    wd = (rng.standard_normal((E, I, H)) / math.sqrt(I)).astype(np.float32)
    out = oracle.round_trip(x, logits, k, E, R, wg, wu, wd)
    part = oracle.rank_partials(out["y_disp"], out["w"], out["ids"], out["slot_to_row"], E, R)
    assert part.shape == (R, T, H)
    for r in range(R):
        ref = _dense_moe_rank(x.astype(np.float64), logits, k, wg.astype(np.float64), wu.astype(np.float64),
                              wd.astype(np.float64), r, E // R)
        np.testing.assert_allclose(part[r], ref, rtol=1e-5, atol=1e-6)  # weights are float32-rounded
    np.testing.assert_allclose(oracle.reduce_ranks(part), out["y"], rtol=0, atol=1e-12)


def test_ep_plan_worked_example_top1():
    """The pages' Top-1 round trip as two source ranks: who sends what where, and what each
    destination receives (A2 goes to GPU 1, B1 to GPU 0, E2 receives A2 and B2)."""
    g = _load("ep_exchange.json")
    E, R, c = g["E"], g["R"], g["top1"]
    ex = c["expected"]
    plans = []
    for s in range(R):
        ids = np.array(c["ids"][s], np.int32)
        p = oracle.ep_plan(ids, np.ones_like(ids, np.float32), E, R)
        for key in ("send_counts", "send_offsets", "slot_send_row", "row_token", "row_ids"):
            assert p[key].tolist() == ex[key][s], (s, key)
        plans.append(p)
    # destination d receives sources 0..R-1 in turn: rank 0 gets A1, B1; rank 1 gets A2, B2
    names = "AB"
    for d in range(R):
        got = []
        for s in range(R):
            lo, hi = plans[s]["send_offsets"][d], plans[s]["send_offsets"][d + 1]
            got += [[names[s], int(t)] for t in plans[s]["row_token"][lo:hi]]
        assert got == ex["received_tokens"][d]


def test_ep_plan_top2_shares_input_delivery():
    """A2's two results come from two GPUs (one row to each); A3's two experts share GPU 1,
    so its row goes there once and carries both local experts: 3 rows for 4 choices."""
    g = _load("ep_exchange.json")
    c = g["top2_shared"]
    ex = c["expected"]
    E, R = g["E"], g["R"]
    logits = np.full((2, E), -30.0, np.float32)
    logits[0, 0], logits[0, 2] = math.log(7 / 3), 0.0
    logits[1, 2], logits[1, 3] = math.log(3 / 2), 0.0
    ids, w = oracle.route(logits, c["k"])
    assert ids.tolist() == c["ids"]
    np.testing.assert_allclose(w, c["w"], atol=1e-6, rtol=0)
    p = oracle.ep_plan(ids, w, E, R)
    for key in ("send_counts", "send_offsets", "slot_send_row", "row_token", "row_ids"):
        assert p[key].tolist() == ex[key], key
    np.testing.assert_allclose(p["row_w"], ex["row_w"], atol=1e-6, rtol=0)
    assert len(p["row_token"]) == ex["rows_sent_for_four_choices"]


def _ep_case(sizes, H, I, E, k, R, seed, bias=0.0):
    rng = np.random.default_rng(seed)
    xs = [rng.standard_normal((T, H)).astype(np.float32) for T in sizes]
    lg = [rng.standard_normal((T, E)).astype(np.float32) for T in sizes]
    for a in lg:
        a[:, :E // R] += bias  # experts of rank 0 hot: many tokens share delivery there
    wg = (rng.standard_normal((E, H, I)) / math.sqrt(H)).astype(np.float32)
    wu = (rng.standard_normal((E, H, I)) / math.sqrt(H)).astype(np.float32)
    wd = (rng.standard_normal((E, I, H)) / math.sqrt(I)).astype(np.float32)
    return xs, lg, wg, wu, wd


@pytest.mark.parametrize("sizes,H,I,E,k,R,bias", [((5, 7), 8, 12, 4, 2, 2, 0.0), ((9, 3, 6), 16, 8, 6, 3, 3, 1.5),
                                                  ((4, 4, 4, 4), 8, 8, 8, 4, 4, 2.0), ((6, 0), 8, 8, 4, 1, 2, 0.0)])
def test_ep_round_trip_equals_single_gpu_round_trip(sizes, H, I, E, k, R, bias):
    """The exchange over R source ranks gives each token the output the one-GPU round trip gives
    it (tokens of all ranks concatenated in rank order), and the plan's invariants hold: one row
    per (token, destination holding any of its experts), every choice carried exactly once."""
    xs, lg, wg, wu, wd = _ep_case(sizes, H, I, E, k, R, seed=sum(sizes) + E, bias=bias)
    ep = oracle.ep_round_trip(xs, lg, k, E, R, wg, wu, wd)
    ref = oracle.round_trip(np.concatenate(xs), np.concatenate(lg), k, E, R, wg, wu, wd)
    np.testing.assert_allclose(np.concatenate(ep["y"]), ref["y"], rtol=0, atol=1e-12 * max(1.0, np.abs(ref["y"]).max()))
    EL = E // R
    for s, (p, (ids, w)) in enumerate(zip(ep["plans"], ep["routes"])):
        pairs = {(t, int(e) // EL) for t in range(ids.shape[0]) for e in ids[t]}
        assert int(p["send_offsets"][-1]) == len(pairs)
        carried = sorted((int(p["row_token"][r]), int(p["row_ids"][r, i]) + EL * d)
                         for d in range(R) for r in range(p["send_offsets"][d], p["send_offsets"][d + 1])
                         for i in range(k) if p["row_ids"][r, i] >= 0)
        assert carried == sorted((t, int(e)) for t in range(ids.shape[0]) for e in ids[t])


def test_ffn_bf16_weights_widen_exactly():
    rng = np.random.default_rng(5)
    H, I, E = 16, 24, 2
    wg = rng.standard_normal((E, H, I)).astype(np.float32)
    wu = rng.standard_normal((E, H, I)).astype(np.float32)
    wd = rng.standard_normal((E, I, H)).astype(np.float32)
    to_bf = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)  # truncation: exactly representable
    from_bf = lambda b: (b.astype(np.uint32) << 16).view(np.float32)
    x = to_bf(rng.standard_normal((3, H)).astype(np.float32))
    e = np.array([1, 0, 1], np.int32)
    y_b = oracle.ffn_rows(x, e, to_bf(wg), to_bf(wu), to_bf(wd), H, I)
    y_f = oracle.ffn_rows(from_bf(x), e, from_bf(to_bf(wg)), from_bf(to_bf(wu)), from_bf(to_bf(wd)), H, I)
    assert (y_b == y_f).all()


def test_identity_experts_reproduce_input():
    rng = np.random.default_rng(11)
    for k in (1, 2, 4):
        T, E, H = 50, 8, 16
        x = rng.standard_normal((T, H))
        ids, w = oracle.route(rng.standard_normal((T, E)).astype(np.float32), k)
        d = oracle.dispatch_index(ids, E, 4)
        xd = oracle.dispatch_rows(x, k, d["slot_to_row"])  # identity experts: y_disp := x_disp
        y = oracle.combine(xd, w, d["slot_to_row"])
        if k == 1:
            assert (y == x).all()
        else:
            np.testing.assert_allclose(y, x, rtol=0, atol=1e-6 * np.abs(x).max())


# ---------------------------------------------------------------------------
# Router affinities: "Expert Parallelism (EP)", "Router Weights" -- every token
# scored against all E experts, logits = x W_r^T + bias.
# ---------------------------------------------------------------------------
def test_router_logits_hand_example():
    # x = [[1, 2], [3, -1]], router rows e0 = (1, 0), e1 = (1, 1), e2 = (0, -2),
    # bias (0.5, 0, -1): worked by hand
    x = np.array([[1, 2], [3, -1]], np.float32)
    w = np.array([[1, 0], [1, 1], [0, -2]], np.float32)
    lg = oracle.router_logits(x, w, [0.5, 0.0, -1.0])
    assert lg.tolist() == [[1.5, 3.0, -5.0], [3.5, 2.0, 1.0]]


def test_router_logits_one_hot_rows_select_columns():
    # a one-hot router row picks one activation column: catches transposed or
    # shifted indices
    rng = np.random.default_rng(3)
    T, H, E = 7, 11, 5
    x = rng.standard_normal((T, H)).astype(np.float32)
    cols = [4, 0, 10, 4, 7]
    w = np.zeros((E, H), np.float32)
    for e, c in enumerate(cols):
        w[e, c] = 1.0
    lg = oracle.router_logits(x, w)
    assert (lg == x[:, cols]).all()


def test_router_logits_bias_only_and_bf16_widening():
    # zero activations give the bias; bf16 bits widen exactly (1.5, -2, 0.25)
    lg = oracle.router_logits(np.zeros((2, 3), np.float32), np.ones((4, 3), np.float32), [1, -2, 0.25, 0])
    assert lg.tolist() == [[1.0, -2.0, 0.25, 0.0]] * 2
    xb = np.array([[0x3FC0, 0xC000, 0x3E80]], np.uint16)    # 1.5, -2, 0.25
    wb = np.array([[0x3F80, 0x3F80, 0x4080]], np.uint16)    # 1, 1, 4
    assert oracle.router_logits(xb, wb).tolist() == [[1.5 - 2.0 + 1.0]]


def test_router_then_route_reproduces_worked_example():
    # identity router (H = E): the logits are the activations, so routing the
    # worked example's logits through the router gives the page's choices
    g = _load("ep_worked_example.json")
    x = np.array(g["logits"], np.float32)
    lg = oracle.router_logits(x, np.eye(g["E"], dtype=np.float32))
    ids, w = oracle.route(lg, g["k"])
    assert ids.tolist() == g["expected"]["topk_ids"]
    assert w.tolist() == g["expected"]["topk_w"]


# ---------------------------------------------------------------- EPLB (expert placement with replicas)
# "什么是专家并行（Expert Parallelism）？", 工作机制 / 边界与常见误解 (third point): a balancer
# redistributes hot and cold experts over the GPUs.  The expected values below are worked by hand
# from the reading stated in the oracle (greedy replica counts, even integer split of an expert's
# load over its replicas, heaviest share first onto the least-loaded rank with a free slot).

def test_eplb_hand_example_one_hot_expert():
    # loads [8,1,...,1], 2 ranks x 5 slots: both extra replicas go to expert 0 (8/1, then 8/2 > 1);
    # shares 3,3,2 then seven 1s; placement r0,r1,r0 (tie),r1,r1,r0 (tie),r1,r0 (tie),r1,r0 (r1 full)
    p = oracle.eplb_plan([8, 1, 1, 1, 1, 1, 1, 1], 2, 5)
    assert p["phys_to_logical"].tolist() == [0, 0, 3, 5, 7, 0, 1, 2, 4, 6]
    assert p["replica_offsets"].tolist() == [0, 3, 4, 5, 6, 7, 8, 9, 10]
    assert p["replicas"].tolist() == [0, 5, 1, 6, 7, 2, 8, 3, 9, 4]
    assert p["rank_load"].tolist() == [8, 7]
    # the static layout of the pages would put experts 0-3 on rank 0: loads 11 and 4
    ids = np.array([[0], [0], [0], [1], [0], [9]], np.int32)
    phys = oracle.eplb_remap(ids, 8, p["replica_offsets"], p["replicas"])
    # token t goes to replica t mod 3 of expert 0 (phys 0, 5, 1), expert 1 has one replica, 9 is no expert
    assert phys.ravel().tolist() == [0, 5, 1, 6, 5, -1]


def test_eplb_equal_loads_without_extra_slots_alternate_ranks():
    # 8 experts, 2 ranks x 4 slots, equal loads: no replicas; experts in id order alternate ranks
    p = oracle.eplb_plan([5] * 8, 2, 4)
    assert p["phys_to_logical"].tolist() == [0, 2, 4, 6, 1, 3, 5, 7]
    assert p["replica_offsets"].tolist() == list(range(9))
    assert p["rank_load"].tolist() == [20, 20]


def test_eplb_remainders_go_to_the_first_replicas():
    # one expert of load 7 over 3 slots on 1 rank: shares 3, 2, 2 (7 = 3 + 2 + 2)
    p = oracle.eplb_plan([7], 1, 3)
    assert p["replica_offsets"].tolist() == [0, 3]
    assert p["replicas"].tolist() == [0, 1, 2]
    assert p["rank_load"].tolist() == [7]
    # two experts 10 and 4 on 2 ranks x 2 slots: extras to 10 (10/1 > 4, then 10/2 = 5 > 4);
    # shares 4, 3, 3 (expert 0) and 4 (expert 1); order (0,0,4) -> r0 slot 0, (1,0,4) -> r1 slot 2,
    # (0,1,3) -> r0 slot 1 (tie 4/4), (0,2,3) -> r1 slot 3
    p = oracle.eplb_plan([10, 4], 2, 2)
    assert p["replica_offsets"].tolist() == [0, 3, 4]
    assert p["replicas"].tolist() == [0, 1, 3, 2]
    assert p["phys_to_logical"].tolist() == [0, 0, 1, 0]
    assert p["rank_load"].tolist() == [7, 7]


@pytest.mark.parametrize("E,R,slots,seed", [(32, 8, 5, 1), (256, 32, 9, 2), (20, 4, 6, 3), (7, 3, 3, 4)])
def test_eplb_plan_invariants(E, R, slots, seed):
    rng = np.random.default_rng(seed)
    load = (rng.zipf(1.3, E) * 17).astype(np.int64) % 5000
    p = oracle.eplb_plan(load, R, slots)
    P = R * slots
    p2l, off, reps = p["phys_to_logical"], p["replica_offsets"], p["replicas"]
    n = np.diff(off)
    assert n.min() >= 1 and n.sum() == P and off[0] == 0
    assert sorted(reps.tolist()) == list(range(P))             # every physical slot used once
    for e in range(E):
        assert (p2l[reps[off[e]:off[e + 1]]] == e).all()          # replicas point back to their expert
    assert np.bincount(p2l, minlength=E).tolist() == n.tolist()
    # greedy replica counts: no expert holding an extra replica would have less load per replica
    # than another expert would with one more replica
    for a in range(E):
        if n[a] > 1:
            for b in range(E):
                assert load[a] * n[b] >= load[b] * (n[a] - 1)
    # the expected rank loads add up to the total; the plan never loads a rank above the static
    # layout's heaviest rank
    assert p["rank_load"].sum() == load.sum()
    static = load[: (E // R) * R].reshape(R, -1).sum(1).max() if E % R == 0 else None
    if static is not None:
        assert p["rank_load"].max() <= static
