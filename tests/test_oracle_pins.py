"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against something independent: hand-worked
examples (tests/golden), exact rational arithmetic, closed forms, brute force
over all subsets, a different algorithm for the same result, or invariants the
pages state.  All of it runs on the CPU.
"""
import heapq
import itertools
import json
import math
import os
from collections import Counter
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_routing_gate_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------------------------------------
# rounding
# ------------------------------------------------------------------------------------------------

def test_round_bf16_ties_and_library():
    # hand cases: spacing of bf16 at 1.0 is 2^-7
    assert O.round_bf16(1 + 2.0 ** -8) == 1.0                       # midpoint -> even (1.0)
    assert O.round_bf16(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6         # midpoint -> even mantissa
    assert O.round_bf16(1 + 2.0 ** -8 + 2.0 ** -30) == 1 + 2.0 ** -7  # just above the midpoint
    assert O.round_bf16(-3.0) == -3.0 and O.round_bf16(0.0) == 0.0
    # torch's fp32 -> bf16 conversion (round to nearest even) on fp32 inputs
    v = torch.randn(100000, generator=torch.Generator().manual_seed(1), dtype=torch.float32) * 7
    ref = v.to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_bf16(v.numpy()), ref)


def _round_f32_exact(q: Fraction) -> float:
    """Correctly rounded fp32 of an exact rational, by comparing the two fp32 neighbours exactly."""
    f = np.float32(float(q))
    cands = [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - q),
                                     int(np.frombuffer(np.float32(c).tobytes(), np.uint32)[0]) & 1))
    return float(best)


# ------------------------------------------------------------------------------------------------
# logits and affinities
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("general_fp32", [True, False])
def test_logits_exact_rational(general_fp32):
    cfg = W.CONFIGS["tiny"].replace(gate_general_fp32=general_fp32)
    x, wg, _, off = W.make_router_inputs(cfg)
    x = x.float().numpy().astype(np.float64)
    wg = wg.numpy().astype(np.float64)
    l = O.router_logits(x, wg)
    rng = np.random.default_rng(5)
    for _ in range(40):
        t, e = int(rng.integers(cfg.T)), int(rng.integers(cfg.n_experts))
        exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(x[t], wg[e]))
        assert float(l[t, e]) == _round_f32_exact(exact)


def test_affinity_closed_forms():
    l = np.array([0.0, 50.0, -50.0, 2.0, -2.0, 1e-3], np.float32)
    s = O.affinity(l, "sigmoid")
    assert s[0] == np.float32(0.5)
    assert s[1] == np.float32(1.0)
    assert s[2] == np.float32(math.exp(-50.0) / (1 + math.exp(-50.0)))
    assert abs(float(s[3]) + float(s[4]) - 1.0) <= 2 ** -24          # sigma(l) + sigma(-l) = 1
    sp = O.affinity(l, "sqrtsoftplus")
    assert sp[0] == np.float32(math.sqrt(math.log(2.0)))              # softplus(0) = ln 2
    assert sp[1] == np.float32(math.sqrt(50.0 + math.log1p(math.exp(-50.0))))
    assert abs(float(sp[2]) / math.exp(-25.0) - 1.0) < 1e-6          # sqrt(log1p(e^-50)) ~ e^-25
    # sqrt(softplus(l)) is increasing and positive
    grid = np.linspace(-20, 20, 4001).astype(np.float32)
    g = O.affinity(grid, "sqrtsoftplus").astype(np.float64)
    assert np.all(g > 0) and np.all(np.diff(g) >= 0)
    sm = O.affinity(np.zeros((3, 8), np.float32), "softmax")
    assert np.all(sm == np.float32(1 / 8))
    sm = O.affinity(np.array([[0.0, math.log(3.0)]], np.float32), "softmax")
    assert np.allclose(sm, [[0.25, 0.75]], rtol=1e-6)


# ------------------------------------------------------------------------------------------------
# selection
# ------------------------------------------------------------------------------------------------

def _brute_force_select(b, G, g, k, has_bias):
    """Best group set by total group score over all C(G, g) sets, then the best k-subset of the kept
    experts by total score over all subsets.  Group score: max over pairs of b_i + b_j (with bias), or
    max b (without)."""
    E = len(b)
    per = E // G
    if G > 1:
        def gscore(gi):
            members = [float(b[gi * per + i]) for i in range(per)]
            if has_bias:
                return max(float(np.float32(np.float32(members[i]) + np.float32(members[j])))
                           for i in range(per) for j in range(per) if i != j)
            return max(members)
        gs = [gscore(gi) for gi in range(G)]
        best_groups = max(itertools.combinations(range(G), g), key=lambda c: sum(gs[i] for i in c))
        cand = [e for e in range(E) if e // per in best_groups]
    else:
        best_groups = (0,)
        cand = list(range(E))
    best = max(itertools.combinations(cand, k), key=lambda c: sum(float(b[e]) for e in c))
    return set(best), set(best_groups)


@pytest.mark.parametrize("has_bias", [True, False])
def test_selection_brute_force_tiny(has_bias):
    cfg = W.CONFIGS["tiny"]
    rng = np.random.default_rng(11)
    for _ in range(64):
        b = rng.normal(0.5, 0.1, cfg.n_experts).astype(np.float32)
        e, kept, _, _ = O.select_experts(b, cfg.n_groups, cfg.n_limited_groups, cfg.topk, has_bias)
        want, want_groups = _brute_force_select(b, cfg.n_groups, cfg.n_limited_groups, cfg.topk, has_bias)
        assert set(e.tolist()) == want
        assert set(kept.tolist()) == want_groups
        assert np.all(np.diff(b[e].astype(np.float64)) <= 0)   # descending score order


def test_selection_no_groups_is_plain_sort():
    rng = np.random.default_rng(3)
    for E, k in [(16, 4), (384, 6), (256, 8)]:
        b = rng.normal(size=E).astype(np.float32)
        b[::7] = b[0]   # plant exact ties
        e, _, _, _ = O.select_experts(b, 1, 1, k, True)
        want = [i for _, i in sorted((-float(v), i) for i, v in enumerate(b))][:k]
        assert e.tolist() == want


def test_gate_hand_examples():
    for ex in _golden("gate_hand_examples.json")["examples"]:
        s = np.array(ex["s"], np.float32)
        bias = None if ex["bias"] is None else np.array(ex["bias"], np.float32)
        b = s if bias is None else (s + bias).astype(np.float32)
        e, kept, _, _ = O.select_experts(b, ex["n_groups"], ex["n_limited_groups"], ex["topk"], bias is not None)
        assert e.tolist() == ex["indices"], ex["name"]
        assert sorted(kept.tolist()) == sorted(ex["kept_groups"]), ex["name"]
        w = O.gate_weights(s[e], True, ex["route_scale"])
        assert np.allclose(w, ex["weights"], rtol=2e-7, atol=0), ex["name"]


def test_gate_invariants_all_configs_small():
    for name in ["tiny", "v3_prefill", "v4_skew"]:
        cfg = W.CONFIGS[name].replace(T=48)
        x, wg, bias, off = W.make_router_inputs(cfg)
        hp = O.Hyper.of(cfg)
        g = O.gate(x.float().numpy(), wg.numpy(), hp,
                   None if bias is None else bias.numpy(), None if off is None else off.numpy())
        per = cfg.n_experts // cfg.n_groups
        for t in range(cfg.T):
            idx = g.indices[t]
            assert len(set(idx.tolist())) == cfg.topk                       # k distinct experts
            if cfg.n_groups > 1:
                assert set((idx // per).tolist()) <= set(g.kept_groups[t].tolist())   # inside kept groups
            w = g.weights[t].astype(np.float64)
            assert abs(w.sum() / cfg.route_scale - 1.0) < 1e-6                # renormalised then scaled
            # the bias never enters the weights: they are the unbiased scores, renormalised
            s = g.scores[t, idx].astype(np.float64)
            assert np.allclose(w, s / s.sum() * cfg.route_scale, rtol=1e-6)


def test_bias_shift_invariance():
    # a bias equal for every expert changes nothing; the bias only perturbs the selection
    cfg = W.CONFIGS["tiny"]
    x, wg, bias, _ = W.make_router_inputs(cfg)
    hp = O.Hyper.of(cfg)
    g0 = O.gate(x.float().numpy(), wg.numpy(), hp, np.zeros(cfg.n_experts, np.float32))
    g1 = O.gate(x.float().numpy(), wg.numpy(), hp, np.full(cfg.n_experts, 0.25, np.float32))
    assert np.array_equal(g0.indices, g1.indices)
    assert np.array_equal(g0.weights, g1.weights)
    # a large bias on one expert forces it into every token's selection, weights still unbiased
    big = np.zeros(cfg.n_experts, np.float32)
    big[5] = 10.0
    g2 = O.gate(x.float().numpy(), wg.numpy(), hp, big)
    assert np.all((g2.indices == 5).any(axis=1))
    assert np.all(g2.indices[:, 0] == 5)
    assert np.all(g2.weights.sum(axis=1) <= cfg.route_scale * (1 + 1e-6))


def test_softmax_not_renormalised():
    hp = O.Hyper(16, 1, 1, 4, "softmax", 2.0)
    rng = np.random.default_rng(0)
    x = O.round_bf16(rng.normal(size=(8, 32)))
    wg = rng.normal(0, 0.2, (16, 32)).astype(np.float32)
    g = O.gate(x, wg, hp)
    for t in range(8):
        assert np.allclose(g.weights[t], g.scores[t, g.indices[t]] * 2.0, rtol=1e-7)
        assert g.scores[t].astype(np.float64).sum() == pytest.approx(1.0, rel=1e-6)


def test_hash_gate_uses_table_order():
    rng = np.random.default_rng(1)
    m, n, k, d = 50, 16, 3, 32
    table = np.stack([rng.permutation(n)[:k] for _ in range(m)]).astype(np.int32)
    ids = rng.integers(0, m, 20)
    x = O.round_bf16(rng.normal(size=(20, d)))
    wg = O.round_bf16(rng.normal(0, 0.1, (n, d))).astype(np.float32)
    idx, w = O.hash_gate(ids, table, x, wg, route_scale=1.5)
    assert np.array_equal(idx, table[ids])
    assert np.allclose(w.astype(np.float64).sum(axis=1), 1.5, rtol=1e-6)
    s = 1 / (1 + np.exp(-(x @ wg.astype(np.float64).T)))
    for t in range(20):
        sel = s[t, table[ids[t]]]
        assert np.allclose(w[t], sel / sel.sum() * 1.5, rtol=1e-6)


# ------------------------------------------------------------------------------------------------
# tid2eid
# ------------------------------------------------------------------------------------------------

def test_tid2eid_hand_examples():
    for ex in _golden("tid2eid_hand_examples.json")["examples"]:
        p = np.array(ex["p32"], np.float64) / 32.0
        table, f = O.build_tid2eid(p, ex["n"], ex["k"])
        assert table.tolist() == ex["rows"], ex["name"]
        assert (f * 32).tolist() == ex["f32"], ex["name"]
        assert O.balance(f) == (ex["max_vio"], ex["min_vio"]), ex["name"]


def _greedy_with_heap(p, n, k):
    """The same greedy rule on a binary heap keyed by (load, expert): an independent data structure."""
    order = sorted(range(len(p)), key=lambda i: (-p[i], i))
    heap = [(0.0, j) for j in range(n)]
    heapq.heapify(heap)
    table = np.zeros((len(p), k), np.int32)
    for i in order:
        picked = [heapq.heappop(heap) for _ in range(k)]
        table[i] = [j for _, j in picked]
        q = p[i] / k
        for load, j in picked:
            heapq.heappush(heap, (load + q, j))
    f = np.zeros(n)
    for load, j in heap:
        f[j] = load
    return table, f


def test_tid2eid_matches_heap_greedy_page_setting():
    # the page's own setting: m=80000 tokens, 128 experts, top-4, p ~ 1/(10+i)
    m, n, k = 80000, 128, 4
    p = 1.0 / (10.0 + np.arange(m))
    p /= p.sum()
    t1, f1 = O.build_tid2eid(p, n, k)
    t2, f2 = _greedy_with_heap(p.tolist(), n, k)
    assert np.array_equal(t1, t2)
    assert np.array_equal(f1, f2)
    mx, mn = O.balance(f1)
    assert 0.0 <= mx < 1e-3 and -1e-3 < mn <= 0.0     # near-perfect balance, as the page reports
    assert abs(f1.sum() - 1.0) < 1e-12


@pytest.mark.slow
def test_tid2eid_extreme_case_closed_form():
    # the hash layer's vocabulary: p_1 / k far above 1/n, the page's "extreme case".  The k experts
    # that take the most frequent token are never again among the lightest, so their load is exactly
    # p_1 / k and max_vio = n p_1 / k - 1.
    cfg = W.CONFIGS["hash"]
    p = W.token_frequencies(cfg)
    n, k = cfg.n_experts, cfg.topk
    assert p[0] / k > 1.0 / n
    table, f = O.build_tid2eid(p, n, k)
    assert sorted(table[0].tolist()) == list(range(k))
    assert np.all(f[:k] == p[0] / k)
    mx, mn = O.balance(f)
    assert mx == f.max() * n - 1 and mx == p[0] / k * n - 1
    assert abs(mx - 4.6871) < 1e-4
    assert np.all([len(set(r)) == k for r in table[:2000].tolist()])
    assert abs(f.sum() - 1.0) < 1e-12
    # every other token avoids the k heavy experts
    assert not np.isin(table[1:], np.arange(k)).any()


# ------------------------------------------------------------------------------------------------
# dispatch
# ------------------------------------------------------------------------------------------------

def test_dispatch_invariants():
    rng = np.random.default_rng(2)
    T, E, k = 200, 16, 4
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    counts, offsets, row_of_slot, tok_of_row = O.dispatch(idx, E)
    c = Counter(idx.reshape(-1).tolist())
    assert counts.tolist() == [c.get(e, 0) for e in range(E)]
    assert counts.sum() == T * k and offsets[-1] == T * k and offsets[0] == 0
    assert sorted(row_of_slot.tolist()) == list(range(T * k))           # a bijection
    for s in range(T * k):
        t, e, r = s // k, idx[s // k, s % k], row_of_slot[s]
        assert offsets[e] <= r < offsets[e + 1]                          # row inside its expert's block
        assert tok_of_row[r] == t
    for e in range(E):
        blk = tok_of_row[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(blk) > 0)                                 # stable: token order kept


# ------------------------------------------------------------------------------------------------
# experts and combine: an identity-like layer
# ------------------------------------------------------------------------------------------------

def identity_like_expert(d, inter, scale):
    """w1 = [+I; -I; 0], w3 = all rows e_{d-1}, w2 = scale [I | -I]: since silu(u) - silu(-u) = u,
    expert(x)_i = scale * x_i for i < d-1 when x_{d-1} = 1 (up to the bf16 rounding of h)."""
    n = d - 1
    assert inter >= 2 * n
    w1 = np.zeros((inter, d))
    w1[np.arange(n), np.arange(n)] = 1.0
    w1[n + np.arange(n), np.arange(n)] = -1.0
    w3 = np.zeros((inter, d))
    w3[:, d - 1] = 1.0
    w2 = np.zeros((d, inter))
    w2[np.arange(n), np.arange(n)] = scale
    w2[np.arange(n), n + np.arange(n)] = -scale
    return w1, w3, w2


def _identity_bound(x, scale):
    # bf16 unit roundoff u = 2^-8.  h+- = bf16(silu(+-x)) err <= u|silu(+-x)|, and |silu(x)| + |silu(-x)| = |x|,
    # so |s(h+ - h-) - s x| <= u s|x|; rounding o to bf16 adds u (s|x| + u s|x|).
    u = 2.0 ** -8
    return scale * np.abs(x) * (u + u * (1 + u)) * 1.001


def test_identity_like_expert():
    rng = np.random.default_rng(4)
    d, inter = 64, 128
    x = O.round_bf16(rng.normal(size=(32, d)) * 2)
    x[:, d - 1] = 1.0
    for scale in [0.25, 1.0, 3.0]:
        o = O.swiglu_expert(x, *identity_like_expert(d, inter, scale))
        assert np.all(o[:, d - 1] == 0)
        err = np.abs(o[:, :d - 1] - scale * x[:, :d - 1])
        assert np.all(err <= _identity_bound(x[:, :d - 1], scale))


def test_identity_like_layer_recovers_weighted_sum():
    cfg = W.CONFIGS["tiny"].replace(dim=64)
    rng = np.random.default_rng(6)
    d, E = cfg.dim, cfg.n_experts
    x = O.round_bf16(rng.normal(size=(cfg.T, d)))
    x[:, d - 1] = 1.0
    wg = rng.normal(0, 0.1, (E, d)).astype(np.float32)
    bias = rng.normal(0, 0.01, E).astype(np.float32)
    scales = {e: (e + 1) / 4.0 for e in range(E)}
    scales[E] = 0.5                                      # shared expert
    experts = {e: identity_like_expert(d, cfg.inter_dim, s) for e, s in scales.items()}
    hp = O.Hyper.of(cfg)
    y, idx, w, counts = O.moe_forward(x, hp, lambda e: experts[e], wg, bias)
    factor = np.array([sum(float(w[t, j]) * scales[int(idx[t, j])] for j in range(cfg.topk)) + scales[E]
                       for t in range(cfg.T)])
    want = factor[:, None] * x[:, :d - 1]
    err = np.abs(y[:, :d - 1] - want)
    # each expert output is within 2u s_e|x| of s_e x (see _identity_bound); fp32 products and sums add
    # ~2^-24; the final bf16 rounding adds u|y|.  So |y - F x| <= (2u + u(1 + 2u)) F|x|, u = 2^-8.
    u = 2.0 ** -8
    bound = np.abs(want) * (2 * u + u * (1 + 2 * u)) * 1.001 + 1e-12
    assert np.all(err <= bound)
    assert np.all(y[:, d - 1] == 0)
    assert counts.sum() == cfg.T * cfg.topk
    # routing to a wrong expert would move the factor by at least 1/4 of a slot weight
    assert np.min(np.abs(np.diff(sorted(scales[e] for e in range(E))))) >= 0.25


def test_expert_matches_fp64_library_matmul():
    # the special case of a library GEMM: torch fp64 matmuls on the CPU, rounding points applied after
    cfg = W.CONFIGS["tiny"]
    x, _, _, _ = W.make_router_inputs(cfg)
    w1, w3, w2 = W.expert_weights(cfg, 3)
    xd, a, b, c = (t.double() for t in (x, w1, w3, w2))
    zg = (xd @ a.T).float().double()
    zv = (xd @ b.T).float().double()
    h = (torch.nn.functional.silu(zg) * zv).float().bfloat16().double()
    ref = (h @ c.T).float().bfloat16().double().numpy()
    got = O.swiglu_expert(xd.numpy(), a.numpy(), b.numpy(), c.numpy())
    # double rounding fp64->fp32->bf16 on the torch side may differ by one bf16 ulp on rare elements
    ulp = np.abs(ref) * 2.0 ** -7
    assert np.all(np.abs(got - ref) <= ulp)
    assert np.mean(got == ref) > 0.99


def test_logit_offset_is_an_extra_input_column():
    # adding c_e to every logit is the same as appending a constant-1 input column with router weights c:
    # one fp32 rounding of x.W + c versus two (x.W rounded first, then the sum), so they differ by at most
    # half an fp32 ulp of x.W plus half an ulp of the result each
    cfg = W.CONFIGS["v4_skew"].replace(T=32, dim=256)
    x, wg, _, off = W.make_router_inputs(cfg)
    xd, wd, c = x.double().numpy(), wg.double().numpy(), off.double().numpy()
    got = O.router_logits(xd, wd, off.numpy()).astype(np.float64)
    plain = O.router_logits(xd, wd)
    aug = O.router_logits(np.hstack([xd, np.ones((cfg.T, 1))]), np.hstack([wd, c[:, None]])).astype(np.float64)
    ulp = lambda v: np.spacing(np.abs(v).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(got - aug) <= 0.5 * ulp(plain) + ulp(aug))
    assert np.abs(got - plain.astype(np.float64)).max() > 0.5
    # a large offset on one expert puts it first for every token, with its affinity taken after the offset
    big = np.zeros(cfg.n_experts, np.float32)
    big[3] = 20.0
    g = O.gate(xd, wd, O.Hyper.of(cfg), None, big)
    assert np.all(g.indices[:, 0] == 3)
    assert np.all(g.scores[:, 3] > 4.4)      # sqrt(softplus(l + 20)) ~ sqrt(20 + l), |l| < 1


def test_swiglu_clamp_closed_forms():
    # identity-like expert: o_i = s (silu(min(x_i, L)) - silu(min(-x_i, L))) * clamp(x_{d-1}, -L, L)
    d, inter, s, L = 64, 128, 0.5, 10.0
    w1, w3, w2 = identity_like_expert(d, inter, s)
    rng = np.random.default_rng(12)
    x = O.round_bf16(rng.uniform(-40, 40, size=(64, d)))
    x[:, d - 1] = 1.0
    big = O.swiglu_expert(x, w1, w3, w2, limit=1e30)
    assert np.array_equal(big, O.swiglu_expert(x, w1, w3, w2))          # no clamp in reach: unchanged
    o = O.swiglu_expert(x, w1, w3, w2, limit=L)[:, :d - 1]
    xv = x[:, :d - 1]
    u = 2.0 ** -8
    small = np.abs(xv) < L - 0.5
    assert np.all(np.abs(o[small] - s * xv[small]) <= s * np.abs(xv[small]) * 2.1 * u)   # inside: identity
    # outside the limit the gate branch saturates: |o| -> s * L * sigmoid(L) (the other branch ~ 0)
    sat = s * L / (1.0 + math.exp(-L))
    far = np.abs(xv) > L + 2
    assert np.all(np.abs(np.abs(o[far]) - sat) <= sat * 2.1 * u + s * 1e-3)
    assert np.all(np.sign(o[far]) == np.sign(xv[far]))
    # the value branch is clamped too: x_{d-1} = 20 enters as 10
    x2 = x.copy()
    x2[:, d - 1] = 20.0
    o2 = O.swiglu_expert(x2, w1, w3, w2, limit=L)[:, :d - 1]
    assert np.all(np.abs(o2[small] - 10 * s * xv[small]) <= 10 * s * np.abs(xv[small]) * 2.1 * u)


def test_weight_in_expert_matches_weight_in_combine():
    # handing each row its routing weight inside the expert computes the same layer, up to rounding
    cfg = W.CONFIGS["tiny"].replace(dim=64)
    rng = np.random.default_rng(13)
    d, E = cfg.dim, cfg.n_experts
    x = O.round_bf16(rng.normal(size=(cfg.T, d)))
    x[:, d - 1] = 1.0
    wg = rng.normal(0, 0.1, (E, d)).astype(np.float32)
    scales = {e: (e + 1) / 4.0 for e in range(E)}
    scales[E] = 0.5
    experts = {e: identity_like_expert(d, cfg.inter_dim, sc) for e, sc in scales.items()}
    hp = O.Hyper.of(cfg)
    y_out, idx, w, _ = O.moe_forward(x, hp, lambda e: experts[e], wg)
    y_in, idx2, w2, _ = O.moe_forward(x, hp, lambda e: experts[e], wg, weight_in_expert=True)
    assert np.array_equal(idx, idx2) and np.array_equal(w, w2)
    factor = np.array([sum(float(w[t, j]) * scales[int(idx[t, j])] for j in range(cfg.topk)) + scales[E]
                       for t in range(cfg.T)])
    want = factor[:, None] * x[:, :d - 1]
    u = 2.0 ** -8
    for y in (y_out, y_in):
        assert np.all(np.abs(y[:, :d - 1] - want) <= np.abs(want) * (2 * u + u * (1 + 2 * u)) * 1.001 + 1e-12)
    assert not np.array_equal(y_out, y_in)       # different rounding points, same layer


# ------------------------------------------------------------------------------------------------
# next rows: n-gram hash routing, randomised greedy, bias update
# ------------------------------------------------------------------------------------------------

def test_ngram_hand_examples():
    ex = _golden("ngram_hand_examples.json")
    pairs = np.array(ex["pairs"])
    got = O.ngram_experts(pairs[:, 0], pairs[:, 1], ex["primes"], ex["n"])
    assert got.tolist() == ex["experts"]
    assert O.primes_above(10, 2) == ex["primes"]


def test_ngram_balances_the_extreme_case():
    # "How was DeepSeek V4's tid2eid derived?", section "An extreme case": where the top token alone
    # exceeds the balanced level (no 1-gram table gets max_vio below p_1 n / k - 1 = 4.69 here), hashing
    # 2-grams spreads the load.  Ids are a seeded permutation of frequency ranks, as in a vocabulary
    # whose ids do not follow frequency: with id 0 the most frequent token, the printed hash sends all k
    # slots of every pair (0, b) to the one expert b mod n, the degenerate case the section's caveat
    # about a bad hash covers.
    cfg = W.CONFIGS["hash"]
    p = W.token_frequencies(cfg)
    rng = np.random.default_rng(21)
    primes = O.primes_above(cfg.hash_vocab, cfg.topk)
    assert len(set(primes)) == cfg.topk and min(primes) > cfg.hash_vocab
    bound_1gram = p[0] * cfg.n_experts / cfg.topk - 1.0
    perm = rng.permutation(cfg.hash_vocab)
    zipf_ids = perm[rng.choice(cfg.hash_vocab, size=400001, p=p)]
    uniform_ids = rng.integers(0, cfg.hash_vocab, size=400001)
    for ids, limit in ((zipf_ids, 0.25 * bound_1gram), (uniform_ids, 0.1)):
        e = O.ngram_experts(ids[:-1], ids[1:], primes, cfg.n_experts)
        assert e.shape == (ids.size - 1, cfg.topk)
        load = np.bincount(e.reshape(-1), minlength=cfg.n_experts) / e.size
        mx, mn = O.balance(load)
        assert mx < limit and mn > -0.5, (mx, mn, limit)
    assert O.balance(O.build_tid2eid(p, cfg.n_experts, cfg.topk)[1])[0] >= bound_1gram - 1e-9


def test_best_tid2eid_keeps_least_max_vio():
    m, n, k = 3000, 32, 3
    p = 1.0 / (5.0 + np.arange(m))
    p /= p.sum()
    rng = np.random.default_rng(4)
    orders = [rng.permutation(m) for _ in range(5)]
    table, f, r = O.best_tid2eid(p, n, k, orders)
    vios = [O.balance(O.build_tid2eid(p, n, k, o)[1])[0] for o in orders]
    assert vios[r] == min(vios) and r == int(np.argmin(vios))
    t0, f0 = O.build_tid2eid(p, n, k, orders[r])
    assert np.array_equal(table, t0) and np.array_equal(f, f0)
    # the descending order as the only run is the plain greedy
    td, fd, rd = O.best_tid2eid(p, n, k, [np.argsort(-p, kind="stable")])
    assert rd == 0 and np.array_equal(td, O.build_tid2eid(p, n, k)[0])


def test_bias_update_balances_a_routing_loop():
    # "From One Giant FFN...", section 6: nudging biases against the load must reduce the imbalance of
    # a fixed biased router over steps (a wrong sign would amplify it)
    rng = np.random.default_rng(7)
    T, E, k = 512, 32, 4
    skew = np.linspace(-0.3, 0.3, E)
    s = (rng.random((T, E)) * 0.2 + 0.4 + skew).astype(np.float32)
    bias = np.zeros(E, np.float32)

    def loads(b):
        sel = np.argsort(-(s + b), axis=1, kind="stable")[:, :k]
        return np.bincount(sel.reshape(-1), minlength=E)

    var0 = np.var(loads(bias))
    for _ in range(400):
        c = loads(bias)
        nb = O.update_bias(bias, c, T, k, 0.002)
        over, under = c * E > T * k, c * E < T * k
        assert np.all(nb[over] < bias[over]) and np.all(nb[under] > bias[under])
        assert np.all(nb[~over & ~under] == bias[~over & ~under])
        bias = nb
    assert np.var(loads(bias)) < 0.1 * var0


# ------------------------------------------------------------------------------------------------
# MXFP4 expert weights ("From One Giant FFN to 384 Tiny Experts", section 11.6)
# ------------------------------------------------------------------------------------------------

def test_e2m1_and_ue8m0_match_an_independent_decoder():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    codes = np.arange(16, dtype=np.uint8)
    want = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = O.e2m1_value(codes)
    assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))
    s = np.arange(255, dtype=np.uint8)
    assert np.array_equal(O.ue8m0_value(s), s.view(ml_dtypes.float8_e8m0fnu).astype(np.float64))
    assert np.isnan(O.ue8m0_value(255))


def test_mxfp4_hand_examples():
    ex = _golden("mxfp4_hand_examples.json")
    for row in ex["rows"]:
        v = O.mxfp4_dequant(np.array([row["packed"]], np.uint8), np.array([row["scales"]], np.uint8))
        assert v.tolist() == [row["values"]], row["working"]
    neg0 = O.mxfp4_dequant(np.array([ex["rows"][0]["packed"]], np.uint8), np.array([[127, 125]], np.uint8))
    assert np.signbit(neg0[0, 2])


def test_mxfp4_decoded_weights_are_bf16_exact():
    # every E2M1 value times a scale in [2, 252] is a normal bf16 number, so an MXFP4 expert computes
    # exactly as the bf16 expert holding the decoded weights
    codes = np.arange(256, dtype=np.uint8).reshape(8, 32)
    for s in (2, 100, 127, 200, 252):
        v = O.mxfp4_dequant(codes, np.full((8, 2), s, np.uint8))
        assert np.array_equal(O.round_bf16(v), v)
        nz = np.abs(v[v != 0])
        assert nz.min() >= 2.0 ** -126 and nz.max() < 2.0 ** 128


def test_mxfp4_generator_covers_every_code():
    pk, sc = W.mxfp4_matrix(64, 256, 0.01, 5, 0, 0)
    pk = pk.numpy()
    codes = np.concatenate([(pk & 0xF).ravel(), (pk >> 4).ravel()])
    assert set(np.unique(codes).tolist()) == set(range(16))
    v = O.mxfp4_dequant(pk, sc.numpy())
    assert 0.003 < v.std() < 0.03


def test_best_tid2eid_ties_keep_the_earlier_run():
    m, n, k = 400, 16, 2
    p = 1.0 / (2.0 + np.arange(m))
    p /= p.sum()
    rng = np.random.default_rng(9)
    a, b = rng.permutation(m), rng.permutation(m)
    va = O.balance(O.build_tid2eid(p, n, k, a)[1])[0]
    vb = O.balance(O.build_tid2eid(p, n, k, b)[1])[0]
    best, worse = (a, b) if va <= vb else (b, a)
    assert O.best_tid2eid(p, n, k, [worse, best, best])[2] == 1
    assert O.best_tid2eid(p, n, k, [best, worse, best])[2] == 0


def _exact_swiglu_1x1(x: float, w: float, limit):
    """bf16 output of a 1x1 SwiGLU expert (w1 = w3 = w2 = [[1]]) on input x with row weight w, from
    50-digit decimal arithmetic (an exp independent of numpy's) and one rounding to bf16 of h; the
    down projection by 1 is exact.  Returns None when h lies too near a bf16 rounding boundary."""
    import decimal
    ctx = decimal.Context(prec=50)
    g = v = decimal.Decimal(float(np.float32(x)))
    if limit is not None:
        L = decimal.Decimal(limit)
        g = min(g, L)
        v = max(min(v, L), -L)
    a = ctx.multiply(ctx.multiply(ctx.divide(g, ctx.add(1, ctx.exp(-g))), v), decimal.Decimal(float(np.float32(w))))
    f = float(a)
    r = float(O.round_bf16(f))
    up = float(O.round_bf16(f * (1 + 1e-12))) if f else r
    dn = float(O.round_bf16(f * (1 - 1e-12))) if f else r
    return r if up == dn == r else None


@pytest.mark.parametrize("limit", [None, 2.0])
def test_swiglu_single_rounding_against_decimal(limit):
    # "From One Giant FFN...", sections 1 and 11.4 and "DeepSeek V4.1 - Add shared" (weight inside the
    # expert): h = bf16(silu(min(g, L)) * clip(v, -L, L) * w), rounded once
    rng = np.random.default_rng(31)
    xs = rng.uniform(-6.0, 6.0, 400).astype(np.float32)
    ws = rng.uniform(0.05, 3.0, 400).astype(np.float32)
    one = np.ones((1, 1))
    got = O.swiglu_expert(xs.astype(np.float64)[:, None], one, one, one, limit=limit, row_weight=ws)[:, 0]
    checked = 0
    for x, w, y in zip(xs, ws, got):
        want = _exact_swiglu_1x1(float(x), float(w), limit)
        if want is None:
            continue
        assert y == want, (x, w, y, want)
        checked += 1
    assert checked > 380


def test_primes_above_are_strictly_greater_than_m():
    # the 2-gram hash takes one prime q_j > m per choice (tid2eid page, "An extreme case"); m itself
    # may be prime, and must then be skipped.  Against a sieve of Eratosthenes.
    limit = 400
    sieve = np.ones(limit, bool)
    sieve[:2] = False
    for i in range(2, int(limit ** 0.5) + 1):
        if sieve[i]:
            sieve[i * i::i] = False
    primes = np.nonzero(sieve)[0]
    for m in (1, 2, 7, 13, 97, 100, 211):
        want = [int(q) for q in primes[primes > m][:5]]
        assert O.primes_above(m, 5) == want, m


def test_combine_rounds_its_fp32_sum_once_to_bf16():
    # the layer output is the fp32 accumulator cast to the activations' bf16 (moe-forward:
    # y.type_as(x)), round to nearest, ties to even.  One token, one feature, one routed expert whose
    # bf16 output is 1.0: the fp32 sums below are exact, and only the final cast changes them.
    cases = [  # (weight, shared term, expected bf16 output)
        (1.0 + 2.0 ** -10, 0.0, 1.0),                 # below half an ulp of bf16 at 1.0: down
        (1.0 + 2.0 ** -8, 0.0, 1.0),                  # exactly half an ulp: tie to the even 1.0
        (1.0 + 3 * 2.0 ** -8, 0.0, 1.0 + 2.0 ** -6),  # tie between 1+2^-7 and 1+2^-6: to even
        (1.0, 2.0 ** -8 + 2.0 ** -12, 1.0 + 2.0 ** -7),  # just above half an ulp: up
    ]
    for w, sh, want in cases:
        y = O.combine(1, 1, np.array([[0]]), np.array([[w]], np.float32), {0: {0: np.array([1.0])}},
                      np.array([[sh]]))
        assert float(y[0, 0]) == want, (w, sh, float(y[0, 0]))


# ------------------------------------------------------------------------------------------------
# FP8 (E4M3) activations with UE8M0 block scales ("From One Giant FFN to 384 Tiny Experts", 11.6)
# ------------------------------------------------------------------------------------------------
def test_e4m3_decode_matches_ml_dtypes():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    codes = np.arange(256, dtype=np.uint8)
    want = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = O.e4m3_value(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.array_equal(got[~np.isnan(got)], want[~np.isnan(want)])
    assert np.array_equal(np.signbit(got[~np.isnan(got)]), np.signbit(want[~np.isnan(want)]))


def test_e4m3_rounding_matches_ml_dtypes():
    # nearest value, ties to the even mantissa, signed zeros: each block holds 448 first (so its
    # scale is 2^0 and the other 31 elements are rounded as they are), against ml_dtypes' own
    # conversion of random values in range, every midpoint between neighbouring E4M3 values, the
    # table itself and the subnormals
    ml_dtypes = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(11)
    table = O.e4m3_value(np.arange(127))
    mids = (table[1:] + table[:-1]) / 2
    q = np.concatenate([rng.uniform(-448, 448, 31000), rng.normal(0, 1, 31000), rng.normal(0, 2 ** -7, 31000),
                        mids, -mids, table, -table, [0.0, -0.0, 2.0 ** -10, -2.0 ** -10, 3 * 2.0 ** -11]])
    q = np.concatenate([q, np.zeros((-len(q)) % 31)])
    blocks = np.concatenate([np.full((len(q) // 31, 1), 448.0), q.reshape(-1, 31)], axis=1)
    codes, scales = O.quantize_e4m3_block(blocks)
    assert np.all(scales == 127)
    want = q.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(codes[:, 1:].reshape(-1), want)


def test_mx_block_hand_examples():
    ex = _golden("mx_e4m3_hand_examples.json")
    for b in ex["blocks"]:
        v = np.zeros((1, 32))
        for pos, val in b["values"].items():
            v[0, int(pos)] = -0.0 if val == "-0" else float(val)
        codes, scales = O.quantize_e4m3_block(v)
        assert scales.shape == (1, 1) and int(scales[0, 0]) == b["scale"], b["why"]
        for pos, code in b["codes"].items():
            assert int(codes[0, int(pos)]) == code, b["why"]


def test_mx_block_scale_is_the_least_that_does_not_saturate():
    rng = np.random.default_rng(12)
    v = rng.normal(0, 1, (40, 256)) * np.exp2(rng.integers(-30, 30, (40, 1)))
    v[3, 32:64] = 0.0
    codes, scales = O.quantize_e4m3_block(v)
    amax = np.abs(v).reshape(40, 8, 32).max(axis=2)
    e = scales.astype(np.int64) - 127
    nz = amax > 0
    assert np.all(448.0 * np.exp2(e[nz]) >= amax[nz])            # nothing saturates
    assert np.all(448.0 * np.exp2(e[nz] - 1) < amax[nz])         # and no smaller scale would do
    assert scales[3, 1] == 0 and np.all(codes[3, 32:64] == 0)
    # the blocks run along rows: quantising the transpose gives other scales
    assert not np.array_equal(O.quantize_e4m3_block(v[:32, :32].T.copy())[1][:, 0], scales[:32, 0])
    # rounding error within half an E4M3 step: 2^-4 relative for normals, 2^-10 * scale below 2^-6
    d = O.e4m3_block_dequant(codes, scales)
    sc = np.repeat(np.exp2(e), 32, axis=1)
    q = np.abs(v) / sc
    bound = np.where(q >= 2.0 ** -6, 2.0 ** -4 * np.abs(v), 2.0 ** -10 * sc)
    assert np.all(np.abs(d - v) <= bound * (1 + 1e-12))
    # values already on the grid come back unchanged (a block whose maximum rounded down to
    # 448 * 2^(e-1) takes the smaller scale the second time, on which the same values lie)
    assert np.array_equal(O.e4m3_block_dequant(*O.quantize_e4m3_block(d)), d)


def test_mx_expert_identity_like_layer():
    # The identity-like expert (silu(u) - silu(-u) = u) on FP8 activations.  x lies on the E4M3 grid
    # of its block scale 2^-6 (its largest entry is 448 * 2^-6), so quantising x is exact and the two
    # projections give exactly +x_i and -x_i; lane d-1 holds a constant 1 that feeds every value
    # branch.  h = (silu(x), silu(-x)) is quantised in blocks of 32 along I, so the output
    # o_i = s (hq_i - hq_{n+i}) differs from s x_i by at most the two quantisation errors of h (half an
    # E4M3 step each: 2^-4 of the value, or 2^-10 of the block scale below 2^-6 of it) plus one bf16
    # rounding -- and, h's quantisation being coarser than bf16, beyond bf16 rounding somewhere (an
    # expert that skipped quantising h would not).
    d = n = 32
    I = 2 * n
    rng = np.random.default_rng(13)
    grid = O.e4m3_value(np.arange(1, 127))
    x = rng.choice(grid, size=(24, d)) * np.exp2(-6.0) * rng.choice([-1.0, 1.0], size=(24, d))
    x[:, 0] = 448.0 * np.exp2(-6.0)
    x[:, d - 1] = 1.0
    assert np.array_equal(O.e4m3_block_dequant(*O.quantize_e4m3_block(x)), x)
    s = 0.5
    w1 = np.zeros((I, d)); w3 = np.zeros((I, d)); w2 = np.zeros((d, I))
    data = np.arange(d - 1)                     # lanes 0 .. d-2 carry data
    w1[data, data] = 1.0
    w1[n + data, data] = -1.0
    w3[:, d - 1] = 1.0
    w2[data, data] = s
    w2[data, n + data] = -s
    o = O.mx_swiglu_expert(x, w1, w3, w2)
    xd = x[:, data]
    h_hi, h_lo = O.silu(xd), O.silu(-xd)        # h_i and h_{n+i}; the rest of h is silu(0) = 0
    scale = np.exp2(np.ceil(np.log2(np.maximum(np.abs(h_hi).max(axis=1), np.abs(h_lo).max(axis=1)) / 448.0)))
    half_step = 2.0 ** -4 * (np.abs(h_hi) + np.abs(h_lo)) + 2.0 ** -10 * 2 * scale[:, None] * 2
    err = np.abs(o[:, data] - s * xd)
    assert np.all(err <= s * half_step + 2.0 ** -8 * np.abs(o[:, data]))
    assert np.any(err > 2.0 ** -8 * np.abs(s * xd))                   # the quantisation of h is visible
    assert np.all(o[:, d - 1] == 0)
