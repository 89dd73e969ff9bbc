"""Parity of the CUDA library (called through its C ABI) with the CPU oracle, on a B200.

Small cases span several tiles and ragged tails and are compared element by element; the five
synthetic layers are run at full size in the launch configuration the benchmark times, with
routing compared for every token and layer outputs for a seeded sample of tokens.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_routing_gate_b200 import build as B
from mixture_experts_routing_gate_b200 import workloads as W
from parity import (assert_outputs_close, compare_routing, expert_fetcher, np64, oracle_by_expert, oracle_gate_of,
                    rounding_slack)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    B.build()
    from mixture_experts_routing_gate_b200 import moe
    return moe


def _gate_gpu(M, cfg, x, wg, bias, off, options=0):
    desc = M.layer_desc(cfg, options=options)
    T = x.shape[0]
    ws = M.Workspace(desc, T)
    w = torch.full((T, cfg.topk), -1.0, dtype=torch.float32, device="cuda")
    idx = torch.full((T, cfg.topk), -1, dtype=torch.int32, device="cuda")
    M.moe_gate(desc, x, wg, bias, off, w, idx, ws)
    M.check_device_errors(ws, "moe_gate")
    return idx.cpu().numpy(), w.cpu().numpy()


# ------------------------------------------------------------------------------------------------
# gate
# ------------------------------------------------------------------------------------------------
GATE_CASES = [("tiny", 64), ("tiny", 300), ("tiny", 1), ("v3_prefill", 4096), ("v3_prefill", 131),
              ("v3_decode", 64), ("v4_skew", 16384), ("v4_skew", 200)]


@pytest.mark.parametrize("name,T", GATE_CASES)
def test_gate_parity(M, name, T, options=0):
    cfg = W.CONFIGS[name].replace(T=T)
    x, wg, bias, off = W.make_router_inputs(cfg, device="cuda")
    idx, w = _gate_gpu(M, cfg, x, wg, bias, off, options)
    g = oracle_gate_of(cfg, x, wg, bias, off)
    exempt, _ = compare_routing(cfg, g, idx, w, None if bias is None else bias.cpu().numpy())
    assert len(exempt) <= max(2, T // 200), f"unexpectedly many near-tied tokens: {len(exempt)}"


@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("name,T", [("tiny", 300), ("v3_prefill", 4096), ("v4_skew", 200)])
def test_gate_prepared_planes_bit_identical(M, name, T, single):
    """Router weights prepared once (moe_gate_prepare) route exactly as when split on every call:
    general fp32 weights (tiny: three planes) and bf16-valued ones (one plane), both router paths."""
    cfg = W.CONFIGS[name].replace(T=T)
    x, wg, bias, off = W.make_router_inputs(cfg, device="cuda")
    opt = M.MOE_OPT_ROUTER_ONE_CTA if single else 0
    idx0, w0 = _gate_gpu(M, cfg, x, wg, bias, off, opt)
    desc = M.layer_desc(cfg, options=opt)
    keep = M.prepare_gate(desc, wg)
    flag = int(keep[:4].view(torch.int32).item())
    assert flag == (1 if cfg.gate_general_fp32 else 0)
    ws = M.Workspace(desc, T)
    w = torch.full((T, cfg.topk), -1.0, dtype=torch.float32, device="cuda")
    idx = torch.full((T, cfg.topk), -1, dtype=torch.int32, device="cuda")
    M.moe_gate(desc, x, wg, bias, off, w, idx, ws)
    M.check_device_errors(ws, "moe_gate")
    assert np.array_equal(idx.cpu().numpy(), idx0)
    assert np.array_equal(w.cpu().numpy(), w0)


@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("name,T", [("tiny", 300), ("v3_prefill", 4096), ("v3_prefill", 8192), ("v3_decode", 64),
                                    ("v4_skew", 200)])
def test_gate_both_router_paths(M, name, T, single):
    # the split-K cluster router (cluster sizes 4, 4, 2, 8, 8 here) and, forced, the one-CTA-per-tile one
    test_gate_parity(M, name, T, options=M.MOE_OPT_ROUTER_ONE_CTA if single else 0)


@pytest.mark.parametrize("variant", ["no_bias_groups", "softmax", "groups_384", "sqrtsoftplus_groups",
                                     "groups_16", "groups_2_e32", "e64_groups_4", "e128_groups_8",
                                     "groups_3_e48", "e80", "e512_k8"])
def test_gate_variants(M, variant):
    base = W.CONFIGS["tiny"].replace(T=260)
    cfg = {
        "no_bias_groups": base.replace(bias_std=None),
        "softmax": base.replace(score_func="softmax", bias_std=None, route_scale=2.0),
        "groups_384": W.CONFIGS["v4_skew"].replace(T=300, n_groups=8, n_limited_groups=3, dim=512,
                                                   score_func="sigmoid"),
        "sqrtsoftplus_groups": base.replace(score_func="sqrtsoftplus", gate_general_fp32=False),
        # one lane per group in the cluster router's epilogue
        "groups_16": W.CONFIGS["v3_prefill"].replace(T=300, dim=512, n_groups=16, n_limited_groups=5),
        "groups_2_e32": base.replace(n_experts=32, n_groups=2, n_limited_groups=1, topk=6),
        "e64_groups_4": base.replace(n_experts=64, n_groups=4, n_limited_groups=2, topk=6, dim=512),
        "e128_groups_8": base.replace(n_experts=128, n_groups=8, n_limited_groups=3, topk=8, dim=1024, T=700),
        # layouts the cluster router does not take (G not dividing 16, E / 16 = 5): the one-CTA router
        "groups_3_e48": base.replace(n_experts=48, n_groups=3, n_limited_groups=2, topk=5),
        "e80": base.replace(n_experts=80, n_groups=1, n_limited_groups=1, topk=8),
        # the largest layout the library takes: 512 experts (two N = 256 MMAs), top-8
        "e512_k8": base.replace(n_experts=512, n_groups=8, n_limited_groups=4, topk=8, dim=512, T=300),
    }[variant]
    x, wg, bias, off = W.make_router_inputs(cfg, device="cuda")
    idx, w = _gate_gpu(M, cfg, x, wg, bias, off)
    g = oracle_gate_of(cfg, x, wg, bias, off)
    compare_routing(cfg, g, idx, w, None if bias is None else bias.cpu().numpy())


# ------------------------------------------------------------------------------------------------
# hash gate
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("single", [False, True])
def test_hash_gate_parity(M, single):
    # the cluster router with the table's experts picked out of all logits and, forced, one warp per
    # token computing just the k dot products
    cfg = W.CONFIGS["hash"]
    p = W.token_frequencies(cfg)
    table_lib, _ = M.moe_build_tid2eid(p, cfg.n_experts, cfg.topk)
    table_ora, _ = O.build_tid2eid(p, cfg.n_experts, cfg.topk)
    assert np.array_equal(table_lib, table_ora)
    ids = W.sample_token_ids(cfg, p)
    x, wg, _, _ = W.make_router_inputs(cfg, device="cuda")
    desc = M.layer_desc(cfg, options=M.MOE_OPT_ROUTER_ONE_CTA if single else 0)
    ws = M.Workspace(desc, cfg.T)
    w = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device="cuda")
    M.moe_hash_gate(desc, torch.from_numpy(ids).cuda(), torch.from_numpy(table_lib).cuda(), x, wg, w, idx, ws)
    M.check_device_errors(ws, "moe_hash_gate")
    i_ora, w_ora = O.hash_gate(ids, table_ora, np64(x), np64(wg), cfg.route_scale)
    assert np.array_equal(idx.cpu().numpy(), i_ora)
    np.testing.assert_allclose(w.cpu().numpy(), w_ora, rtol=2e-5, atol=2e-6)


def test_hash_gate_flags_bad_token_id(M):
    cfg = W.CONFIGS["hash"].replace(T=16, dim=256)
    vocab = 100
    table = torch.zeros((vocab, cfg.topk), dtype=torch.int32, device="cuda")
    table[:, :] = torch.arange(cfg.topk, dtype=torch.int32, device="cuda")
    ids = torch.arange(cfg.T, dtype=torch.int32, device="cuda")
    ids[5] = vocab + 7
    x, wg, _, _ = W.make_router_inputs(cfg, device="cuda")
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, cfg.T)
    w = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device="cuda")
    M.moe_hash_gate(desc, ids, table, x, wg, w, idx, ws)
    st, info = M.moe_get_error(ws)
    assert st == M.MOE_ERR_DEVICE and info == vocab + 7
    assert M.moe_get_error(ws) == (M.MOE_OK, 0)   # cleared by the read


# ------------------------------------------------------------------------------------------------
# 2-gram hash gate and the bias update
# ------------------------------------------------------------------------------------------------
def _ngram_gpu(M, cfg, prev, ids, primes, vocab, x, wg, options=0):
    desc = M.layer_desc(cfg, options=options)
    T = ids.shape[0]
    ws = M.Workspace(desc, T)
    w = torch.full((T, cfg.topk), -1.0, dtype=torch.float32, device="cuda")
    idx = torch.full((T, cfg.topk), -1, dtype=torch.int32, device="cuda")
    M.moe_ngram_gate(desc, torch.from_numpy(prev).cuda(), torch.from_numpy(ids).cuda(), primes, vocab, x, wg, w, idx,
                     ws)
    return idx.cpu().numpy(), w.cpu().numpy(), ws


@pytest.mark.parametrize("single", [False, True])
def test_ngram_gate_parity(M, single):
    # the hash layer's vocabulary and Zipf ids, sequences of 2048 tokens whose first token follows id 0
    # (ids are frequency ranks, so pairs (0, b) repeat one expert k times: duplicates are covered)
    cfg = W.CONFIGS["hash"]
    p = W.token_frequencies(cfg)
    ids = W.sample_token_ids(cfg, p)
    prev = np.concatenate([[0], ids[:-1]]).astype(np.int32)
    prev[::2048] = 0
    primes = O.primes_above(cfg.hash_vocab, cfg.topk)
    x, wg, _, _ = W.make_router_inputs(cfg, device="cuda")
    idx, w, ws = _ngram_gpu(M, cfg, prev, ids, primes, cfg.hash_vocab, x, wg,
                            options=M.MOE_OPT_ROUTER_ONE_CTA if single else 0)
    M.check_device_errors(ws, "moe_ngram_gate")
    i_ora, w_ora = O.ngram_gate(prev, ids, primes, np64(x), np64(wg), cfg.route_scale)
    assert np.array_equal(idx, i_ora)
    assert any(len(set(r)) < cfg.topk for r in i_ora.tolist())
    np.testing.assert_allclose(w, w_ora, rtol=2e-5, atol=2e-6)


def test_ngram_gate_wide_ids_and_primes(M):
    # ids up to 2^31 - 2 and primes just below 2^32: a * q + b needs the full 64 bits
    cfg = W.CONFIGS["hash"].replace(T=1000, dim=512, n_experts=384, topk=8, route_scale=1.5)
    vocab = 2 ** 31 - 1
    rng = np.random.default_rng(31)
    ids = rng.integers(vocab - 10 ** 6, vocab, cfg.T).astype(np.int32)
    prev = rng.integers(0, vocab, cfg.T).astype(np.int32)
    prev[:3] = vocab - 1
    primes = O.primes_above(2 ** 32 - 600, cfg.topk)
    assert max(primes) < 2 ** 32
    x, wg, _, _ = W.make_router_inputs(cfg, device="cuda")
    idx, w, ws = _ngram_gpu(M, cfg, prev, ids, primes, vocab, x, wg)
    M.check_device_errors(ws, "moe_ngram_gate")
    i_ora, w_ora = O.ngram_gate(prev, ids, primes, np64(x), np64(wg), cfg.route_scale)
    assert np.array_equal(idx, i_ora)
    np.testing.assert_allclose(w, w_ora, rtol=2e-5, atol=2e-6)


def test_ngram_gate_flags_bad_previous_id(M):
    cfg = W.CONFIGS["hash"].replace(T=16, dim=256)
    vocab = 100
    ids = np.arange(cfg.T, dtype=np.int32)
    prev = np.zeros(cfg.T, np.int32)
    prev[9] = -3
    x, wg, _, _ = W.make_router_inputs(cfg, device="cuda")
    _, _, ws = _ngram_gpu(M, cfg, prev, ids, O.primes_above(vocab, cfg.topk), vocab, x, wg)
    st, info = M.moe_get_error(ws)
    assert st == M.MOE_ERR_DEVICE and info == -3


@pytest.mark.parametrize("E,T,k", [(256, 4096, 8), (384, 16384, 6), (16, 64, 4)])
def test_update_bias_parity(M, E, T, k):
    rng = np.random.default_rng(E + T)
    level = T * k / E
    counts = rng.poisson(level, E).astype(np.int32)
    if float(level).is_integer():
        counts[::7] = int(level)   # exactly balanced experts keep their bias
    counts[1] = 0
    bias = rng.normal(0.0, 0.01, E).astype(np.float32)
    cfg = W.CONFIGS["tiny"].replace(n_experts=E, topk=k, n_groups=1, n_limited_groups=1)
    desc = M.layer_desc(cfg)
    b_gpu = torch.from_numpy(bias).cuda()
    M.moe_update_bias(desc, T, torch.from_numpy(counts).cuda(), b_gpu, 0.001)
    want = O.update_bias(bias, counts, T, k, 0.001)
    assert np.array_equal(b_gpu.cpu().numpy(), want)
    M.moe_update_bias(desc, T, torch.from_numpy(counts).cuda(), b_gpu, 0.0)   # gamma 0: the frozen phase
    assert np.array_equal(b_gpu.cpu().numpy(), want)


def test_bias_update_loop_balances_the_gate(M):
    # gate -> dispatch counts -> bias update, repeated on the device: a router whose logits favour
    # the first experts must end far closer to balance (the control loop of the bias-update rule)
    cfg = W.CONFIGS["tiny"].replace(T=2048, dim=256, n_experts=64, n_groups=1, n_limited_groups=1, topk=4)
    x, wg, _, _ = W.make_router_inputs(cfg, device="cuda")
    off = torch.linspace(0.8, -0.8, cfg.n_experts, device="cuda", dtype=torch.float32)
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, cfg.T)
    bias = torch.zeros(cfg.n_experts, dtype=torch.float32, device="cuda")
    w = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device="cuda")
    S = cfg.T * cfg.topk
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    offsets = torch.empty(cfg.n_experts + 1, dtype=torch.int32, device="cuda")
    ros = torch.empty(S, dtype=torch.int32, device="cuda")
    tor = torch.empty(S, dtype=torch.int32, device="cuda")
    xp = torch.empty((S, cfg.dim), dtype=torch.bfloat16, device="cuda")
    spread = []
    for step in range(300):
        M.moe_gate(desc, x, wg, bias, off, w, idx, ws)
        M.moe_dispatch(desc, idx, x, counts, offsets, ros, tor, xp, ws)
        if step in (0, 299):
            spread.append(int(counts.max() - counts.min()))
            b_before = bias.cpu().numpy()
            c_host = counts.cpu().numpy()
        M.moe_update_bias(desc, cfg.T, counts, bias, 0.002)
        if step == 0:
            assert np.array_equal(bias.cpu().numpy(), O.update_bias(b_before, c_host, cfg.T, cfg.topk, 0.002))
    M.check_device_errors(ws, "bias update loop")
    assert spread[1] < 0.2 * spread[0], spread


# ------------------------------------------------------------------------------------------------
# dispatch
# ------------------------------------------------------------------------------------------------
def _skewed_indices(T, E, k, seed):
    """Distinct experts per token drawn with Zipf-like expert popularity (some experts empty)."""
    rng = np.random.default_rng(seed)
    pop = 1.0 / np.arange(1, E + 1) ** 1.2
    pop[E // 2:E // 2 + 3] = 0.0   # a few experts nobody picks
    pop /= pop.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=pop) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k,d", [(300, 16, 4, 256), (4096, 256, 8, 7168), (1, 384, 6, 512), (2000, 384, 6, 128)])
def test_dispatch_parity(M, T, E, k, d):
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d)
    idx = _skewed_indices(T, E, k, seed=T + E)
    x = W.normal_bf16((T, d), 1.0, 7, W.TID_X, device="cuda")
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, T)
    S = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ros = torch.empty(S, dtype=torch.int32, device="cuda")
    tor = torch.empty(S, dtype=torch.int32, device="cuda")
    xp = torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    M.moe_dispatch(desc, torch.from_numpy(idx).cuda(), x, counts, offsets, ros, tor, xp, ws)
    M.check_device_errors(ws, "moe_dispatch")
    c, o, r, t = O.dispatch(idx, E)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offsets.cpu().numpy(), o)
    assert np.array_equal(ros.cpu().numpy(), r)
    assert np.array_equal(tor.cpu().numpy(), t)
    assert torch.equal(xp, x[torch.from_numpy(t).cuda().long()])


def test_dispatch_flags_bad_expert(M):
    cfg = W.CONFIGS["tiny"].replace(T=40)
    idx = _skewed_indices(cfg.T, cfg.n_experts, cfg.topk, 1)
    idx[3, 2] = cfg.n_experts + 5
    x = W.normal_bf16((cfg.T, cfg.dim), 1.0, 7, W.TID_X, device="cuda")
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, cfg.T)
    S = cfg.T * cfg.topk
    out = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (cfg.n_experts, cfg.n_experts + 1, S, S)]
    xp = torch.empty((S, cfg.dim), dtype=torch.bfloat16, device="cuda")
    M.moe_dispatch(desc, torch.from_numpy(idx).cuda(), x, *out, xp, ws)
    st, info = M.moe_get_error(ws)
    assert st == M.MOE_ERR_DEVICE and info == cfg.n_experts + 5
    assert int(out[1][-1]) == S   # still a valid permutation: the bad id was clamped


# ------------------------------------------------------------------------------------------------
# experts
# ------------------------------------------------------------------------------------------------
EXPERT_CASES = [
    (300, 16, 4, 256, 384),     # single-CTA kernels (I % 256 != 0, d % 512 != 0)
    (1, 16, 4, 128, 128),       # one token
    (700, 32, 6, 384, 256),     # CTA-pair up projection, single-CTA down projection
    (600, 16, 4, 512, 512),     # CTA-pair kernels for both
    (1000, 32, 8, 1024, 768),   # CTA-pair kernels, several feature blocks, 256-row token chunks
    (3000, 16, 4, 512, 512),    # CTA-pair kernels, 256-row chunks, experts spanning several chunks
    (2500, 16, 4, 768, 256),    # CTA-pair, one w2 tile per CTA (d an odd multiple of 256), 256-row chunks
    (400, 16, 4, 256, 256),     # CTA-pair, one w2 tile per CTA, 128-row chunks
    (1, 16, 4, 512, 256),       # CTA-pair kernels, one token (chunk of 1 row)
]


GATHER_CASES = [c for c in EXPERT_CASES if c[4] % 256 == 0]   # the CTA-pair up projection


@pytest.mark.parametrize("T,E,k,d,I", EXPERT_CASES)
def test_expert_ffn_parity(M, T, E, k, d, I, gather=False, options=0):
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d,
                                    inter_dim=I, w_std=0.05)
    li = W.make_layer(cfg, device="cuda")
    idx = _skewed_indices(T, E, k, seed=3 * T + E)
    desc = M.layer_desc(cfg, options=options)
    ws = M.Workspace(desc, T)
    S = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ros = torch.empty(S, dtype=torch.int32, device="cuda")
    tor = torch.empty(S, dtype=torch.int32, device="cuda")
    xp = None if gather else torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    M.moe_dispatch(desc, torch.from_numpy(idx).cuda(), li.x, counts, offsets, ros, tor, xp, ws)
    out_perm = torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    out_sh = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    if gather:
        M.moe_expert_ffn_gather(desc, tor, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws)
    else:
        M.moe_expert_ffn(desc, xp, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws)
    M.check_device_errors(ws, "moe_expert_ffn")
    c, o, r, tok = O.dispatch(idx, E)
    if gather:   # dispatch without x_perm still writes the whole permutation
        assert np.array_equal(offsets.cpu().numpy(), o) and np.array_equal(tor.cpu().numpy(), tok)
    if T >= 300:
        assert c.max() > 128 and (c == 0).any()  # several token chunks and an empty expert
    x = np64(li.x)
    got = np64(out_perm)
    fetch = expert_fetcher(li)
    for e in range(E):
        if c[e] == 0:
            continue
        ref = O.swiglu_expert(x[tok[o[e]:o[e + 1]]], *fetch(e))
        assert_outputs_close(got[o[e]:o[e + 1]], ref, f"expert {e}", per_element=True)
    assert_outputs_close(np64(out_sh), O.swiglu_expert(x, *fetch(E)), "shared expert", per_element=True)


@pytest.mark.parametrize("T,E,k,d,I", GATHER_CASES)
def test_expert_ffn_gather_parity(M, T, E, k, d, I):
    # the up projection reads its routed rows of x through tok_of_row (tile::gather4), no x_perm
    test_expert_ffn_parity(M, T, E, k, d, I, gather=True)


@pytest.mark.parametrize("T,E,k,d,I,limit,weighted", [(3000, 16, 4, 512, 512, 0.0, False),
                                                      (700, 32, 6, 384, 256, 0.5, True),
                                                      (1, 16, 4, 512, 256, 0.0, True)])
def test_expert_ffn_gather_bit_identical(M, T, E, k, d, I, limit, weighted):
    # gathering from x feeds the tensor cores the same rows in the same order as x_perm does
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d,
                                    inter_dim=I, w_std=0.05, swiglu_limit=limit)
    li = W.make_layer(cfg, device="cuda")
    idx = torch.from_numpy(_skewed_indices(T, E, k, seed=7 * T + E)).cuda()
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, T)
    S = T * k
    rw = W.uniform(S, 13, 90).to(torch.float32).cuda() * 2.0 if weighted else None
    outs = []
    for gather in (False, True):
        counts = torch.empty(E, dtype=torch.int32, device="cuda")
        offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        ros = torch.empty(S, dtype=torch.int32, device="cuda")
        tor = torch.empty(S, dtype=torch.int32, device="cuda")
        xp = None if gather else torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
        M.moe_dispatch(desc, idx, li.x, counts, offsets, ros, tor, xp, ws)
        out_perm = torch.full((S, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        out_sh = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        if gather:
            M.moe_expert_ffn_gather(desc, tor, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws,
                                    row_weights=rw)
        else:
            M.moe_expert_ffn(desc, xp, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws, row_weights=rw)
        M.check_device_errors(ws, "expert ffn")
        outs.append((out_perm, out_sh, ros, tor))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


def test_forward_fused_gather_bit_identical(M):
    # moe_forward with the gather fused into the up projection, and with dispatch writing x_perm
    cfg = W.CONFIGS["v3_decode"]
    li = W.make_layer(cfg, device="cuda")
    ys = []
    for opt in (0, M.MOE_OPT_FUSED_GATHER):   # the second: the experts gather the rows of x themselves
        ys.append(_forward_gpu(M, cfg, li, options=opt)[0])
    assert torch.equal(ys[0], ys[1])


@pytest.mark.parametrize("single", [False, True])
def test_expert_ffn_both_kernel_paths(M, single):
    # the same CTA-pair-capable shape through the CTA-pair kernels and, forced, the single-CTA ones
    test_expert_ffn_parity(M, 640, 32, 6, 512, 512, options=M.MOE_OPT_GEMM_ONE_CTA if single else 0)


@pytest.mark.parametrize("T,E,k,d,I", [(400, 16, 4, 512, 512), (300, 16, 4, 256, 384)])
def test_expert_ffn_clamp_and_row_weights(M, T, E, k, d, I):
    # the V4-style expert ("From One Giant FFN...", section 11.4; "DeepSeek V4.1 - Add shared"): SwiGLU
    # clamp, and each routed row's weight applied to h; the limit is chosen to clip many values
    limit = 0.5
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d,
                                    inter_dim=I, w_std=0.05, swiglu_limit=limit)
    li = W.make_layer(cfg, device="cuda")
    idx = _skewed_indices(T, E, k, seed=5 * T + E)
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, T)
    S = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ros = torch.empty(S, dtype=torch.int32, device="cuda")
    tor = torch.empty(S, dtype=torch.int32, device="cuda")
    xp = torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    M.moe_dispatch(desc, torch.from_numpy(idx).cuda(), li.x, counts, offsets, ros, tor, xp, ws)
    rw = W.uniform(S, 11, 90).to(torch.float32).cuda() * 2.0
    out_perm = torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    out_sh = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    M.moe_expert_ffn(desc, xp, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws, row_weights=rw)
    M.check_device_errors(ws, "moe_expert_ffn")
    c, o, r, tok = O.dispatch(idx, E)
    x = np64(li.x)
    got = np64(out_perm)
    rwn = rw.cpu().numpy()
    fetch = expert_fetcher(li)
    clipped = 0
    for e in range(E):
        if c[e] == 0:
            continue
        rows = slice(o[e], o[e + 1])
        w1, w3, w2 = fetch(e)
        ref = O.swiglu_expert(x[tok[rows]], w1, w3, w2, limit=limit, row_weight=rwn[rows])
        assert_outputs_close(got[rows], ref, f"expert {e}", per_element=True)
        clipped += int((np.abs(x[tok[rows]] @ w3.T) > limit).sum())
    assert clipped > 0
    w1, w3, w2 = fetch(E)
    assert_outputs_close(np64(out_sh), O.swiglu_expert(x, w1, w3, w2, limit=limit), "shared expert",
                         per_element=True)


@pytest.mark.parametrize("base,T", [("tiny", 200), ("v4_skew", 256)])
def test_forward_v4_style_expert(M, base, T):
    # whole layer with the clamp and the weight handed to the expert (combine sums unweighted outputs)
    over = dict(T=T, swiglu_limit=0.5, weight_in_expert=True, w_std=0.05)
    if base == "v4_skew":
        over.update(dim=512, inter_dim=256)
    cfg = W.CONFIGS[base].replace(**over)
    li = W.make_layer(cfg, device="cuda")
    y, iw, ww, cw = _forward_gpu(M, cfg, li)
    hp = O.Hyper.of(cfg)
    bias = None if li.bias is None else li.bias.cpu().numpy()
    off = None if li.logit_offset is None else li.logit_offset.cpu().numpy()
    g = O.gate(np64(li.x), np64(li.w_gate), hp, bias, off)
    exempt, counts = compare_routing(cfg, g, iw, ww, bias)
    assert np.array_equal(cw, counts)
    terms = {}
    y_ref, _, _, _ = O.moe_forward(np64(li.x), hp, expert_fetcher(li), np64(li.w_gate), bias, off, terms=terms,
                                   swiglu_limit=0.5, weight_in_expert=True)
    keep = np.setdiff1d(np.arange(T), exempt)
    slack = rounding_slack(y_ref, terms)
    assert_outputs_close(np64(y)[keep], y_ref[keep], "y", slack=slack[keep])


def test_identity_like_layer_on_gpu(M):
    # The oracle's closed-form pin, run through the library: w1 = [+I; -I; 0], w3 rows = e_{d-1},
    # w2 = s_e [I | -I] make expert e return s_e * x (up to bf16 rounding of h) when x_{d-1} = 1.
    cfg = W.CONFIGS["tiny"].replace(T=200, dim=128, inter_dim=256)
    d, I, E = cfg.dim, cfg.inter_dim, cfg.n_experts
    n = d - 1
    scales = [(e + 1) / 4.0 for e in range(E)] + [0.5]
    w1 = np.zeros((E + 1, I, d)); w3 = np.zeros((E + 1, I, d)); w2 = np.zeros((E + 1, d, I))
    for e, s in enumerate(scales):
        w1[e, np.arange(n), np.arange(n)] = 1.0
        w1[e, n + np.arange(n), np.arange(n)] = -1.0
        w3[e, :, d - 1] = 1.0
        w2[e, np.arange(n), np.arange(n)] = s
        w2[e, np.arange(n), n + np.arange(n)] = -s
    x, wg, bias, _ = W.make_router_inputs(cfg, device="cuda")
    x[:, d - 1] = 1.0
    dev = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()
    w1t, w3t, w2t = dev(w1), dev(w3), dev(w2)
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, cfg.T)
    y = torch.empty_like(x)
    wout = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
    iout = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device="cuda")
    M.moe_forward(desc, x, wg, w1t, w3t, w2t, y, ws, bias=bias, weights_out=wout, indices_out=iout)
    M.check_device_errors(ws, "moe_forward")
    iw, ww = iout.cpu().numpy(), wout.cpu().numpy().astype(np.float64)
    factor = np.array([sum(ww[t, j] * scales[iw[t, j]] for j in range(cfg.topk)) + scales[E] for t in range(cfg.T)])
    xv = np64(x)[:, :n]
    want = factor[:, None] * xv
    u = 2.0 ** -8
    err = np.abs(np64(y)[:, :n] - want)
    assert np.all(err <= np.abs(want) * (2 * u + u * (1 + 2 * u)) * 1.001 + 1e-12)
    assert np.all(np64(y)[:, d - 1] == 0)
    # and the routing itself is the oracle's
    g = oracle_gate_of(cfg, x, wg, bias, None)
    compare_routing(cfg, g, iw, ww.astype(np.float32), bias.cpu().numpy())


# ------------------------------------------------------------------------------------------------
# whole layer
# ------------------------------------------------------------------------------------------------
def _forward_gpu(M, cfg, li, table=None, options=0):
    desc = M.layer_desc(cfg, options=options)
    ws = M.Workspace(desc, cfg.T)
    y = torch.empty_like(li.x)
    wout = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
    iout = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device="cuda")
    cout = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    kw = {}
    if table is not None:
        kw = dict(token_ids=li.token_ids, tid2eid=torch.from_numpy(table).cuda())
    M.moe_forward(desc, li.x, li.w_gate, li.w1, li.w3, li.w2, y, ws, bias=li.bias, logit_offset=li.logit_offset,
                  weights_out=wout, indices_out=iout, counts_out=cout, **kw)
    M.check_device_errors(ws, "moe_forward")
    return y, iout.cpu().numpy(), wout.cpu().numpy(), cout.cpu().numpy()


@pytest.mark.parametrize("T", [64, 257])
def test_forward_tiny_every_token(M, T):
    cfg = W.CONFIGS["tiny"].replace(T=T)
    li = W.make_layer(cfg, device="cuda")
    y, iw, ww, cw = _forward_gpu(M, cfg, li)
    hp = O.Hyper.of(cfg)
    g = oracle_gate_of(cfg, li.x, li.w_gate, li.bias, li.logit_offset)
    exempt, counts = compare_routing(cfg, g, iw, ww, li.bias.cpu().numpy())
    assert np.array_equal(cw, counts)
    terms = {}
    y_ref, _, _, _ = O.moe_forward(np64(li.x), hp, expert_fetcher(li), np64(li.w_gate), li.bias.cpu().numpy(),
                                   terms=terms)
    keep = np.setdiff1d(np.arange(T), exempt)
    slack = rounding_slack(y_ref, terms)
    assert_outputs_close(np64(y)[keep], y_ref[keep], "y", slack=slack[keep])


def test_forward_max_experts_and_topk(M):
    # the largest expert count and top-k the library accepts (E = 512, k = 8), most experts holding
    # a token or two, through the whole forward: every token's routing and output
    cfg = W.CONFIGS["tiny"].replace(T=300, n_experts=512, n_groups=8, n_limited_groups=4, topk=8, dim=512,
                                    inter_dim=256)
    li = W.make_layer(cfg, device="cuda")
    y, iw, ww, cw = _forward_gpu(M, cfg, li)
    hp = O.Hyper.of(cfg)
    g = oracle_gate_of(cfg, li.x, li.w_gate, li.bias, li.logit_offset)
    exempt, counts = compare_routing(cfg, g, iw, ww, li.bias.cpu().numpy())
    assert np.array_equal(cw, counts)
    terms = {}
    y_ref, _, _, _ = O.moe_forward(np64(li.x), hp, expert_fetcher(li), np64(li.w_gate), li.bias.cpu().numpy(),
                                   terms=terms)
    keep = np.setdiff1d(np.arange(cfg.T), exempt)
    slack = rounding_slack(y_ref, terms)
    assert_outputs_close(np64(y)[keep], y_ref[keep], "y", slack=slack[keep])


FULL = ["v3_prefill", "hash", "v3_decode", "v4_skew"]


def _staged_gpu(M, cfg, li, table=None):
    """The layer through its four stage entry points, in the launch sequence the benchmark times:
    returns every intermediate output."""
    desc = M.layer_desc(cfg)
    T, k, E, d = cfg.T, cfg.topk, cfg.n_experts, cfg.dim
    S = T * k
    ws = M.Workspace(desc, T)
    i32 = dict(dtype=torch.int32, device="cuda")
    bf = dict(dtype=torch.bfloat16, device="cuda")
    o = dict(weights=torch.empty((T, k), dtype=torch.float32, device="cuda"), indices=torch.empty((T, k), **i32),
             counts=torch.full((E,), -1, **i32), offsets=torch.full((E + 1,), -1, **i32),
             ros=torch.full((S,), -1, **i32), tor=torch.full((S,), -1, **i32), x_perm=torch.empty((S, d), **bf),
             out_perm=torch.full((S, d), float("nan"), **bf), out_sh=torch.full((T, d), float("nan"), **bf),
             y=torch.full((T, d), float("nan"), **bf))
    if table is not None:
        M.moe_hash_gate(desc, li.token_ids, torch.from_numpy(table).cuda(), li.x, li.w_gate, o["weights"],
                        o["indices"], ws)
    else:
        M.moe_gate(desc, li.x, li.w_gate, li.bias, li.logit_offset, o["weights"], o["indices"], ws)
    M.moe_dispatch(desc, o["indices"], li.x, o["counts"], o["offsets"], o["ros"], o["tor"], o["x_perm"], ws)
    M.moe_expert_ffn(desc, o["x_perm"], o["offsets"], li.x, li.w1, li.w3, li.w2, o["out_perm"], o["out_sh"], ws)
    M.moe_combine(desc, T, o["out_perm"], o["ros"], o["weights"], o["out_sh"], o["y"])
    M.check_device_errors(ws, "staged forward")
    return o


def _whole_experts(counts: np.ndarray, n: int, seed: int):
    """n experts chosen by seed among those with rows, always including the heaviest and the lightest
    (a single token chunk)."""
    live = np.nonzero(counts)[0]
    pick = {int(live[np.argmax(counts[live])]), int(live[np.argmin(counts[live])])}
    order = live[np.argsort(W.uniform(len(live), seed, W.TID_SAMPLE).numpy(), kind="stable")]
    for e in order:
        if len(pick) >= n:
            break
        pick.add(int(e))
    return sorted(pick)


@pytest.mark.parametrize("name", FULL)
def test_forward_full_size(M, name):
    # Full size, in the benchmark's launch configuration: routing and counts for every token; the
    # dispatch permutation bit for bit; 16 whole experts (the heaviest, the lightest and 14 by seed)
    # and the shared expert over all T tokens element by element; y on 256 sampled tokens; and
    # moe_forward's y bit-identical to the staged calls'.
    cfg = W.CONFIGS[name]
    li = W.make_layer(cfg, device="cuda")
    table = None
    if cfg.is_hash:
        table, _ = M.moe_build_tid2eid(li.p, cfg.n_experts, cfg.topk)
    o = _staged_gpu(M, cfg, li, table)
    y_fwd, iw_fwd, _, cw_fwd = _forward_gpu(M, cfg, li, table)
    assert torch.equal(y_fwd, o["y"]), "moe_forward and the staged entry points disagree"
    iw, ww = o["indices"].cpu().numpy(), o["weights"].cpu().numpy()
    cw = o["counts"].cpu().numpy()
    assert np.array_equal(iw, iw_fwd) and np.array_equal(cw, cw_fwd)
    hp = O.Hyper.of(cfg)
    x64 = np64(li.x)
    wg64 = np64(li.w_gate)
    # routing and counts: every token
    if cfg.is_hash:
        t_ora, _ = O.build_tid2eid(li.p, cfg.n_experts, cfg.topk)
        assert np.array_equal(table, t_ora)
        ids = li.token_ids.cpu().numpy()
        i_ora, w_ora = O.hash_gate(ids, t_ora, x64, wg64, cfg.route_scale)
        assert np.array_equal(iw, i_ora)
        np.testing.assert_allclose(ww, w_ora, rtol=2e-5, atol=2e-6)
        exempt, counts = np.zeros(0, int), np.bincount(i_ora.reshape(-1), minlength=cfg.n_experts)
    else:
        bias = None if li.bias is None else li.bias.cpu().numpy()
        off = None if li.logit_offset is None else li.logit_offset.cpu().numpy()
        g = O.gate(x64, wg64, hp, bias, off)
        exempt, counts = compare_routing(cfg, g, iw, ww, bias)
        i_ora, w_ora = g.indices, g.weights
    assert np.array_equal(cw, counts)
    assert cw.sum() == cfg.T * cfg.topk
    # dispatch of the GPU's routing: bit for bit, and x_perm rows are rows of x
    c, off_o, ros_o, tok_o = O.dispatch(iw, cfg.n_experts)
    assert np.array_equal(o["offsets"].cpu().numpy(), off_o)
    assert np.array_equal(o["ros"].cpu().numpy(), ros_o)
    assert np.array_equal(o["tor"].cpu().numpy(), tok_o)
    assert torch.equal(o["x_perm"], li.x[torch.from_numpy(tok_o).cuda().long()])
    # experts: whole experts and the shared expert element by element; y on a sample of tokens
    whole = _whole_experts(c, 16, seed=cfg.seed + 200)
    rows = np.setdiff1d(W.sample_rows(cfg.T, 256, seed=cfg.seed + 100), exempt)
    ref_whole, y_ref, terms, shared_ref = oracle_by_expert(x64, expert_fetcher(li), i_ora, w_ora, cfg.n_experts,
                                                           rows, whole, tok_o, off_o)
    for e in whole:
        assert_outputs_close(np64(o["out_perm"][off_o[e]:off_o[e + 1]]), ref_whole[e],
                             f"{name} expert {e} ({c[e]} rows)", per_element=True)
    assert_outputs_close(np64(o["out_sh"]), shared_ref, f"{name} shared expert ({cfg.T} rows)", per_element=True)
    r = assert_outputs_close(np64(o["y"])[rows], y_ref, f"{name} y ({len(rows)} sampled tokens)",
                             slack=rounding_slack(y_ref, terms))
    print(f"{name}: experts {whole} rows {c[whole].tolist()}; max |y - y_oracle| / rms = {r:.4f} over "
          f"{len(rows)} tokens")
    # every output row is finite and written
    assert torch.isfinite(o["y"].float()).all() and torch.isfinite(o["out_perm"].float()).all()


def test_generator_gives_the_same_inputs_on_cpu_and_gpu():
    # the seeded inputs are a pure function of (seed, tensor, expert, index): regenerated on the CPU
    # they equal the GPU's, so the oracle can rebuild any single expert on its own
    for fn in (lambda dev: W.normal_bf16((257, 384), 0.02, 9, W.TID_W1, 5, device=dev),
               lambda dev: W.normal_f32((64, 512), 0.006, 1, W.TID_W_GATE, device=dev),
               lambda dev: W.uniform(1000, 3, W.TID_SAMPLE, device=dev)):
        assert torch.equal(fn("cpu"), fn("cuda").cpu())
    for a, b in zip(W.mxfp4_matrix(128, 512, 0.01, 2, 1, 7, device="cpu"),
                    W.mxfp4_matrix(128, 512, 0.01, 2, 1, 7, device="cuda")):
        assert torch.equal(a, b.cpu())


def test_concurrent_forwards_on_two_streams(M):
    # two layers in flight at once on two streams, each with its own workspace (the library keeps no
    # other state): both outputs equal the single-stream results bit for bit
    cfg_a = W.CONFIGS["tiny"].replace(T=300, dim=512, inter_dim=512)
    cfg_b = W.CONFIGS["v3_prefill"].replace(T=512, n_experts=32, n_groups=8, n_limited_groups=4, seed=11)
    outs = {}
    for name, cfg in (("a", cfg_a), ("b", cfg_b)):
        li = W.make_layer(cfg, device="cuda")
        desc = M.layer_desc(cfg)
        ref_ws, ws = M.Workspace(desc, cfg.T), M.Workspace(desc, cfg.T)
        y_ref, y = torch.empty_like(li.x), torch.empty_like(li.x)
        M.moe_forward(desc, li.x, li.w_gate, li.w1, li.w3, li.w2, y_ref, ref_ws, bias=li.bias,
                      logit_offset=li.logit_offset)
        torch.cuda.synchronize()
        outs[name] = (cfg, li, desc, ws, y_ref, y)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for _ in range(3):
        for s, name in zip(streams, ("a", "b")):
            cfg, li, desc, ws, y_ref, y = outs[name]
            with torch.cuda.stream(s):
                M.moe_forward(desc, li.x, li.w_gate, li.w1, li.w3, li.w2, y, ws, bias=li.bias,
                              logit_offset=li.logit_offset, stream=s)
    torch.cuda.synchronize()
    for name in ("a", "b"):
        cfg, li, desc, ws, y_ref, y = outs[name]
        M.check_device_errors(ws, f"forward {name}")
        assert torch.equal(y, y_ref), name


@pytest.mark.parametrize("name", ["v3_decode", "tiny"])
def test_forward_replays_from_a_cuda_graph(M, name):
    # moe_forward issues only stream work (no allocation, no host synchronisation), so a serving loop
    # can capture it once in a CUDA graph and replay it on new inputs written into the same buffers
    cfg = W.CONFIGS[name]
    li = W.make_layer(cfg, device="cuda")
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, cfg.T)
    x = li.x.clone()
    y = torch.empty_like(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def fwd(y_out, w):
        M.moe_forward(desc, x, li.w_gate, li.w1, li.w3, li.w2, y_out, w, bias=li.bias,
                      logit_offset=li.logit_offset, stream=s)

    with torch.cuda.stream(s):
        fwd(y, ws)   # first call outside the capture: one-time host setup
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fwd(y, ws)
    ws_ref = M.Workspace(desc, cfg.T)
    y_ref = torch.empty_like(x)
    for seed in (101, 202):
        x.copy_(W.normal_bf16(tuple(x.shape), 1.0, seed, W.TID_X, device="cuda"))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            fwd(y_ref, ws_ref)
        torch.cuda.synchronize()
        M.check_device_errors(ws, "graph replay")
        M.check_device_errors(ws_ref, "direct call")
        assert torch.equal(y, y_ref), seed
    del g
