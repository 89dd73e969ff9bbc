"""Parity of the MXFP4 expert-weight path ("From One Giant FFN to 384 Tiny Experts", section 11.6)
with the CPU oracle, through the C ABI, on a B200.

Two activation precisions: by default the activations are MX-quantised to E4M3 with UE8M0 scales per
32 elements and the experts run on the block-scaled tensor cores (kind::mxf8f6f4: E2M1 weights x E4M3
activations); with MOE_OPT_MXFP4_BF16_ACTIVATIONS the activations stay bf16 and the weights are
decoded to bf16 inside the GEMM.  The oracle decodes every expert's E2M1 codes and UE8M0 scales by
their plain definition and runs the matching expert (O.mx_swiglu_expert, or the bf16 O.swiglu_expert
on the decoded weights, which are exact in bf16).  Expert outputs are compared element by element on
small layers that span several tiles and ragged tails, and layer outputs on sampled tokens of the
synthetic layers.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_routing_gate_b200 import build as B
from mixture_experts_routing_gate_b200 import workloads as W
from parity import assert_outputs_close, compare_routing, mx_flip_slack, np64, rounding_slack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    B.build()
    from mixture_experts_routing_gate_b200 import moe
    return moe


def _skewed_indices(T, E, k, seed):
    """Distinct experts per token drawn with Zipf-like expert popularity (some experts empty)."""
    rng = np.random.default_rng(seed)
    pop = 1.0 / np.arange(1, E + 1) ** 1.2
    pop[E // 2:E // 2 + 3] = 0.0
    pop /= pop.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=pop) for _ in range(T)]).astype(np.int32)


def _decoded_fetcher(w):
    """Oracle-side decode of one expert's MXFP4 weights (copied from the device one expert at a time)."""
    def fetch(e):
        return tuple(O.mxfp4_dequant(q[e].cpu().numpy(), s[e].cpu().numpy())
                     for q, s in ((w.w1, w.w1s), (w.w3, w.w3s), (w.w2, w.w2s)))
    return fetch


ACTS = ["e4m3", "bf16"]


def _options(M, act):
    return 0 if act == "e4m3" else M.MOE_OPT_MXFP4_BF16_ACTIVATIONS


def _expert_ref(act):
    return O.mx_swiglu_expert if act == "e4m3" else O.swiglu_expert


def _check_expert(act, got, xr, weights, what, limit=None, row_weight=None):
    """One expert's rows against the oracle; on E4M3 activations an element beyond the bar may be
    explained by h codes the kernel can round either way (mx_flip_slack)."""
    ref = _expert_ref(act)(xr, *weights, limit=limit, row_weight=row_weight)
    slack = mx_flip_slack(xr, *weights, limit=limit, row_weight=row_weight, y_ref=ref) if act == "e4m3" else None
    return assert_outputs_close(got, ref, what, per_element=True, slack=slack)


def _run_experts(M, cfg, T, idx, w, row_weights=None, gather=False, act="e4m3", token_chunk=0):
    E, k, d = cfg.n_experts, cfg.topk, cfg.dim
    x = W.normal_bf16((T, d), 1.0, cfg.seed, W.TID_X, device="cuda")
    desc = M.layer_desc(cfg, options=_options(M, act), token_chunk=token_chunk)
    ws = M.Workspace(desc, T)
    S = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ros = torch.empty(S, dtype=torch.int32, device="cuda")
    tor = torch.empty(S, dtype=torch.int32, device="cuda")
    xp = None if gather else torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    M.moe_dispatch(desc, torch.from_numpy(idx).cuda(), x, counts, offsets, ros, tor, xp, ws)
    out_perm = torch.full((S, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    out_sh = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    if gather:
        M.moe_expert_ffn_mxfp4_gather(desc, tor, offsets, x, w, out_perm, out_sh, ws, row_weights=row_weights)
    else:
        M.moe_expert_ffn_mxfp4(desc, xp, offsets, x, w, out_perm, out_sh, ws, row_weights=row_weights)
    return x, out_perm, out_sh, ws


MXFP4_CASES = [
    (600, 16, 4, 512, 512),     # 256-row token chunks (experts average 150 rows)
    (3000, 16, 4, 512, 512),    # experts spanning several 256-row chunks
    (2500, 16, 4, 1536, 1024),  # several feature blocks in both GEMMs; scale rows of 48 and 32 bytes
    (100, 32, 4, 512, 1024),    # 128-row chunks (experts average 12.5 rows)
    (64, 16, 4, 512, 512),      # E4M3: T <= 64, one CTA per tile (64-row chunks); hot experts of up to 64 rows
    (40, 32, 4, 1536, 1024),    # E4M3: one CTA per tile, several feature blocks in both GEMMs
    (96, 16, 4, 512, 1024),     # E4M3: T <= 96, so 96-row chunks with two accumulator buffers
    (97, 16, 4, 512, 512),      # E4M3: one token more, 224-row chunks again
    (1, 16, 4, 512, 512),       # one token
]


@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("T,E,k,d,I", MXFP4_CASES)
def test_expert_ffn_mxfp4_parity(M, T, E, k, d, I, act):
    _expert_parity(M, T, E, k, d, I, act)


@pytest.mark.parametrize("T,E,k,d,I", [(600, 16, 4, 512, 512), (3000, 16, 4, 1024, 512), (300, 64, 6, 512, 512)])
def test_expert_ffn_mxfp4_two_buffer_chunks(M, T, E, k, d, I):
    """Chunks of 96 rows chosen by the caller (token_chunk): experts spanning several chunks, tiles
    alternating between the two accumulator buffers, ragged last chunks."""
    _expert_parity(M, T, E, k, d, I, "e4m3", token_chunk=96)


def _expert_parity(M, T, E, k, d, I, act, token_chunk=0):
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d,
                                    inter_dim=I, w_std=0.05, seed=40 + T)
    w = W.make_mxfp4_weights(cfg, device="cuda")
    idx = _skewed_indices(T, E, k, seed=7 * T + E)
    x, out_perm, out_sh, ws = _run_experts(M, cfg, T, idx, w, act=act, token_chunk=token_chunk)
    M.check_device_errors(ws, "moe_expert_ffn_mxfp4")
    c, o, _, tok = O.dispatch(idx, E)
    if T >= 600:
        assert c.max() > 128 and (c == 0).any()
    x64 = np64(x)
    got = np64(out_perm)
    fetch = _decoded_fetcher(w)
    for e in range(E):
        if c[e] == 0:
            continue
        _check_expert(act, got[o[e]:o[e + 1]], x64[tok[o[e]:o[e + 1]]], fetch(e), f"expert {e}")
    _check_expert(act, np64(out_sh), x64, fetch(E), "shared expert")


@pytest.mark.parametrize("act", ACTS)
def test_expert_ffn_mxfp4_clamp_and_row_weights(M, act):
    T, E, k, d, I = 500, 16, 4, 512, 512
    limit = 0.5
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d,
                                    inter_dim=I, w_std=0.05, seed=77, swiglu_limit=limit)
    w = W.make_mxfp4_weights(cfg, device="cuda")
    idx = _skewed_indices(T, E, k, seed=99)
    rw = W.uniform(T * k, 12, 90).to(torch.float32).cuda() * 2.0
    x, out_perm, out_sh, ws = _run_experts(M, cfg, T, idx, w, row_weights=rw, act=act)
    M.check_device_errors(ws, "moe_expert_ffn_mxfp4")
    c, o, _, tok = O.dispatch(idx, E)
    x64 = np64(x)
    got = np64(out_perm)
    rwn = rw.cpu().numpy()
    fetch = _decoded_fetcher(w)
    for e in range(E):
        if c[e] == 0:
            continue
        _check_expert(act, got[o[e]:o[e + 1]], x64[tok[o[e]:o[e + 1]]], fetch(e), f"expert {e}", limit=limit,
                      row_weight=rwn[o[e]:o[e + 1]])
    _check_expert(act, np64(out_sh), x64, fetch(E), "shared expert", limit=limit)


@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("T,E,k,d,I", [(3000, 16, 4, 512, 512), (100, 32, 4, 512, 1024), (1, 16, 4, 512, 512)])
def test_expert_ffn_mxfp4_gather_bit_identical(M, T, E, k, d, I, act):
    # routed rows gathered from x by the up projection give the results of the x_perm path, bit for bit
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d,
                                    inter_dim=I, w_std=0.05, seed=60 + T)
    w = W.make_mxfp4_weights(cfg, device="cuda")
    idx = _skewed_indices(T, E, k, seed=11 * T + E)
    rw = W.uniform(T * k, 17, 90).to(torch.float32).cuda() * 2.0
    _, p0, s0, ws0 = _run_experts(M, cfg, T, idx, w, row_weights=rw, act=act)
    _, p1, s1, ws1 = _run_experts(M, cfg, T, idx, w, row_weights=rw, gather=True, act=act)
    M.check_device_errors(ws0, "moe_expert_ffn_mxfp4")
    M.check_device_errors(ws1, "moe_expert_ffn_mxfp4_gather")
    assert torch.equal(p0, p1) and torch.equal(s0, s1)


@pytest.mark.parametrize("act", ACTS)
def test_mxfp4_scale_out_of_range_is_reported(M, act):
    T, E, k, d, I = 64, 16, 4, 512, 512
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d,
                                    inter_dim=I, w_std=0.05, seed=5)
    w = W.make_mxfp4_weights(cfg, device="cuda")
    w.w2s[E, 3, 1] = 253   # the shared expert always runs, so this block is always decoded
    idx = _skewed_indices(T, E, k, seed=1)
    _, _, _, ws = _run_experts(M, cfg, T, idx, w, act=act)
    st, info = M.moe_get_error(ws)
    assert st == M.MOE_ERR_DEVICE and info == 0x10000 + 253


def test_forward_mxfp4_v3_prefill(M, act="e4m3"):
    # the V3-shaped prefill layer with MXFP4 experts: routing of every token, outputs of sampled tokens
    cfg = W.CONFIGS["v3_prefill"]
    x, wg, bias, off = W.make_router_inputs(cfg, device="cuda")
    w = W.make_mxfp4_weights(cfg, device="cuda")
    desc = M.layer_desc(cfg, options=_options(M, act))
    ws = M.Workspace(desc, cfg.T)
    y = torch.empty_like(x)
    wout = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
    iout = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device="cuda")
    cout = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    M.moe_forward_mxfp4(desc, x, wg, w, y, ws, bias=bias, logit_offset=off, weights_out=wout, indices_out=iout,
                        counts_out=cout)
    M.check_device_errors(ws, "moe_forward_mxfp4")
    hp = O.Hyper.of(cfg)
    x64, wg64, b = np64(x), np64(wg), bias.cpu().numpy()
    g = O.gate(x64, wg64, hp, b, None)
    exempt, counts = compare_routing(cfg, g, iout.cpu().numpy(), wout.cpu().numpy(), b)
    assert np.array_equal(cout.cpu().numpy(), counts)
    rows = np.setdiff1d(W.sample_rows(cfg.T, 16, seed=cfg.seed + 300), exempt)
    terms = {}
    y_ref, _, _, _ = O.moe_forward(x64[rows], hp, _decoded_fetcher(w), wg64, b, None, terms=terms,
                                   mx_activations=act == "e4m3")
    r = assert_outputs_close(np64(y)[rows], y_ref, "v3_prefill mxfp4 y (sampled rows)",
                             slack=rounding_slack(y_ref, terms))
    print(f"v3_prefill mxfp4: max |y - y_oracle| / rms = {r:.4f} over {len(rows)} sampled tokens")
    assert torch.isfinite(y.float()).all()


def _forward_mxfp4(M, cfg, x, wg, bias, off, w, token_ids=None, tid2eid=None, act="e4m3"):
    desc = M.layer_desc(cfg, options=_options(M, act))
    ws = M.Workspace(desc, cfg.T)
    y = torch.empty_like(x)
    wout = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device="cuda")
    iout = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device="cuda")
    cout = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    M.moe_forward_mxfp4(desc, x, wg, w, y, ws, bias=bias, logit_offset=off, token_ids=token_ids, tid2eid=tid2eid,
                        weights_out=wout, indices_out=iout, counts_out=cout)
    M.check_device_errors(ws, "moe_forward_mxfp4")
    return y, iout.cpu().numpy(), wout.cpu().numpy(), cout.cpu().numpy()


def test_forward_mxfp4_hash_layer(M):
    # the hash-routed layer (tid2eid from the greedy builder) with MXFP4 experts
    cfg = W.CONFIGS["hash"].replace(T=2048)
    p = W.token_frequencies(cfg)
    table, _ = M.moe_build_tid2eid(p, cfg.n_experts, cfg.topk)
    ids = W.sample_token_ids(cfg, p)
    x, wg, _, _ = W.make_router_inputs(cfg, device="cuda")
    w = W.make_mxfp4_weights(cfg, device="cuda")
    y, iw, ww, cw = _forward_mxfp4(M, cfg, x, wg, None, None, w, token_ids=torch.from_numpy(ids).cuda(),
                                   tid2eid=torch.from_numpy(table).cuda())
    x64, wg64 = np64(x), np64(wg)
    i_ora, w_ora = O.hash_gate(ids, table, x64, wg64, cfg.route_scale)
    assert np.array_equal(iw, i_ora)
    np.testing.assert_allclose(ww, w_ora, rtol=2e-5, atol=2e-6)
    assert np.array_equal(cw, np.bincount(i_ora.reshape(-1), minlength=cfg.n_experts))
    rows = W.sample_rows(cfg.T, 8, seed=cfg.seed + 400)
    terms = {}
    y_ref, _, _, _ = O.moe_forward(x64[rows], O.Hyper.of(cfg), _decoded_fetcher(w), wg64, terms=terms,
                                   token_ids=ids[rows], tid2eid=table, mx_activations=True)
    r = assert_outputs_close(np64(y)[rows], y_ref, "hash mxfp4 y (sampled rows)", slack=rounding_slack(y_ref, terms))
    print(f"hash mxfp4: max |y - y_oracle| / rms = {r:.4f} over {len(rows)} sampled tokens")


@pytest.mark.parametrize("act", ACTS)
def test_forward_mxfp4_v4_style_expert(M, act):
    # the V4-shaped skewed layer with MXFP4 experts, the SwiGLU clamp and the weight inside each expert
    cfg = W.CONFIGS["v4_skew"].replace(T=2048, swiglu_limit=10.0, weight_in_expert=True)
    x, wg, bias, off = W.make_router_inputs(cfg, device="cuda")
    w = W.make_mxfp4_weights(cfg, device="cuda")
    y, iw, ww, cw = _forward_mxfp4(M, cfg, x, wg, bias, off, w, act=act)
    hp = O.Hyper.of(cfg)
    x64, wg64, b, o = np64(x), np64(wg), bias.cpu().numpy(), off.cpu().numpy()
    g = O.gate(x64, wg64, hp, b, o)
    exempt, counts = compare_routing(cfg, g, iw, ww, b)
    assert np.array_equal(cw, counts)
    rows = np.setdiff1d(W.sample_rows(cfg.T, 8, seed=cfg.seed + 500), exempt)
    terms = {}
    y_ref, _, _, _ = O.moe_forward(x64[rows], hp, _decoded_fetcher(w), wg64, b, o, terms=terms,
                                   swiglu_limit=10.0, weight_in_expert=True, mx_activations=act == "e4m3")
    r = assert_outputs_close(np64(y)[rows], y_ref, "v4 mxfp4 y (sampled rows)", slack=rounding_slack(y_ref, terms))
    print(f"v4_skew mxfp4 {act} (clamp, weight inside): max |y - y_oracle| / rms = {r:.4f} over {len(rows)} tokens")


@pytest.mark.parametrize("act", ACTS)
def test_forward_mxfp4_v3_decode(M, act):
    # the decode batch (T=64, 2 rows per expert on average) with MXFP4 experts: routing of every
    # token, outputs of every token
    cfg = W.CONFIGS["v3_decode"]
    x, wg, bias, off = W.make_router_inputs(cfg, device="cuda")
    w = W.make_mxfp4_weights(cfg, device="cuda")
    y, iw, ww, cw = _forward_mxfp4(M, cfg, x, wg, bias, off, w, act=act)
    hp = O.Hyper.of(cfg)
    x64, wg64, b = np64(x), np64(wg), bias.cpu().numpy()
    g = O.gate(x64, wg64, hp, b, None)
    exempt, counts = compare_routing(cfg, g, iw, ww, b)
    assert np.array_equal(cw, counts)
    rows = np.setdiff1d(np.arange(cfg.T), exempt)
    terms = {}
    y_ref, _, _, _ = O.moe_forward(x64[rows], hp, _decoded_fetcher(w), wg64, b, None, terms=terms,
                                   mx_activations=act == "e4m3")
    r = assert_outputs_close(np64(y)[rows], y_ref, "v3_decode mxfp4 y", slack=rounding_slack(y_ref, terms))
    print(f"v3_decode mxfp4 {act}: max |y - y_oracle| / rms = {r:.4f} over {len(rows)} tokens")
