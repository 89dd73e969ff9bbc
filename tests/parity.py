"""Helpers shared by the GPU parity tests: run the oracle on CPU copies of the generated inputs and
compare the library's outputs with it.

Rules (the routing parity rule of the layer):
* routing indices match the oracle exactly for every token that is not near-tied -- a token is
  exempt when its oracle k-th and (k+1)-th masked selection scores, or its last kept and first
  dropped group scores, differ by less than 1e-5; an exempt token's GPU choice must still be one
  of the valid near-tied choices; inside a token's k experts the order may differ only between
  experts whose scores are within 1e-5;
* expert counts match exactly once the exempt tokens' GPU choices are substituted;
* gate weights agree to fp32 rounding of the score arithmetic;
* layer outputs agree within max|err| <= 2e-2 * rms(y_oracle), except for final bf16 rounding flips
  (within two bf16 ulps, at most one element in 10^4), and mean|err| <= 2e-3 * rms; a single
  expert's outputs also element by element within one bf16 ulp plus a small absolute term.
"""
from __future__ import annotations

import itertools

import numpy as np
import torch

import oracle as O
from oracle.moe_oracle import _e4m3_round   # the oracle's nearest-E4M3 rounding, at a given scale
from mixture_experts_routing_gate_b200 import workloads as W

TIE = 1e-5


def np64(t: torch.Tensor) -> np.ndarray:
    """fp64 numpy copy of a tensor (the widening is exact for bf16 and fp32 inputs)."""
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_gate_of(cfg, x, w_gate, bias, off) -> O.GateResult:
    return O.gate(np64(x), np64(w_gate), O.Hyper.of(cfg),
                  None if bias is None else bias.cpu().numpy(), None if off is None else off.cpu().numpy())


def _valid_near_tie(cfg, b_row: np.ndarray, gpu_idx: np.ndarray, has_bias: bool) -> bool:
    """True if gpu_idx is the top-k of some group selection whose groups are within TIE of the cut,
    up to TIE among the experts."""
    k, G, g, E = cfg.topk, cfg.n_groups, cfg.n_limited_groups, cfg.n_experts
    if len(set(gpu_idx.tolist())) != k:
        return False
    per = E // G
    if G > 1:
        grp = b_row.reshape(G, per).astype(np.float64)
        gs = np.sort(grp, axis=1)[:, ::-1]
        gscore = gs[:, 0] + gs[:, 1] if has_bias else gs[:, 0]
        cut = np.sort(gscore)[::-1][g - 1]
        cands = [c for c in itertools.combinations(range(G), g) if all(gscore[i] >= cut - TIE for i in c)]
    else:
        cands = [(0,)]
        per = E
    for c in cands:
        allowed = np.zeros(E, bool)
        for gi in c:
            allowed[gi * per:(gi + 1) * per] = True
        if not allowed[gpu_idx].all():
            continue
        masked = np.where(allowed, b_row.astype(np.float64), -np.inf)
        kth = np.sort(masked)[::-1][k - 1]
        if np.all(masked[gpu_idx] >= kth - TIE):
            return True
    return False


def compare_routing(cfg, g: O.GateResult, idx_gpu: np.ndarray, w_gpu: np.ndarray, bias=None):
    """Asserts the routing rule; returns (exempt tokens, expected counts).

    Non-exempt tokens: the set of experts is the oracle's exactly, and the order is the oracle's
    except between experts whose oracle selection scores are within TIE of each other (their fp32
    order is decided by summation-order rounding); weights are compared expert by expert.
    """
    idx_gpu = np.asarray(idx_gpu).astype(np.int64)
    w_gpu = np.asarray(w_gpu, np.float32)
    T = g.indices.shape[0]
    exempt = g.exempt(TIE)
    ok = np.ones(T, bool)
    ok[exempt] = False
    b = g.scores if bias is None else (g.scores + np.asarray(bias, np.float32)).astype(np.float32)
    same_set = np.array([np.array_equal(np.sort(idx_gpu[t]), np.sort(g.indices[t])) for t in range(T)])
    bad = np.nonzero(ok & ~same_set)[0]
    assert bad.size == 0, f"{bad.size} non-exempt tokens chose other experts, e.g. token {bad[:5]}: " \
                          f"gpu {idx_gpu[bad[:1]]} oracle {g.indices[bad[:1]]} gaps {g.expert_gap[bad[:3]]}"
    reordered = np.nonzero(ok & (idx_gpu != g.indices).any(axis=1))[0]
    for t in reordered:
        sg = b[t, idx_gpu[t]].astype(np.float64)
        so = b[t, g.indices[t]].astype(np.float64)
        assert np.all(np.abs(sg - so) < TIE), f"token {t}: order differs beyond near-ties: {idx_gpu[t]} vs {g.indices[t]}"
    for t in exempt:
        assert _valid_near_tie(cfg, b[t], idx_gpu[t], bias is not None), f"exempt token {t}: invalid choice"
    # weights, matched by expert: fp32 score arithmetic, differences from summation order only
    og = np.argsort(idx_gpu[ok], axis=1, kind="stable")
    oo = np.argsort(g.indices[ok], axis=1, kind="stable")
    wg = np.take_along_axis(w_gpu[ok], og, axis=1)
    wo = np.take_along_axis(g.weights[ok], oo, axis=1)
    np.testing.assert_allclose(wg, wo, rtol=2e-5, atol=2e-6 * cfg.route_scale)
    # counts, with the exempt tokens' GPU choices substituted
    ref_idx = g.indices.copy()
    ref_idx[exempt] = idx_gpu[exempt]
    return exempt, np.bincount(ref_idx.reshape(-1), minlength=cfg.n_experts)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(a)).astype(int) - 7)


def rounding_slack(y_ref: np.ndarray, terms: dict) -> np.ndarray:
    """Per element, the change one bf16 rounding flip in each rounded input of y could make:
    ulp(y) + sum_j w_j ulp(o_j) + ulp(o_shared), from the oracle's own summands."""
    slack = bf16_ulp(y_ref).copy()
    for t, row in enumerate(terms["routed"]):
        for w, o in row:
            slack[t] += abs(w) * bf16_ulp(o)
    if terms.get("shared") is not None:
        slack += bf16_ulp(terms["shared"])
    return slack


def assert_outputs_close(y_gpu: np.ndarray, y_ref: np.ndarray, what: str, per_element: bool = False,
                         slack: np.ndarray = None):
    """The layer's output bar, max|err| <= 2e-2 rms(y_ref), applied to every element except bf16
    rounding flips: an element may exceed the bar only if its error is within `slack` (by default
    two bf16 ulps of y; for a layer output, one ulp of y plus one ulp of every bf16 expert output
    that feeds it, weighted -- see rounding_slack), and at most one element in 10^4 may do so.
    Also mean|err| <= 2e-3 rms.

    Why the exception: both sides round every expert output and y to bf16 after fp32 sums whose
    order differs at the last bit; when |y| or an expert output exceeds ~4 rms(y), one of its ulps
    is larger than 2e-2 rms, so a single rounding flip of a large value can cross the bar.
    With per_element (one expert's output, a single bf16 rounding after fp32 accumulation), also
    99.9 % of elements within one bf16 ulp plus 2e-3 rms.  Returns max|err| / rms.
    """
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    err = np.abs(y_gpu - y_ref)
    over = err > 2e-2 * rms
    lim = 2 * bf16_ulp(y_ref) if slack is None else slack
    flips = over & (err <= lim)
    assert not np.any(over & ~flips), f"{what}: max err {err[over & ~flips].max()} > 2e-2 * rms {rms} " \
                                      f"and beyond one rounding flip of its inputs"
    assert flips.sum() <= max(1, err.size // 10000), f"{what}: {flips.sum()} rounding flips above 2e-2 rms"
    assert float(err.mean()) <= 2e-3 * rms + 1e-30, f"{what}: mean err {err.mean()} > 2e-3 * rms {rms}"
    if per_element:
        lim = 2.0 ** -7 * np.abs(y_ref) + 2e-3 * rms
        frac = float(np.mean(err <= lim)) if err.size else 1.0
        assert frac >= 0.999, f"{what}: only {frac:.5f} of elements within one bf16 ulp + 2e-3 rms"
    return float(err.max(initial=0.0) / rms) if rms else 0.0


def mx_flip_slack(xr, w1, w3, w2, limit=None, row_weight=None, y_ref=None, ulps: int = 16) -> np.ndarray:
    """Per-element slack [n, d] of one expert computed on E4M3 activations (O.mx_swiglu_expert) for
    the h codes that the kernel may round to the other neighbour.

    The kernel accumulates g and v in fp32 in its own order (the products of E4M3 and E2M1 values
    are exact) and evaluates silu in fp32 with the fast exponential, so its h may differ from the
    oracle's by up to about `ulps` fp32 ulps of the sum of the products' magnitudes, carried through
    silu(g) * v, plus the fast silu's relative error.  Within that reach an h element may take the neighbouring E4M3 code, and a
    block whose maximum may cross a power-of-two boundary may take the other scale (every element
    of it then re-rounded on the other grid).  The largest move of each element's quantised value
    over those cases, times |w2[c, i]|, summed over the row, bounds the change of y[r, c]; the
    slack adds two bf16 ulps for the output's own rounding.  Which code the kernel picks for such
    an element is not unique; everything else the test compares is."""
    xr = np.asarray(xr, np.float64)
    w1, w3, w2 = (np.asarray(a, np.float64) for a in (w1, w3, w2))
    act = O.mx_swiglu_hidden(xr, w1, w3, limit, row_weight)
    xq = O.e4m3_block_dequant(*O.quantize_e4m3_block(xr))
    u = 2.0 ** -24
    dg = ulps * u * (np.abs(xq) @ np.abs(w1).T)
    dv = ulps * u * (np.abs(xq) @ np.abs(w3).T)
    g, v = xq @ w1.T, xq @ w3.T
    if limit is not None:
        g, v = np.minimum(g, limit), np.clip(v, -limit, limit)
    sig = 1.0 / (1.0 + np.exp(-g))
    rw = 1.0 if row_weight is None else np.abs(np.asarray(row_weight, np.float64))[:, None]
    # silu in fp32 with the fast exponential and division: their documented maximum errors (2 + 1.17|z|
    # ulps for exp(z), 2 ulps for the division) bound its relative error by about (4 + 1.2|g|) ulps
    dact = (np.abs(sig * (1.0 + g * (1.0 - sig)) * v) * dg + np.abs(g * sig) * dv) * rw + \
        (4.0 + 1.2 * np.abs(g)) * 2.0 ** -23 * np.abs(act)
    n, I = act.shape
    blk = lambda a: a.reshape(n, I // 32, 32)
    amax_hi = blk(np.abs(act) + dact).max(axis=2)
    amax_lo = blk(np.maximum(np.abs(act) - dact, 0.0)).max(axis=2)

    def least_exp(amax):
        _, ex = np.frexp(amax)
        e = ex.astype(np.int64) - 9
        e = np.where(np.ldexp(448.0, e) >= amax, e, e + 1)
        return np.where(amax == 0, -127, np.clip(e, -127, 127))

    def qval(a, e):   # a quantised on the grid of block scale 2^e (saturating at 448 * 2^e)
        sc = np.repeat(np.ldexp(1.0, e), 32, axis=1)
        return O.e4m3_value(_e4m3_round(a / sc)) * sc

    chosen = O.e4m3_block_dequant(*O.quantize_e4m3_block(act))
    gap = np.zeros_like(act)
    for e in (least_exp(amax_lo), least_exp(amax_hi)):
        for a in (act - dact, act + dact):
            gap = np.maximum(gap, np.abs(qval(a, e) - chosen))
    flip = gap @ np.abs(w2).T
    if y_ref is None:
        y_ref = O.round_bf16(chosen @ w2.T)
    return flip + 2 * bf16_ulp(np.abs(np.asarray(y_ref, np.float64)) + flip)


def expert_fetcher(li: W.LayerInputs):
    """Oracle-side access to the generated expert weights (copied from the device one expert at a time)."""
    def fetch(e):
        return np64(li.w1[e]), np64(li.w3[e]), np64(li.w2[e])
    return fetch


def oracle_by_expert(x64: np.ndarray, fetch, indices: np.ndarray, weights: np.ndarray, E: int, sample_rows,
                     whole_experts, tok_of_row: np.ndarray, offsets: np.ndarray):
    """The oracle's expert outputs for a full-size layer, each expert's weights fetched once.

    Returns (whole, y_sample, terms, shared):
    * whole[e]  = O.swiglu_expert on every row routed to e (in dispatch's row order), for e in whole_experts;
    * y_sample  = O.combine of the sampled tokens' expert outputs and their shared-expert rows
                  (the layer output y for those tokens, as O.moe_forward computes it);
    * terms     = the summands of y_sample (for rounding_slack);
    * shared    = O.swiglu_expert of the shared expert on all T tokens.
    """
    sample_rows = np.asarray(sample_rows)
    idx_s = np.asarray(indices)[sample_rows]
    w_s = np.asarray(weights, np.float32)[sample_rows]
    need = sorted(set(idx_s.reshape(-1).tolist()) | set(int(e) for e in whole_experts))
    whole, outs = {}, {}
    for e in need:
        w1, w3, w2 = fetch(e)
        if e in whole_experts:
            rows = slice(int(offsets[e]), int(offsets[e + 1]))
            whole[e] = O.swiglu_expert(x64[tok_of_row[rows]], w1, w3, w2)
        toks = np.nonzero((idx_s == e).any(axis=1))[0]
        if toks.size:
            o = O.swiglu_expert(x64[sample_rows[toks]], w1, w3, w2)
            outs[e] = {int(t): o[r] for r, t in enumerate(toks)}
    shared = O.swiglu_expert(x64, *fetch(E))
    y_sample = O.combine(len(sample_rows), x64.shape[1], idx_s, w_s, outs, shared[sample_rows])
    terms = {"routed": [[(float(w_s[t, j]), outs[int(idx_s[t, j])][t]) for j in range(idx_s.shape[1])]
                        for t in range(len(sample_rows))],
             "shared": shared[sample_rows]}
    return whole, y_sample, terms, shared
