"""Plain CPU oracle of the MoE layer forward (numpy, fp64) -- test infrastructure.

Only the tests, the package smoke self-check and the benchmark's CPU-baseline
leg may import this module.  It shares nothing with the CUDA library.

What it restates, and where each step comes from (pages cited by title):

* "DeepSeek-V3.2-Exp - Routing weights", gate-forward excerpt: router logits
  ``linear(x.float(), weight.float())``, sigmoid / softmax affinity, a bias
  added for selection only, group-limited top-k (groups scored by the sum of
  their two best biased scores, or by the max without a bias), top-k experts,
  the unbiased scores gathered, renormalised (sigmoid) and scaled.
* "From One Giant FFN to 384 Tiny Experts", section 11.2: the Sqrt(Softplus)
  affinity of DeepSeek-V4; section 11.1: hash routing by token id; section 1:
  the SwiGLU expert ``W_down(SiLU(W_gate u) * W_up u)``; section 6: the bias
  perturbs only the top-k cut.
* "DeepSeek-V3.2-Exp - Routing weights", moe-forward excerpt, and
  "DeepSeek V4.1 - Add shared": bincount of the chosen experts, the per-expert
  gather ``x[idx]``, the fp32 accumulator ``y[idx] += expert(x[idx]) * w``,
  the shared expert added for every token, the cast back to the input dtype.
* "From One Giant FFN to 384 Tiny Experts", section 11.6: expert weights in
  the OCP MXFP4 format, E2M1 elements sharing one power-of-two (UE8M0) scale
  per block of 32 along a row; the expert computes with the decoded weights,
  on bf16 activations or on FP8 (E4M3) activations MX-quantised with UE8M0
  scales per 32 elements ("FP8 for everything else").
* "How was DeepSeek V4's tid2eid derived?", sections "Mathematical
  formulation" (eq. 1, eq. 2), the greedy rule and "Reference implementation":
  tokens in descending frequency each take the k currently lightest experts,
  each of which gains p_i / k; balance is measured by max_vio / min_vio.

Precision (the pages fix fp32 scores and a bf16 model):
* logits: fp64 dot products of bf16 x and fp32 router weights, rounded once to
  fp32 (for bf16-valued weights every product is exact in fp64, so this is the
  fp32 rounding of the true dot product up to fp64 summation error);
* affinities evaluated in fp64 from the fp32 logit and rounded to fp32;
  selection scores, group scores, renormalisation and scaling in fp32 with
  IEEE round-to-nearest-even, as torch computes them on fp32 tensors;
* expert: both projections in fp64 rounded to fp32, ``silu(z_g) * z_v`` in
  fp64 rounded to bf16, down projection in fp64 rounded to bf16;
* combine: fp32 products and sums in ascending expert order, the shared
  expert last, one final rounding to bf16.

Readings of the pages taken here (each one is also listed in the design
notes): ties in every top-k go to the lower index; sqrt-softplus weights are
renormalised like sigmoid ones; w1 is the gate branch and w3 the value branch;
the routing weight multiplies the bf16 expert output in the combine; the greedy
builder breaks load ties by the lower expert index.

Parity pins (tests/test_oracle_pins.py): brute force over all group and expert
subsets on tiny inputs; the no-group case against a plain descending sort;
exact rational arithmetic for logits; closed forms of the affinities; the
greedy builder on hand-worked examples, against a heap-based re-implementation
and against the closed form of the "extreme case"; dispatch invariants; an
identity-like expert layer whose output is known in closed form; the E2M1,
E4M3 and UE8M0 decodes and the E4M3 rounding against ml_dtypes; hand-worked MX
blocks; the least-scale and half-step properties of the MX quantiser; an
identity-like expert on FP8 activations with a derived error bound.  Every
function below is pinned by at least one of them.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional, Sequence

import numpy as np

__all__ = [
    "round_bf16", "round_f32", "router_logits", "affinity", "select_experts",
    "gate_weights", "GateResult", "gate", "hash_gate", "build_tid2eid", "balance",
    "best_tid2eid", "primes_above", "ngram_experts", "ngram_gate", "update_bias",
    "dispatch", "silu", "swiglu_expert", "combine", "moe_forward", "Hyper",
    "e2m1_value", "ue8m0_value", "mxfp4_dequant", "e4m3_value", "quantize_e4m3_block",
    "e4m3_block_dequant", "mx_swiglu_hidden", "mx_swiglu_expert",
]


# ----------------------------------------------------------------------------------------------
# rounding helpers
# ----------------------------------------------------------------------------------------------

def round_bf16(a) -> np.ndarray:
    """Round to the nearest bf16 value (8 significant bits), ties to even; result held in fp64."""
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)                       # a = m * 2**e with 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # np.rint rounds half to even


def round_f32(a) -> np.ndarray:
    """Round to fp32 (numpy's fp64 -> fp32 conversion is round-to-nearest-even)."""
    return np.asarray(a, dtype=np.float64).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class Hyper:
    """The routing hyper-parameters a Gate is built with (gate-init excerpt)."""
    n_experts: int
    n_groups: int
    n_limited_groups: int
    topk: int
    score_func: str = "sigmoid"
    route_scale: float = 1.0
    renorm: Optional[bool] = None            # default: sigmoid and sqrtsoftplus renormalise

    @property
    def do_renorm(self) -> bool:
        if self.renorm is not None:
            return self.renorm
        return self.score_func in ("sigmoid", "sqrtsoftplus")

    @staticmethod
    def of(obj) -> "Hyper":
        return Hyper(obj.n_experts, obj.n_groups, obj.n_limited_groups, obj.topk,
                     obj.score_func, obj.route_scale)


# ----------------------------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------------------------

def router_logits(x, w_gate, logit_offset=None) -> np.ndarray:
    """l[t, e] = fp32( sum_i x[t, i] * W[e, i] ), accumulated in fp64.

    gate-forward: ``linear(x.float(), self.weight.float())``.  An optional
    per-expert offset (the skewed synthetic layer's knob) is added to the fp32
    logit before the affinity.
    """
    l = round_f32(np.asarray(x, np.float64) @ np.asarray(w_gate, np.float64).T)
    if logit_offset is not None:
        l = (l + np.asarray(logit_offset, np.float32)).astype(np.float32)
    return l


def affinity(l, score_func: str) -> np.ndarray:
    """Affinity scores s from fp32 logits, evaluated in fp64 and rounded to fp32.

    sigmoid (gate-forward; "From One Giant FFN...", section 7),
    sqrt(softplus) (same essay, section 11.2),
    softmax over the experts (gate-forward, score_func == "softmax").
    """
    l = np.asarray(l, np.float64)
    if score_func == "sigmoid":
        s = 1.0 / (1.0 + np.exp(-l))
    elif score_func == "sqrtsoftplus":
        softplus = np.maximum(l, 0.0) + np.log1p(np.exp(-np.abs(l)))
        s = np.sqrt(softplus)
    elif score_func == "softmax":
        z = np.exp(l - l.max(axis=-1, keepdims=True))
        s = z / z.sum(axis=-1, keepdims=True)
    else:
        raise ValueError(score_func)
    return round_f32(s)


def _descending(v) -> np.ndarray:
    """Indices of v by value descending, equal values by index ascending."""
    return np.argsort(-np.asarray(v), kind="stable")


def select_experts(b, n_groups: int, n_limited_groups: int, topk: int, has_bias: bool):
    """Group-limited top-k of one token's selection scores b [E] (fp32).

    gate-forward: view the scores as [G, E/G]; score each group by the sum of
    its two largest entries when a bias exists, else by its largest; keep the
    ``n_limited_groups`` best groups, set the rest to -inf; take the top-k.
    Returns (experts [k] in descending score order, kept groups, expert gap,
    group gap) where the gaps are the differences between the last kept and
    the first dropped score (inf when nothing is dropped).
    """
    b = np.asarray(b, np.float32)
    E = b.shape[0]
    group_gap = np.inf
    kept = np.arange(n_groups)
    if n_groups > 1:
        per = b.reshape(n_groups, E // n_groups)
        if has_bias:
            top2 = np.sort(per, axis=1)[:, ::-1][:, :2]
            gscore = (top2[:, 0] + top2[:, 1]).astype(np.float32)
        else:
            gscore = per.max(axis=1)
        gorder = _descending(gscore)
        kept = np.sort(gorder[:n_limited_groups])
        if n_groups > n_limited_groups:
            group_gap = float(gscore[gorder[n_limited_groups - 1]]) - float(gscore[gorder[n_limited_groups]])
        masked = np.full_like(per, -np.inf)
        masked[kept] = per[kept]
        b = masked.reshape(E)
    order = _descending(b)
    experts = order[:topk]
    expert_gap = np.inf
    if E > topk and np.isfinite(b[order[topk]]):
        expert_gap = float(b[order[topk - 1]]) - float(b[order[topk]])
    return experts, kept, expert_gap, group_gap


def gate_weights(s_sel, do_renorm: bool, route_scale: float) -> np.ndarray:
    """Gate values of one token from the unbiased scores of its chosen experts (fp32).

    gate-forward: ``weights = original_scores.gather(...)``; for renormalising
    score functions divide by their sum (accumulated in the experts' output
    order); then multiply by route_scale.
    """
    w = np.asarray(s_sel, np.float32).copy()
    if do_renorm:
        total = np.float32(0.0)
        for v in w:
            total = np.float32(total + v)
        w = (w / total).astype(np.float32)
    return (w * np.float32(route_scale)).astype(np.float32)


@dataclasses.dataclass
class GateResult:
    indices: np.ndarray       # [T, k] int64, descending selection score
    weights: np.ndarray       # [T, k] fp32
    scores: np.ndarray        # [T, E] fp32 unbiased affinities
    expert_gap: np.ndarray    # [T] fp64: k-th minus (k+1)-th masked selection score
    group_gap: np.ndarray     # [T] fp64: last kept minus first dropped group score
    kept_groups: np.ndarray   # [T, n_limited_groups]

    def exempt(self, threshold: float = 1e-5) -> np.ndarray:
        """Tokens whose selection is decided by a near-tie (index list)."""
        return np.nonzero((self.expert_gap < threshold) | (self.group_gap < threshold))[0]


def gate(x, w_gate, hp: Hyper, bias=None, logit_offset=None) -> GateResult:
    """Gate.forward for a batch of tokens x [T, d]."""
    s = affinity(router_logits(x, w_gate, logit_offset), hp.score_func)
    b = s if bias is None else (s + np.asarray(bias, np.float32)).astype(np.float32)
    T = s.shape[0]
    idx = np.zeros((T, hp.topk), np.int64)
    wts = np.zeros((T, hp.topk), np.float32)
    eg = np.zeros(T)
    gg = np.zeros(T)
    kept = np.zeros((T, max(hp.n_limited_groups, 1) if hp.n_groups > 1 else 1), np.int64)
    for t in range(T):
        e, kg, eg[t], gg[t] = select_experts(b[t], hp.n_groups, hp.n_limited_groups, hp.topk, bias is not None)
        idx[t] = e
        kept[t, :len(kg)] = kg
        wts[t] = gate_weights(s[t, e], hp.do_renorm, hp.route_scale)
    return GateResult(idx, wts, s, eg, gg, kept)


def hash_gate(token_ids, tid2eid, x, w_gate, route_scale: float, score_func: str = "sigmoid",
              do_renorm: bool = True):
    """Hash-routed gate: experts = tid2eid[token_id] in table order ("From One Giant FFN...",
    section 11.1; "How was DeepSeek V4's tid2eid derived?"); weights = affinities of those
    experts, renormalised and scaled as in gate-forward.  Returns (indices [T,k], weights [T,k])."""
    tid2eid = np.asarray(tid2eid)
    idx = tid2eid[np.asarray(token_ids, np.int64)].astype(np.int64)
    s = affinity(router_logits(x, w_gate), score_func)
    wts = np.stack([gate_weights(s[t, idx[t]], do_renorm, route_scale) for t in range(idx.shape[0])]) \
        if idx.shape[0] else np.zeros((0, tid2eid.shape[1]), np.float32)
    return idx, wts


# ----------------------------------------------------------------------------------------------
# tid2eid
# ----------------------------------------------------------------------------------------------

def _k_lightest(f, k: int) -> np.ndarray:
    """The k experts of least load, by (load, expert index) ascending."""
    return np.argsort(f, kind="stable")[:k]


def build_tid2eid(p, n_experts: int, k: int, order: Optional[Sequence[int]] = None):
    """Greedy tid2eid ("How was DeepSeek V4's tid2eid derived?", greedy rule under eq. 2).

    Tokens are visited by descending frequency p (equal frequencies by token id),
    or in ``order`` when given (the randomised variant).  Each visited token is
    assigned the k experts currently carrying the least load, which each gain
    p_i / k.  Returns (table [m, k] int32, loads f [n] fp64).
    """
    p = np.asarray(p, np.float64)
    m = p.shape[0]
    visit = _descending(p) if order is None else np.asarray(order)
    f = np.zeros(n_experts, np.float64)
    table = np.zeros((m, k), np.int32)
    for i in visit:
        chosen = _k_lightest(f, k)
        table[i] = chosen
        f[chosen] += p[i] / k
    return table, f


def balance(f):
    """(max_vio, min_vio) = (n * max f - 1, n * min f - 1) (same page, reference implementation)."""
    f = np.asarray(f, np.float64)
    n = f.shape[0]
    return float(f.max() * n - 1.0), float(f.min() * n - 1.0)


def best_tid2eid(p, n_experts: int, k: int, orders):
    """The randomised variant (same page, after the reference implementation): build one table per
    visiting order (the caller draws the random permutations) and keep the one of least max_vio
    (equal max_vio: the earlier order).  Returns (table, loads, index of the kept order)."""
    best = None
    for r, order in enumerate(orders):
        table, f = build_tid2eid(p, n_experts, k, order)
        mx = balance(f)[0]
        if best is None or mx < best[3]:
            best = (table, f, r, mx)
    return best[0], best[1], best[2]


def primes_above(m: int, k: int):
    """The k smallest primes greater than m, by trial division."""
    out = []
    q = m + 1
    while len(out) < k:
        if q > 1 and all(q % f for f in range(2, int(q ** 0.5) + 1)):
            out.append(q)
        q += 1
    return out


def ngram_experts(prev_ids, ids, primes, n_experts: int) -> np.ndarray:
    """2-gram hash routing (tid2eid page, "An extreme case"): for the pair (a, b) of the previous and
    the current token, expert j = (a * q_j + b) mod n with one prime q_j > m per choice.  Duplicate
    experts are allowed.  Returns [T, k] int64."""
    prev_ids = [int(v) for v in np.asarray(prev_ids).reshape(-1)]
    ids = [int(v) for v in np.asarray(ids).reshape(-1)]
    return np.array([[(a * int(q) + b) % n_experts for q in primes] for a, b in zip(prev_ids, ids)], np.int64)


def ngram_gate(prev_ids, ids, primes, x, w_gate, route_scale: float, score_func: str = "sigmoid",
               do_renorm: bool = True):
    """Gate of a 2-gram hash layer: experts from ngram_experts, weights as in hash_gate (a duplicate
    expert contributes its score once per occurrence)."""
    idx = ngram_experts(prev_ids, ids, primes, np.asarray(w_gate).shape[0])
    s = affinity(router_logits(x, w_gate), score_func)
    wts = np.stack([gate_weights(s[t, idx[t]], do_renorm, route_scale) for t in range(idx.shape[0])]) \
        if idx.shape[0] else np.zeros((0, len(primes)), np.float32)
    return idx, wts


def update_bias(bias, counts, T: int, k: int, gamma: float) -> np.ndarray:
    """Auxiliary-loss-free balancing ("From One Giant FFN...", section 6): an expert whose load is
    above the balanced level T*k/E loses gamma from its bias, one below it gains gamma; one exactly
    at it keeps its bias.  fp32 arithmetic."""
    bias = np.asarray(bias, np.float32).copy()
    counts = np.asarray(counts, np.int64)
    E = bias.shape[0]
    g = np.float32(gamma)
    for e in range(E):
        if counts[e] * E > T * k:
            bias[e] = np.float32(bias[e] - g)
        elif counts[e] * E < T * k:
            bias[e] = np.float32(bias[e] + g)
    return bias


# ----------------------------------------------------------------------------------------------
# dispatch, experts, combine
# ----------------------------------------------------------------------------------------------

def dispatch(indices, n_experts: int):
    """bincount + stable permutation into per-expert contiguous rows (moe-forward excerpt).

    Slot s = t * k + j.  Row r of the permuted matrix belongs to expert e when
    offsets[e] <= r < offsets[e+1]; within a block rows keep slot order.
    Returns counts [E], offsets [E+1], row_of_slot [T*k], tok_of_row [T*k].
    """
    indices = np.asarray(indices, np.int64)
    k = indices.shape[1] if indices.ndim == 2 else 1
    flat = indices.reshape(-1)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    slot_of_row = np.argsort(flat, kind="stable")
    row_of_slot = np.empty_like(slot_of_row)
    row_of_slot[slot_of_row] = np.arange(flat.shape[0])
    return counts, offsets, row_of_slot, slot_of_row // k


def e2m1_value(code) -> np.ndarray:
    """E2M1 (FFN essay section 11.6, the OCP MXFP4 element): bit 3 sign, bits 2-1 exponent with
    bias 1, bit 0 mantissa.  Exponent field 0 is subnormal: 0.5 * m; otherwise
    2^(e-1) * (1 + m/2).  Returns fp64 values of the 4-bit codes."""
    code = np.asarray(code, np.int64)
    sign = np.where(code & 8, -1.0, 1.0)
    e = (code >> 1) & 3
    m = (code & 1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, (e - 1).astype(np.int64)))
    return sign * mag


def ue8m0_value(s) -> np.ndarray:
    """UE8M0 block scale: 2^(s - 127) for s in 0..254 (255 is NaN in the format)."""
    s = np.asarray(s, np.int64)
    return np.where(s == 255, np.nan, np.ldexp(1.0, s - 127))


def mxfp4_dequant(packed, scales) -> np.ndarray:
    """Decode an MXFP4 matrix: packed [R, K/2] uint8 holding element 2j in the low nibble and
    element 2j+1 in the high nibble of byte j; scales [R, K/32] uint8, block b covering elements
    32b .. 32b+31 of its row.  Returns fp64 [R, K] = e2m1(code) * 2^(scale - 127)."""
    packed = np.asarray(packed, np.uint8)
    R, half = packed.shape
    codes = np.empty((R, 2 * half), np.uint8)
    codes[:, 0::2] = packed & 0xF
    codes[:, 1::2] = packed >> 4
    values = e2m1_value(np.arange(16))[codes]        # the definition, evaluated once per code
    return values * np.repeat(ue8m0_value(scales), 32, axis=1)


def e4m3_value(code) -> np.ndarray:
    """E4M3 (the OCP FP8 "E4M3" element, finite-only variant): bit 7 sign, bits 6-3 exponent with
    bias 7, bits 2-0 mantissa.  Exponent field 0 is subnormal: 2^-6 * m/8; otherwise
    2^(e-7) * (1 + m/8); exponent 15 with mantissa 7 is NaN (no infinities).  Returns fp64."""
    code = np.asarray(code, np.int64)
    sign = np.where(code & 0x80, -1.0, 1.0)
    e = (code >> 3) & 15
    m = (code & 7).astype(np.float64)
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)))
    mag = np.where((e == 15) & ((code & 7) == 7), np.nan, mag)
    return sign * mag


def _e4m3_round(q) -> np.ndarray:
    """Nearest E4M3 code of each value of q (|q| <= 448), ties to the even code (the mantissa's
    last bit), found by comparing with the table of all non-negative finite E4M3 values."""
    q = np.asarray(q, np.float64)
    table = e4m3_value(np.arange(127))               # codes 0..126: 0 .. 448, increasing
    a = np.abs(q)
    hi = np.clip(np.searchsorted(table, a, side="left"), 0, 126)   # first table value >= |q|
    lo = np.clip(hi - 1, 0, 126)
    d_lo, d_hi = a - table[lo], table[hi] - a
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    pick = np.where(a == table[hi], hi, pick)
    return (pick | np.where(np.signbit(q), 0x80, 0)).astype(np.uint8)   # the sign is kept, -0 too


def quantize_e4m3_block(v, block: int = 32):
    """MX quantisation of activations ("From One Giant FFN to 384 Tiny Experts", section 11.6: expert
    weights in FP4, everything else computed in FP8 E4M3 with power-of-two UE8M0 block scales).

    Each row of v [R, K] is cut into blocks of 32 consecutive elements.  Reading (the page fixes
    the formats, not the exponent rule): a block's scale is 2^e with e the least integer such that
    448 * 2^e >= max|v| over the block (448 is E4M3's largest finite value), so no element
    saturates; an all-zero block takes e = -127; e is kept in [-127, 127].  Each element is v / 2^e
    rounded to the nearest E4M3 value, ties to even.
    Returns (codes [R, K] uint8 E4M3 bit patterns, scales [R, K/32] uint8 with byte e + 127)."""
    v = np.asarray(v, np.float64)
    R, K = v.shape
    blocks = v.reshape(R, K // block, block)
    amax = np.abs(blocks).max(axis=2)
    _, ex = np.frexp(amax)                            # amax = f * 2^ex with f in [0.5, 1)
    e = ex.astype(np.int64) - 1 - 8                   # floor(log2 amax) - 8
    e = np.where(np.ldexp(448.0, e) >= amax, e, e + 1)
    e = np.where(amax == 0, -127, np.clip(e, -127, 127))
    q = blocks / np.ldexp(1.0, e)[:, :, None]
    codes = _e4m3_round(q).reshape(R, K)
    return codes, (e + 127).astype(np.uint8)


def e4m3_block_dequant(codes, scales, block: int = 32) -> np.ndarray:
    """Values of an MX-quantised matrix: e4m3(code) * 2^(scale - 127), one scale per 32 elements."""
    return e4m3_value(codes) * np.repeat(ue8m0_value(scales), block, axis=1)


def mx_swiglu_hidden(xr, w1, w3, limit: Optional[float] = None, row_weight=None) -> np.ndarray:
    """The hidden activations h [n, I] of mx_swiglu_expert before their MX quantisation: the input
    rows MX-quantised along d (quantize_e4m3_block) times the decoded expert weights w1, w3 [I, d]
    (the MXFP4 weights' exact values), both projections rounded to fp32, then h = silu(g) * v with
    the clamp and row weight of swiglu_expert ("From One Giant FFN to 384 Tiny Experts", section 11.6)."""
    xr = np.asarray(xr, np.float64)
    xq = e4m3_block_dequant(*quantize_e4m3_block(xr))
    gate_z = round_f32(xq @ np.asarray(w1, np.float64).T).astype(np.float64)
    value_z = round_f32(xq @ np.asarray(w3, np.float64).T).astype(np.float64)
    if limit is not None:
        gate_z = np.minimum(gate_z, limit)
        value_z = np.clip(value_z, -limit, limit)
    act = silu(gate_z) * value_z
    if row_weight is not None:
        act = act * np.asarray(row_weight, np.float32).astype(np.float64)[:, None]
    return act


def mx_swiglu_expert(xr, w1, w3, w2, limit: Optional[float] = None, row_weight=None) -> np.ndarray:
    """One SwiGLU expert computed on FP8 activations ("From One Giant FFN to 384 Tiny Experts",
    section 11.6): h from mx_swiglu_hidden is MX-quantised along I and the down projection with
    w2 [d, I] is rounded to bf16."""
    act = mx_swiglu_hidden(xr, w1, w3, limit, row_weight)
    hq = e4m3_block_dequant(*quantize_e4m3_block(act))
    return round_bf16(hq @ np.asarray(w2, np.float64).T)


def silu(z):
    """SiLU(z) = z * sigmoid(z) in fp64 ("From One Giant FFN...", section 1)."""
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(-z))


def swiglu_expert(xr, w1, w3, w2, limit: Optional[float] = None, row_weight=None) -> np.ndarray:
    """One SwiGLU expert on rows xr [n, d]: w2( silu(w1 x) * (w3 x) ), with w1/w3 [I, d], w2 [d, I].

    Gate and value projections rounded to fp32, the product to bf16, the down
    projection to bf16 (the rounding points of a bf16 expert with fp32
    accumulation).  Returns fp64 values that are bf16-exact.

    ``limit`` ("From One Giant FFN...", section 11.4, swiglu_limit): the gate
    branch is capped above at limit and the value branch clamped to
    [-limit, limit] before the product.  ``row_weight`` [n] ("DeepSeek V4.1 -
    Add shared": the routing weight handed to the expert): each row's h is
    multiplied by its weight before the single bf16 rounding.
    """
    xr = np.asarray(xr, np.float64)
    zg = round_f32(xr @ np.asarray(w1, np.float64).T).astype(np.float64)
    zv = round_f32(xr @ np.asarray(w3, np.float64).T).astype(np.float64)
    if limit is not None:
        zg = np.minimum(zg, limit)
        zv = np.clip(zv, -limit, limit)
    a = silu(zg) * zv
    if row_weight is not None:
        a = a * np.asarray(row_weight, np.float32).astype(np.float64)[:, None]
    h = round_bf16(a)
    return round_bf16(h @ np.asarray(w2, np.float64).T)


def combine(T: int, d: int, indices, weights, expert_out: dict, shared_out) -> np.ndarray:
    """y = bf16( sum over experts e ascending of fp32(o_e[t] * w) + shared[t] ), fp32 accumulator.

    moe-forward: ``y = zeros(fp32); for i: y[idx] += expert(x[idx]) * weights[idx, top]``;
    ``y += shared_experts(x)``; ``y.type_as(x)``.  ``expert_out[e]`` maps
    token -> output row (bf16-exact fp64) for the tokens routed to e; with
    ``weights`` None the expert outputs already carry their weights ("DeepSeek
    V4.1 - Add shared": ``y[idx] += expert(x[idx], weights[idx, top])``).
    """
    indices = np.asarray(indices)
    weights = None if weights is None else np.asarray(weights, np.float32)
    y = np.zeros((T, d), np.float32)
    for e in sorted(expert_out):
        rows = expert_out[e]
        for t, j in zip(*np.nonzero(indices == e)):
            o = rows[(t, j)] if (t, j) in rows else rows[t]
            term = o.astype(np.float32) if weights is None else (o.astype(np.float32) * weights[t, j]).astype(np.float32)
            y[t] = (y[t] + term).astype(np.float32)
    if shared_out is not None:
        y = (y + np.asarray(shared_out, np.float32)).astype(np.float32)
    return round_bf16(y)


def moe_forward(x, hp: Hyper, expert: Callable[[int], tuple], w_gate, bias=None, logit_offset=None,
                token_ids=None, tid2eid=None, shared: bool = True, terms: Optional[dict] = None,
                swiglu_limit: Optional[float] = None, weight_in_expert: bool = False,
                mx_activations: bool = False):
    """The MoE layer forward for tokens x [T, d] (bf16-valued).

    ``expert(e)`` returns (w1, w3, w2) of routed expert e, and of the shared
    expert for e == n_experts; each is fetched once, only when some token needs it.
    Returns (y [T, d] bf16-exact fp64, indices, weights, counts).  When ``terms``
    is a dict it receives the summands of y: terms["routed"][t] = [(w_j, o_j), ...]
    and terms["shared"] = the shared expert's rows.  ``swiglu_limit`` clamps every
    expert (shared included); ``weight_in_expert`` hands each routed row its
    weight inside the expert instead of weighting the output in the combine.
    ``mx_activations`` computes every expert (shared included) on FP8 activations
    (mx_swiglu_expert: x and h MX-quantised) with the weights ``expert`` returns.
    """
    expert_fn = mx_swiglu_expert if mx_activations else swiglu_expert
    x = np.asarray(x, np.float64)
    T, d = x.shape
    if tid2eid is not None:
        indices, weights = hash_gate(token_ids, tid2eid, x, w_gate, hp.route_scale, hp.score_func, hp.do_renorm)
    else:
        g = gate(x, w_gate, hp, bias, logit_offset)
        indices, weights = g.indices, g.weights
    counts = np.bincount(indices.reshape(-1), minlength=hp.n_experts)
    outs = {}
    for e in np.nonzero(counts)[0]:
        w1, w3, w2 = expert(int(e))
        if weight_in_expert:
            toks, tops = np.nonzero(indices == e)
            o = expert_fn(x[toks], w1, w3, w2, swiglu_limit, weights[toks, tops])
            outs[int(e)] = {(int(t), int(j)): o[r] for r, (t, j) in enumerate(zip(toks, tops))}
        else:
            toks = np.nonzero((indices == e).any(axis=1))[0]
            o = expert_fn(x[toks], w1, w3, w2, swiglu_limit)
            outs[int(e)] = {int(t): o[r] for r, t in enumerate(toks)}
    shared_out = None
    if shared:
        w1, w3, w2 = expert(hp.n_experts)
        shared_out = expert_fn(x, w1, w3, w2, swiglu_limit)
    y = combine(T, d, indices, None if weight_in_expert else weights, outs, shared_out)
    if terms is not None:
        def _term(t, j):
            rows = outs[int(indices[t, j])]
            if weight_in_expert:
                return (1.0, rows[(t, j)])
            return (float(weights[t, j]), rows[t])
        terms["routed"] = [[_term(t, j) for j in range(indices.shape[1])] for t in range(T)]
        terms["shared"] = shared_out
    return y, indices, weights, counts
