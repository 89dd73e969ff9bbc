"""The comparison helpers of the GPU parity tests, checked on the CPU: the slack allowed for E4M3
rounding flips of the hidden activations (parity.mx_flip_slack) must cover what a computation in the
kernel's precision (fp32 accumulation in another order, fp32 SwiGLU) can produce, and must not hide a
wrong result."""
import numpy as np
import pytest

import oracle as O
from parity import assert_outputs_close, bf16_ulp, mx_flip_slack


def _f32_expert(xr, w1, w3, w2, perm, rng_err):
    """The expert on E4M3 activations in fp32 arithmetic with the K sums taken in another order
    (a permutation of d): how a kernel's fp32 accumulators can differ from the oracle's."""
    xq = O.e4m3_block_dequant(*O.quantize_e4m3_block(xr))[:, perm]

    def f32_sum(w):   # 32-term partial products (exact here), added one after another in fp32
        w = w[:, perm]
        acc = np.zeros((xq.shape[0], w.shape[0]), np.float32)
        for k in range(0, xq.shape[1], 32):
            acc = acc + (xq[:, k:k + 32] @ w[:, k:k + 32].T).astype(np.float32)
        return acc
    g, v = f32_sum(w1), f32_sum(w3)
    # silu with an approximate exponential: a relative error within (2 + 1.17|g|) fp32 ulps
    e = np.exp(-g.astype(np.float64)) * (1.0 + (2.0 + 1.17 * np.abs(g)) * 2.0 ** -23 * rng_err.uniform(-1, 1, g.shape))
    act = ((g / (1.0 + e)).astype(np.float32)) * v
    hq = O.e4m3_block_dequant(*O.quantize_e4m3_block(act.astype(np.float64))).astype(np.float32)
    return O.round_bf16((hq @ w2.astype(np.float32).T).astype(np.float64)), act


@pytest.fixture(scope="module")
def case():
    rng = np.random.default_rng(3)
    n, d, I = 3000, 1024, 512
    xr = O.round_bf16(rng.standard_normal((n, d)))
    dec = lambda r, c: O.mxfp4_dequant(rng.integers(0, 256, (r, c // 2), dtype=np.uint8),
                                       rng.integers(120, 124, (r, c // 32), dtype=np.uint8))
    w1, w3, w2 = dec(I, d), dec(I, d), dec(d, I)
    perm = rng.permutation(d)
    y32, act32 = _f32_expert(xr, w1, w3, w2, perm, np.random.default_rng(4))
    return xr, w1, w3, w2, y32, act32


def test_flip_slack_covers_fp32_emulation(case):
    xr, w1, w3, w2, y32, _ = case
    ref = O.mx_swiglu_expert(xr, w1, w3, w2)
    slack = mx_flip_slack(xr, w1, w3, w2, y_ref=ref)
    assert_outputs_close(y32, ref, "fp32 emulation", per_element=True, slack=slack)


def test_flip_slack_covers_h_moved_to_the_edge_of_its_reach(case):
    """Kernels whose h sits at either end of the reach the slack assumes (every element moved up, or
    every element moved down, by that much; block scales recomputed): every ambiguous code flips at
    once, and the slack still covers every element."""
    xr, w1, w3, w2, _, _ = case
    ref = O.mx_swiglu_expert(xr, w1, w3, w2)
    slack = mx_flip_slack(xr, w1, w3, w2, y_ref=ref)
    act = O.mx_swiglu_hidden(xr, w1, w3)
    # the reach mx_flip_slack derives, recomputed here from its stated bound with ulps = 16
    xq = O.e4m3_block_dequant(*O.quantize_e4m3_block(xr))
    g, v = xq @ w1.T, xq @ w3.T
    sig = 1.0 / (1.0 + np.exp(-g))
    dg = 16 * 2.0 ** -24 * (np.abs(xq) @ np.abs(w1).T)
    dv = 16 * 2.0 ** -24 * (np.abs(xq) @ np.abs(w3).T)
    dact = np.abs(sig * (1 + g * (1 - sig)) * v) * dg + np.abs(g * sig) * dv + (4 + 1.2 * np.abs(g)) * 2.0 ** -23 * np.abs(act)
    bar = 2e-2 * np.sqrt(np.mean(ref ** 2))
    flips = 0
    for moved in (act + 0.999 * dact, act - 0.999 * dact):
        codes, scales = O.quantize_e4m3_block(moved)
        flips += int((O.e4m3_block_dequant(codes, scales) != O.e4m3_block_dequant(*O.quantize_e4m3_block(act))).sum())
        y = O.round_bf16(O.e4m3_block_dequant(codes, scales) @ w2.T)
        err = np.abs(y - ref)
        assert np.all(err <= np.maximum(slack, bar)), float(np.max(err - np.maximum(slack, bar)))
    assert flips > 0


def test_flip_slack_does_not_hide_a_wrong_expert(case):
    xr, w1, w3, w2, y32, _ = case
    ref = O.mx_swiglu_expert(xr, w1, w3, w2)
    slack = mx_flip_slack(xr, w1, w3, w2, y_ref=ref)
    # the h-flip allowance exceeds the plain allowance (the bar, or two bf16 ulps of y) on a minority of
    # elements (rows with an h element within reach of a rounding boundary), and then by little; the
    # element-count, mean-error and 99.9 % checks of assert_outputs_close do not use it at all
    rms = np.sqrt(np.mean(ref ** 2))
    plain = np.maximum(2e-2 * rms, 2 * bf16_ulp(ref))
    assert np.mean(slack > plain) < 0.15
    assert np.max(slack) < 10 * 2e-2 * rms
    # a dropped block of w2 columns, a sign error in the value branch, a transposed row order: all fail
    for bad in (O.mx_swiglu_expert(xr, w1, w3, np.where(np.arange(w2.shape[1]) < 32, 0.0, w2)),
                O.mx_swiglu_expert(xr, w1, -w3, w2),
                y32[::-1]):
        with pytest.raises(AssertionError):
            assert_outputs_close(bad, ref, "mutant", per_element=True, slack=slack)
