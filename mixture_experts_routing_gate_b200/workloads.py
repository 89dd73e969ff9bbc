"""Seeded synthetic MoE-layer workloads.

This module only draws inputs: activations, router and expert weights, the
selection bias, the per-expert logit offset of the skewed layer, and the token
ids and token frequencies of the hash-routed layer.  It holds none of the
layer's arithmetic, so that both the CPU oracle and the CUDA path can be fed
from it without sharing any computation.

Every tensor is drawn from a counter-based generator: element ``i`` of tensor
``(seed, tensor_id, expert_id)`` is a pure function of those four integers.
Consequences:

* any single expert's weights can be regenerated alone (the oracle never has to
  hold a 22 GB weight set);
* the same call gives the same values on the CPU and on a GPU (integer hashing
  is exact on both; the Box-Muller transform runs in fp64, where the two
  devices' ``log``/``cos`` agree to an ulp or so, far below the bf16/fp32
  rounding applied afterwards).

Generator: a 32-bit integer finaliser (xor-shift / multiply, the "lowbias32"
constants published in C. Wellons' hash-prospector) applied to the element
index and a per-tensor key gives two uniform 32-bit words, which the
Box-Muller transform turns into one standard normal.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

_M32 = 0xFFFFFFFF

# tensor ids of the generator streams
TID_X = 1
TID_W_GATE = 2
TID_BIAS = 3
TID_LOGIT_OFFSET = 4
TID_W1 = 5
TID_W3 = 6
TID_W2 = 7
TID_TOKEN_IDS = 8
TID_SAMPLE = 9
TID_FP4_CODES = 10   # + 0 / 1 / 2 for w1 / w3 / w2
TID_FP4_SCALES = 13  # + 0 / 1 / 2


def _mix32_int(h: int) -> int:
    h &= _M32
    h ^= h >> 16
    h = (h * 0x7FEB352D) & _M32
    h ^= h >> 15
    h = (h * 0x846CA68B) & _M32
    h ^= h >> 16
    return h


def _mix32(h: torch.Tensor) -> torch.Tensor:
    # h: int64 tensor holding values in [0, 2^32). Products wrap modulo 2^64,
    # and the mask keeps the low 32 bits, exactly as uint32 arithmetic would.
    h = h ^ (h >> 16)
    h = (h * 0x7FEB352D) & _M32
    h = h ^ (h >> 15)
    h = (h * 0x846CA68B) & _M32
    return h ^ (h >> 16)


def stream_key(seed: int, tensor_id: int, expert_id: int = 0) -> tuple[int, int]:
    k = 0x9E3779B9
    for v in (seed, tensor_id, expert_id):
        k = _mix32_int(k ^ (v & _M32))
    return k, _mix32_int(k ^ 0x85EBCA6B)


def _uniform_pair(n: int, start: int, key: tuple[int, int], device) -> tuple[torch.Tensor, torch.Tensor]:
    i = torch.arange(start, start + n, dtype=torch.int64, device=device)
    lo = i & _M32
    hi = i >> 32
    h1 = _mix32(_mix32(lo ^ key[0]) ^ hi)
    h2 = _mix32(h1 ^ key[1])
    return h1, h2


def normal(shape, seed: int, tensor_id: int, expert_id: int = 0, device="cpu",
           chunk: int = 1 << 24) -> torch.Tensor:
    """Standard normal fp64 tensor of ``shape`` from stream (seed, tensor_id, expert_id)."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(n, dtype=torch.float64, device=device)
    key = stream_key(seed, tensor_id, expert_id)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        h1, h2 = _uniform_pair(m, s, key, device)
        u1 = (h1.to(torch.float64) + 0.5) * (2.0 ** -32)
        u2 = h2.to(torch.float64) * (2.0 ** -32)
        out[s:s + m] = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
    return out.view(*shape)


def uniform(n: int, seed: int, tensor_id: int, expert_id: int = 0, device="cpu") -> torch.Tensor:
    """Uniform fp64 values in (0, 1)."""
    h1, _ = _uniform_pair(n, 0, stream_key(seed, tensor_id, expert_id), device)
    return (h1.to(torch.float64) + 0.5) * (2.0 ** -32)


def normal_bf16(shape, std: float, seed: int, tensor_id: int, expert_id: int = 0,
                device="cpu", out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """N(0, std^2) drawn in fp64, rounded once to fp32 and then RNE to bf16."""
    v = (normal(shape, seed, tensor_id, expert_id, device) * std).to(torch.float32).to(torch.bfloat16)
    if out is not None:
        out.copy_(v)
        return out
    return v


def normal_f32(shape, std: float, seed: int, tensor_id: int, expert_id: int = 0, device="cpu") -> torch.Tensor:
    return (normal(shape, seed, tensor_id, expert_id, device) * std).to(torch.float32)


# Probabilities of the eight E2M1 magnitude codes 0..7 in synthetic MXFP4 weights: a bell-shaped
# histogram peaking at the small codes, with the largest code rare, as in blocks whose shared scale
# is set by the block's largest entry.  The root mean square of the coded magnitudes is about 1.8.
_FP4_MAG_P = (0.22, 0.20, 0.18, 0.14, 0.11, 0.08, 0.05, 0.02)
_FP4_RMS = 1.8


def mxfp4_matrix(rows: int, cols: int, std: float, seed: int, which: int, expert_id: int = 0, device="cpu",
                 jitter: int = 1):
    """Synthetic MXFP4 weights of a [rows, cols] matrix: (packed [rows, cols/2] uint8 with element 2j
    in the low nibble of byte j, scales [rows, cols/32] uint8).  Codes: magnitude from _FP4_MAG_P and a
    uniform sign; UE8M0 scales 127 + round(log2(std / 1.8)) plus a uniform offset in [-jitter, jitter],
    so that the decoded weights have roughly the standard deviation std."""
    n = rows * cols
    h1, h2 = _uniform_pair(n, 0, stream_key(seed, TID_FP4_CODES + which, expert_id), device)
    cdf = torch.tensor(np.cumsum(_FP4_MAG_P)[:-1] * 2.0 ** 32, dtype=torch.float64, device=device)
    mag = torch.bucketize(h1.to(torch.float64), cdf, right=True)
    code = (mag | ((h2 & 1) << 3)).to(torch.uint8).view(rows, cols)
    packed = code[:, 0::2] | (code[:, 1::2] << 4)
    base = 127 + int(round(math.log2(std / _FP4_RMS)))
    hs, _ = _uniform_pair(rows * (cols // 32), 0, stream_key(seed, TID_FP4_SCALES + which, expert_id), device)
    scales = (base - jitter + (hs % (2 * jitter + 1))).to(torch.uint8).view(rows, cols // 32)
    return packed.contiguous(), scales.contiguous()


@dataclasses.dataclass
class Mxfp4Weights:
    """Stacked MXFP4 expert weights, shared expert last (index E)."""
    w1: torch.Tensor   # [E+1, I, d/2] uint8
    w1s: torch.Tensor  # [E+1, I, d/32] uint8
    w3: torch.Tensor
    w3s: torch.Tensor
    w2: torch.Tensor   # [E+1, d, I/2]
    w2s: torch.Tensor  # [E+1, d, I/32]


def expert_mxfp4(cfg: "LayerConfig", e: int, device="cpu"):
    """((w1, w1s), (w3, w3s), (w2, w2s)) of expert e (e == E: the shared expert)."""
    I, d = cfg.inter_dim, cfg.dim
    return (mxfp4_matrix(I, d, cfg.w_std, cfg.seed, 0, e, device),
            mxfp4_matrix(I, d, cfg.w_std, cfg.seed, 1, e, device),
            mxfp4_matrix(d, I, cfg.w_std, cfg.seed, 2, e, device))


def make_mxfp4_weights(cfg: "LayerConfig", device="cpu") -> Mxfp4Weights:
    E, I, d = cfg.n_experts, cfg.inter_dim, cfg.dim
    u8 = dict(dtype=torch.uint8, device=device)
    w = Mxfp4Weights(torch.empty((E + 1, I, d // 2), **u8), torch.empty((E + 1, I, d // 32), **u8),
                     torch.empty((E + 1, I, d // 2), **u8), torch.empty((E + 1, I, d // 32), **u8),
                     torch.empty((E + 1, d, I // 2), **u8), torch.empty((E + 1, d, I // 32), **u8))
    for e in range(E + 1):
        (a, a_s), (b, b_s), (c, c_s) = expert_mxfp4(cfg, e, device)
        w.w1[e].copy_(a); w.w1s[e].copy_(a_s)
        w.w3[e].copy_(b); w.w3s[e].copy_(b_s)
        w.w2[e].copy_(c); w.w2s[e].copy_(c_s)
    return w


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """One synthetic MoE layer: shapes, routing hyper-parameters and value distributions."""
    name: str
    seed: int
    T: int                      # tokens in the batch
    dim: int                    # d
    n_experts: int              # E routed experts
    n_groups: int               # G
    n_limited_groups: int       # groups kept per token
    topk: int                   # k
    inter_dim: int              # I (routed and shared experts alike)
    score_func: str             # "sigmoid" | "sqrtsoftplus" | "softmax"
    route_scale: float
    w_std: float                # expert weights
    gate_std: float             # router weight
    gate_general_fp32: bool     # router weight drawn as general fp32 (else bf16-valued)
    bias_std: Optional[float]   # selection bias, None = no bias
    x_std: float = 1.0
    logit_offset_std: Optional[float] = None   # per-expert logit offset (skew), None = none
    hash_vocab: int = 0         # >0: hash-routed layer over a vocabulary of this size
    zipf_s: float = 1.1         # token frequency p_i ~ i^-zipf_s for the hash layer
    n_shared: int = 1
    swiglu_limit: float = 0.0   # > 0: SwiGLU clamp of every expert
    weight_in_expert: bool = False  # routing weight applied to h inside each routed expert

    @property
    def renorm(self) -> bool:
        return self.score_func in ("sigmoid", "sqrtsoftplus")

    @property
    def is_hash(self) -> bool:
        return self.hash_vocab > 0

    def replace(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": LayerConfig(
        name="tiny", seed=0, T=64, dim=256, n_experts=16, n_groups=4, n_limited_groups=2, topk=4,
        inter_dim=128, score_func="sigmoid", route_scale=1.0, w_std=0.02, gate_std=0.02,
        gate_general_fp32=True, bias_std=0.01),
    "v3_prefill": LayerConfig(
        name="v3_prefill", seed=1, T=4096, dim=7168, n_experts=256, n_groups=8, n_limited_groups=4,
        topk=8, inter_dim=2048, score_func="sigmoid", route_scale=2.5, w_std=0.006, gate_std=0.006,
        gate_general_fp32=False, bias_std=0.01),
    "hash": LayerConfig(
        name="hash", seed=2, T=8192, dim=4096, n_experts=256, n_groups=1, n_limited_groups=1, topk=6,
        inter_dim=2048, score_func="sigmoid", route_scale=1.0, w_std=0.01, gate_std=0.01,
        gate_general_fp32=False, bias_std=None, hash_vocab=129280, zipf_s=1.1),
    "v3_decode": LayerConfig(
        name="v3_decode", seed=3, T=64, dim=7168, n_experts=256, n_groups=8, n_limited_groups=4,
        topk=8, inter_dim=2048, score_func="sigmoid", route_scale=2.5, w_std=0.006, gate_std=0.006,
        gate_general_fp32=False, bias_std=0.01),
    "v4_skew": LayerConfig(
        name="v4_skew", seed=4, T=16384, dim=5120, n_experts=384, n_groups=1, n_limited_groups=1,
        topk=6, inter_dim=1536, score_func="sqrtsoftplus", route_scale=1.5, w_std=0.01, gate_std=0.01,
        gate_general_fp32=False, bias_std=0.01, logit_offset_std=1.0),
}


def token_frequencies(cfg: LayerConfig) -> np.ndarray:
    """p_i proportional to i^-s over token ids 0..m-1 (id i-1 has rank i), fp64, sums to 1."""
    p = np.arange(1, cfg.hash_vocab + 1, dtype=np.float64) ** (-cfg.zipf_s)
    return p / p.sum()


def sample_token_ids(cfg: LayerConfig, p: np.ndarray) -> np.ndarray:
    """T token ids drawn from p by inverse-CDF sampling of the generator's uniforms (int32)."""
    u = uniform(cfg.T, cfg.seed, TID_TOKEN_IDS).numpy()
    cdf = np.cumsum(p)
    ids = np.searchsorted(cdf, u * cdf[-1], side="right")
    return np.minimum(ids, cfg.hash_vocab - 1).astype(np.int32)


@dataclasses.dataclass
class LayerInputs:
    cfg: LayerConfig
    x: torch.Tensor                      # [T, d] bf16
    w_gate: torch.Tensor                 # [E, d] fp32
    bias: Optional[torch.Tensor]         # [E] fp32
    logit_offset: Optional[torch.Tensor]  # [E] fp32
    w1: torch.Tensor                     # [E+1, I, d] bf16, shared expert last
    w3: torch.Tensor                     # [E+1, I, d] bf16
    w2: torch.Tensor                     # [E+1, d, I] bf16
    token_ids: Optional[torch.Tensor] = None   # [T] int32 (hash layer)
    p: Optional[np.ndarray] = None             # [m] fp64 token frequencies (hash layer)


def make_router_inputs(cfg: LayerConfig, device="cpu"):
    """x, w_gate, bias, logit_offset for ``cfg`` on ``device``."""
    E, d = cfg.n_experts, cfg.dim
    x = normal_bf16((cfg.T, d), cfg.x_std, cfg.seed, TID_X, device=device)
    if cfg.gate_general_fp32:
        w_gate = normal_f32((E, d), cfg.gate_std, cfg.seed, TID_W_GATE, device=device)
    else:
        # a bf16 parameter read through .float(): bf16-exact values held in fp32
        w_gate = normal_bf16((E, d), cfg.gate_std, cfg.seed, TID_W_GATE, device=device).to(torch.float32)
    bias = None if cfg.bias_std is None else normal_f32((E,), cfg.bias_std, cfg.seed, TID_BIAS, device=device)
    off = None if cfg.logit_offset_std is None else normal_f32(
        (E,), cfg.logit_offset_std, cfg.seed, TID_LOGIT_OFFSET, device=device)
    return x, w_gate, bias, off


def expert_weights(cfg: LayerConfig, e: int, device="cpu"):
    """(w1 [I,d], w3 [I,d], w2 [d,I]) bf16 of expert e (e == E is the shared expert)."""
    I, d = cfg.inter_dim, cfg.dim
    w1 = normal_bf16((I, d), cfg.w_std, cfg.seed, TID_W1, e, device=device)
    w3 = normal_bf16((I, d), cfg.w_std, cfg.seed, TID_W3, e, device=device)
    w2 = normal_bf16((d, I), cfg.w_std, cfg.seed, TID_W2, e, device=device)
    return w1, w3, w2


def make_layer(cfg: LayerConfig, device="cpu", bf16_experts: bool = True) -> LayerInputs:
    """All inputs of one layer on ``device`` (the expert weights are generated expert by expert;
    bf16_experts=False leaves w1 / w3 / w2 as None, for layers run with MXFP4 experts)."""
    x, w_gate, bias, off = make_router_inputs(cfg, device)
    E, I, d = cfg.n_experts, cfg.inter_dim, cfg.dim
    w1 = w3 = w2 = None
    if bf16_experts:
        w1 = torch.empty((E + 1, I, d), dtype=torch.bfloat16, device=device)
        w3 = torch.empty((E + 1, I, d), dtype=torch.bfloat16, device=device)
        w2 = torch.empty((E + 1, d, I), dtype=torch.bfloat16, device=device)
        for e in range(E + 1):
            normal_bf16((I, d), cfg.w_std, cfg.seed, TID_W1, e, device=device, out=w1[e])
            normal_bf16((I, d), cfg.w_std, cfg.seed, TID_W3, e, device=device, out=w3[e])
            normal_bf16((d, I), cfg.w_std, cfg.seed, TID_W2, e, device=device, out=w2[e])
    li = LayerInputs(cfg, x, w_gate, bias, off, w1, w3, w2)
    if cfg.is_hash:
        li.p = token_frequencies(cfg)
        li.token_ids = torch.from_numpy(sample_token_ids(cfg, li.p)).to(device)
    return li


def sample_rows(n_total: int, n_sample: int, seed: int) -> np.ndarray:
    """A seeded, sorted sample of distinct row indices (used to pick tokens to check one by one)."""
    if n_sample >= n_total:
        return np.arange(n_total)
    u = uniform(n_total, seed, TID_SAMPLE).numpy()
    return np.sort(np.argsort(u, kind="stable")[:n_sample])
