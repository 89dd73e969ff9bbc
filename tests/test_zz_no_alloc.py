"""moe_dispatch_static: the dispatch for callers that cannot allocate device memory.

Such callers (a plugin given only its input and output buffers by a framework that owns all device
memory, or a loop that may not take an allocation's implicit synchronisation) cannot pass the
workspace moe_dispatch needs; moe_dispatch_static keeps that scratch in a fixed array of the
library's own device memory instead.  This test calls it through the C ABI twice in a row, on two
different batches, and checks every output against moe_dispatch's on the same inputs: the shared
array keeps the previous call's contents, and the second call must not see them.  It also checks
that sizes beyond the array are refused before anything is launched.

This file is collected last so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest
import torch

from mixture_experts_routing_gate_b200 import build as B
from mixture_experts_routing_gate_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _indices(T, E, k, seed):
    rng = np.random.default_rng(seed)
    pop = 1.0 / np.arange(1, E + 1) ** 1.1
    pop /= pop.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=pop) for _ in range(T)]).astype(np.int32)


def _run(M, fn, desc, idx, x, E, with_ws):
    return _run_t(M, fn, desc, torch.from_numpy(idx).cuda(), x, E, with_ws)


def _run_t(M, fn, desc, idx_t, x, E, with_ws):
    T, d = x.shape
    S = idx_t.numel()
    outs = [torch.full((n,), -7, dtype=torch.int32, device="cuda") for n in (E, E + 1, S, S)]
    xp = torch.zeros((S, d), dtype=torch.bfloat16, device="cuda")
    if with_ws:
        ws = M.Workspace(desc, T)
        fn(desc, idx_t, x, *outs, xp, ws)
    else:
        fn(desc, idx_t, x, *outs, xp)
    torch.cuda.synchronize()
    return [o.cpu() for o in outs], xp


def test_static_dispatch_matches_workspace_dispatch_twice():
    B.build()
    from mixture_experts_routing_gate_b200 import moe as M
    cases = [("v3_prefill", 4096, 256, 8, 7168, 1), ("v4_skew", 2048, 384, 6, 512, 2)]
    for name, T, E, k, d, seed in cases:          # two calls in a row, different shapes and data
        cfg = W.CONFIGS[name].replace(T=T, dim=d)
        desc = M.layer_desc(cfg)
        idx = _indices(T, E, k, seed)
        x = W.normal_bf16((T, d), 1.0, seed, W.TID_X, device="cuda")
        ref, xp_ref = _run(M, M.moe_dispatch, desc, idx, x, E, with_ws=True)
        got, xp_got = _run(M, M.moe_dispatch_static, desc, idx, x, E, with_ws=False)
        for r, g in zip(ref, got):
            assert torch.equal(r, g)
        assert torch.equal(xp_ref, xp_got)
    # without x_perm (the permutation only, for moe_expert_ffn_gather): the same index outputs
    S = idx.size
    outs = [torch.full((n,), -7, dtype=torch.int32, device="cuda") for n in (E, E + 1, S, S)]
    M.moe_dispatch_static(desc, torch.from_numpy(idx).cuda(), x, *outs, None)
    torch.cuda.synchronize()
    for r, g in zip(ref, outs):
        assert torch.equal(r, g.cpu())
    assert int(got[1][-1]) == T * k


def test_static_dispatch_rejects_sizes_beyond_its_scratch():
    B.build()
    from mixture_experts_routing_gate_b200 import moe as M
    # T*k = 2^21 slots cut into ceil(2^21 / 8192) = 256 histogram blocks: 256 * E = 131072 > 131040,
    # the scratch's limit.  Real, valid buffers are passed, so the call would be harmless even if the
    # check were missing.
    T, E, k, d = 262144, 512, 8, 128
    assert -(-T * k // 8192) * E > 131040
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d)
    desc = M.layer_desc(cfg)
    S = T * k
    idx = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    outs = [torch.full((n,), -7, dtype=torch.int32, device="cuda") for n in (E, E + 1, S, S)]
    xp = torch.full((S, d), -7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(M.MoeError) as exc:
        M.moe_dispatch_static(desc, idx, x, *outs, xp)
    assert exc.value.status == M.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    for o in outs:                                  # nothing was written
        assert bool((o == -7).all())
    assert bool((xp == -7.0).all())
    # one slot fewer per block row fits: T*k = 255 * 8192 slots -> 255 blocks * 512 = 130560
    T2 = 255 * 8192 // k
    desc2 = M.layer_desc(cfg.replace(T=T2))
    rows = np.arange(T2, dtype=np.int64)[:, None] * 7 + np.arange(k)[None, :] * (E // k)
    idx2 = torch.from_numpy((rows % E).astype(np.int32)).cuda()   # k distinct experts per token
    ref, xp_ref = _run_t(M, M.moe_dispatch, desc2, idx2, x[:T2], E, with_ws=True)
    got, xp_got = _run_t(M, M.moe_dispatch_static, desc2, idx2, x[:T2], E, with_ws=False)
    for r, g in zip(ref, got):
        assert torch.equal(r, g)
    assert torch.equal(xp_ref, xp_got)
