"""Failure detection on the GPU without a GPU fault: a wait that can never complete runs out.

The test build of the library (libmoe_testhooks.so, the same sources compiled with -DMOE_TEST_HOOKS)
exports moe_test_set_stall: while it is set, the CTA-pair expert GEMMs issue no loads, so the MMA
thread's wait for the first stage and the epilogue's wait for the first accumulator can never
complete.  The product library has no such hook.  Every such wait is bounded (about two seconds of
SM clock): it records MOE_ERR_TIMEOUT with the wait's site in the workspace error word, raises the
CTA's abort flag so that the other roles stop waiting too, and the kernel returns.  The host reads
the status through moe_get_error, and the same context then runs the layer correctly.  Nothing
traps and nothing is left in flight.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_routing_gate_b200 import build as B
from mixture_experts_routing_gate_b200 import workloads as W
from parity import assert_outputs_close, expert_fetcher, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    B.build()
    from mixture_experts_routing_gate_b200 import moe
    return moe


@pytest.fixture()
def hooks(M, monkeypatch):
    """The binding's entry points routed to the test build for the duration of one test."""
    import ctypes
    test_lib = M.load_library(B.build(test_hooks=True))
    test_lib.moe_test_set_stall.argtypes = [ctypes.c_int]
    test_lib.moe_test_set_stall.restype = None
    monkeypatch.setattr(M, "lib", test_lib)
    yield test_lib
    test_lib.moe_test_set_stall(0)


def test_stalled_expert_gemm_times_out_and_the_context_recovers(M, hooks):
    T, E, k, d, I = 300, 16, 4, 512, 512
    cfg = W.CONFIGS["tiny"].replace(T=T, n_experts=E, n_groups=1, n_limited_groups=1, topk=k, dim=d, inter_dim=I,
                                    w_std=0.05)
    li = W.make_layer(cfg, device="cuda")
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    desc = M.layer_desc(cfg)
    ws = M.Workspace(desc, T)
    S = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ros = torch.empty(S, dtype=torch.int32, device="cuda")
    tor = torch.empty(S, dtype=torch.int32, device="cuda")
    xp = torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    M.moe_dispatch(desc, torch.from_numpy(idx).cuda(), li.x, counts, offsets, ros, tor, xp, ws)
    M.check_device_errors(ws, "moe_dispatch")
    out_perm = torch.empty((S, d), dtype=torch.bfloat16, device="cuda")
    out_sh = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")

    hooks.moe_test_set_stall(1)
    t0 = time.perf_counter()
    M.moe_expert_ffn(desc, xp, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws)
    st, info = M.moe_get_error(ws)   # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert st == M.MOE_ERR_TIMEOUT, (st, info)
    assert info in (213, 214), info          # the MMA thread's or the epilogue's wait gave up
    assert elapsed < 60.0
    assert M.moe_get_error(ws) == (M.MOE_OK, 0)   # cleared by the read

    hooks.moe_test_set_stall(0)
    M.moe_expert_ffn(desc, xp, offsets, li.x, li.w1, li.w3, li.w2, out_perm, out_sh, ws)
    M.check_device_errors(ws, "moe_expert_ffn after the stalled call")
    c, o, _, tok = O.dispatch(idx, E)
    x = np64(li.x)
    fetch = expert_fetcher(li)
    e = int(np.argmax(c))
    assert_outputs_close(np64(out_perm)[o[e]:o[e + 1]], O.swiglu_expert(x[tok[o[e]:o[e + 1]]], *fetch(e)),
                         f"expert {e}", per_element=True)
    assert_outputs_close(np64(out_sh), O.swiglu_expert(x, *fetch(E)), "shared expert", per_element=True)
