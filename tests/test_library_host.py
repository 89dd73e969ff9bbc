"""Host-side checks of libmoe that need no GPU: exports, argument validation, the tid2eid builder.

The tid2eid builder is host code of the library, so it is compared with the oracle bit for bit
(tables and loads) on the hand-worked examples, the tid2eid page's own setting and the hash layer's
vocabulary.  No call here launches a kernel.
"""
import ctypes
import json
import os
import re

import numpy as np
import pytest

import oracle as O
from mixture_experts_routing_gate_b200 import build as B
from mixture_experts_routing_gate_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    B.build()
    from mixture_experts_routing_gate_b200 import moe as M
    return M


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(moe):
    declared = _declared_functions()
    assert "moe_forward" in declared and "moe_gate" in declared
    for name in declared:
        assert hasattr(moe.lib, name), name
        assert ctypes.cast(getattr(moe.lib, name), ctypes.c_void_p).value
    assert set(declared) == set(moe.EXPORTS)


def test_status_strings(moe):
    for s in range(8):
        assert moe.lib.moe_status_str(s).decode().startswith("MOE_")


def test_workspace_bytes_and_desc_checks(moe):
    cfg = W.CONFIGS["v3_prefill"]
    d = moe.layer_desc(cfg)
    n = moe.moe_workspace_bytes(d, cfg.T)
    S = cfg.T * cfg.topk
    # at least the permuted activations, the intermediate h and the permuted outputs
    assert n >= S * cfg.dim * 2 * 2 + (S + cfg.T) * cfg.inter_dim * 2
    assert moe.moe_workspace_bytes(d, 0) > 0
    assert moe.moe_workspace_bytes(d, -1) == 0
    for bad in [dict(n_experts=250), dict(topk=9), dict(dim=100), dict(inter_dim=1000), dict(n_groups=3),
                dict(n_limited_groups=9), dict(n_shared=2), dict(n_experts=1024), dict(topk=33)]:
        c = moe.layer_desc(cfg)
        for k, v in bad.items():
            setattr(c, k, v)
        assert moe.moe_workspace_bytes(c, 16) == 0, bad


def test_entry_points_reject_bad_arguments_before_launch(moe):
    cfg = W.CONFIGS["tiny"]
    d = moe.layer_desc(cfg)
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: every call below must fail its argument checks first
    lib = moe.lib
    assert lib.moe_gate(ctypes.byref(d), 4, None, None, None, None, None, None, fake, 1 << 30, None) == moe.MOE_ERR_INVALID
    assert lib.moe_gate(ctypes.byref(d), -1, fake, fake, None, None, fake, fake, fake, 1 << 30, None) == moe.MOE_ERR_INVALID
    # misaligned activation pointer
    assert lib.moe_gate(ctypes.byref(d), 4, P((1 << 20) + 2), fake, None, None, fake, fake, fake, 1 << 30,
                        None) == moe.MOE_ERR_INVALID
    # workspace too small / missing
    assert lib.moe_gate(ctypes.byref(d), 4, fake, fake, None, None, fake, fake, fake, 16, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_gate(ctypes.byref(d), 4, fake, fake, None, None, fake, fake, None, 1 << 30, None) == moe.MOE_ERR_WORKSPACE
    bad = moe.layer_desc(cfg)
    bad.n_shared = 0
    assert lib.moe_forward(ctypes.byref(bad), 4, fake, None, None, 0, fake, None, None, fake, fake, fake, fake,
                           None, None, None, fake, 1 << 30, None) == moe.MOE_ERR_UNSUPPORTED
    # hash forward needs both the ids and the table
    assert lib.moe_forward(ctypes.byref(d), 4, fake, fake, None, 10, fake, None, None, fake, fake, fake, fake,
                           None, None, None, fake, 1 << 30, None) == moe.MOE_ERR_INVALID
    assert lib.moe_build_tid2eid(None, 5, 4, 2, None, None) == moe.MOE_ERR_INVALID
    p = np.array([0.5, np.nan])
    t = np.zeros((2, 1), np.int32)
    assert lib.moe_build_tid2eid(p.ctypes.data, 2, 4, 1, t.ctypes.data, None) == moe.MOE_ERR_INVALID
    assert lib.moe_build_tid2eid(p.ctypes.data, 2, 4, 5, t.ctypes.data, None) == moe.MOE_ERR_INVALID


def test_tid2eid_hand_examples(moe):
    with open(os.path.join(ROOT, "tests", "golden", "tid2eid_hand_examples.json")) as f:
        for ex in json.load(f)["examples"]:
            p = np.array(ex["p32"], np.float64) / 32
            table, loads = moe.moe_build_tid2eid(p, ex["n"], ex["k"])
            assert table.tolist() == ex["rows"], ex["name"]
            assert (loads * 32).tolist() == ex["f32"], ex["name"]


def test_tid2eid_matches_oracle_page_setting(moe):
    m, n, k = 80000, 128, 4
    p = 1.0 / (10.0 + np.arange(m))
    p /= p.sum()
    t_lib, f_lib = moe.moe_build_tid2eid(p, n, k)
    t_ora, f_ora = O.build_tid2eid(p, n, k)
    assert np.array_equal(t_lib, t_ora)
    assert np.array_equal(f_lib, f_ora)


@pytest.mark.slow
def test_tid2eid_matches_oracle_hash_vocab(moe):
    cfg = W.CONFIGS["hash"]
    p = W.token_frequencies(cfg)
    t_lib, f_lib = moe.moe_build_tid2eid(p, cfg.n_experts, cfg.topk)
    t_ora, f_ora = O.build_tid2eid(p, cfg.n_experts, cfg.topk)
    assert np.array_equal(t_lib, t_ora)
    assert np.array_equal(f_lib, f_ora)
    assert O.balance(f_lib) == O.balance(f_ora)


def test_tid2eid_unsorted_and_tied_frequencies(moe):
    rng = np.random.default_rng(8)
    p = rng.integers(1, 6, 3000).astype(np.float64)   # many exact ties, unsorted
    p /= 1024.0
    t_lib, f_lib = moe.moe_build_tid2eid(p, 37, 5)
    t_ora, f_ora = O.build_tid2eid(p, 37, 5)
    assert np.array_equal(t_lib, t_ora) and np.array_equal(f_lib, f_ora)
    t0, f0 = moe.moe_build_tid2eid(np.zeros(0), 8, 2)
    assert t0.shape == (0, 2) and np.all(f0 == 0)


def test_tid2eid_best_matches_oracle(moe):
    rng = np.random.default_rng(12)
    m, n, k = 5000, 64, 4
    p = 1.0 / (3.0 + np.arange(m)) ** 1.05
    p /= p.sum()
    orders = np.stack([rng.permutation(m) for _ in range(6)]).astype(np.int32)
    orders[4] = orders[1]                       # an exact tie: the earlier run must stay
    orders[5] = np.argsort(-p, kind="stable")   # the plain greedy among the runs
    t_lib, f_lib, vio, kept = moe.moe_build_tid2eid_best(p, n, k, orders)
    t_ora, f_ora, kept_ora = O.best_tid2eid(p, n, k, list(orders))
    assert kept == kept_ora
    assert np.array_equal(t_lib, t_ora) and np.array_equal(f_lib, f_ora)
    assert vio.tolist() == [O.balance(O.build_tid2eid(p, n, k, o)[1])[0] for o in orders]
    assert vio[4] == vio[1]


def test_next_rows_reject_bad_arguments_before_launch(moe):
    cfg = W.CONFIGS["hash"]
    d = moe.layer_desc(cfg)
    lib = moe.lib
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: every call below must fail its argument checks first
    vocab = cfg.hash_vocab
    good = O.primes_above(vocab, cfg.topk)

    def ngram(primes, v=vocab, desc=d):
        q = np.asarray(primes, np.int64)
        return lib.moe_ngram_gate(ctypes.byref(desc), 4, fake, fake, q.ctypes.data, v, fake, fake, fake, fake,
                                  fake, 1 << 30, None)

    assert ngram(good[:-1] + [good[0]]) == moe.MOE_ERR_INVALID          # repeated prime
    assert ngram(good[:-1] + [vocab + 1 if vocab % 2 else vocab + 2]) == moe.MOE_ERR_INVALID  # even: not prime
    assert ngram([7] + good[1:]) == moe.MOE_ERR_INVALID                  # prime below the vocabulary
    assert ngram(good[:-1] + [4294967311]) == moe.MOE_ERR_INVALID        # prime above 2^32
    assert ngram(good, v=0) == moe.MOE_ERR_INVALID
    soft = moe.layer_desc(cfg)
    soft.score_func = moe.SCORE_FUNCS["softmax"]
    assert ngram(good, desc=soft) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_ngram_gate(ctypes.byref(d), 4, fake, fake, None, vocab, fake, fake, fake, fake, fake, 1 << 30,
                              None) == moe.MOE_ERR_INVALID
    for gamma in (-0.001, float("nan"), float("inf")):
        assert lib.moe_update_bias(ctypes.byref(d), 16, fake, fake, gamma, None) == moe.MOE_ERR_INVALID
    assert lib.moe_update_bias(ctypes.byref(d), 16, None, fake, 0.001, None) == moe.MOE_ERR_INVALID
    assert lib.moe_update_bias(ctypes.byref(d), -1, fake, fake, 0.001, None) == moe.MOE_ERR_INVALID
    p = np.full(4, 0.25)
    t = np.zeros((4, 2), np.int32)
    bad_orders = np.array([[0, 1, 2, 2]], np.int32)
    assert lib.moe_build_tid2eid_best(p.ctypes.data, 4, 8, 2, bad_orders.ctypes.data, 1, t.ctypes.data, None, None,
                                      None) == moe.MOE_ERR_INVALID
    out_of_range = np.array([[0, 1, 2, 4]], np.int32)
    assert lib.moe_build_tid2eid_best(p.ctypes.data, 4, 8, 2, out_of_range.ctypes.data, 1, t.ctypes.data, None,
                                      None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_build_tid2eid_best(p.ctypes.data, 4, 8, 2, bad_orders.ctypes.data, 0, t.ctypes.data, None, None,
                                      None) == moe.MOE_ERR_INVALID


def test_gather_entry_points_reject_bad_arguments_before_launch(moe):
    lib = moe.lib
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: every call below must fail its argument checks first
    good = moe.Mxfp4Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    # the gathered up projection runs on the CTA-pair kernel only: inter_dim % 256 == 0
    d = moe.layer_desc(W.CONFIGS["tiny"].replace(dim=256, inter_dim=384))
    assert lib.moe_expert_ffn_gather(ctypes.byref(d), 4, fake, fake, None, fake, fake, fake, fake, fake, fake, fake,
                                     1 << 30, None) == moe.MOE_ERR_UNSUPPORTED
    d = moe.layer_desc(W.CONFIGS["tiny"].replace(dim=512, inter_dim=512), options=moe.MOE_OPT_GEMM_ONE_CTA)
    assert lib.moe_expert_ffn_gather(ctypes.byref(d), 4, fake, fake, None, fake, fake, fake, fake, fake, fake, fake,
                                     1 << 30, None) == moe.MOE_ERR_UNSUPPORTED
    d = moe.layer_desc(W.CONFIGS["tiny"].replace(dim=512, inter_dim=512))
    # missing row map, weights, outputs; misaligned x; short workspace
    assert lib.moe_expert_ffn_gather(ctypes.byref(d), 4, None, fake, None, fake, fake, fake, fake, fake, fake, fake,
                                     1 << 30, None) == moe.MOE_ERR_INVALID
    assert lib.moe_expert_ffn_gather(ctypes.byref(d), 4, fake, fake, None, fake, None, fake, fake, fake, fake, fake,
                                     1 << 30, None) == moe.MOE_ERR_INVALID
    assert lib.moe_expert_ffn_gather(ctypes.byref(d), 4, fake, fake, None, fake, fake, fake, fake, None, fake, fake,
                                     1 << 30, None) == moe.MOE_ERR_INVALID
    assert lib.moe_expert_ffn_gather(ctypes.byref(d), 4, fake, fake, None, P((1 << 20) + 2), fake, fake, fake, fake,
                                     fake, fake, 1 << 30, None) == moe.MOE_ERR_INVALID
    assert lib.moe_expert_ffn_gather(ctypes.byref(d), 4, fake, fake, None, fake, fake, fake, fake, fake, fake, fake,
                                     16, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_expert_ffn_mxfp4_gather(ctypes.byref(d), 4, fake, fake, None, fake, None, fake, fake, fake,
                                           1 << 30, None) == moe.MOE_ERR_INVALID
    assert lib.moe_expert_ffn_mxfp4_gather(ctypes.byref(d), 4, None, fake, None, fake, ctypes.byref(good), fake,
                                           fake, fake, 1 << 30, None) == moe.MOE_ERR_INVALID
    d = moe.layer_desc(W.CONFIGS["tiny"].replace(dim=512, inter_dim=256))   # MXFP4 needs I % 512 == 0
    assert lib.moe_expert_ffn_mxfp4_gather(ctypes.byref(d), 4, fake, fake, None, fake, ctypes.byref(good), fake,
                                           fake, fake, 1 << 30, None) == moe.MOE_ERR_UNSUPPORTED
    # T == 0 needs no pointers at all
    assert lib.moe_expert_ffn_gather(ctypes.byref(d), 0, None, None, None, None, None, None, None, None, None, fake,
                                     1 << 30, None) == moe.MOE_OK


def test_mxfp4_entry_points_reject_bad_arguments_before_launch(moe):
    lib = moe.lib
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced: every call below must fail its argument checks first
    good = moe.Mxfp4Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    # inter_dim and dim must be multiples of 512
    for dim, inter in ((256, 128), (512, 256), (768, 512)):
        d = moe.layer_desc(W.CONFIGS["tiny"].replace(dim=dim, inter_dim=inter))
        assert lib.moe_expert_ffn_mxfp4(ctypes.byref(d), 4, fake, fake, None, fake, ctypes.byref(good), fake, fake,
                                        fake, 1 << 30, None) == moe.MOE_ERR_UNSUPPORTED
    d = moe.layer_desc(W.CONFIGS["tiny"].replace(dim=512, inter_dim=512))
    assert lib.moe_expert_ffn_mxfp4(ctypes.byref(d), 4, fake, fake, None, fake, None, fake, fake, fake, 1 << 30,
                                    None) == moe.MOE_ERR_INVALID
    for field in ("w1", "w1_scale", "w3", "w3_scale", "w2", "w2_scale"):
        bad = moe.Mxfp4Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
        setattr(bad, field, (1 << 20) + 8)    # misaligned
        assert lib.moe_expert_ffn_mxfp4(ctypes.byref(d), 4, fake, fake, None, fake, ctypes.byref(bad), fake, fake,
                                        fake, 1 << 30, None) == moe.MOE_ERR_INVALID, field
        setattr(bad, field, None)
        assert lib.moe_forward_mxfp4(ctypes.byref(d), 4, fake, None, None, 0, fake, None, None, ctypes.byref(bad),
                                     fake, None, None, None, fake, 1 << 30, None) == moe.MOE_ERR_INVALID, field
    assert lib.moe_forward_mxfp4(ctypes.byref(d), 4, fake, None, None, 0, fake, None, None, None, fake, None, None,
                                 None, fake, 1 << 30, None) == moe.MOE_ERR_INVALID
    assert lib.moe_forward_mxfp4(ctypes.byref(d), 4, fake, None, None, 0, fake, None, None, ctypes.byref(good), fake,
                                 None, None, None, fake, 16, None) == moe.MOE_ERR_WORKSPACE


def test_tid2eid_table_file_round_trip_and_checks(moe, tmp_path):
    # a table built once is kept in a file and read back for every forward; the file carries the
    # sizes and a hash of the frequencies it was built from
    rng = np.random.default_rng(5)
    m, n, k = 1000, 16, 3
    p = rng.random(m)
    p /= p.sum()
    table, _ = moe.moe_build_tid2eid(p, n, k)
    path = str(tmp_path / "t.bin")
    moe.moe_tid2eid_save(path, table, n, p)
    assert moe.moe_tid2eid_header(path) == (m, k, n)
    assert np.array_equal(moe.moe_tid2eid_load(path, p), table)
    assert np.array_equal(moe.moe_tid2eid_load(path), table)              # no frequency check
    q = p.copy()
    q[17] *= 1.0 + 2.0 ** -40                                              # other frequencies
    with pytest.raises(moe.MoeError) as e:
        moe.moe_tid2eid_load(path, q)
    assert e.value.status == moe.MOE_ERR_INVALID
    lib = moe.lib
    out = np.zeros((m, k), np.int32)
    for dims in ((m + 1, k, n), (m, k + 1, n), (m, k, n + 1)):            # sizes the file does not hold
        assert lib.moe_tid2eid_load(path.encode(), out.ctypes.data, *dims, None) == moe.MOE_ERR_INVALID
    raw = bytearray(open(path, "rb").read())
    assert len(raw) == 32 + 4 * m * k and raw[:8] == b"MOETID01"
    bad = bytearray(raw)
    bad[32 + 4 * 5:32 + 4 * 6] = (n + 3).to_bytes(4, "little")           # an expert id out of range
    open(path, "wb").write(bytes(bad))
    out[:] = -7
    assert lib.moe_tid2eid_load(path.encode(), out.ctypes.data, m, k, n, None) == moe.MOE_ERR_INVALID
    assert np.all(out == -7)                                              # a refused file writes nothing
    open(path, "wb").write(bytes(raw[:-4]))                                # truncated
    assert lib.moe_tid2eid_load(path.encode(), out.ctypes.data, m, k, n, None) == moe.MOE_ERR_INVALID
    open(path, "wb").write(bytes(raw) + b"\0")                            # trailing bytes
    assert lib.moe_tid2eid_load(path.encode(), out.ctypes.data, m, k, n, None) == moe.MOE_ERR_INVALID
    open(path, "wb").write(b"NOTATABL" + bytes(raw[8:]))                  # not a table file
    with pytest.raises(moe.MoeError) as e:
        moe.moe_tid2eid_header(path)
    assert e.value.status == moe.MOE_ERR_INVALID
    with pytest.raises(moe.MoeError) as e:
        moe.moe_tid2eid_load(str(tmp_path / "missing.bin"))
    assert e.value.status == moe.MOE_ERR_IO
    # saved without frequencies: loads without the check, fails the check when p is given
    moe.moe_tid2eid_save(path, table, n)
    assert np.array_equal(moe.moe_tid2eid_load(path), table)
    with pytest.raises(moe.MoeError):
        moe.moe_tid2eid_load(path, p)
    # an id outside [0, n) is refused before anything is written
    path2 = str(tmp_path / "t2.bin")
    t2 = table.copy()
    t2[3, 1] = n
    with pytest.raises(moe.MoeError) as e:
        moe.moe_tid2eid_save(path2, t2, n, p)
    assert e.value.status == moe.MOE_ERR_INVALID and not os.path.exists(path2)


def test_token_chunk_families(moe):
    """token_chunk: 128 / 256 for the bf16 tensor-core kernels, 96 / 224 for the block-scaled ones; any
    other value is invalid, a value of the other family unsupported (both before the workspace check)."""
    lib = moe.lib
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced
    good = moe.Mxfp4Weights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    cfg = W.CONFIGS["tiny"].replace(dim=512, inter_dim=512)
    want = {0: ("ws", "ws"), 96: ("unsup", "ws"), 128: ("ws", "unsup"), 224: ("unsup", "ws"),
            256: ("ws", "unsup"), 64: ("inv", "inv"), 192: ("inv", "inv")}
    code = {"ws": moe.MOE_ERR_WORKSPACE, "unsup": moe.MOE_ERR_UNSUPPORTED, "inv": moe.MOE_ERR_INVALID}
    for chunk, (bf16_want, mx_want) in want.items():
        d = moe.layer_desc(cfg, token_chunk=chunk)
        assert lib.moe_expert_ffn(ctypes.byref(d), 4, fake, fake, None, fake, fake, fake, fake, fake, fake, fake,
                                  16, None) == code[bf16_want], chunk
        assert lib.moe_expert_ffn_mxfp4(ctypes.byref(d), 4, fake, fake, None, fake, ctypes.byref(good), fake, fake,
                                        fake, 16, None) == code[mx_want], chunk
        # MXFP4 weights on bf16 activations run the bf16 tensor-core kernels: their family
        d = moe.layer_desc(cfg, options=moe.MOE_OPT_MXFP4_BF16_ACTIVATIONS, token_chunk=chunk)
        assert lib.moe_expert_ffn_mxfp4(ctypes.byref(d), 4, fake, fake, None, fake, ctypes.byref(good), fake, fake,
                                        fake, 16, None) == code[bf16_want], chunk


def test_gate_prepare_rejects_bad_arguments(moe):
    lib = moe.lib
    P = ctypes.c_void_p
    fake = P(1 << 20)  # never dereferenced
    cfg = W.CONFIGS["v3_prefill"]
    d = moe.layer_desc(cfg)
    assert lib.moe_gate_prepared_bytes(ctypes.byref(d)) == 1024 + 3 * cfg.n_experts * cfg.dim * 2
    assert lib.moe_gate_prepare(ctypes.byref(d), None, fake, None) == moe.MOE_ERR_INVALID
    assert lib.moe_gate_prepare(ctypes.byref(d), fake, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_gate_prepare(ctypes.byref(d), fake, P((1 << 20) + 8), None) == moe.MOE_ERR_INVALID
    assert lib.moe_gate_prepare(ctypes.byref(d), P((1 << 20) + 4), fake, None) == moe.MOE_ERR_INVALID
    # a misaligned prepared pointer in the descriptor fails every entry point's descriptor check
    d.gate_prepared = (1 << 20) + 8
    assert lib.moe_gate(ctypes.byref(d), 4, fake, fake, None, None, fake, fake, fake, 1 << 30, None) == \
        moe.MOE_ERR_INVALID
    assert lib.moe_gate_prepared_bytes(ctypes.byref(d)) == 0
