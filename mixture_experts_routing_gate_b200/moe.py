"""Python binding of libmoe (include/moe.h): argument marshalling only.

Each function has the name of the C entry point it calls, takes torch tensors (device tensors
unless noted) and passes their data pointers, the sizes and the current CUDA stream.  Every value
is computed by the CUDA library; a non-OK status raises MoeError.  Importing this module raises
ImportError when libmoe.so has not been built -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m mixture_experts_routing_gate_b200.build`")

# ------------------------------------------------------------------------------------------------
# types
# ------------------------------------------------------------------------------------------------
(MOE_OK, MOE_ERR_INVALID, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_WORKSPACE, MOE_ERR_DEVICE, MOE_ERR_TIMEOUT,
 MOE_ERR_IO) = range(8)
SCORE_FUNCS = {"sigmoid": 0, "sqrtsoftplus": 1, "softmax": 2}


# moe_layer_desc.options bits (kernel choices; the values computed do not depend on them)
MOE_OPT_ROUTER_ONE_CTA = 1   # one CTA per 128 tokens instead of the split-K cluster router
MOE_OPT_GEMM_ONE_CTA = 2     # single-CTA expert GEMMs instead of CTA pairs (bf16 weights)
MOE_OPT_FUSED_GATHER = 4     # moe_forward: the up projection gathers rows of x, no x_perm
MOE_OPT_MXFP4_BF16_ACTIVATIONS = 8   # MXFP4 weights with bf16 activations (decoded on the SMs)


class LayerDesc(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int), ("n_experts", ctypes.c_int), ("n_groups", ctypes.c_int),
                ("n_limited_groups", ctypes.c_int), ("topk", ctypes.c_int), ("inter_dim", ctypes.c_int),
                ("n_shared", ctypes.c_int), ("score_func", ctypes.c_int), ("route_scale", ctypes.c_float),
                ("renorm", ctypes.c_int), ("swiglu_limit", ctypes.c_float), ("weight_in_expert", ctypes.c_int),
                ("options", ctypes.c_int), ("token_chunk", ctypes.c_int), ("gate_prepared", ctypes.c_void_p)]


def layer_desc(cfg, options: int = 0, token_chunk: int = 0) -> LayerDesc:
    """moe_layer_desc from any object with the LayerConfig attribute names; ``options`` ORs MOE_OPT_*
    kernel choices, ``token_chunk`` (0; 128 or 256 for the bf16 tensor-core GEMMs, 96 or 224 for the
    block-scaled ones) fixes the CTA-pair GEMMs' token-chunk rows.  gate_prepared starts NULL (see
    prepare_gate)."""
    renorm = getattr(cfg, "renorm", cfg.score_func in ("sigmoid", "sqrtsoftplus"))
    return LayerDesc(cfg.dim, cfg.n_experts, cfg.n_groups, cfg.n_limited_groups, cfg.topk, cfg.inter_dim,
                     getattr(cfg, "n_shared", 1), SCORE_FUNCS[cfg.score_func], float(cfg.route_scale), int(renorm),
                     float(getattr(cfg, "swiglu_limit", 0.0) or 0.0), int(bool(getattr(cfg, "weight_in_expert", False))),
                     int(options), int(token_chunk))


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, info: Optional[int] = None):
        self.status = status
        msg = f"{where}: {lib.moe_status_str(status).decode()}"
        if info is not None:
            msg += f" (info={info})"
        super().__init__(msg)


class Mxfp4Weights(ctypes.Structure):
    """moe_mxfp4_weights: device pointers of the packed E2M1 codes and UE8M0 scales."""
    _fields_ = [("w1", ctypes.c_void_p), ("w1_scale", ctypes.c_void_p), ("w3", ctypes.c_void_p),
                ("w3_scale", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("w2_scale", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.POINTER(LayerDesc)
_W4 = ctypes.POINTER(Mxfp4Weights)
_SIG = {
    "moe_workspace_bytes": (ctypes.c_size_t, [_D, _I]),
    "moe_workspace_init": (_I, [_P, ctypes.c_size_t, _P]),
    "moe_gate_prepared_bytes": (ctypes.c_size_t, [_D]),
    "moe_gate_prepare": (_I, [_D, _P, _P, _P]),
    "moe_gate": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_hash_gate": (_I, [_D, _I, _P, _P, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_ngram_gate": (_I, [_D, _I, _P, _P, _P, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_build_tid2eid": (_I, [_P, _I, _I, _I, _P, _P]),
    "moe_build_tid2eid_best": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _P, ctypes.POINTER(ctypes.c_int32)]),
    "moe_tid2eid_save": (_I, [ctypes.c_char_p, _P, _I, _I, _I, _P]),
    "moe_tid2eid_header": (_I, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                ctypes.POINTER(ctypes.c_int)]),
    "moe_tid2eid_load": (_I, [ctypes.c_char_p, _P, _I, _I, _I, _P]),
    "moe_dispatch": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_dispatch_static": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_expert_ffn": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_expert_ffn_mxfp4": (_I, [_D, _I, _P, _P, _P, _P, _W4, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_expert_ffn_gather": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_expert_ffn_mxfp4_gather": (_I, [_D, _I, _P, _P, _P, _P, _W4, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_combine": (_I, [_D, _I, _P, _P, _P, _P, _P, _P]),
    "moe_forward": (_I, [_D, _I, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_forward_mxfp4": (_I, [_D, _I, _P, _P, _P, _I, _P, _P, _P, _W4, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_update_bias": (_I, [_D, _I, _P, _P, ctypes.c_float, _P]),
    "moe_get_error": (_I, [_P, _P, ctypes.POINTER(ctypes.c_int32)]),
    "moe_status_str": (ctypes.c_char_p, [_I]),
}


def load_library(path: str) -> ctypes.CDLL:
    """Opens a build of libmoe and declares the signatures of its entry points.  The module's `lib` is
    the in-tree libmoe.so; the tests also open the test build (libmoe_testhooks.so) this way."""
    handle = ctypes.CDLL(path)
    for name, (res, args) in _SIG.items():
        f = getattr(handle, name)
        f.restype = res
        f.argtypes = args
    return handle


lib = load_library(_LIB_PATH)
EXPORTS = tuple(_SIG)


# ------------------------------------------------------------------------------------------------
# marshalling helpers
# ------------------------------------------------------------------------------------------------
def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return t.data_ptr()


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _dev(t: Optional[torch.Tensor], dtype, name: str):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


# ------------------------------------------------------------------------------------------------
# workspace
# ------------------------------------------------------------------------------------------------
def moe_workspace_bytes(desc: LayerDesc, T: int) -> int:
    return int(lib.moe_workspace_bytes(ctypes.byref(desc), T))


class Workspace:
    """A device workspace of moe_workspace_bytes(desc, T) bytes (1 KiB aligned), error word cleared."""

    def __init__(self, desc: LayerDesc, T: int, device=None):
        n = moe_workspace_bytes(desc, T)
        if n == 0:
            raise MoeError(MOE_ERR_INVALID, "moe_workspace_bytes")
        self.buf = torch.empty(n + 1024, dtype=torch.uint8, device=device or "cuda")
        off = (-self.buf.data_ptr()) % 1024
        self.tensor = self.buf[off:off + n]
        self.nbytes = n
        _check(lib.moe_workspace_init(self.ptr, n, _stream()), "moe_workspace_init")

    @property
    def ptr(self) -> int:
        return self.tensor.data_ptr()


def moe_workspace_init(ws: Workspace, stream=None):
    _check(lib.moe_workspace_init(ws.ptr, ws.nbytes, _stream(stream)), "moe_workspace_init")


# ------------------------------------------------------------------------------------------------
# entry points
# ------------------------------------------------------------------------------------------------
def prepare_gate(desc, w_gate: torch.Tensor, stream=None) -> torch.Tensor:
    """moe_gate_prepare into a new device buffer, which it points desc.gate_prepared at; the caller
    keeps the returned buffer alive while desc is used (and prepares again when w_gate changes)."""
    _dev(w_gate, torch.float32, "w_gate")
    buf = torch.empty(lib.moe_gate_prepared_bytes(ctypes.byref(desc)), dtype=torch.uint8, device=w_gate.device)
    _check(lib.moe_gate_prepare(ctypes.byref(desc), _ptr(w_gate), buf.data_ptr(), _stream(stream)), "moe_gate_prepare")
    desc.gate_prepared = buf.data_ptr()
    return buf


def moe_gate(desc, x, w_gate, bias, logit_offset, weights, indices, ws: Workspace, stream=None):
    _dev(x, torch.bfloat16, "x"); _dev(w_gate, torch.float32, "w_gate")
    _dev(bias, torch.float32, "bias"); _dev(logit_offset, torch.float32, "logit_offset")
    _dev(weights, torch.float32, "weights"); _dev(indices, torch.int32, "indices")
    _check(lib.moe_gate(ctypes.byref(desc), x.shape[0], _ptr(x), _ptr(w_gate), _ptr(bias), _ptr(logit_offset),
                        _ptr(weights), _ptr(indices), ws.ptr, ws.nbytes, _stream(stream)), "moe_gate")


def moe_hash_gate(desc, token_ids, tid2eid, x, w_gate, weights, indices, ws: Workspace, stream=None):
    _dev(token_ids, torch.int32, "token_ids"); _dev(tid2eid, torch.int32, "tid2eid")
    _dev(x, torch.bfloat16, "x"); _dev(w_gate, torch.float32, "w_gate")
    _check(lib.moe_hash_gate(ctypes.byref(desc), x.shape[0], _ptr(token_ids), _ptr(tid2eid), tid2eid.shape[0],
                             _ptr(x), _ptr(w_gate), _ptr(weights), _ptr(indices), ws.ptr, ws.nbytes,
                             _stream(stream)), "moe_hash_gate")


def moe_ngram_gate(desc, prev_ids, token_ids, primes, vocab: int, x, w_gate, weights, indices, ws: Workspace,
                   stream=None):
    """2-gram hash gate; primes is a host sequence of desc.topk primes in (vocab, 2^32)."""
    _dev(prev_ids, torch.int32, "prev_ids"); _dev(token_ids, torch.int32, "token_ids")
    _dev(x, torch.bfloat16, "x"); _dev(w_gate, torch.float32, "w_gate")
    q = np.ascontiguousarray(np.asarray(primes, dtype=np.int64))
    if q.shape != (desc.topk,):
        raise ValueError(f"primes: expected {desc.topk} values, got shape {q.shape}")
    _check(lib.moe_ngram_gate(ctypes.byref(desc), x.shape[0], _ptr(prev_ids), _ptr(token_ids), q.ctypes.data,
                              int(vocab), _ptr(x), _ptr(w_gate), _ptr(weights), _ptr(indices), ws.ptr, ws.nbytes,
                              _stream(stream)), "moe_ngram_gate")


def moe_build_tid2eid_best(p: np.ndarray, n_experts: int, k: int, orders: np.ndarray):
    """Host call: orders [runs, m] int32 permutations.  Returns (tid2eid, loads, max_vio [runs], kept)."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    m = p.shape[0]
    orders = np.ascontiguousarray(orders, dtype=np.int32)
    if orders.ndim != 2 or orders.shape[1] != m:
        raise ValueError(f"orders: expected [runs, {m}], got {orders.shape}")
    runs = orders.shape[0]
    table = np.zeros((m, k), np.int32)
    loads = np.zeros(n_experts, np.float64)
    vio = np.zeros(runs, np.float64)
    kept = ctypes.c_int32(-1)
    _check(lib.moe_build_tid2eid_best(p.ctypes.data, m, n_experts, k, orders.ctypes.data, runs, table.ctypes.data,
                                      loads.ctypes.data, vio.ctypes.data, ctypes.byref(kept)),
           "moe_build_tid2eid_best")
    return table, loads, vio, int(kept.value)


def moe_update_bias(desc, T: int, counts, bias, gamma: float, stream=None):
    """In-place bias[e] -= / += gamma for experts above / below the balanced load T*k/E."""
    _dev(counts, torch.int32, "counts"); _dev(bias, torch.float32, "bias")
    _check(lib.moe_update_bias(ctypes.byref(desc), int(T), _ptr(counts), _ptr(bias), float(gamma), _stream(stream)),
           "moe_update_bias")


def moe_tid2eid_save(path: str, tid2eid: np.ndarray, n_experts: int, p: Optional[np.ndarray] = None):
    """Host call: writes tid2eid [m, k] to a table file (with the hash of p when given)."""
    t = np.ascontiguousarray(tid2eid, dtype=np.int32)
    pp = None if p is None else np.ascontiguousarray(p, dtype=np.float64)
    if pp is not None and pp.shape[0] != t.shape[0]:
        raise ValueError(f"p: expected [{t.shape[0]}], got {pp.shape}")
    _check(lib.moe_tid2eid_save(os.fsencode(path), t.ctypes.data, t.shape[0], t.shape[1], n_experts,
                                None if pp is None else pp.ctypes.data), "moe_tid2eid_save")


def moe_tid2eid_header(path: str):
    """Host call: (m, k, n_experts) of a table file."""
    m, k, n = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.moe_tid2eid_header(os.fsencode(path), ctypes.byref(m), ctypes.byref(k), ctypes.byref(n)),
           "moe_tid2eid_header")
    return m.value, k.value, n.value


def moe_tid2eid_load(path: str, p: Optional[np.ndarray] = None) -> np.ndarray:
    """Host call: the table [m, k] int32 of a file, checked against the frequencies p when given."""
    m, k, n = moe_tid2eid_header(path)
    pp = None if p is None else np.ascontiguousarray(p, dtype=np.float64)
    if pp is not None and pp.shape[0] != m:
        raise MoeError(MOE_ERR_INVALID, "moe_tid2eid_load: p has the wrong length")
    t = np.zeros((m, k), np.int32)
    _check(lib.moe_tid2eid_load(os.fsencode(path), t.ctypes.data, m, k, n, None if pp is None else pp.ctypes.data),
           "moe_tid2eid_load")
    return t


def moe_build_tid2eid(p: np.ndarray, n_experts: int, k: int):
    """Host call: returns (tid2eid [m, k] int32, loads [n_experts] fp64) as numpy arrays."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    m = p.shape[0]
    table = np.zeros((m, k), np.int32)
    loads = np.zeros(n_experts, np.float64)
    _check(lib.moe_build_tid2eid(p.ctypes.data, m, n_experts, k, table.ctypes.data, loads.ctypes.data),
           "moe_build_tid2eid")
    return table, loads


def moe_dispatch(desc, indices, x, counts, offsets, row_of_slot, tok_of_row, x_perm, ws: Workspace, stream=None):
    """x_perm may be None: the permutation only, for moe_expert_ffn_gather."""
    _dev(indices, torch.int32, "indices"); _dev(x, torch.bfloat16, "x"); _dev(x_perm, torch.bfloat16, "x_perm")
    _check(lib.moe_dispatch(ctypes.byref(desc), x.shape[0], _ptr(indices), _ptr(x), _ptr(counts), _ptr(offsets),
                            _ptr(row_of_slot), _ptr(tok_of_row), _ptr(x_perm), ws.ptr, ws.nbytes,
                            _stream(stream)), "moe_dispatch")


def moe_dispatch_static(desc, indices, x, counts, offsets, row_of_slot, tok_of_row, x_perm, stream=None):
    """moe_dispatch with the library's own fixed scratch instead of a workspace (allocates nothing)."""
    _dev(indices, torch.int32, "indices"); _dev(x, torch.bfloat16, "x"); _dev(x_perm, torch.bfloat16, "x_perm")
    _check(lib.moe_dispatch_static(ctypes.byref(desc), x.shape[0], _ptr(indices), _ptr(x), _ptr(counts),
                                   _ptr(offsets), _ptr(row_of_slot), _ptr(tok_of_row), _ptr(x_perm),
                                   _stream(stream)), "moe_dispatch_static")


def moe_expert_ffn(desc, x_perm, offsets, x, w1, w3, w2, out_perm, out_shared, ws: Workspace, row_weights=None,
                   stream=None):
    for t, n in ((x_perm, "x_perm"), (x, "x"), (w1, "w1"), (w3, "w3"), (w2, "w2"), (out_perm, "out_perm"),
                 (out_shared, "out_shared")):
        _dev(t, torch.bfloat16, n)
    _dev(row_weights, torch.float32, "row_weights")
    _check(lib.moe_expert_ffn(ctypes.byref(desc), x.shape[0], _ptr(x_perm), _ptr(offsets), _ptr(row_weights),
                              _ptr(x), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(out_perm), _ptr(out_shared), ws.ptr,
                              ws.nbytes, _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_gather(desc, tok_of_row, offsets, x, w1, w3, w2, out_perm, out_shared, ws: Workspace,
                          row_weights=None, stream=None):
    """moe_expert_ffn reading routed row r from x[tok_of_row[r]] (no x_perm)."""
    for t, n in ((x, "x"), (w1, "w1"), (w3, "w3"), (w2, "w2"), (out_perm, "out_perm"), (out_shared, "out_shared")):
        _dev(t, torch.bfloat16, n)
    _dev(tok_of_row, torch.int32, "tok_of_row")
    _dev(row_weights, torch.float32, "row_weights")
    _check(lib.moe_expert_ffn_gather(ctypes.byref(desc), x.shape[0], _ptr(tok_of_row), _ptr(offsets),
                                     _ptr(row_weights), _ptr(x), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(out_perm),
                                     _ptr(out_shared), ws.ptr, ws.nbytes, _stream(stream)), "moe_expert_ffn_gather")


def moe_combine(desc, T, out_perm, row_of_slot, weights, out_shared, y, stream=None):
    _check(lib.moe_combine(ctypes.byref(desc), T, _ptr(out_perm), _ptr(row_of_slot), _ptr(weights), _ptr(out_shared),
                           _ptr(y), _stream(stream)), "moe_combine")


def moe_forward(desc, x, w_gate, w1, w3, w2, y, ws: Workspace, bias=None, logit_offset=None, token_ids=None,
                tid2eid=None, weights_out=None, indices_out=None, counts_out=None, stream=None):
    vocab = 0 if tid2eid is None else tid2eid.shape[0]
    _check(lib.moe_forward(ctypes.byref(desc), x.shape[0], _ptr(x), _ptr(token_ids), _ptr(tid2eid), vocab,
                           _ptr(w_gate), _ptr(bias), _ptr(logit_offset), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(y),
                           _ptr(weights_out), _ptr(indices_out), _ptr(counts_out), ws.ptr, ws.nbytes,
                           _stream(stream)), "moe_forward")


def mxfp4_weights(w) -> Mxfp4Weights:
    """moe_mxfp4_weights from any object with uint8 CUDA tensors w1, w1s, w3, w3s, w2, w2s."""
    for name in ("w1", "w1s", "w3", "w3s", "w2", "w2s"):
        _dev(getattr(w, name), torch.uint8, name)
    return Mxfp4Weights(_ptr(w.w1), _ptr(w.w1s), _ptr(w.w3), _ptr(w.w3s), _ptr(w.w2), _ptr(w.w2s))


def moe_expert_ffn_mxfp4(desc, x_perm, offsets, x, w, out_perm, out_shared, ws: Workspace, row_weights=None,
                         stream=None):
    """moe_expert_ffn with MXFP4 weights ``w`` (see mxfp4_weights)."""
    for t, n in ((x_perm, "x_perm"), (x, "x"), (out_perm, "out_perm"), (out_shared, "out_shared")):
        _dev(t, torch.bfloat16, n)
    _dev(row_weights, torch.float32, "row_weights")
    mw = mxfp4_weights(w)
    _check(lib.moe_expert_ffn_mxfp4(ctypes.byref(desc), x.shape[0], _ptr(x_perm), _ptr(offsets), _ptr(row_weights),
                                    _ptr(x), ctypes.byref(mw), _ptr(out_perm), _ptr(out_shared), ws.ptr, ws.nbytes,
                                    _stream(stream)), "moe_expert_ffn_mxfp4")


def moe_expert_ffn_mxfp4_gather(desc, tok_of_row, offsets, x, w, out_perm, out_shared, ws: Workspace,
                                row_weights=None, stream=None):
    """moe_expert_ffn_mxfp4 reading routed row r from x[tok_of_row[r]] (no x_perm)."""
    for t, n in ((x, "x"), (out_perm, "out_perm"), (out_shared, "out_shared")):
        _dev(t, torch.bfloat16, n)
    _dev(tok_of_row, torch.int32, "tok_of_row")
    _dev(row_weights, torch.float32, "row_weights")
    mw = mxfp4_weights(w)
    _check(lib.moe_expert_ffn_mxfp4_gather(ctypes.byref(desc), x.shape[0], _ptr(tok_of_row), _ptr(offsets),
                                           _ptr(row_weights), _ptr(x), ctypes.byref(mw), _ptr(out_perm),
                                           _ptr(out_shared), ws.ptr, ws.nbytes, _stream(stream)),
           "moe_expert_ffn_mxfp4_gather")


def moe_forward_mxfp4(desc, x, w_gate, w, y, ws: Workspace, bias=None, logit_offset=None, token_ids=None,
                      tid2eid=None, weights_out=None, indices_out=None, counts_out=None, stream=None):
    """moe_forward with MXFP4 expert weights ``w`` (see mxfp4_weights)."""
    vocab = 0 if tid2eid is None else tid2eid.shape[0]
    mw = mxfp4_weights(w)
    _check(lib.moe_forward_mxfp4(ctypes.byref(desc), x.shape[0], _ptr(x), _ptr(token_ids), _ptr(tid2eid), vocab,
                                 _ptr(w_gate), _ptr(bias), _ptr(logit_offset), ctypes.byref(mw), _ptr(y),
                                 _ptr(weights_out), _ptr(indices_out), _ptr(counts_out), ws.ptr, ws.nbytes,
                                 _stream(stream)), "moe_forward_mxfp4")


def moe_get_error(ws: Workspace, stream=None):
    """(status, info) of the first bad value a kernel saw since the last call; clears it."""
    info = ctypes.c_int32(0)
    st = lib.moe_get_error(ws.ptr, _stream(stream), ctypes.byref(info))
    return int(st), int(info.value)


def check_device_errors(ws: Workspace, where: str = "kernels", stream=None):
    st, info = moe_get_error(ws, stream)
    if st != MOE_OK:
        raise MoeError(st, where, info)
