"""fp64 CPU oracle for the speculative-decoding verify/accept step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` leg of ``bench.py`` may import this
package.  The product (the CUDA library and its Python binding) never imports
it, and it imports nothing from the product: the two share no code.  The only
module both sides use is the seeded input generator
(``speculative_decoding_verify_temperature_b200.workloads``), which holds no
verify arithmetic.

The arithmetic lives in ``spec_oracle.c`` (plain C, fp64); this file is the
ctypes marshalling around it.  Array conventions:

* logits / probability arrays are numpy arrays of shape ``[B, R, stride]``
  where ``stride >= V`` is the row stride in elements; dtype ``float32`` means
  f32 input and ``uint16`` means bf16 bit patterns;
* integer arrays are ``int32``, uniforms ``float32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spec_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

F32, BF16 = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile ``spec_oracle.c`` into ``liboracle.so`` next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        P = ctypes.c_void_p
        i32, i64, f32, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        L.oracle_chain.restype = None
        L.oracle_chain.argtypes = [i32, i32, i32, P, i32, i64, P, i32, i32, i64,
                                   P, P, P, P, P, P, P, P, P, P, P, i32]
        L.oracle_tree_greedy.restype = None
        L.oracle_tree_greedy.argtypes = [i32, i32, i32, i32, P, i32, i64, P, P, P, P, P, P, i32]
        L.oracle_tree_sample.restype = None
        L.oracle_tree_sample.argtypes = [i32, i32, i32, i32, P, i32, i64, P, P, P, P, P, P, i64,
                                         f32, f32, P, P, P, P, P, P, P, i32]
        L.oracle_tree_sample_filtered.restype = None
        L.oracle_tree_sample_filtered.argtypes = [i32, i32, i32, i32, P, i32, i64, P, P, P, P, P, P, i64,
                                                  f32, f32, P, P, P, P, P, P, P, P, P, P, i32]
        L.oracle_chain_filtered.restype = None
        L.oracle_chain_filtered.argtypes = [i32, i32, i32, P, i32, i64, P, i32, i32, i64,
                                            P, P, P, P, P, P, P, P, P, P, P, P, P, P, i32]
        L.oracle_filter_row.restype = i32
        L.oracle_filter_row.argtypes = [P, i32, i32, f64, i32, f64, P, P]
        L.oracle_tree_mss.restype = None
        L.oracle_tree_mss.argtypes = [i32, i32, i32, i32, P, i32, i64, P, P, P, P, P, P, i64,
                                      P, P, P, P, P, P, P, i32]
        L.oracle_softmax_row.restype = i32
        L.oracle_softmax_row.argtypes = [P, i32, i32, f64, P]
        L.oracle_inverse_cdf.restype = i32
        L.oracle_inverse_cdf.argtypes = [P, i32, f64, P, P]
        L.oracle_set_mutation.restype = None
        L.oracle_set_mutation.argtypes = [i32]
        _lib = L
    return _lib


def set_mutation(m: int) -> None:
    """Plant deliberate mistake ``m`` (0 = none).  For the pin-sensitivity tests only."""
    lib().oracle_set_mutation(int(m))


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"logits must be float32 or uint16 (bf16 bits), got {a.dtype}")


def _c(a: np.ndarray, dtype=None) -> np.ndarray:
    a = np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def chain(target, draft, draft_is_probs, draft_tokens, temperature, coins, final_u, V=None,
          nthreads: int = 0, top_k=None, top_p=None) -> dict:
    """Chain verify (acceptance rules 1-3).  ``target`` is ``[B, gamma+1, stride]``,
    ``draft`` ``[B, gamma, dstride]`` (logits, or f32 probabilities when
    ``draft_is_probs``).  With ``top_k`` / ``top_p`` (per sequence, ``[B]``) the
    target rows and draft-logit rows are top-k / top-p filtered first."""
    target = _c(target)
    draft = _c(draft)
    B, R, ts = target.shape
    gamma = R - 1
    ds = draft.shape[2]
    V = ts if V is None else int(V)
    if draft_is_probs and draft.dtype != np.float32:
        raise TypeError("draft probabilities must be float32")
    draft_tokens = _c(draft_tokens, np.int32).reshape(B, gamma)
    temperature = _c(temperature, np.float32).reshape(B)
    coins = _c(coins, np.float32).reshape(B, gamma)
    final_u = _c(final_u, np.float32).reshape(B)
    out = dict(
        tokens=np.empty((B, gamma + 1), np.int32),
        num_accepted=np.empty(B, np.int32),
        px=np.empty((B, gamma), np.float64),
        qx=np.empty((B, gamma), np.float64),
        S=np.empty(B, np.float64),
        dmargin=np.empty(B, np.float64),
        cmargin=np.empty(B, np.float64),
    )
    if B == 0:
        return out
    if top_k is None and top_p is None:
        lib().oracle_chain(B, gamma, V, _ptr(target), _dtype_code(target), ts,
                           _ptr(draft), F32 if draft_is_probs else _dtype_code(draft),
                           int(bool(draft_is_probs)), ds,
                           _ptr(draft_tokens), _ptr(temperature), _ptr(coins), _ptr(final_u),
                           _ptr(out["tokens"]), _ptr(out["num_accepted"]), _ptr(out["px"]),
                           _ptr(out["qx"]), _ptr(out["S"]), _ptr(out["dmargin"]),
                           _ptr(out["cmargin"]), int(nthreads))
        return out
    tk = _c(np.zeros(B, np.int32) if top_k is None else top_k, np.int32).reshape(B)
    tp = _c(np.ones(B, np.float32) if top_p is None else top_p, np.float32).reshape(B)
    out["fmargin"] = np.empty(B, np.float64)
    lib().oracle_chain_filtered(B, gamma, V, _ptr(target), _dtype_code(target), ts,
                                _ptr(draft), F32 if draft_is_probs else _dtype_code(draft),
                                int(bool(draft_is_probs)), ds,
                                _ptr(draft_tokens), _ptr(temperature), _ptr(coins), _ptr(final_u),
                                _ptr(tk), _ptr(tp),
                                _ptr(out["tokens"]), _ptr(out["num_accepted"]), _ptr(out["px"]),
                                _ptr(out["qx"]), _ptr(out["S"]), _ptr(out["dmargin"]),
                                _ptr(out["cmargin"]), _ptr(out["fmargin"]), int(nthreads))
    return out


def filter_row(row: np.ndarray, T: float, top_k: int, top_p: float, V=None):
    """The oracle's top-k / top-p filtered temperature softmax of one row:
    ``(p, margin)``, or ``None`` for an invalid row or filter."""
    row = _c(row)
    V = row.shape[-1] if V is None else int(V)
    p = np.empty(V, np.float64)
    m = np.empty(1, np.float64)
    r = lib().oracle_filter_row(_ptr(row), _dtype_code(row), V, float(np.float32(T)), int(top_k), float(top_p),
                                _ptr(p), _ptr(m))
    return None if r else (p, float(m[0]))


def tree_greedy(target, tokens, parents, max_depth: int, V=None, nthreads: int = 0) -> dict:
    """Greedy tree verify.  ``target`` is ``[B, N, stride]``; ``tokens``/``parents`` ``[B, N]``."""
    target = _c(target)
    B, N, ts = target.shape
    V = ts if V is None else int(V)
    tokens = _c(tokens, np.int32).reshape(B, N)
    parents = _c(parents, np.int32).reshape(B, N)
    W = max_depth + 1
    out = dict(
        accept_index=np.empty((B, W), np.int32),
        tokens=np.empty((B, W), np.int32),
        num_accepted=np.empty(B, np.int32),
        argmax=np.empty((B, N), np.int32),
    )
    if B == 0:
        return out
    lib().oracle_tree_greedy(B, N, V, max_depth, _ptr(target), _dtype_code(target), ts,
                             _ptr(tokens), _ptr(parents), _ptr(out["accept_index"]),
                             _ptr(out["tokens"]), _ptr(out["num_accepted"]),
                             _ptr(out["argmax"]), int(nthreads))
    return out


def tree_sample(target, tokens, parents, temperature, coins, final_u, max_depth: int,
                draft_probs=None, threshold_single: float = 1.0, threshold_acc: float = 1.0,
                V=None, nthreads: int = 0, top_k=None, top_p=None) -> dict:
    """Target-only tree sampling.  ``coins`` is ``[B, N]`` (coin of the visited node),
    ``draft_probs`` ``None`` (zeros) or f32 ``[B, N, dstride]``.  With ``top_k`` /
    ``top_p`` (per sequence, ``[B]``) every node's target row is top-k / top-p
    filtered first (the result then has ``fmargin``)."""
    target = _c(target)
    B, N, ts = target.shape
    V = ts if V is None else int(V)
    tokens = _c(tokens, np.int32).reshape(B, N)
    parents = _c(parents, np.int32).reshape(B, N)
    temperature = _c(temperature, np.float32).reshape(B)
    coins = _c(coins, np.float32).reshape(B, N)
    final_u = _c(final_u, np.float32).reshape(B)
    dstride = 0
    if draft_probs is not None:
        draft_probs = _c(draft_probs, np.float32)
        dstride = draft_probs.shape[2]
    W = max_depth + 1
    out = dict(
        accept_index=np.empty((B, W), np.int32),
        tokens=np.empty((B, W), np.int32),
        num_accepted=np.empty(B, np.int32),
        pchild=np.empty((B, N), np.float64),
        S=np.empty(B, np.float64),
        dmargin=np.empty(B, np.float64),
        cmargin=np.empty(B, np.float64),
    )
    if B == 0:
        return out
    if top_k is None and top_p is None:
        lib().oracle_tree_sample(B, N, V, max_depth, _ptr(target), _dtype_code(target), ts,
                                 _ptr(tokens), _ptr(parents), _ptr(temperature), _ptr(coins),
                                 _ptr(final_u), _ptr(draft_probs), dstride,
                                 float(threshold_single), float(threshold_acc),
                                 _ptr(out["accept_index"]), _ptr(out["tokens"]),
                                 _ptr(out["num_accepted"]), _ptr(out["pchild"]), _ptr(out["S"]),
                                 _ptr(out["dmargin"]), _ptr(out["cmargin"]), int(nthreads))
        return out
    tk = _c(np.zeros(B, np.int32) if top_k is None else top_k, np.int32).reshape(B)
    tp = _c(np.ones(B, np.float32) if top_p is None else top_p, np.float32).reshape(B)
    out["fmargin"] = np.empty(B, np.float64)
    lib().oracle_tree_sample_filtered(B, N, V, max_depth, _ptr(target), _dtype_code(target), ts,
                                      _ptr(tokens), _ptr(parents), _ptr(temperature), _ptr(coins),
                                      _ptr(final_u), _ptr(draft_probs), dstride,
                                      float(threshold_single), float(threshold_acc), _ptr(tk), _ptr(tp),
                                      _ptr(out["accept_index"]), _ptr(out["tokens"]),
                                      _ptr(out["num_accepted"]), _ptr(out["pchild"]), _ptr(out["S"]),
                                      _ptr(out["dmargin"]), _ptr(out["cmargin"]), _ptr(out["fmargin"]),
                                      int(nthreads))
    return out


def tree_mss(target, tokens, parents, temperature, coins, final_u, max_depth: int, draft_probs,
             V=None, nthreads: int = 0) -> dict:
    """Tree verification with a draft distribution (SpecInfer multi-step speculative
    sampling).  ``coins`` is ``[B, N]`` (coin of the tested child), ``draft_probs``
    f32 ``[B, N, dstride]`` (row n = the distribution n's children were drawn from)."""
    target = _c(target)
    B, N, ts = target.shape
    V = ts if V is None else int(V)
    tokens = _c(tokens, np.int32).reshape(B, N)
    parents = _c(parents, np.int32).reshape(B, N)
    temperature = _c(temperature, np.float32).reshape(B)
    coins = _c(coins, np.float32).reshape(B, N)
    final_u = _c(final_u, np.float32).reshape(B)
    draft_probs = _c(draft_probs, np.float32)
    W = max_depth + 1
    out = dict(
        accept_index=np.empty((B, W), np.int32),
        tokens=np.empty((B, W), np.int32),
        num_accepted=np.empty(B, np.int32),
        ptest=np.empty((B, N), np.float64),
        S=np.empty(B, np.float64),
        dmargin=np.empty(B, np.float64),
        cmargin=np.empty(B, np.float64),
    )
    if B == 0:
        return out
    lib().oracle_tree_mss(B, N, V, max_depth, _ptr(target), _dtype_code(target), ts,
                          _ptr(tokens), _ptr(parents), _ptr(temperature), _ptr(coins),
                          _ptr(final_u), _ptr(draft_probs), draft_probs.shape[2],
                          _ptr(out["accept_index"]), _ptr(out["tokens"]),
                          _ptr(out["num_accepted"]), _ptr(out["ptest"]), _ptr(out["S"]),
                          _ptr(out["dmargin"]), _ptr(out["cmargin"]), int(nthreads))
    return out


def softmax_row(row: np.ndarray, T: float, V=None) -> np.ndarray | None:
    """The oracle's temperature softmax of one row (None for an invalid row)."""
    row = _c(row)
    V = row.shape[0] if V is None else int(V)
    p = np.empty(V, np.float64)
    rc = lib().oracle_softmax_row(_ptr(row), _dtype_code(row), V, float(np.float32(T)), _ptr(p))
    return None if rc else p


def inverse_cdf(w: np.ndarray, u: float):
    """The oracle's inverse-CDF draw: (index, S, margin)."""
    w = _c(w, np.float64)
    S = ctypes.c_double()
    m = ctypes.c_double()
    j = lib().oracle_inverse_cdf(_ptr(w), w.shape[0], float(u), ctypes.byref(S), ctypes.byref(m))
    return j, S.value, m.value
