"""Python binding of libspecverify: the C ABI of ``include/spec_verify.h`` with the
same names, taking torch CUDA tensors.  Argument marshalling only -- every step
of the verify path runs in the library's sm_100a kernels; there is no CPU
fallback, and a missing library raises.

Tensor conventions: logits/probabilities are ``[B, R, S]`` with unit stride in
the last dim and ``stride(0) == R * stride(1)`` (rows equally spaced); the row
stride passed to the library is ``stride(1)``.  Outputs are allocated with
``torch.empty`` when not given.  All calls run on ``torch.cuda.current_stream()``
unless a stream is given.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SPEC_VERIFY_LIB selects another build of the library, e.g. the bounds-checked
# libspecverify_debug.so next to this file.
LIB_PATH = os.environ.get("SPEC_VERIFY_LIB") or os.path.join(_HERE, "libspecverify.so")

SPEC_OK, SPEC_ERR_INVALID_ARG, SPEC_ERR_UNSUPPORTED, SPEC_ERR_CUDA = 0, 1, 2, 3
SPEC_ERR_DEVICE_INPUT, SPEC_ERR_TIMEOUT, SPEC_ERR_WORKSPACE, SPEC_ERR_COPY_IN_FLIGHT = 4, 5, 6, 7
SPEC_F32, SPEC_BF16 = 0, 1
SPEC_ENTRY_CHAIN, SPEC_ENTRY_TREE_GREEDY, SPEC_ENTRY_TREE_SAMPLE, SPEC_ENTRY_TREE_MSS = 0, 1, 2, 3

_lib = None


class SpecError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = lib().spec_last_error_detail().decode()
        msg = lib().spec_status_string(status).decode()
        super().__init__(f"{where}: {msg} ({status}){': ' + detail if detail else ''}")


def lib():
    """Load libspecverify.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m speculative_decoding_verify_temperature_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        for sfx in ("", "_lazy"):
            f = getattr(L, "spec_verify_chain" + sfx)
            f.restype = i32
            f.argtypes = [i32, i32, i32, P, i32, i64, P, i32, i32, i64, P, P, P, P, P, P, P, P, sz, P]
            f = getattr(L, "spec_verify_tree_greedy" + sfx)
            f.restype = i32
            f.argtypes = [i32, i32, i32, i32, P, i32, i64, P, P, P, P, P, P, sz, P]
            f = getattr(L, "spec_verify_tree_sample" + sfx)
            f.restype = i32
            f.argtypes = [i32, i32, i32, i32, P, i32, i64, P, P, P, P, P, P, i64,
                          f32, f32, P, P, P, P, P, sz, P]
        for name in ("spec_verify_tree_mss", "spec_verify_tree_mss_lazy"):
            f = getattr(L, name)
            f.restype = i32
            f.argtypes = [i32, i32, i32, i32, P, i32, i64, P, P, P, P, P, P, i64, P, P, P, P, P, sz, P]
        for name in ("spec_verify_tree_sample_filtered", "spec_verify_tree_sample_filtered_lazy"):
            f = getattr(L, name)
            f.restype = i32
            f.argtypes = [i32, i32, i32, i32, P, i32, i64, P, P, P, P, P, P, i64,
                          f32, f32, P, P, P, P, P, P, P, sz, P]
        for name in ("spec_verify_chain_filtered", "spec_verify_chain_filtered_lazy"):
            f = getattr(L, name)
            f.restype = i32
            f.argtypes = [i32, i32, i32, P, i32, i64, P, i32, i32, i64, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.spec_vp_record_bytes.restype = sz
        L.spec_vp_record_bytes.argtypes = []
        L.spec_vp_chain_stats.restype = i32
        L.spec_vp_chain_stats.argtypes = [i32, i32, i32, i32, P, i32, i64, P, i32, i32, i64, P, P, P, P, sz, P]
        L.spec_vp_chain_decide.restype = i32
        L.spec_vp_chain_decide.argtypes = [i32, i32, i32, i32, i32, P, i32, P, P, P, P, P, P, P, sz, P]
        L.spec_vp_chain_residual.restype = i32
        L.spec_vp_chain_residual.argtypes = [i32, i32, i32, i32, i32, P, i32, i64, P, i32, i32, i64, P, P, P, sz, P]
        L.spec_vp_chain_sample.restype = i32
        L.spec_vp_chain_sample.argtypes = [i32, i32, i32, i32, i32, i32, P, i32, i64, P, i32, i32, i64,
                                           P, P, P, P, P, P, sz, P]
        L.spec_vp_chain_finish.restype = i32
        L.spec_vp_chain_finish.argtypes = [i32, i32, i32, P, P, P, sz, P]
        L.spec_workspace_bytes.restype = sz
        L.spec_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.spec_workspace_init.restype = i32
        L.spec_workspace_init.argtypes = [P, sz, P]
        L.spec_read_device_status.restype = i32
        L.spec_read_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int), P]
        L.spec_status_string.restype = ctypes.c_char_p
        L.spec_status_string.argtypes = [i32]
        L.spec_last_error_detail.restype = ctypes.c_char_p
        L.spec_last_error_detail.argtypes = []
        L.spec_profile_events.restype = i32
        L.spec_profile_events.argtypes = [P, P]
        L.spec_debug_wait_budget.restype = i32
        L.spec_debug_wait_budget.argtypes = [ctypes.c_longlong]
        L.spec_launch_count.restype = ctypes.c_ulonglong
        L.spec_launch_count.argtypes = []
        L.spec_debug_bounds_hits.restype = i32
        L.spec_debug_bounds_hits.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)]
        L.spec_debug_filter_path.restype = i32
        L.spec_debug_filter_path.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_ulonglong)]
        _lib = L
    return _lib


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SPEC_BF16
    if t.dtype == torch.float32:
        return SPEC_F32
    raise TypeError(f"logits must be bf16 or f32, got {t.dtype}")


def _rows(t: torch.Tensor, name: str) -> int:
    """Row stride (elements) of a [B, R, S] tensor whose rows are equally spaced.
    Strides of size-1 dims carry no information and are ignored."""
    if t.dim() != 3 or (t.shape[2] > 1 and t.stride(2) != 1):
        raise ValueError(f"{name} must be [B, R, S] with unit stride in the last dim")
    B, R, S = t.shape
    if R > 1:
        rs = t.stride(1)
    elif B > 1:
        rs = t.stride(0)
    else:
        q = 16 // t.element_size()
        rs = -(-S // q) * q
    if B > 1 and R > 1 and t.stride(0) != R * rs:
        raise ValueError(f"{name}: rows must be equally spaced (stride(0) == R * stride(1))")
    return rs


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != SPEC_OK:
        raise SpecError(status, where)


def spec_workspace_bytes(entry: int, B: int, rows: int, V: int) -> int:
    return int(lib().spec_workspace_bytes(entry, B, rows, V))


def spec_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(lib().spec_workspace_init(_p(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)), "spec_workspace_init")


def spec_read_device_status(workspace: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int(0)
    _check(lib().spec_read_device_status(_p(workspace), ctypes.byref(v), _stream(stream)),
           "spec_read_device_status")
    return v.value


def spec_profile_events(start=None, stop=None) -> None:
    """Record ``start``/``stop`` (torch.cuda.Event) around the row kernel of later
    calls on this thread; ``spec_profile_events()`` switches it off."""
    for ev in (start, stop):
        if ev is not None and not ev.cuda_event:
            ev.record()                        # torch creates the CUDA event on first record
    a = None if start is None else ctypes.c_void_p(start.cuda_event)
    b = None if stop is None else ctypes.c_void_p(stop.cuda_event)
    _check(lib().spec_profile_events(a, b), "spec_profile_events")


def spec_launch_count() -> int:
    """Kernels launched (or captured) by the library from this host thread so far."""
    return int(lib().spec_launch_count())


def spec_debug_bounds_hits() -> int | None:
    """Failed device-side bounds checks since the last call (synchronises the
    device), or None when the loaded library was built without them."""
    v = ctypes.c_ulonglong(0)
    st = lib().spec_debug_bounds_hits(ctypes.byref(v))
    if st == SPEC_ERR_UNSUPPORTED:
        return None
    _check(st, "spec_debug_bounds_hits")
    return int(v.value)


def spec_debug_wait_budget(tries: int = -1) -> None:
    """Testing hook: polls of the first wait for each bulk copy the finalize
    kernels issue, for later calls on this thread (0 = give up at once and take
    the timeout path; negative = the default budget)."""
    _check(lib().spec_debug_wait_budget(int(tries)), "spec_debug_wait_budget")


def spec_debug_filter_path(mode: int = -1, read: bool = False) -> tuple[int, int, int] | None:
    """Testing hook for the bf16 top-k / top-p filters, for later calls on this
    thread: mode 0 = candidates first (the default) and count rows by path,
    1 = whole-row paths only and count, -1 = the default without counting.
    With read=True, returns (rows the candidates resolved at the first cut,
    rows left to a whole-row path, rows resolved at the deeper cut) since the
    last read on the current device and resets them (synchronises the
    device)."""
    if not read:
        _check(lib().spec_debug_filter_path(int(mode), None), "spec_debug_filter_path")
        return None
    v = (ctypes.c_ulonglong * 3)()
    _check(lib().spec_debug_filter_path(int(mode), v), "spec_debug_filter_path")
    return int(v[0]), int(v[1]), int(v[2])


class Workspace:
    """Caller-owned scratch for one entry point and shape, zero-filled on creation
    (and re-created whenever the shape changes)."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.key = None
        self.buf = None

    def get(self, entry: int, B: int, rows: int, V: int, stream=None) -> torch.Tensor:
        key = (entry, B, rows, V)
        if key != self.key:
            n = spec_workspace_bytes(entry, B, rows, V)
            if n == 0:
                raise ValueError(f"no workspace size for {key}")
            self.buf = torch.empty(n, dtype=torch.uint8, device=self.device)
            spec_workspace_init(self.buf, stream)
            self.key = key
        return self.buf


_default_ws = {}


def _ws(workspace, entry, B, rows, V, device, stream):
    if workspace is not None:
        return workspace
    w = _default_ws.setdefault((device, entry), Workspace(device))
    return w.get(entry, B, rows, V, stream)


def spec_verify_chain(target, draft, draft_tokens, temperature, coins, final_u, *,
                      draft_is_probs: bool = False, V: int | None = None, out_tokens=None,
                      out_num_accepted=None, diag=None, workspace=None, stream=None,
                      _name: str = "spec_verify_chain"):
    """Chain verify of one round.  Returns ``(out_tokens [B, gamma+1], out_num_accepted [B])``."""
    B, R, S = target.shape
    gamma = R - 1
    V = S if V is None else int(V)
    dev = target.device
    if out_tokens is None:
        out_tokens = torch.empty((B, gamma + 1), dtype=torch.int32, device=dev)
    if out_num_accepted is None:
        out_num_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
    ws = _ws(workspace, SPEC_ENTRY_CHAIN, B, gamma, V, dev, stream)
    st = getattr(lib(), _name)(
        B, gamma, V, _p(target), _dtype(target), _rows(target, "target"),
        _p(draft), SPEC_F32 if draft_is_probs else _dtype(draft), int(bool(draft_is_probs)),
        _rows(draft, "draft"), _p(draft_tokens), _p(temperature), _p(coins), _p(final_u),
        _p(out_tokens), _p(out_num_accepted), _p(diag), _p(ws), ws.numel(), _stream(stream))
    _check(st, _name)
    return out_tokens, out_num_accepted


def spec_verify_tree_greedy(target, tokens, parents, max_depth: int, *, V: int | None = None,
                            out_accept_index=None, out_tokens=None, out_num_accepted=None,
                            workspace=None, stream=None, _name: str = "spec_verify_tree_greedy"):
    """Greedy tree verify.  Returns ``(accept_index, tokens, num_accepted)``."""
    B, N, S = target.shape
    V = S if V is None else int(V)
    dev = target.device
    W = max_depth + 1
    if out_accept_index is None:
        out_accept_index = torch.empty((B, W), dtype=torch.int32, device=dev)
    if out_tokens is None:
        out_tokens = torch.empty((B, W), dtype=torch.int32, device=dev)
    if out_num_accepted is None:
        out_num_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
    ws = _ws(workspace, SPEC_ENTRY_TREE_GREEDY, B, N, V, dev, stream)
    st = getattr(lib(), _name)(
        B, N, V, max_depth, _p(target), _dtype(target), _rows(target, "target"), _p(tokens),
        _p(parents), _p(out_accept_index), _p(out_tokens), _p(out_num_accepted), _p(ws), ws.numel(),
        _stream(stream))
    _check(st, _name)
    return out_accept_index, out_tokens, out_num_accepted


def spec_verify_tree_sample(target, tokens, parents, temperature, coins, final_u, max_depth: int, *,
                            draft_probs=None, threshold_single: float = 1.0,
                            threshold_acc: float = 1.0, V: int | None = None,
                            out_accept_index=None, out_tokens=None, out_num_accepted=None,
                            diag=None, workspace=None, stream=None, _name: str = "spec_verify_tree_sample"):
    """Target-only tree sampling.  Returns ``(accept_index, tokens, num_accepted)``."""
    B, N, S = target.shape
    V = S if V is None else int(V)
    dev = target.device
    W = max_depth + 1
    if out_accept_index is None:
        out_accept_index = torch.empty((B, W), dtype=torch.int32, device=dev)
    if out_tokens is None:
        out_tokens = torch.empty((B, W), dtype=torch.int32, device=dev)
    if out_num_accepted is None:
        out_num_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
    ws = _ws(workspace, SPEC_ENTRY_TREE_SAMPLE, B, N, V, dev, stream)
    dstride = _rows(draft_probs, "draft_probs") if draft_probs is not None else 0
    st = getattr(lib(), _name)(
        B, N, V, max_depth, _p(target), _dtype(target), _rows(target, "target"), _p(tokens),
        _p(parents), _p(temperature), _p(coins), _p(final_u), _p(draft_probs), dstride,
        float(threshold_single), float(threshold_acc), _p(out_accept_index), _p(out_tokens),
        _p(out_num_accepted), _p(diag), _p(ws), ws.numel(), _stream(stream))
    _check(st, _name)
    return out_accept_index, out_tokens, out_num_accepted


def spec_verify_tree_sample_filtered(target, tokens, parents, temperature, coins, final_u, max_depth: int,
                                     top_k=None, top_p=None, *, draft_probs=None, threshold_single: float = 1.0,
                                     threshold_acc: float = 1.0, V: int | None = None, out_accept_index=None,
                                     out_tokens=None, out_num_accepted=None, diag=None, workspace=None,
                                     stream=None, _name: str = "spec_verify_tree_sample_filtered"):
    """Target-only tree sampling on top-k / top-p filtered node rows; ``top_k`` int32
    ``[B]`` (0 = off) and ``top_p`` f32 ``[B]`` (1 = off), either may be None (not
    both).  Returns ``(accept_index, tokens, num_accepted)``."""
    if top_k is None and top_p is None:
        raise ValueError("give top_k, top_p or both")
    if top_k is not None and top_k.dtype != torch.int32:
        raise TypeError("top_k must be int32")
    if top_p is not None and top_p.dtype != torch.float32:
        raise TypeError("top_p must be float32")
    B, N, S = target.shape
    V = S if V is None else int(V)
    dev = target.device
    W = max_depth + 1
    if out_accept_index is None:
        out_accept_index = torch.empty((B, W), dtype=torch.int32, device=dev)
    if out_tokens is None:
        out_tokens = torch.empty((B, W), dtype=torch.int32, device=dev)
    if out_num_accepted is None:
        out_num_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
    ws = _ws(workspace, SPEC_ENTRY_TREE_SAMPLE, B, N, V, dev, stream)
    dstride = _rows(draft_probs, "draft_probs") if draft_probs is not None else 0
    st = getattr(lib(), _name)(
        B, N, V, max_depth, _p(target), _dtype(target), _rows(target, "target"), _p(tokens),
        _p(parents), _p(temperature), _p(coins), _p(final_u), _p(draft_probs), dstride,
        float(threshold_single), float(threshold_acc), _p(top_k), _p(top_p), _p(out_accept_index),
        _p(out_tokens), _p(out_num_accepted), _p(diag), _p(ws), ws.numel(), _stream(stream))
    _check(st, _name)
    return out_accept_index, out_tokens, out_num_accepted


def spec_verify_tree_sample_filtered_lazy(*args, **kw):
    """Row-on-demand filtered tree sampling: the arguments and results of
    ``spec_verify_tree_sample_filtered``, filtering only the rows the walk reaches;
    ``diag`` holds NaN for children of unvisited nodes."""
    return spec_verify_tree_sample_filtered(*args, _name="spec_verify_tree_sample_filtered_lazy", **kw)


def spec_verify_chain_lazy(*args, **kw):
    """Row-on-demand chain verify: the arguments and results of ``spec_verify_chain``
    (bit-identical for valid inputs); ``diag`` entries of positions after the first
    rejection are NaN."""
    return spec_verify_chain(*args, _name="spec_verify_chain_lazy", **kw)


def spec_verify_tree_greedy_lazy(*args, **kw):
    """Row-on-demand greedy tree verify: the arguments and results of
    ``spec_verify_tree_greedy``."""
    return spec_verify_tree_greedy(*args, _name="spec_verify_tree_greedy_lazy", **kw)


def spec_verify_tree_sample_lazy(*args, **kw):
    """Row-on-demand target-only tree sampling: the arguments and results of
    ``spec_verify_tree_sample``; ``diag`` holds NaN for children of unvisited nodes."""
    return spec_verify_tree_sample(*args, _name="spec_verify_tree_sample_lazy", **kw)


def spec_verify_tree_mss(target, tokens, parents, temperature, coins, final_u, max_depth: int, draft_probs, *,
                         V: int | None = None, out_accept_index=None, out_tokens=None, out_num_accepted=None,
                         diag=None, workspace=None, stream=None, _name: str = "spec_verify_tree_mss"):
    """Tree verification with a draft distribution (multi-step speculative sampling).
    ``coins`` ``[B, N]`` holds the uniform of each child's test; ``draft_probs`` f32
    ``[B, N, S]`` row n is the distribution node n's children were drawn from.
    Returns ``(accept_index, tokens, num_accepted)``."""
    B, N, S = target.shape
    V = S if V is None else int(V)
    dev = target.device
    W = max_depth + 1
    if out_accept_index is None:
        out_accept_index = torch.empty((B, W), dtype=torch.int32, device=dev)
    if out_tokens is None:
        out_tokens = torch.empty((B, W), dtype=torch.int32, device=dev)
    if out_num_accepted is None:
        out_num_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
    if draft_probs.dtype != torch.float32:
        raise TypeError("draft_probs must be float32")
    ws = _ws(workspace, SPEC_ENTRY_TREE_MSS, B, N, V, dev, stream)
    st = getattr(lib(), _name)(
        B, N, V, max_depth, _p(target), _dtype(target), _rows(target, "target"), _p(tokens), _p(parents),
        _p(temperature), _p(coins), _p(final_u), _p(draft_probs), _rows(draft_probs, "draft_probs"),
        _p(out_accept_index), _p(out_tokens), _p(out_num_accepted), _p(diag), _p(ws), ws.numel(),
        _stream(stream))
    _check(st, _name)
    return out_accept_index, out_tokens, out_num_accepted


def spec_verify_tree_mss_lazy(*args, **kw):
    """Row-on-demand multi-step speculative sampling: the arguments and results of
    ``spec_verify_tree_mss``, reading only the rows of the visited nodes."""
    return spec_verify_tree_mss(*args, _name="spec_verify_tree_mss_lazy", **kw)


def spec_verify_chain_filtered(target, draft, draft_tokens, temperature, coins, final_u, top_k=None, top_p=None, *,
                               draft_is_probs: bool = False, V: int | None = None, out_tokens=None,
                               out_num_accepted=None, diag=None, workspace=None, stream=None,
                               _name: str = "spec_verify_chain_filtered"):
    """Chain verify under top-k / top-p filtered temperature sampling; ``top_k`` int32
    ``[B]`` (0 = off) and ``top_p`` f32 ``[B]`` (1 = off), either may be None (not
    both).  Returns ``(out_tokens [B, gamma+1], out_num_accepted [B])``."""
    B, R, S = target.shape
    gamma = R - 1
    V = S if V is None else int(V)
    dev = target.device
    if top_k is None and top_p is None:
        raise ValueError("give top_k, top_p or both")
    if out_tokens is None:
        out_tokens = torch.empty((B, gamma + 1), dtype=torch.int32, device=dev)
    if out_num_accepted is None:
        out_num_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
    if top_k is not None and top_k.dtype != torch.int32:
        raise TypeError("top_k must be int32")
    if top_p is not None and top_p.dtype != torch.float32:
        raise TypeError("top_p must be float32")
    ws = _ws(workspace, SPEC_ENTRY_CHAIN, B, gamma, V, dev, stream)
    st = getattr(lib(), _name)(
        B, gamma, V, _p(target), _dtype(target), _rows(target, "target"),
        _p(draft), SPEC_F32 if draft_is_probs else _dtype(draft), int(bool(draft_is_probs)),
        _rows(draft, "draft"), _p(draft_tokens), _p(temperature), _p(coins), _p(final_u), _p(top_k), _p(top_p),
        _p(out_tokens), _p(out_num_accepted), _p(diag), _p(ws), ws.numel(), _stream(stream))
    _check(st, _name)
    return out_tokens, out_num_accepted


def spec_verify_chain_filtered_lazy(*args, **kw):
    """spec_verify_chain_filtered as a row-on-demand level walk: only the rows the
    decisions reach get statistics and filter records; same outputs for valid
    inputs (diagnostics only where evaluated)."""
    return spec_verify_chain_filtered(*args, _name="spec_verify_chain_filtered_lazy", **kw)



# ----------------------------------------------------------------------------- vocabulary-parallel chain

def spec_vp_record_bytes() -> int:
    return int(lib().spec_vp_record_bytes())


def _vp_ws(workspace, B, gamma, Vs, dev, stream):
    return _ws(workspace, SPEC_ENTRY_CHAIN, B, gamma, Vs, dev, stream)


def spec_vp_chain_stats(target, draft, draft_tokens, temperature, *, vocab_offset: int, draft_is_probs=False,
                        V_shard=None, rec_out=None, workspace=None, stream=None):
    """Step 1 on one rank: per-row shard statistics, ``uint8 [B, 2*gamma+1, record]``."""
    B, R, S = target.shape
    gamma = R - 1
    Vs = S if V_shard is None else int(V_shard)
    if rec_out is None:
        rec_out = torch.empty((B, 2 * gamma + 1, spec_vp_record_bytes()), dtype=torch.uint8, device=target.device)
    ws = _vp_ws(workspace, B, gamma, Vs, target.device, stream)
    st = lib().spec_vp_chain_stats(B, gamma, Vs, int(vocab_offset), _p(target), _dtype(target), _rows(target, "target"),
                                   _p(draft), SPEC_F32 if draft_is_probs else _dtype(draft), int(bool(draft_is_probs)),
                                   _rows(draft, "draft"), _p(draft_tokens), _p(temperature), _p(rec_out), _p(ws),
                                   ws.numel(), _stream(stream))
    _check(st, "spec_vp_chain_stats")
    return rec_out


def spec_vp_chain_decide(rec_all, draft_tokens, temperature, coins, *, V: int, V_shard: int, draft_is_probs=False,
                         out_tokens=None, out_num_accepted=None, diag=None, workspace=None, stream=None):
    """Step 2 (identical on every rank): ``(out_tokens, out_num_accepted)`` with the
    last token still -1."""
    world, B, R2, _ = rec_all.shape
    gamma = (R2 - 1) // 2
    dev = rec_all.device
    if out_tokens is None:
        out_tokens = torch.empty((B, gamma + 1), dtype=torch.int32, device=dev)
    if out_num_accepted is None:
        out_num_accepted = torch.empty((B,), dtype=torch.int32, device=dev)
    ws = _vp_ws(workspace, B, gamma, int(V_shard), dev, stream)
    st = lib().spec_vp_chain_decide(B, gamma, int(V), int(V_shard), world, _p(rec_all), int(bool(draft_is_probs)),
                                    _p(draft_tokens), _p(temperature), _p(coins), _p(out_tokens),
                                    _p(out_num_accepted), _p(diag), _p(ws), ws.numel(), _stream(stream))
    _check(st, "spec_vp_chain_decide")
    return out_tokens, out_num_accepted


def spec_vp_chain_residual(target, draft, rec_all, *, rank: int, draft_is_probs=False, V_shard=None,
                           mass_out=None, workspace=None, stream=None):
    """Step 3 on one rank: the shard's part of the last distribution's mass, f64 ``[B]``."""
    B, R, S = target.shape
    gamma = R - 1
    Vs = S if V_shard is None else int(V_shard)
    world = rec_all.shape[0]
    if mass_out is None:
        mass_out = torch.empty((B,), dtype=torch.float64, device=target.device)
    ws = _vp_ws(workspace, B, gamma, Vs, target.device, stream)
    st = lib().spec_vp_chain_residual(B, gamma, Vs, world, int(rank), _p(target), _dtype(target),
                                      _rows(target, "target"), _p(draft),
                                      SPEC_F32 if draft_is_probs else _dtype(draft), int(bool(draft_is_probs)),
                                      _rows(draft, "draft"), _p(rec_all), _p(mass_out), _p(ws), ws.numel(),
                                      _stream(stream))
    _check(st, "spec_vp_chain_residual")
    return mass_out


def spec_vp_chain_sample(target, draft, final_u, rec_all, mass_all, *, vocab_offset: int, rank: int,
                         draft_is_probs=False, V_shard=None, tok_out=None, diag=None, workspace=None, stream=None):
    """Step 4 on one rank: int32 ``[B]``, the global token id where this shard holds
    u*S, else -1."""
    B, R, S = target.shape
    gamma = R - 1
    Vs = S if V_shard is None else int(V_shard)
    world = rec_all.shape[0]
    if tok_out is None:
        tok_out = torch.empty((B,), dtype=torch.int32, device=target.device)
    ws = _vp_ws(workspace, B, gamma, Vs, target.device, stream)
    st = lib().spec_vp_chain_sample(B, gamma, Vs, int(vocab_offset), world, int(rank), _p(target), _dtype(target),
                                    _rows(target, "target"), _p(draft),
                                    SPEC_F32 if draft_is_probs else _dtype(draft), int(bool(draft_is_probs)),
                                    _rows(draft, "draft"), _p(final_u), _p(rec_all), _p(mass_all), _p(tok_out),
                                    _p(diag), _p(ws), ws.numel(), _stream(stream))
    _check(st, "spec_vp_chain_sample")
    return tok_out


def spec_vp_chain_finish(tok, out_tokens, *, V_shard: int, workspace=None, stream=None):
    """Step 5: the reduced token into position k of ``out_tokens``."""
    B, W = out_tokens.shape
    ws = _vp_ws(workspace, B, W - 1, int(V_shard), out_tokens.device, stream)
    st = lib().spec_vp_chain_finish(B, W - 1, int(V_shard), _p(tok), _p(out_tokens), _p(ws), ws.numel(),
                                    _stream(stream))
    _check(st, "spec_vp_chain_finish")
    return out_tokens


class TorchExchange:
    """The three exchanges of a vocabulary-parallel round over a torch.distributed
    process group (NCCL on GPUs)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather(self, t):
        parts = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts)

    def all_reduce_max(self, t):
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)
        return t


def spec_verify_chain_vocab_parallel(target, draft, draft_tokens, temperature, coins, final_u, *, vocab_offset: int,
                                     V: int, draft_is_probs=False, exchange=None, ops=None, out_tokens=None,
                                     out_num_accepted=None, diag=None, workspace=None, stream=None):
    """One chain round with the vocabulary sharded over the ranks of ``exchange``
    (default: the torch.distributed world).  ``target`` / ``draft`` are this
    rank's shard ``[B, R, V_shard]``; the others are replicated.  Returns
    ``(out_tokens [B, gamma+1], out_num_accepted [B])`` on every rank.  ``ops``
    replaces the five device steps (tests of the exchange logic only)."""
    ex = exchange or TorchExchange()
    o = ops or _VP_OPS
    Vs = target.shape[2]
    rec = o.stats(target, draft, draft_tokens, temperature, vocab_offset=vocab_offset, draft_is_probs=draft_is_probs,
                  V_shard=Vs, workspace=workspace, stream=stream)
    rec_all = ex.all_gather(rec)
    out_tokens, out_num_accepted = o.decide(rec_all, draft_tokens, temperature, coins, V=V, V_shard=Vs,
                                            draft_is_probs=draft_is_probs, out_tokens=out_tokens,
                                            out_num_accepted=out_num_accepted, diag=diag, workspace=workspace,
                                            stream=stream)
    mass = o.residual(target, draft, rec_all, rank=ex.rank, draft_is_probs=draft_is_probs, V_shard=Vs,
                      workspace=workspace, stream=stream)
    mass_all = ex.all_gather(mass)
    tok = o.sample(target, draft, final_u, rec_all, mass_all, vocab_offset=vocab_offset, rank=ex.rank,
                   draft_is_probs=draft_is_probs, V_shard=Vs, diag=diag, workspace=workspace, stream=stream)
    tok = ex.all_reduce_max(tok)
    o.finish(tok, out_tokens, V_shard=Vs, workspace=workspace, stream=stream)
    return out_tokens, out_num_accepted


class _VpOps:
    stats = staticmethod(spec_vp_chain_stats)
    decide = staticmethod(spec_vp_chain_decide)
    residual = staticmethod(spec_vp_chain_residual)
    sample = staticmethod(spec_vp_chain_sample)
    finish = staticmethod(spec_vp_chain_finish)


_VP_OPS = _VpOps()
