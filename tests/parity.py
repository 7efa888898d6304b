"""Parity helpers: run the CUDA path and the fp64 oracle on the same bytes and
compare them element by element.

Comparison rule (the verify step's stated tolerance): accepted lengths and
emitted token ids must be identical, except on sequences the oracle marks as
near-ties -- a decision with |coin - ratio| < 1e-6 (or |coin - prob_acc/theta|,
|p - theta_single| < 1e-6), an inverse-CDF draw whose uniform lies within 1e-6
(relative to the mass) of a cell boundary, or a residual mass below 1e-6.
Flagged sequences are counted and reported, never dropped silently.
Intermediate probabilities (the diagnostics) must match within 1e-5 relative.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TIE_TOL = 1e-6
RTOL = 1e-5
ATOL = 1e-30


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


# ----------------------------------------------------------------------------- chain

def _sel(inp_tensor, rows):
    if rows is None:
        return slice(None)
    return torch.as_tensor(np.asarray(rows), device=inp_tensor.device, dtype=torch.long)


def _rows_np(rows):
    return slice(None) if rows is None else np.asarray(rows)


def oracle_chain(inp, rows=None, nthreads=0):
    sel = _sel(inp.target, rows)
    return oracle.chain(to_np(inp.target[sel]), to_np(inp.draft[sel]), inp.draft_is_probs,
                        to_np(inp.draft_tokens[sel]), to_np(inp.temperature[sel]),
                        to_np(inp.coins[sel]), to_np(inp.final_u[sel]), V=inp.V, nthreads=nthreads)


def _fn(name, lazy):
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    return getattr(sv, name + ("_lazy" if lazy else ""))


def gpu_chain(inp, workspace=None, lazy=False):
    B, g = inp.B, inp.gamma
    diag = torch.full((B, 2 * g + 1), float("nan"), device=inp.target.device)
    toks, na = _fn("spec_verify_chain", lazy)(
        inp.target, inp.draft, inp.draft_tokens, inp.temperature, inp.coins, inp.final_u,
        draft_is_probs=inp.draft_is_probs, V=inp.V, diag=diag, workspace=workspace)
    torch.cuda.synchronize()
    d = diag.cpu().numpy().astype(np.float64)
    return dict(tokens=toks.cpu().numpy(), num_accepted=na.cpu().numpy(),
                px=d[:, :g], qx=d[:, g:2 * g], S=d[:, 2 * g])


def oracle_chain_filtered(inp, top_k, top_p, rows=None, nthreads=0):
    sel = _sel(inp.target, rows)
    tk = None if top_k is None else to_np(top_k[sel])
    tp = None if top_p is None else to_np(top_p[sel])
    if tk is None:
        tk = np.zeros(len(to_np(inp.temperature[sel])), np.int32)
    return oracle.chain(to_np(inp.target[sel]), to_np(inp.draft[sel]), inp.draft_is_probs,
                        to_np(inp.draft_tokens[sel]), to_np(inp.temperature[sel]),
                        to_np(inp.coins[sel]), to_np(inp.final_u[sel]), V=inp.V, nthreads=nthreads,
                        top_k=tk, top_p=tp)


def gpu_chain_filtered(inp, top_k, top_p, workspace=None, with_diag=True, lazy=False):
    B, g = inp.B, inp.gamma
    diag = torch.full((B, 2 * g + 1), float("nan"), device=inp.target.device) if with_diag else None
    toks, na = _fn("spec_verify_chain_filtered", lazy)(inp.target, inp.draft, inp.draft_tokens, inp.temperature,
                                                       inp.coins, inp.final_u, top_k, top_p,
                                                       draft_is_probs=inp.draft_is_probs, V=inp.V, diag=diag,
                                                       workspace=workspace)
    torch.cuda.synchronize()
    d = diag.cpu().numpy().astype(np.float64) if with_diag else np.full((B, 2 * g + 1), np.nan)
    return dict(tokens=toks.cpu().numpy(), num_accepted=na.cpu().numpy(),
                px=d[:, :g], qx=d[:, g:2 * g], S=d[:, 2 * g])


def chain_flags(o, gamma):
    k = o["num_accepted"]
    f = (o["dmargin"] < TIE_TOL) | (o["cmargin"] < TIE_TOL) | ((k >= 0) & (k < gamma) & (o["S"] < TIE_TOL))
    if "fmargin" in o:                         # a top-p set decided within the tolerance
        f |= o["fmargin"] < TIE_TOL
    return f


def compare_chain(g, o, gamma, rows=None):
    """Returns (n_flagged, n_mismatch_unflagged, details)."""
    rows = _rows_np(rows)
    gk = g["num_accepted"][rows]
    gt = g["tokens"][rows]
    flags = chain_flags(o, gamma)
    same = (gk == o["num_accepted"]) & (gt == o["tokens"]).all(axis=1)
    bad = ~same & ~flags
    det = dict(bad_rows=np.nonzero(bad)[0][:10].tolist())
    # diagnostics on valid sequences
    valid = o["num_accepted"] >= 0
    gpx, gqx, gS = g["px"][rows], g["qx"][rows], g["S"][rows]
    if valid.any():
        np.testing.assert_allclose(gpx[valid], o["px"][valid], rtol=RTOL, atol=ATOL)
        np.testing.assert_allclose(gqx[valid], o["qx"][valid], rtol=RTOL, atol=ATOL)
        ok_s = valid & same & ~flags
        np.testing.assert_allclose(gS[ok_s], o["S"][ok_s], rtol=RTOL, atol=1e-12)
    inval = ~valid
    assert (gk[inval] == -1).all() and (gt[inval] == -1).all(), "invalid sequences must be all -1"
    return int(flags.sum()), int(bad.sum()), det


# ----------------------------------------------------------------------------- trees

def oracle_greedy(inp, rows=None, nthreads=0):
    sel = _sel(inp.target, rows)
    return oracle.tree_greedy(to_np(inp.target[sel]), to_np(inp.tokens[sel]), to_np(inp.parents[sel]),
                              inp.max_depth, V=inp.V, nthreads=nthreads)


def gpu_greedy(inp, workspace=None, lazy=False):
    ai, ot, na = _fn("spec_verify_tree_greedy", lazy)(inp.target, inp.tokens, inp.parents, inp.max_depth,
                                                      V=inp.V, workspace=workspace)
    torch.cuda.synchronize()
    return dict(accept_index=ai.cpu().numpy(), tokens=ot.cpu().numpy(), num_accepted=na.cpu().numpy())


def oracle_sample(inp, rows=None, nthreads=0, threshold_single=1.0, threshold_acc=1.0, top_k=None, top_p=None):
    sel = _sel(inp.target, rows)
    dp = None if inp.draft_probs is None else to_np(inp.draft_probs[sel])
    tk = None if top_k is None else to_np(top_k[sel])
    tp = None if top_p is None else to_np(top_p[sel])
    return oracle.tree_sample(to_np(inp.target[sel]), to_np(inp.tokens[sel]), to_np(inp.parents[sel]),
                              to_np(inp.temperature[sel]), to_np(inp.coins[sel]), to_np(inp.final_u[sel]),
                              inp.max_depth, draft_probs=dp, threshold_single=threshold_single,
                              threshold_acc=threshold_acc, V=inp.V, nthreads=nthreads, top_k=tk, top_p=tp)


def gpu_sample(inp, workspace=None, threshold_single=1.0, threshold_acc=1.0, lazy=False, top_k=None, top_p=None,
               with_diag=True):
    B, N = inp.B, inp.N
    diag = torch.full((B, N + 1), float("nan"), device=inp.target.device) if with_diag else None
    if top_k is not None or top_p is not None:
        ai, ot, na = _fn("spec_verify_tree_sample_filtered", lazy)(
            inp.target, inp.tokens, inp.parents, inp.temperature, inp.coins, inp.final_u, inp.max_depth,
            top_k, top_p, draft_probs=inp.draft_probs, threshold_single=threshold_single,
            threshold_acc=threshold_acc, V=inp.V, diag=diag, workspace=workspace)
    else:
        ai, ot, na = _fn("spec_verify_tree_sample", lazy)(
            inp.target, inp.tokens, inp.parents, inp.temperature, inp.coins, inp.final_u, inp.max_depth,
            draft_probs=inp.draft_probs, threshold_single=threshold_single, threshold_acc=threshold_acc,
            V=inp.V, diag=diag, workspace=workspace)
    torch.cuda.synchronize()
    d = diag.cpu().numpy().astype(np.float64) if with_diag else np.full((B, N + 1), np.nan)
    return dict(accept_index=ai.cpu().numpy(), tokens=ot.cpu().numpy(), num_accepted=na.cpu().numpy(),
                pchild=d[:, :N], S=d[:, N])


def compare_tree(g, o, rows=None, sample=False):
    sel = _rows_np(rows)
    gk, gt, ga = g["num_accepted"][sel], g["tokens"][sel], g["accept_index"][sel]
    if sample:
        flags = (o["dmargin"] < TIE_TOL) | (o["cmargin"] < TIE_TOL)
        if "fmargin" in o:                     # a top-p set decided within the tolerance
            flags |= o["fmargin"] < TIE_TOL
    else:
        flags = np.zeros(len(gk), bool)
    same = (gk == o["num_accepted"]) & (gt == o["tokens"]).all(axis=1) & (ga == o["accept_index"]).all(axis=1)
    bad = ~same & ~flags
    valid = o["num_accepted"] >= 0
    if sample and valid.any():
        gp = g["pchild"][sel]
        np.testing.assert_allclose(gp[valid], o["pchild"][valid], rtol=RTOL, atol=ATOL)
        ok_s = valid & same & ~flags
        np.testing.assert_allclose(g["S"][sel][ok_s], o["S"][ok_s], rtol=RTOL, atol=1e-12)
    inval = ~valid
    assert (gk[inval] == -1).all() and (gt[inval] == -1).all()
    return int(flags.sum()), int(bad.sum()), dict(bad_rows=np.nonzero(bad)[0][:10].tolist())


# ----------------------------------------------------------------------------- trees with a draft distribution

def oracle_mss(inp, rows=None, nthreads=0):
    sel = _sel(inp.target, rows)
    return oracle.tree_mss(to_np(inp.target[sel]), to_np(inp.tokens[sel]), to_np(inp.parents[sel]),
                           to_np(inp.temperature[sel]), to_np(inp.coins[sel]), to_np(inp.final_u[sel]),
                           inp.max_depth, to_np(inp.draft_probs[sel]), V=inp.V, nthreads=nthreads)


def gpu_mss(inp, workspace=None, lazy=False):
    B, N = inp.B, inp.N
    diag = torch.full((B, N + 1), -7.0, device=inp.target.device)
    ai, ot, na = _fn("spec_verify_tree_mss", lazy)(inp.target, inp.tokens, inp.parents, inp.temperature, inp.coins,
                                         inp.final_u, inp.max_depth, inp.draft_probs, V=inp.V, diag=diag,
                                         workspace=workspace)
    torch.cuda.synchronize()
    d = diag.cpu().numpy().astype(np.float64)
    return dict(accept_index=ai.cpu().numpy(), tokens=ot.cpu().numpy(), num_accepted=na.cpu().numpy(),
                ptest=d[:, :N], S=d[:, N])


def compare_mss(g, o, rows=None):
    """Walk outputs bit-exact except on oracle-flagged near-ties; p(x) at every test
    within RTOL (and NaN exactly where the oracle tested nothing); the final
    residual mass within RTOL on matching, unflagged sequences."""
    sel = _rows_np(rows)
    gk, gt, ga = g["num_accepted"][sel], g["tokens"][sel], g["accept_index"][sel]
    flags = (o["dmargin"] < TIE_TOL) | (o["cmargin"] < TIE_TOL)
    same = (gk == o["num_accepted"]) & (gt == o["tokens"]).all(axis=1) & (ga == o["accept_index"]).all(axis=1)
    bad = ~same & ~flags
    valid = o["num_accepted"] >= 0
    ok_rows = valid & same & ~flags
    gp = g["ptest"][sel]
    if ok_rows.any():
        tested = ~np.isnan(o["ptest"][ok_rows])
        assert (np.isnan(gp[ok_rows]) == ~tested).all(), "tested children differ"
        np.testing.assert_allclose(gp[ok_rows][tested], o["ptest"][ok_rows][tested], rtol=RTOL, atol=1e-12)
        np.testing.assert_allclose(g["S"][sel][ok_rows], o["S"][ok_rows], rtol=RTOL, atol=1e-12)
    inval = ~valid
    assert (gk[inval] == -1).all() and (gt[inval] == -1).all()
    assert np.isnan(gp[inval]).all()
    return int(flags.sum()), int(bad.sum()), dict(bad_rows=np.nonzero(bad)[0][:10].tolist())


# ----------------------------------------------------------------------------- runners with the oracle's signature

def gpu_chain_runner(target, draft, draft_is_probs, draft_tokens, temperature, coins, final_u, V=None,
                     nthreads=0, lazy=False, top_k=None, top_p=None):
    """Same call signature and result keys as ``oracle.chain`` (numpy in, numpy out),
    executed by the CUDA library.  Used to run the oracle's statistical pins
    through the GPU path."""
    spec_verify_chain = _fn("spec_verify_chain", lazy)
    dev = torch.device("cuda")

    def t(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    tg = _pad_rows(t(target))
    dr = _pad_rows(t(draft))
    B, R, S = target.shape
    V = S if V is None else V
    args = (tg, dr, t(np.asarray(draft_tokens, np.int32)), t(np.asarray(temperature, np.float32).reshape(B)),
            t(np.asarray(coins, np.float32)), t(np.asarray(final_u, np.float32).reshape(B)))
    if top_k is not None or top_p is not None:
        from speculative_decoding_verify_temperature_b200 import spec_verify as sv
        tk = None if top_k is None else t(np.asarray(top_k, np.int32).reshape(B))
        tp = None if top_p is None else t(np.asarray(top_p, np.float32).reshape(B))
        toks, na = _fn("spec_verify_chain_filtered", lazy)(*args, tk, tp, draft_is_probs=draft_is_probs, V=V)
    else:
        toks, na = spec_verify_chain(*args, draft_is_probs=draft_is_probs, V=V)
    return dict(tokens=toks.cpu().numpy(), num_accepted=na.cpu().numpy())


def gpu_tree_sample_runner(target, tokens, parents, temperature, coins, final_u, max_depth, draft_probs=None,
                           threshold_single=1.0, threshold_acc=1.0, V=None, nthreads=0, lazy=False,
                           top_k=None, top_p=None):
    spec_verify_tree_sample = _fn("spec_verify_tree_sample", lazy)
    dev = torch.device("cuda")

    def t(a):
        a = np.array(a, order="C", copy=True)          # writable, whatever view it came as
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    B, N, S = target.shape
    V = S if V is None else V
    dp = None if draft_probs is None else _pad_rows(t(draft_probs))
    args = (_pad_rows(t(target)), t(np.asarray(tokens, np.int32)), t(np.asarray(parents, np.int32)),
            t(np.asarray(temperature, np.float32).reshape(B)), t(np.asarray(coins, np.float32)),
            t(np.asarray(final_u, np.float32).reshape(B)), max_depth)
    diag = torch.full((B, N + 1), float("nan"), device=dev)
    if top_k is not None or top_p is not None:
        ai, ot, na = _fn("spec_verify_tree_sample_filtered", lazy)(
            *args, None if top_k is None else t(np.asarray(top_k, np.int32)),
            None if top_p is None else t(np.asarray(top_p, np.float32)), draft_probs=dp,
            threshold_single=threshold_single, threshold_acc=threshold_acc, V=V, diag=diag)
    else:
        ai, ot, na = spec_verify_tree_sample(*args, draft_probs=dp, threshold_single=threshold_single,
                                             threshold_acc=threshold_acc, V=V, diag=diag)
    d = diag.cpu().numpy().astype(np.float64)
    return dict(accept_index=ai.cpu().numpy(), tokens=ot.cpu().numpy(), num_accepted=na.cpu().numpy(),
                pchild=d[:, :N])


def gpu_tree_greedy_runner(target, tokens, parents, max_depth, V=None, nthreads=0, lazy=False):
    spec_verify_tree_greedy = _fn("spec_verify_tree_greedy", lazy)
    dev = torch.device("cuda")

    def t(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    B, N, S = target.shape
    V = S if V is None else V
    ai, ot, na = spec_verify_tree_greedy(_pad_rows(t(target)), t(np.asarray(tokens, np.int32)),
                                         t(np.asarray(parents, np.int32)), max_depth, V=V)
    return dict(accept_index=ai.cpu().numpy(), tokens=ot.cpu().numpy(), num_accepted=na.cpu().numpy())


def _pad_rows(x: torch.Tensor) -> torch.Tensor:
    """Copy [B, R, V] into storage whose row stride is a multiple of 16 bytes."""
    B, R, V = x.shape
    q = 16 // x.element_size()
    S = -(-V // q) * q
    if S == V and x.is_contiguous():
        return x
    out = torch.zeros((B, R, S), dtype=x.dtype, device=x.device)
    out[:, :, :V] = x
    return out


def gpu_tree_mss_runner(target, tokens, parents, temperature, coins, final_u, max_depth, draft_probs, V=None,
                        nthreads=0, lazy=False):
    """``oracle.tree_mss``'s signature, executed by the CUDA library."""
    spec_verify_tree_mss = _fn("spec_verify_tree_mss", lazy)
    dev = torch.device("cuda")

    def t(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    B, N, S = target.shape
    V = S if V is None else V
    ai, ot, na = spec_verify_tree_mss(_pad_rows(t(target)), t(np.asarray(tokens, np.int32)),
                                         t(np.asarray(parents, np.int32)),
                                         t(np.asarray(temperature, np.float32).reshape(B)),
                                         t(np.asarray(coins, np.float32)),
                                         t(np.asarray(final_u, np.float32).reshape(B)), max_depth,
                                         _pad_rows(t(np.asarray(draft_probs, np.float32))), V=V)
    return dict(accept_index=ai.cpu().numpy(), tokens=ot.cpu().numpy(), num_accepted=na.cpu().numpy())
