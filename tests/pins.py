"""Pins for the fp64 oracle: checks against what the pages and the mathematics
fix, independent of how the oracle computes.

* ``chain_bruteforce`` / ``tree_bruteforce`` -- exact output distribution of the
  first K generated tokens, by enumerating every draft sequence and every cell
  of the uniforms' breakpoint partition (the oracle's output is constant on
  each cell, so it is evaluated once at the cell midpoint).  The result must
  equal the target's own autoregressive distribution (lossless-ness, the
  "why lossless" argument of the spec_origins page) to 1e-12.
* ``chain_closed_form_exact`` -- with the same (p, q) at every position the
  exact E[#tokens per round] equals (1 - beta^(gamma+1)) / (1 - beta),
  beta = sum min(p, q) (spec_origins page, "closed form").
* ``chain_chisquare`` / ``tree_chisquare`` -- 10^6 simulated rounds with random
  uniforms; chi-square of the first K tokens against the exact product
  distribution.
* ``greedy_equivalence`` -- speculative greedy over random trees emits exactly
  the sequence of plain argmax decoding (Blockwise "verify" paragraph).

Each function returns a small report dict with an ``ok`` flag so that the
mutation tests can assert that a planted mistake makes it fail.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
from scipy import special, stats

import oracle


# ----------------------------------------------------------------------------- toy models

class ToyModel:
    """Prefix-dependent target p(.|h) and draft q(.|h) tables over a tiny vocab.

    Target rows are dyadic distributions (multiples of 1/64, zeros allowed),
    handed to the verify step as f32 logits T*log(p) (-inf for zeros), so that
    the temperature softmax at T gives p back.  Draft rows are either dyadic
    probabilities (``draft_kind="probs"``, exact in f32) or f32 logits d whose
    softmax(d/T) is the draft distribution (``"logits"``).  With ``iid=True``
    every prefix shares one (p, q) pair."""

    def __init__(self, V: int, seed: int, draft_kind: str = "probs", iid: bool = False,
                 denom: int = 64, T: float = 1.0, position_only: bool = False):
        self.V, self.seed, self.draft_kind, self.iid, self.denom = V, seed, draft_kind, iid, denom
        self.position_only = position_only
        self.T = float(np.float32(T))
        self._p, self._q = {}, {}

    def key(self, prefix):
        if self.iid:
            return ()
        if self.position_only:
            return (-1 - len(prefix),)
        return tuple(int(t) for t in prefix)

    def _rng(self, tag: int, prefix):
        key = self.key(prefix)
        return np.random.default_rng([self.seed, tag, len(key)] + [t + 1 + (1 << 20) for t in key])

    def _dyadic(self, rng) -> np.ndarray:
        V, D = self.V, self.denom
        c = rng.multinomial(D, rng.dirichlet(rng.uniform(0.2, 1.5, V)))
        if V > 1 and rng.random() < 0.5:               # force a zero now and then
            z = int(rng.integers(V))
            moved, c[z] = c[z], 0
            others = [j for j in range(V) if j != z]
            c[others[int(np.argmax(c[others]))]] += moved
        return c.astype(np.float64) / D

    def p(self, prefix):
        key = self.key(prefix)
        if key not in self._p:
            probs = self._dyadic(self._rng(1, prefix))
            with np.errstate(divide="ignore"):
                logits = (np.log(probs) * self.T).astype(np.float32)
            self._p[key] = (logits, probs)
        return self._p[key]

    def q(self, prefix):
        key = self.key(prefix)
        if key not in self._q:
            rng = self._rng(2, prefix)
            if self.draft_kind == "probs":
                probs = self._dyadic(rng)
                row = probs.astype(np.float32)
            else:
                row = (rng.normal(0, 1.5, self.V)).astype(np.float32)
                if rng.random() < 0.3:
                    row[rng.integers(self.V)] = -np.inf
                probs = special.softmax(row.astype(np.float64) / self.T)
            self._q[key] = (row, probs)
        return self._q[key]


def _product_distribution(model: ToyModel, K: int) -> dict:
    out = {}
    for seq in itertools.product(range(model.V), repeat=K):
        pr = 1.0
        for i in range(K):
            pr *= model.p(seq[:i])[1][seq[i]]
        out[seq] = pr
    return out


# ----------------------------------------------------------------------------- chain brute force

def _chain_cases(model: ToyModel, prefix, gamma: int):
    V = model.V
    cases = []
    for x in itertools.product(range(V), repeat=gamma):
        wq = 1.0
        for i in range(gamma):
            wq *= model.q(prefix + x[:i])[1][x[i]]
        if wq == 0.0:
            continue
        prow = [model.p(prefix + x[:i]) for i in range(gamma + 1)]
        qrow = [model.q(prefix + x[:i]) for i in range(gamma)]
        a = [min(1.0, prow[i][1][x[i]] / qrow[i][1][x[i]]) for i in range(gamma)]
        for k in range(gamma + 1):
            wk = float(np.prod(a[:k])) * ((1.0 - a[k]) if k < gamma else 1.0)
            if wk <= 0.0:
                continue
            coins = [a[i] / 2 for i in range(k)]
            if k < gamma:
                coins.append((a[k] + 1.0) / 2)
            coins += [0.5] * (gamma - len(coins))
            if k < gamma:
                r = np.maximum(0.0, prow[k][1] - qrow[k][1])
            else:
                r = prow[gamma][1].copy()
            S = r.sum()
            C = np.cumsum(r)
            for j in range(V):
                if r[j] > 0:
                    cases.append(dict(weight=wq * wk * r[j] / S,
                                      target=np.stack([pr[0] for pr in prow]),
                                      draft=np.stack([qr[0] for qr in qrow]),
                                      x=np.array(x, np.int32),
                                      coins=np.array(coins, np.float32),
                                      u=np.float32((C[j] - r[j] / 2) / S)))
    return cases


def _run_chain_cases(model: ToyModel, cases, runner=None):
    target = np.stack([c["target"] for c in cases])
    draft = np.stack([c["draft"] for c in cases])
    x = np.stack([c["x"] for c in cases])
    coins = np.stack([c["coins"] for c in cases])
    u = np.array([c["u"] for c in cases], np.float32)
    T = np.full(len(cases), model.T, np.float32)
    return (runner or oracle.chain)(target, draft, model.draft_kind == "probs", x, T, coins, u)


def chain_bruteforce(V=3, gamma=2, K=3, seed=1, draft_kind="probs", tol=1e-12, T=1.0, runner=None) -> dict:
    """Exact distribution of the first K tokens of repeated chain rounds."""
    model = ToyModel(V, seed, draft_kind, T=T)
    states = {(): 1.0}
    dist = {}
    while states:
        batch, owners = [], []
        for prefix, w in states.items():
            cs = _chain_cases(model, prefix, gamma)
            batch += cs
            owners += [(prefix, w)] * len(cs)
        res = _run_chain_cases(model, batch, runner)
        nxt = {}
        for i, (prefix, w) in enumerate(owners):
            k = int(res["num_accepted"][i])
            if k < 0:
                return dict(ok=False, err=float("inf"), reason="oracle flagged valid input")
            emitted = tuple(int(t) for t in res["tokens"][i, :k + 1])
            h = prefix + emitted
            ww = w * batch[i]["weight"]
            if len(h) >= K:
                dist[h[:K]] = dist.get(h[:K], 0.0) + ww
            else:
                nxt[h] = nxt.get(h, 0.0) + ww
        states = nxt
    want = _product_distribution(model, K)
    err = max(abs(dist.get(s, 0.0) - pv) for s, pv in want.items())
    extra = sum(v for s, v in dist.items() if s not in want)
    err = max(err, extra)
    return dict(ok=err < tol, err=err)


def chain_closed_form_exact(V=4, gamma=3, seed=2, draft_kind="probs", tol=1e-12, runner=None) -> dict:
    """Exact E[tokens per round] with one (p, q) pair at every position versus
    (1 - beta^(gamma+1)) / (1 - beta)."""
    model = ToyModel(V, seed, draft_kind, iid=True)
    cases = _chain_cases(model, (), gamma)
    res = _run_chain_cases(model, cases, runner)
    w = np.array([c["weight"] for c in cases])
    tau = res["num_accepted"].astype(np.float64) + 1.0
    e_tau = float((w * tau).sum())
    beta = float(np.minimum(model.p(())[1], model.q(())[1]).sum())
    want = (1 - beta ** (gamma + 1)) / (1 - beta) if beta < 1 else gamma + 1.0
    err = abs(e_tau - want)
    # Each emitted token of the round must also be distributed as p.
    first = np.zeros(V)
    for i, c in enumerate(cases):
        first[res["tokens"][i, 0]] += c["weight"]
    err_first = float(np.abs(first - model.p(())[1]).max())
    return dict(ok=err < tol and err_first < tol and abs(w.sum() - 1) < tol,
                err=err, e_tau=e_tau, want=want, beta=beta, err_first=err_first)


def chain_closed_form_positional(V=4, gamma=3, seed=9, draft_kind="probs", tol=1e-12) -> dict:
    """Exact E[tokens per round] when (p_i, q_i) depend on the position i only:
    E[tau] = sum_{k=0}^{gamma} prod_{i<k} beta_i, beta_i = sum min(p_i, q_i)
    (the closed form's independence assumption, position by position)."""
    model = ToyModel(V, seed, draft_kind, position_only=True)
    cases = _chain_cases(model, (), gamma)
    res = _run_chain_cases(model, cases)
    w = np.array([c["weight"] for c in cases])
    e_tau = float((w * (res["num_accepted"] + 1.0)).sum())
    betas = [float(np.minimum(model.p((0,) * i)[1], model.q((0,) * i)[1]).sum()) for i in range(gamma)]
    want = sum(float(np.prod(betas[:k])) for k in range(gamma + 1))
    return dict(ok=abs(e_tau - want) < tol, e_tau=e_tau, want=want, betas=betas)


# ----------------------------------------------------------------------------- chain simulation

class _Tables:
    """All prefixes up to length L of a ToyModel, addressed by integer ids
    (id(h + t) = id(h) * (V + 1) + t + 1)."""

    def __init__(self, model: ToyModel, L: int):
        V = model.V
        self.V = V
        size = (V + 1) ** (L + 1)
        self.P = np.zeros((size, V))
        self.PL = np.zeros((size, V), np.float32)
        self.Q = np.zeros((size, V))
        self.QR = np.zeros((size, V), np.float32)
        for n in range(L + 1):
            for h in itertools.product(range(V), repeat=n):
                i = self.id(h)
                self.PL[i], self.P[i] = model.p(h)
                self.QR[i], self.Q[i] = model.q(h)

    def id(self, h):
        i = 0
        for t in h:
            i = i * (self.V + 1) + t + 1
        return i

    def child(self, ids, t):
        return ids * (self.V + 1) + t + 1


def _sample_rows(probs: np.ndarray, rng) -> np.ndarray:
    c = np.cumsum(probs, axis=1)
    u = rng.random(probs.shape[0]) * c[:, -1]
    return np.minimum((c <= u[:, None]).sum(axis=1), probs.shape[1] - 1)


def _uniform24(rng, shape):
    """Uniforms k * 2^-24, k in [1, 2^24): exact in f32, and never 0 -- with u = 0
    the rule u <= p(x)/q(x) would accept a token whose target probability is 0
    (an event of probability 0 for a continuous uniform, 2^-24 on this grid)."""
    return (rng.integers(1, 1 << 24, size=shape) * 2.0 ** -24).astype(np.float32)


def chain_chisquare(V=4, gamma=3, K=3, rounds=1_000_000, seed=3, draft_kind="probs",
                    pmin=1e-3, T=1.0, runner=None) -> dict:
    model = ToyModel(V, seed, draft_kind, T=T)
    tab = _Tables(model, K - 1 + gamma)
    rng = np.random.default_rng(seed + 100)
    n = rounds
    ids = np.zeros(n, np.int64)
    ntok = np.zeros(n, np.int64)
    first = np.zeros((n, K), np.int64)
    active = np.arange(n)
    tau_sum, tau_n = 0.0, 0
    while active.size:
        m = active.size
        h = ids[active]
        x = np.zeros((m, gamma), np.int32)
        rows_t = np.zeros((m, gamma + 1), np.int64)
        rows_q = np.zeros((m, gamma), np.int64)
        cur = h.copy()
        for i in range(gamma):
            rows_t[:, i] = cur
            rows_q[:, i] = cur
            x[:, i] = _sample_rows(tab.Q[cur], rng)
            cur = tab.child(cur, x[:, i])
        rows_t[:, gamma] = cur
        res = (runner or oracle.chain)(tab.PL[rows_t], tab.QR[rows_q], draft_kind == "probs", x,
                           np.full(m, model.T, np.float32), _uniform24(rng, (m, gamma)),
                           _uniform24(rng, m))
        k = res["num_accepted"]
        if (k < 0).any():
            return dict(ok=False, p=0.0, reason="invalid")
        tau_sum += float((k + 1).sum())
        tau_n += m
        for j in range(gamma + 1):
            sel = (k >= j)
            idx = active[sel]
            tok = res["tokens"][sel, j]
            put = ntok[idx] < K
            first[idx[put], ntok[idx[put]]] = tok[put]
            ntok[idx[put]] += 1
            ids[idx] = tab.child(ids[idx], tok)
        active = active[ntok[active] < K]
    return _chisq(first, tab, V, K, pmin) | dict(mean_tau=tau_sum / tau_n)


def _chisq(first, tab, V, K, pmin):
    code = np.zeros(first.shape[0], np.int64)
    for i in range(K):
        code = code * V + first[:, i]
    obs = np.bincount(code, minlength=V ** K).astype(np.float64)
    exp = np.zeros(V ** K)
    for c, seq in enumerate(itertools.product(range(V), repeat=K)):
        pr = 1.0
        for i in range(K):
            pr *= tab.P[tab.id(seq[:i])][seq[i]]
        exp[c] = pr
    exp *= first.shape[0]
    impossible = obs[exp == 0].sum()
    keep = exp >= 5
    o, e = list(obs[keep]), list(exp[keep])
    if (~keep).any() and exp[~keep].sum() > 0:
        o.append(obs[~keep].sum())
        e.append(exp[~keep].sum())
    o, e = np.array(o), np.array(e)
    e *= o.sum() / e.sum()
    chi2, p = stats.chisquare(o, e)
    return dict(ok=bool(p > pmin and impossible == 0), p=float(p), chi2=float(chi2),
                impossible=float(impossible))


def chain_closed_form_mc(V=4, gamma=3, rounds=1_000_000, seed=4, draft_kind="probs",
                         nse=4.0, runner=None) -> dict:
    """Mean tau over simulated rounds with one (p, q) at every position versus the
    closed form, within ``nse`` standard errors."""
    model = ToyModel(V, seed, draft_kind, iid=True)
    (pl, p), (qr, q) = model.p(()), model.q(())
    rng = np.random.default_rng(seed + 7)
    x = np.stack([_sample_rows(np.broadcast_to(q, (rounds, V)), rng) for _ in range(gamma)], 1)
    res = (runner or oracle.chain)(np.broadcast_to(pl, (rounds, gamma + 1, V)),
                       np.broadcast_to(qr, (rounds, gamma, V)), draft_kind == "probs",
                       x.astype(np.int32), np.ones(rounds, np.float32),
                       _uniform24(rng, (rounds, gamma)), _uniform24(rng, rounds))
    tau = res["num_accepted"].astype(np.float64) + 1
    beta = float(np.minimum(p, q).sum())
    want = (1 - beta ** (gamma + 1)) / (1 - beta)
    se = tau.std(ddof=1) / math.sqrt(rounds)
    z = (tau.mean() - want) / se
    return dict(ok=bool(abs(z) < nse), z=float(z), mean=float(tau.mean()), want=want)


# ----------------------------------------------------------------------------- trees

def _tree_for_prefix(model: ToyModel, prefix, parents):
    """Tokens of a fixed-shape tree for ``prefix``: the children of every node
    carry distinct pseudo-random tokens (a deterministic function of the
    prefix)."""
    V = model.V
    rng = np.random.default_rng([model.seed, 99, len(prefix)] + [t + 1 for t in prefix])
    N = len(parents)
    tokens = np.zeros(N, np.int32)
    children = {}
    for n in range(1, N):
        children.setdefault(parents[n], []).append(n)
    for pa, ch in children.items():
        perm = rng.permutation(V)
        for r, c in enumerate(ch):
            tokens[c] = perm[r]
    return tokens, children


def _paths(parents, tokens):
    N = len(parents)
    path = [()] * N
    for n in range(1, N):
        path[n] = path[parents[n]] + (int(tokens[n]),)
    return path


def _tree_cases(model: ToyModel, prefix, parents):
    V = model.V
    tokens, children = _tree_for_prefix(model, prefix, parents)
    path = _paths(parents, tokens)
    N = len(parents)
    target = np.stack([model.p(prefix + path[n])[0] for n in range(N)])
    probs = [model.p(prefix + path[n])[1] for n in range(N)]
    # p_parent(n)(token_n): what the walk must use for node n
    pch = np.array([0.0] + [probs[parents[n]][tokens[n]] for n in range(1, N)])
    cases = []

    def visit(cur, weight, coins):
        p = probs[cur]
        ch = children.get(cur, [])
        A = 0.0
        for c in ch:
            pc = p[tokens[c]]
            lo, A = A, A + pc
            if pc > 0:
                visit(c, weight * pc, coins | {cur: (lo + A) / 2})
        rest = 1.0 - A if ch else 1.0
        if rest <= 1e-15:
            return
        r = p.copy()
        for c in ch:
            r[tokens[c]] = 0.0
        S = r.sum()
        C = np.cumsum(r)
        cc = coins | ({cur: (A + 1.0) / 2} if ch else {})
        for j in range(V):
            if r[j] > 0:
                cv = np.full(N, 0.5, np.float32)
                for node, val in cc.items():
                    cv[node] = val
                cases.append(dict(weight=weight * rest * r[j] / S, target=target, tokens=tokens,
                                  coins=cv, u=np.float32((C[j] - r[j] / 2) / S), pch=pch))

    visit(0, 1.0, {})
    return cases


def tree_bruteforce(V=3, K=3, seed=5, parents=(-1, 0, 0, 1, 1, 2, 3), tol=1e-12,
                    draft_probs_zero=False, T=1.0, runner=None, top_k=None, top_p=None) -> dict:
    """Exact distribution of the first K tokens of repeated target-only tree rounds
    (thresholds 1) against the target's autoregressive distribution -- with
    ``top_k`` / ``top_p``, against the filtered target's (filter_definition), the
    rows handed over unfiltered and the filter left to the verify step."""
    filt = top_k is not None or top_p is not None
    model = ToyModel(V, seed, T=T)
    if filt:
        model = FilteredModel(model, 0 if top_k is None else top_k, 1.0 if top_p is None else top_p)
    parents = np.array(parents, np.int32)
    N = len(parents)
    depth = max(len(p) for p in _paths(parents, np.zeros(N, np.int32)))
    states = {(): 1.0}
    dist = {}
    fmin, perr = np.inf, 0.0
    while states:
        batch, owners = [], []
        for prefix, w in states.items():
            cs = _tree_cases(model, prefix, parents)
            batch += cs
            owners += [(prefix, w)] * len(cs)
        m = len(batch)
        fk = dict(top_k=np.full(m, model.top_k, np.int32), top_p=np.full(m, model.top_p, np.float32)) if filt \
            else {}
        res = (runner or oracle.tree_sample)(np.stack([c["target"] for c in batch]),
                                 np.stack([c["tokens"] for c in batch]),
                                 np.broadcast_to(parents, (m, N)), np.full(m, model.T, np.float32),
                                 np.stack([c["coins"] for c in batch]),
                                 np.array([c["u"] for c in batch], np.float32), depth,
                                 draft_probs=np.zeros((m, N, V), np.float32) if draft_probs_zero else None,
                                 **fk)
        if "fmargin" in res:
            fmin = min(fmin, float(res["fmargin"].min()))
        if filt:                   # the walk's child probabilities are the filtered ones (f32 logits: 1e-6)
            perr = max(perr, float(np.abs(np.asarray(res["pchild"])[:, 1:]
                                          - np.stack([c["pch"] for c in batch])[:, 1:]).max()))
        nxt = {}
        for i, (prefix, w) in enumerate(owners):
            k = int(res["num_accepted"][i])
            if k < 0:
                return dict(ok=False, err=float("inf"))
            h = prefix + tuple(int(t) for t in res["tokens"][i, :k + 1])
            ww = w * batch[i]["weight"]
            if len(h) >= K:
                dist[h[:K]] = dist.get(h[:K], 0.0) + ww
            else:
                nxt[h] = nxt.get(h, 0.0) + ww
        states = nxt
    want = _product_distribution(model, K)
    err = max(abs(dist.get(s, 0.0) - pv) for s, pv in want.items())
    err = max(err, sum(v for s, v in dist.items() if s not in want))
    return dict(ok=err < tol and fmin > 1e-9 and perr < 1e-6, err=err, fmargin=fmin, pchild_err=perr)


def tree_chisquare(V=4, K=3, rounds=1_000_000, seed=6, shapes=None, pmin=1e-3, runner=None) -> dict:
    """Simulated target-only tree rounds (thresholds 1) over a few tree shapes with
    random distinct sibling tokens; chi-square of the first K tokens."""
    shapes = shapes or [(-1, 0, 0, 1, 1, 2), (-1, 0, 1, 2), (-1, 0, 0, 0, 1, 2, 3, 4)]
    model = ToyModel(V, seed)
    maxd = 0
    for s in shapes:
        d = [0] * len(s)
        for n in range(1, len(s)):
            d[n] = d[s[n]] + 1
        maxd = max(maxd, max(d))
    tab = _Tables(model, K - 1 + maxd)
    rng = np.random.default_rng(seed + 11)
    n = rounds
    ids = np.zeros(n, np.int64)
    ntok = np.zeros(n, np.int64)
    first = np.zeros((n, K), np.int64)
    active = np.arange(n)
    while active.size:
        pick = rng.integers(0, len(shapes), active.size)
        for si, shape in enumerate(shapes):
            sub = active[pick == si]
            if sub.size == 0:
                continue
            m = sub.size
            par = np.array(shape, np.int32)
            N = len(par)
            # distinct sibling tokens: per node, a random permutation of the vocab
            perms = np.argsort(rng.random((m, N, V)), axis=2).astype(np.int32)
            tokens = np.zeros((m, N), np.int32)
            rank = np.zeros(N, np.int64)
            seen = {}
            for c in range(1, N):
                r = seen.get(par[c], 0)
                rank[c] = r
                seen[par[c]] = r + 1
            for c in range(1, N):
                tokens[:, c] = perms[:, par[c], rank[c]]
            nid = np.zeros((m, N), np.int64)
            nid[:, 0] = ids[sub]
            for c in range(1, N):
                nid[:, c] = tab.child(nid[:, par[c]], tokens[:, c])
            d = [0] * N
            for c in range(1, N):
                d[c] = d[par[c]] + 1
            res = (runner or oracle.tree_sample)(tab.PL[nid], tokens, np.broadcast_to(par, (m, N)),
                                     np.ones(m, np.float32), _uniform24(rng, (m, N)),
                                     _uniform24(rng, m), max(d))
            k = res["num_accepted"]
            if (k < 0).any():
                return dict(ok=False, p=0.0)
            for j in range(max(d) + 1):
                sel = k >= j
                idx = sub[sel]
                tok = res["tokens"][sel, j]
                put = ntok[idx] < K
                first[idx[put], ntok[idx[put]]] = tok[put]
                ntok[idx[put]] += 1
                ids[idx] = tab.child(ids[idx], tok)
        active = active[ntok[active] < K]
    return _chisq(first, tab, V, K, pmin)


# ----------------------------------------------------------------------------- top-k / top-p filtering

def filter_definition(logits, T, top_k, top_p):
    """Filtered distribution from the definitions in threshold form (independent of
    the oracle's sort-and-accumulate): theta_k = the largest logit value t with
    #{l >= t} >= top_k; theta_p = the largest value t >= theta_k whose set
    {l >= t} carries, under softmax(l/T) renormalised on {l >= theta_k}, a mass
    >= top_p; keep {l >= max(theta_k, theta_p)} and renormalise."""
    l = np.asarray(logits, np.float64)
    V = l.size
    p = special.softmax(l / T)
    vals = np.unique(l)[::-1]                                     # every distinct value, -inf included
    th_k = -np.inf
    if 0 < top_k < V:
        th_k = max(t for t in vals if (l >= t).sum() >= top_k)
    A = l >= th_k
    pa = np.where(A, p, 0.0)
    pa /= pa.sum()
    th = th_k
    if top_p < 1.0:
        th = max(t for t in vals if t >= th_k and pa[l >= t].sum() >= top_p)
    keep = l >= th
    out = np.where(keep, p, 0.0)
    return out / out.sum(), keep


class FilteredModel:
    """A ToyModel seen through top-k / top-p: p() and q() return the raw row given
    to the verify step and the filtered distribution the drafts are drawn from
    and the output must follow (draft probabilities are filtered by the caller
    and handed over as they are)."""

    def __init__(self, model: ToyModel, top_k: int, top_p: float):
        self.m, self.top_k, self.top_p = model, top_k, top_p
        self.V, self.T, self.draft_kind, self.seed = model.V, model.T, model.draft_kind, model.seed

    def p(self, prefix):
        logits, _ = self.m.p(prefix)
        return logits, filter_definition(logits.astype(np.float64), self.T, self.top_k, self.top_p)[0]

    def q(self, prefix):
        row, probs = self.m.q(prefix)
        if self.draft_kind == "probs":
            f = filter_definition(np.log(np.maximum(probs, 1e-300)) + np.where(probs > 0, 0, -np.inf), 1.0,
                                  self.top_k, self.top_p)[0]
            return f.astype(np.float32), f.astype(np.float32).astype(np.float64)
        return row, filter_definition(row.astype(np.float64), self.T, self.top_k, self.top_p)[0]


def chain_filtered_bruteforce(V=4, gamma=2, K=2, seed=1, draft_kind="logits", T=1.0, top_k=3, top_p=0.8,
                              tol=1e-12, runner=None) -> dict:
    """Exact distribution of the first K tokens of repeated chain rounds under
    top-k / top-p filtering against the filtered target's autoregressive
    distribution (the rules keep whatever target distribution they are given)."""
    model = FilteredModel(ToyModel(V, seed, draft_kind, T=T), top_k, top_p)
    states = {(): 1.0}
    dist = {}
    fmin = np.inf
    while states:
        batch, owners = [], []
        for prefix, w in states.items():
            cs = _chain_cases(model, prefix, gamma)
            batch += cs
            owners += [(prefix, w)] * len(cs)
        n = len(batch)
        res = (runner or oracle.chain)(np.stack([c["target"] for c in batch]), np.stack([c["draft"] for c in batch]),
                                       draft_kind == "probs", np.stack([c["x"] for c in batch]),
                                       np.full(n, model.T, np.float32), np.stack([c["coins"] for c in batch]),
                                       np.array([c["u"] for c in batch], np.float32),
                                       top_k=np.full(n, top_k, np.int32), top_p=np.full(n, top_p, np.float32))
        if "fmargin" in res:
            fmin = min(fmin, float(res["fmargin"].min()))
        nxt = {}
        for i, (prefix, w) in enumerate(owners):
            k = int(res["num_accepted"][i])
            if k < 0:
                return dict(ok=False, err=float("inf"), reason="flagged valid input")
            h = prefix + tuple(int(t) for t in res["tokens"][i, :k + 1])
            ww = w * batch[i]["weight"]
            if len(h) >= K:
                dist[h[:K]] = dist.get(h[:K], 0.0) + ww
            else:
                nxt[h] = nxt.get(h, 0.0) + ww
        states = nxt
    want = _product_distribution(model, K)
    err = max(abs(dist.get(s, 0.0) - pv) for s, pv in want.items())
    err = max(err, sum(v for s, v in dist.items() if s not in want))
    return dict(ok=err < tol and fmin > 1e-9, err=err, fmargin=fmin)


def filter_properties(trials=400, seed=3) -> dict:
    """The oracle's filter against the defining properties on random rows (ties,
    signed zeros, -inf entries, bf16 and f32): kept values dominate dropped
    ones; top-k keeps >= top_k tokens with < top_k strictly above its smallest
    kept value; top-p keeps whole groups of equal logits, reaches top_p and
    would fall short without its smallest kept group; kept probabilities are
    scipy's softmax on the kept set; off switches give scipy's softmax."""
    rng = np.random.default_rng(seed)
    worst = 0.0
    for t in range(trials):
        V = int(rng.integers(1, 60))
        kind = rng.integers(3)
        if kind == 0:
            l = rng.integers(-3, 4, V).astype(np.float32)            # many ties
            l[rng.random(V) < 0.1] = -0.0
        elif kind == 1:
            l = rng.normal(0, 2, V).astype(np.float32)
        else:
            l = (rng.normal(0, 2, V).astype(np.float32).view(np.uint32) >> 16 << 16).view(np.float32)
        if V > 2 and rng.random() < 0.2:
            l[rng.integers(V)] = -np.inf
        if not np.isfinite(l).any():
            l[0] = 0.0
        T = float(np.float32(rng.choice([0.5, 1.0, 1.7])))
        K = int(rng.choice([0, 1, 2, 5, V, V + 3]))
        P = float(np.float32(rng.choice([1.0, 0.3, 0.7, 0.95, 1e-6])))
        row = l if rng.random() < 0.5 else (l.view(np.uint32) >> 16).astype(np.uint16)
        lv = l if row.dtype == np.float32 else (row.astype(np.uint32) << 16).view(np.float32)
        res = oracle.filter_row(row, T, K, P)
        if res is None:
            return dict(ok=False, trial=t, reason="valid filter rejected")
        p, margin = res
        lv64 = lv.astype(np.float64)
        keep = p > 0
        base = special.softmax(lv64 / T)
        if (K == 0 or K >= V) and P >= 1.0:
            worst = max(worst, float(np.abs(p - base).max()))
            continue
        if not keep.any() or (keep.any() and (~keep).any() and lv64[keep].min() < lv64[~keep].max()):
            return dict(ok=False, trial=t, reason="a dropped value exceeds a kept one")
        lo = lv64[keep].min()
        if (~keep & (lv64 == lo)).any():
            return dict(ok=False, trial=t, reason="a group of equal values was split")
        if 0 < K < V:
            if keep.sum() < K and P >= 1.0:
                return dict(ok=False, trial=t, reason="top-k kept too few")
            if (lv64 > lo).sum() >= K:
                return dict(ok=False, trial=t, reason="top-k kept too many")
        if P < 1.0:
            A = lv64 >= (np.sort(lv64)[::-1][K - 1] if 0 < K < V else -np.inf)
            pa = np.where(A, base, 0.0)
            pa /= pa.sum()
            if margin > 1e-9:
                if pa[keep].sum() < P:
                    return dict(ok=False, trial=t, reason="top-p mass short of top_p")
                if pa[keep & (lv64 > lo)].sum() >= P:
                    return dict(ok=False, trial=t, reason="top-p set not minimal")
        want = np.where(keep, base, 0.0)
        want /= want.sum()
        worst = max(worst, float(np.abs(p - want).max()))
    return dict(ok=worst < 1e-12, worst=worst)


# ----------------------------------------------------------------------------- trees with a draft distribution (MSS)

def _mss_cases(model: ToyModel, prefix, parents):
    """Every way one round of multi-step speculative sampling can go on a fixed
    tree shape: the children's tokens drawn independently from the draft
    distribution at their parent (weight = product of q), then every cell of
    the coins' and final uniform's breakpoint partition, with its probability
    under the rule (accept child with min(1, p/q), else p <- norm(max(0, p - q))
    and try the next sibling; at the end draw from p)."""
    V = model.V
    N = len(parents)
    children = {}
    for n in range(1, N):
        children.setdefault(int(parents[n]), []).append(n)
    cases = []
    for toks in itertools.product(range(V), repeat=N - 1):
        tokens = np.zeros(N, np.int32)
        tokens[1:] = toks
        path = _paths(parents, tokens)
        wq = 1.0
        for n in range(1, N):
            wq *= model.q(prefix + path[parents[n]])[1][tokens[n]]
        if wq == 0.0:
            continue
        target = np.stack([model.p(prefix + path[n])[0] for n in range(N)])
        draft = np.stack([model.q(prefix + path[n])[0] for n in range(N)]).astype(np.float32)

        def visit(cur, weight, coins):
            p = model.p(prefix + path[cur])[1].copy()
            q = model.q(prefix + path[cur])[1]
            for c in children.get(cur, []):
                x = tokens[c]
                a = min(1.0, p[x] / q[x])
                if a > 0:
                    visit(c, weight * a, coins | {c: a / 2})
                if a >= 1.0:
                    return
                weight *= 1.0 - a
                coins = coins | {c: (1.0 + a) / 2}
                r = np.maximum(0.0, p - q)
                p = r / r.sum()
            C = np.cumsum(p)
            for j in range(V):
                if p[j] > 0:
                    cv = np.full(N, 0.5, np.float32)
                    for node, val in coins.items():
                        cv[node] = val
                    cases.append(dict(weight=wq * weight * p[j], target=target, draft=draft, tokens=tokens,
                                      coins=cv, u=np.float32(C[j] - p[j] / 2)))

        visit(0, 1.0, {})
    return cases


def tree_mss_bruteforce(V=3, K=3, seed=5, parents=(-1, 0, 0, 0, 1, 1), tol=1e-12, T=1.0,
                        runner=None) -> dict:
    """Exact distribution of the first K tokens of repeated multi-step speculative
    sampling rounds (children drawn from q) against the target's autoregressive
    distribution ([origins] "SpecInfer": MSS keeps the target distribution)."""
    model = ToyModel(V, seed, "probs", T=T)
    parents = np.array(parents, np.int32)
    N = len(parents)
    depth = max(len(p) for p in _paths(parents, np.zeros(N, np.int32)))
    states = {(): 1.0}
    dist = {}
    while states:
        batch, owners = [], []
        for prefix, w in states.items():
            cs = _mss_cases(model, prefix, parents)
            batch += cs
            owners += [(prefix, w)] * len(cs)
        m = len(batch)
        res = (runner or oracle.tree_mss)(np.stack([c["target"] for c in batch]),
                                          np.stack([c["tokens"] for c in batch]),
                                          np.broadcast_to(parents, (m, N)), np.full(m, model.T, np.float32),
                                          np.stack([c["coins"] for c in batch]),
                                          np.array([c["u"] for c in batch], np.float32), depth,
                                          np.stack([c["draft"] for c in batch]))
        nxt = {}
        for i, (prefix, w) in enumerate(owners):
            k = int(res["num_accepted"][i])
            if k < 0:
                return dict(ok=False, err=float("inf"))
            h = prefix + tuple(int(t) for t in res["tokens"][i, :k + 1])
            ww = w * batch[i]["weight"]
            if len(h) >= K:
                dist[h[:K]] = dist.get(h[:K], 0.0) + ww
            else:
                nxt[h] = nxt.get(h, 0.0) + ww
        states = nxt
    want = _product_distribution(model, K)
    err = max(abs(dist.get(s, 0.0) - pv) for s, pv in want.items())
    err = max(err, sum(v for s, v in dist.items() if s not in want))
    return dict(ok=err < tol, err=err)


def tree_mss_chisquare(V=4, K=3, rounds=1_000_000, seed=16, shapes=None, pmin=1e-3, runner=None) -> dict:
    """Simulated multi-step speculative sampling rounds over a few tree shapes whose
    children are drawn independently from the draft distribution at their parent
    (duplicate siblings included); chi-square of the first K tokens."""
    shapes = shapes or [(-1, 0, 0, 0, 1, 1), (-1, 0, 1, 2), (-1, 0, 0, 1, 1, 2, 2, 3)]
    model = ToyModel(V, seed, "probs")
    maxd = 0
    for sh in shapes:
        d = [0] * len(sh)
        for n in range(1, len(sh)):
            d[n] = d[sh[n]] + 1
        maxd = max(maxd, max(d))
    tab = _Tables(model, K - 1 + maxd)
    rng = np.random.default_rng(seed + 13)
    n = rounds
    ids = np.zeros(n, np.int64)
    ntok = np.zeros(n, np.int64)
    first = np.zeros((n, K), np.int64)
    active = np.arange(n)
    while active.size:
        pick = rng.integers(0, len(shapes), active.size)
        for si, shape in enumerate(shapes):
            sub = active[pick == si]
            if sub.size == 0:
                continue
            m = sub.size
            par = np.array(shape, np.int32)
            N = len(par)
            tokens = np.zeros((m, N), np.int32)
            nid = np.zeros((m, N), np.int64)
            nid[:, 0] = ids[sub]
            for c in range(1, N):
                tokens[:, c] = _sample_rows(tab.Q[nid[:, par[c]]], rng)
                nid[:, c] = tab.child(nid[:, par[c]], tokens[:, c])
            d = [0] * N
            for c in range(1, N):
                d[c] = d[par[c]] + 1
            res = (runner or oracle.tree_mss)(tab.PL[nid], tokens, np.broadcast_to(par, (m, N)),
                                              np.ones(m, np.float32), _uniform24(rng, (m, N)),
                                              _uniform24(rng, m), max(d), tab.QR[nid])
            k = res["num_accepted"]
            if (k < 0).any():
                return dict(ok=False, p=0.0)
            for j in range(max(d) + 1):
                sel = k >= j
                idx = sub[sel]
                tok = res["tokens"][sel, j]
                put = ntok[idx] < K
                first[idx[put], ntok[idx[put]]] = tok[put]
                ntok[idx[put]] += 1
                ids[idx] = tab.child(ids[idx], tok)
        active = active[ntok[active] < K]
    return _chisq(first, tab, V, K, pmin)


# ----------------------------------------------------------------------------- greedy

def _toy_row(h: int, V: int, levels: int) -> np.ndarray:
    """Small-integer logits (as bf16 bit patterns) from a prefix hash: many ties."""
    rng = np.random.default_rng([h & 0xFFFFFFFF, h >> 32])
    vals = rng.integers(0, levels, V).astype(np.float32)
    return (vals.view(np.uint32) >> 16).astype(np.uint16)


def greedy_equivalence(steps=10_000, V=16, levels=4, seed=7, max_nodes=12, max_depth=4,
                       runner=None) -> dict:
    """Speculative greedy over random trees versus plain argmax decoding of the same
    toy model (lowest index among equal maxima), token for token."""
    MOD = (1 << 61) - 1

    def hnext(h, t):
        return (h * 1000003 + t + 1 + seed) % MOD

    def row_f(h):
        bits = _toy_row(h, V, levels)
        return bits, (bits.astype(np.uint32) << 16).view(np.float32)

    # plain greedy decoding
    plain = []
    h = 0
    while len(plain) < steps:
        _, f = row_f(h)
        t = int(np.argmax(f))                      # numpy: first index of the maximum
        plain.append(t)
        h = hnext(h, t)
    # speculative greedy over random trees
    rng = np.random.default_rng(seed)
    spec = []
    h = 0
    rounds = 0
    while len(spec) < steps:
        N = int(rng.integers(1, max_nodes + 1))
        parents = [-1]
        depth = [0]
        for n in range(1, N):
            cand = [m for m in range(n) if depth[m] < max_depth]
            pa = int(cand[rng.integers(len(cand))])
            parents.append(pa)
            depth.append(depth[pa] + 1)
        hs = [h] + [0] * (N - 1)
        tokens = [0] * N
        rows = [row_f(h)[0]] + [None] * (N - 1)
        for n in range(1, N):
            pa = parents[n]
            if rng.random() < 0.6:
                tokens[n] = int(np.argmax(row_f(hs[pa])[1]))
            else:
                tokens[n] = int(rng.integers(V))
            hs[n] = hnext(hs[pa], tokens[n])
            rows[n] = row_f(hs[n])[0]
        res = (runner or oracle.tree_greedy)(np.stack(rows)[None], np.array([tokens]),
                                             np.array([parents]), max(depth))
        k = int(res["num_accepted"][0])
        if k < 0:
            return dict(ok=False, reason="invalid")
        for t in res["tokens"][0, :k + 1]:
            spec.append(int(t))
            h = hnext(h, int(t))
        rounds += 1
    ok = spec[:steps] == plain
    first_diff = next((i for i in range(steps) if spec[i] != plain[i]), -1)
    return dict(ok=ok, rounds=rounds, first_diff=first_diff)
