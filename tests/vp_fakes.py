"""CPU stand-ins for the five device steps of the vocabulary-parallel chain round,
in fp64 numpy, for testing the exchange logic of
``spec_verify_chain_vocab_parallel`` on gloo ranks without a GPU.  They follow
the same split of the rules as the CUDA steps (per-shard (m, Z) and drafted
values, a combine in rank order, per-shard residual masses, the owner shard
draws) with their own record format; the records are opaque to the
orchestration."""
from __future__ import annotations

import numpy as np
import torch


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


class FakeVpOps:
    def __init__(self):
        self.state = None

    def stats(self, target, draft, draft_tokens, temperature, *, vocab_offset, draft_is_probs, V_shard, **_):
        l = _f64(target)[:, :, :V_shard]
        d = _f64(draft)[:, :, :V_shard]
        x = draft_tokens.cpu().numpy()
        T = temperature.cpu().numpy().astype(np.float64)
        B, R = l.shape[:2]
        g = R - 1
        rec = np.zeros((B, 2 * g + 1, 5))                     # m, Z, val, has, bad
        for b in range(B):
            for r in range(2 * g + 1):
                row = l[b, r] if r <= g else d[b, r - g - 1]
                i = r if r <= g else r - g - 1
                if r <= g or not draft_is_probs:
                    z = row / T[b]
                    m = z.max()
                    rec[b, r, 0] = m
                    rec[b, r, 1] = np.exp(z - m).sum() if np.isfinite(m) else 0.0
                if i < g:
                    j = x[b, i] - vocab_offset
                    if 0 <= j < V_shard:
                        rec[b, r, 2] = row[j]
                        rec[b, r, 3] = 1
        return torch.from_numpy(rec)

    @staticmethod
    def _combine(ra, b, r):
        m = ra[:, b, r, 0].max()
        Z = sum(ra[w, b, r, 1] * np.exp(ra[w, b, r, 0] - m) for w in range(ra.shape[0]) if np.isfinite(ra[w, b, r, 0]))
        return m, Z

    def decide(self, rec_all, draft_tokens, temperature, coins, *, V, V_shard, draft_is_probs, out_tokens=None,
               out_num_accepted=None, **_):
        ra = rec_all.numpy()
        world, B, R2, _ = ra.shape
        g = (R2 - 1) // 2
        x = draft_tokens.cpu().numpy()
        T = temperature.cpu().numpy().astype(np.float64)
        c = coins.cpu().numpy().astype(np.float64)
        toks = np.full((B, g + 1), -1, np.int32)
        ks = np.zeros(B, np.int32)
        self.state = []
        for b in range(B):
            k = g
            for i in range(g):
                m, Z = self._combine(ra, b, i)
                w = int(np.nonzero(ra[:, b, i, 3])[0][0])
                p = np.exp(ra[w, b, i, 2] / T[b] - m) / Z
                wq = int(np.nonzero(ra[:, b, g + 1 + i, 3])[0][0])
                if draft_is_probs:
                    q = ra[wq, b, g + 1 + i, 2]
                else:
                    mq, Zq = self._combine(ra, b, g + 1 + i)
                    q = np.exp(ra[wq, b, g + 1 + i, 2] / T[b] - mq) / Zq
                ratio = p / q if q > 0 else np.inf
                if not c[b, i] <= ratio:
                    k = i
                    break
            toks[b, :k] = x[b, :k]
            ks[b] = k
            mp, Zp = self._combine(ra, b, k)
            mq, Zq = self._combine(ra, b, g + 1 + k) if (k < g and not draft_is_probs) else (0.0, 1.0)
            self.state.append((k, T[b], mp, Zp, mq, Zq))
        return torch.from_numpy(toks), torch.from_numpy(ks)

    def _weights(self, target, draft, b, draft_is_probs, V_shard):
        k, T, mp, Zp, mq, Zq = self.state[b]
        g = target.shape[1] - 1
        p = np.exp(_f64(target)[b, k, :V_shard] / T - mp) / Zp
        if k == g:
            return p
        d = _f64(draft)[b, k, :V_shard]
        q = d if draft_is_probs else np.exp(d / T - mq) / Zq
        return np.maximum(0.0, p - q)

    def residual(self, target, draft, rec_all, *, rank, draft_is_probs, V_shard, **_):
        B = target.shape[0]
        return torch.tensor([self._weights(target, draft, b, draft_is_probs, V_shard).sum() for b in range(B)],
                            dtype=torch.float64)

    def sample(self, target, draft, final_u, rec_all, mass_all, *, vocab_offset, rank, draft_is_probs, V_shard, **_):
        ma = mass_all.numpy()
        u = final_u.cpu().numpy().astype(np.float64)
        B = target.shape[0]
        tok = np.full(B, -1, np.int32)
        for b in range(B):
            t = u[b] * ma[:, b].sum()
            c = 0.0
            owner, before = -1, 0.0
            for w in range(ma.shape[0]):
                if ma[w, b] > 0 and t < c + ma[w, b]:
                    owner, before = w, c
                    break
                c += ma[w, b]
            if owner == rank:
                w8 = self._weights(target, draft, b, draft_is_probs, V_shard)
                C = np.cumsum(w8)
                j = int(np.searchsorted(C, t - before, side="right"))
                tok[b] = vocab_offset + min(j, V_shard - 1)
        return torch.from_numpy(tok)

    def finish(self, tok, out_tokens, **_):
        for b, st in enumerate(self.state):
            out_tokens[b, st[0]] = int(tok[b])
        return out_tokens
