"""Lazy (row-on-demand) entry points: spec_verify_chain_lazy,
spec_verify_tree_greedy_lazy, spec_verify_tree_sample_lazy.

For valid inputs they must emit exactly what the dense entry points emit
(which the other GPU tests pin to the fp64 oracle); they are also compared
with the oracle directly, run through the pins (brute force, chi-square) and
checked for their documented differences: diagnostics only at evaluated
positions, no validation of rows that are never read."""
import functools

import numpy as np
import pytest
import torch

import parity
import pins
from speculative_decoding_verify_temperature_b200 import workloads as wl
from speculative_decoding_verify_temperature_b200 import spec_verify as sv

pytestmark = pytest.mark.gpu


def _q(dt):
    return 16 // (2 if dt == torch.bfloat16 else 4)


def _stride(V, pad, dt):
    return -(-(V + pad) // _q(dt)) * _q(dt)


# ----------------------------------------------------------------------------- chain

def _chain_same(inp):
    """Lazy == dense on tokens and counts; diagnostics equal where the lazy walk
    evaluated them (positions <= k), NaN after."""
    d = parity.gpu_chain(inp)
    z = parity.gpu_chain(inp, lazy=True)
    np.testing.assert_array_equal(z["num_accepted"], d["num_accepted"])
    np.testing.assert_array_equal(z["tokens"], d["tokens"])
    g = inp.gamma
    for b, k in enumerate(d["num_accepted"]):
        if k < 0:
            continue
        ev = min(k + 1, g)
        np.testing.assert_array_equal(z["px"][b, :ev], d["px"][b, :ev])
        np.testing.assert_array_equal(z["qx"][b, :ev], d["qx"][b, :ev])
        assert np.isnan(z["px"][b, ev:]).all() and np.isnan(z["qx"][b, ev:]).all()
        assert z["S"][b] == d["S"][b]
    return z, d


def _chain_vs_oracle(inp, rows=None):
    z = parity.gpu_chain(inp, lazy=True)
    o = parity.oracle_chain(inp, rows)
    sel = parity._rows_np(rows)
    flags = parity.chain_flags(o, inp.gamma)
    zk, zt = z["num_accepted"][sel], z["tokens"][sel]
    same = (zk == o["num_accepted"]) & (zt == o["tokens"]).all(axis=1)
    assert (same | flags).all(), np.nonzero(~same & ~flags)[0][:10]
    assert flags.sum() <= 0.2 * len(zk) + 1
    for i, k in enumerate(o["num_accepted"]):
        if k < 0 or not same[i]:
            continue
        ev = min(k + 1, inp.gamma)
        np.testing.assert_allclose(z["px"][sel][i, :ev], o["px"][i, :ev], rtol=parity.RTOL, atol=parity.ATOL)
        np.testing.assert_allclose(z["qx"][sel][i, :ev], o["qx"][i, :ev], rtol=parity.RTOL, atol=parity.ATOL)
        if not flags[i]:
            np.testing.assert_allclose(z["S"][sel][i], o["S"][i], rtol=parity.RTOL, atol=1e-12)


CHAIN = [
    # B, gamma, V, tdt, draft (dtype or "probs"), stride pad, temperatures
    (3, 1, 1003, torch.bfloat16, torch.bfloat16, 5, (1.0,)),
    (4, 4, 8193, torch.bfloat16, torch.bfloat16, 7, (0.6, 1.0)),
    (2, 16, 20000, torch.bfloat16, torch.bfloat16, 0, (1.3,)),
    (5, 3, 4096 * 3 + 5, torch.float32, torch.float32, 3, (0.8,)),
    (3, 2, 9000, torch.bfloat16, torch.float32, 0, (1.0,)),
    (3, 2, 9000, torch.float32, torch.bfloat16, 0, (1.0,)),
    (6, 5, 30001, torch.bfloat16, "probs", 3, (1.0,)),
    (2, 3, 5000, torch.float32, "probs", 0, (0.7,)),
    (1, 1, 1, torch.float32, torch.float32, 3, (1.0,)),
    (3, 2, 7, torch.bfloat16, torch.bfloat16, 1, (1.0,)),
    (200, 4, 70000, torch.bfloat16, torch.bfloat16, 0, (0.6, 1.0)),     # > one wave: sliced residual
]


@pytest.mark.parametrize("case", CHAIN, ids=lambda c: f"B{c[0]}g{c[1]}V{c[2]}{str(c[3])[-4:]}{str(c[4])[-5:]}")
def test_lazy_chain_equals_dense_and_oracle(case, cuda_device):
    B, gamma, V, tdt, dk, pad, temps = case
    probs = dk == "probs"
    ddt = torch.float32 if probs else dk
    for seed in range(3):
        inp = wl.chain_inputs(B, gamma, V, seed=4000 + seed, device="cuda", target_dtype=tdt, draft_dtype=ddt,
                              draft_is_probs=probs, zipf=True, temperatures=temps,
                              stride=_stride(V, pad, tdt), dstride=_stride(V, pad, ddt))
        _chain_same(inp)
        _chain_vs_oracle(inp, rows=None if B <= 16 else np.arange(0, B, 13))


def test_lazy_chain_workloads(cuda_device):
    """B=64 gamma=5 V=32000 bf16 logits (every sequence vs the oracle) and B=512
    gamma=7 V=129280 bf16 + f32 draft probabilities (48 sequences vs the oracle)."""
    for r in range(2):
        inp = wl.chain_config1(r, "cuda")
        _chain_same(inp)
        _chain_vs_oracle(inp)
    inp = wl.chain_config4(0, "cuda")
    _chain_same(inp)
    _chain_vs_oracle(inp, rows=np.arange(0, 512, 512 // 48)[:48])


def test_lazy_chain_workload0_rounds(cuda_device):
    target, draft = wl.chain_config0_logits("cuda")
    for r in range(200):
        _chain_same(wl.chain_config0_round(r, target, draft, "cuda"))


def test_lazy_chain_through_pins(cuda_device):
    run = functools.partial(parity.gpu_chain_runner, lazy=True)
    for kw in [dict(), dict(draft_kind="logits", seed=11, T=0.7)]:
        r = pins.chain_bruteforce(runner=run, **kw)
        assert r["ok"], (kw, r)
    r = pins.chain_closed_form_exact(runner=run)
    assert r["ok"], r
    r = pins.chain_chisquare(rounds=1_000_000, seed=3, draft_kind="probs", runner=run)
    assert r["ok"], r


def test_lazy_chain_validation(cuda_device):
    """Rows and tokens on the walk are validated; rows after the first rejection
    are not read and so not validated."""
    B, gamma, V = 6, 3, 3000
    inp = wl.chain_inputs(B, gamma, V, seed=5, device="cuda")
    inp.temperature[1] = 0.0                      # bad temperature: always checked
    inp.draft_tokens[2, 0] = V                    # first drafted token out of range
    inp.target[3, 0, 17] = float("nan")           # NaN in the first target row
    # sequence 4: rejected at position 0 for sure (p(x_0) ~ 0), NaN in a later row
    x0 = int(inp.draft_tokens[4, 0])
    inp.target[4, 0, x0] = -1e4
    inp.coins[4, 0] = 0.5
    inp.target[4, 2, 5] = float("nan")
    inp.draft_tokens[4, 2] = -5
    ws = sv.Workspace("cuda")
    buf = ws.get(sv.SPEC_ENTRY_CHAIN, B, gamma, V)
    z = parity.gpu_chain(inp, workspace=buf, lazy=True)
    assert list(z["num_accepted"][1:4]) == [-1] * 3 and (z["tokens"][1:4] == -1).all()
    assert np.isnan(z["px"][1:4]).all()
    assert z["num_accepted"][4] == 0 and z["tokens"][4, 0] >= 0 and (z["tokens"][4, 1:] == -1).all()
    assert sv.spec_read_device_status(buf) & (1 << sv.SPEC_ERR_DEVICE_INPUT)
    d = parity.gpu_chain(inp, lazy=False)
    assert d["num_accepted"][4] == -1             # the dense path reads (and rejects) every row
    for b in (0, 5):
        assert z["num_accepted"][b] == d["num_accepted"][b]
        assert (z["tokens"][b] == d["tokens"][b]).all()


def test_lazy_chain_graph_replay_and_reuse(cuda_device):
    """One workspace across dense and lazy calls, eager and inside a CUDA graph
    replayed with new inputs: the per-level counts start from zero every call."""
    sets = [wl.chain_config1(r, "cuda") for r in range(3)]
    ref = [parity.gpu_chain(s) for s in sets]
    x = sets[0]
    B, g = x.B, x.gamma
    ws = sv.Workspace("cuda")
    buf = ws.get(sv.SPEC_ENTRY_CHAIN, B, g, x.V)
    static = [t.clone() for t in (x.target, x.draft, x.draft_tokens, x.temperature, x.coins, x.final_u)]
    toks = torch.empty((B, g + 1), dtype=torch.int32, device="cuda")
    na = torch.empty((B,), dtype=torch.int32, device="cuda")

    def call(lazy):
        fn = sv.spec_verify_chain_lazy if lazy else sv.spec_verify_chain
        fn(*static, V=x.V, out_tokens=toks, out_num_accepted=na, workspace=buf)

    for lazy in (True, False, True):
        call(lazy)
        torch.cuda.synchronize()
        assert (toks.cpu().numpy() == ref[0]["tokens"]).all()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call(True)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(True)
    for _ in range(2):
        for i, st in enumerate(sets):
            for dst, src in zip(static, (st.target, st.draft, st.draft_tokens, st.temperature, st.coins,
                                         st.final_u)):
                dst.copy_(src)
            graph.replay()
            torch.cuda.synchronize()
            np.testing.assert_array_equal(toks.cpu().numpy(), ref[i]["tokens"])
            np.testing.assert_array_equal(na.cpu().numpy(), ref[i]["num_accepted"])


# ----------------------------------------------------------------------------- trees

def _parents_fn(kind):
    if kind == "random":
        return lambda g: wl.random_tree(20, 4, g)
    if kind == "chain":
        return lambda g: wl.chain_tree(9)
    if kind == "root":
        return lambda g: [-1]
    if kind == "big":
        return lambda g: wl.random_tree(256, 6, g, max_depth=64)
    return None


GREEDY = [
    (4, 1003, torch.bfloat16, "level", None, 5),
    (6, 20000, torch.bfloat16, "random", 3, 0),
    (5, 8192 * 2 + 1, torch.bfloat16, "chain", None, 7),
    (3, 5000, torch.float32, "random", 2, 1),
    (2, 9, torch.bfloat16, "root", None, 0),
    (8, 300, torch.bfloat16, "big", 2, 4),
]


@pytest.mark.parametrize("case", GREEDY, ids=lambda c: f"B{c[0]}V{c[1]}{c[3]}")
def test_lazy_greedy_equals_dense_and_oracle(case, cuda_device):
    B, V, dt, kind, ties, pad = case
    for seed in range(3):
        inp = wl.tree_greedy_inputs(B, V, seed=4200 + seed, device="cuda", parents_fn=_parents_fn(kind),
                                    target_dtype=dt, stride=_stride(V, pad, dt), int_logits=ties, p_match=0.8)
        d = parity.gpu_greedy(inp)
        z = parity.gpu_greedy(inp, lazy=True)
        for key in ("accept_index", "tokens", "num_accepted"):
            np.testing.assert_array_equal(z[key], d[key])
        nflag, nbad, det = parity.compare_tree(z, parity.oracle_greedy(inp))
        assert nbad == 0, det


def test_lazy_greedy_workload2(cuda_device):
    inp = wl.tree_config2(0, "cuda")
    d = parity.gpu_greedy(inp)
    z = parity.gpu_greedy(inp, lazy=True)
    for key in ("accept_index", "tokens", "num_accepted"):
        np.testing.assert_array_equal(z[key], d[key])
    nflag, nbad, det = parity.compare_tree(z, parity.oracle_greedy(inp))
    assert nbad == 0, det


def test_lazy_greedy_equals_argmax_decoding(cuda_device):
    r = pins.greedy_equivalence(steps=2000, runner=functools.partial(parity.gpu_tree_greedy_runner, lazy=True))
    assert r["ok"], r


def test_lazy_greedy_validation(cuda_device):
    inp = wl.tree_greedy_inputs(5, 4000, seed=9, device="cuda", parents_fn=lambda g: wl.random_tree(10, 3, g))
    inp.parents[1, 5] = 7                          # parent after child
    inp.tokens[2, 2] = -3                          # token out of range
    inp.parents[3, 0] = 0                          # root must have parent -1
    inp.target[4, 0, 7] = float("nan")            # NaN in the root row: always read
    z = parity.gpu_greedy(inp, lazy=True)
    assert list(z["num_accepted"][1:]) == [-1] * 4
    assert (z["tokens"][1:] == -1).all() and (z["accept_index"][1:] == -1).all()
    d = parity.gpu_greedy(inp)
    for key in ("accept_index", "tokens", "num_accepted"):
        np.testing.assert_array_equal(z[key], d[key])


def _sample_same(inp, **th):
    d = parity.gpu_sample(inp, **th)
    z = parity.gpu_sample(inp, lazy=True, **th)
    for key in ("accept_index", "tokens", "num_accepted"):
        np.testing.assert_array_equal(z[key], d[key])
    par = inp.parents.cpu().numpy()
    for b in range(inp.B):
        if d["num_accepted"][b] < 0:
            continue
        visited = set(int(n) for n in d["accept_index"][b] if n >= 0)
        ev = np.array([n > 0 and par[b, n] in visited for n in range(inp.N)])
        np.testing.assert_array_equal(z["pchild"][b, ev], d["pchild"][b, ev])
        assert np.isnan(z["pchild"][b, 1:][~ev[1:]]).all()
        assert z["pchild"][b, 0] == 0.0
        assert z["S"][b] == d["S"][b]
    return z


SAMPLE = [
    (4, 1003, torch.bfloat16, "level", None, 0.8, 5),
    (5, 20000, torch.bfloat16, "random", "zeros", 1.0, 0),
    (5, 20000, torch.bfloat16, "random", "random", 1.0, 0),
    (3, 8192 * 2 + 3, torch.float32, "chain", None, 0.6, 1),
    (2, 9, torch.bfloat16, "root", None, 1.0, 0),
    (4, 300, torch.bfloat16, "big", None, 1.7, 4),
    (4, 300, torch.float32, "big", "random", 1.0, 4),
]


@pytest.mark.parametrize("case", SAMPLE, ids=lambda c: f"B{c[0]}V{c[1]}{c[3]}{c[4]}")
def test_lazy_sample_equals_dense_and_oracle(case, cuda_device):
    B, V, dt, kind, dp, T, pad = case
    for seed in range(3):
        inp = wl.tree_sample_inputs(B, V, seed=4300 + seed, device="cuda", parents_fn=_parents_fn(kind),
                                    target_dtype=dt, stride=_stride(V, pad, dt), temperature=T, draft_probs=dp,
                                    zipf=V > 100)
        z = _sample_same(inp)
        o = parity.oracle_sample(inp)
        flags = (o["dmargin"] < parity.TIE_TOL) | (o["cmargin"] < parity.TIE_TOL)
        same = ((z["num_accepted"] == o["num_accepted"]) & (z["tokens"] == o["tokens"]).all(axis=1)
                & (z["accept_index"] == o["accept_index"]).all(axis=1))
        assert (same | flags).all()
        ev = ~np.isnan(z["pchild"])
        np.testing.assert_allclose(z["pchild"][ev], o["pchild"][ev], rtol=parity.RTOL, atol=parity.ATOL)


def test_lazy_sample_thresholds(cuda_device):
    inp = wl.tree_sample_inputs(6, 5000, seed=77, device="cuda")
    for ts, ta in [(0.05, 1.0), (1.0, 0.5), (0.3, 0.7)]:
        _sample_same(inp, threshold_single=ts, threshold_acc=ta)


def test_lazy_sample_workload3(cuda_device):
    inp = wl.tree_config3(0, "cuda")
    z = _sample_same(inp)
    rows = np.arange(0, 128, 8)
    o = parity.oracle_sample(inp, rows=rows)
    flags = (o["dmargin"] < parity.TIE_TOL) | (o["cmargin"] < parity.TIE_TOL)
    same = (z["num_accepted"][rows] == o["num_accepted"]) & (z["tokens"][rows] == o["tokens"]).all(axis=1)
    assert (same | flags).all()


def test_lazy_sample_through_pins(cuda_device):
    run = functools.partial(parity.gpu_tree_sample_runner, lazy=True)
    for kw in [dict(), dict(draft_probs_zero=True, seed=8, T=0.8)]:
        r = pins.tree_bruteforce(runner=run, **kw)
        assert r["ok"], (kw, r)
    r = pins.tree_chisquare(rounds=1_000_000, seed=6, runner=run)
    assert r["ok"], r


def test_lazy_sample_validation(cuda_device):
    inp = wl.tree_sample_inputs(4, 3000, seed=12, device="cuda")
    inp.temperature[1] = float("nan")
    inp.parents[2, 3] = 9
    # sequence 3: NaN in the row of a node the walk cannot reach (a leaf whose
    # parent's children all get rejected is not guaranteed, so use the last
    # node, a leaf: its row is read only if the walk ends there)
    d0 = parity.gpu_sample(inp)
    last = inp.N - 1
    if last not in set(d0["accept_index"][3].tolist()):
        inp.target[3, last, 11] = float("nan")
    z = parity.gpu_sample(inp, lazy=True)
    assert list(z["num_accepted"][1:3]) == [-1, -1]
    assert np.isnan(z["pchild"][1:3]).all()
    assert z["num_accepted"][3] == d0["num_accepted"][3]
    assert (z["tokens"][3] == d0["tokens"][3]).all()
