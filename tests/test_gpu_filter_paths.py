"""The bf16 top-k / top-p filters resolve a row from its candidates (the values
near the row's maximum) and fall back to a whole-row path when the candidates
cannot hold the answer.  Both must give the same record, so every output and
diagnostic is compared bit for bit between the default paths and the
whole-row paths alone (spec_debug_filter_path), on the dense, no-diagnostics
(on-demand tree walk) and lazy entry points; the per-path row counts show
which path ran, and inputs built to overflow or undershoot the candidates
check that the fallback is taken and still agrees with the oracle."""
import numpy as np
import pytest
import torch

import parity
from speculative_decoding_verify_temperature_b200 import spec_verify as sv
from speculative_decoding_verify_temperature_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _run(mode, fn):
    """fn() under filter mode `mode`; returns (outputs, (rows by candidates at
    the first cut, rows by a whole-row path, rows by candidates at the deeper
    cut))."""
    sv.spec_debug_filter_path(mode, read=True)           # reset the counters
    try:
        out = fn()
        rows = sv.spec_debug_filter_path(mode, read=True)
    finally:
        sv.spec_debug_filter_path(-1)
    return out, rows


def _same(a, b):
    assert a.keys() == b.keys()
    for k in a:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def _ab(fn):
    """Default paths vs whole-row paths alone: identical outputs.  Returns the
    default run's row counts."""
    d, rd = _run(0, fn)
    w, rw = _run(1, fn)
    _same(d, w)
    assert rw[0] == 0 and rw[2] == 0 and rw[1] == sum(rd), (rd, rw)
    return rd


def _params(B, seed, ks=(0, 1, 20, 50, 300), ps=(1.0, 0.9, 0.95, 0.5, 0.99)):
    g = np.random.default_rng(seed)
    tk = torch.from_numpy(g.choice(np.array(ks, np.int32), B).astype(np.int32)).cuda()
    tp = torch.from_numpy(g.choice(np.array(ps, np.float32), B).astype(np.float32)).cuda()
    return tk, tp


CHAIN = [
    # B, gamma, V, draft (dtype or "probs"), temperatures, zipf
    (16, 4, 32000, torch.bfloat16, (0.6, 1.0), True),
    (12, 3, 129280, "probs", (1.0,), True),
    (8, 2, 20001, torch.bfloat16, (0.3, 2.0), False),
    (8, 5, 777, torch.bfloat16, (1.0,), False),
]


@pytest.mark.parametrize("case", CHAIN, ids=lambda c: f"B{c[0]}g{c[1]}V{c[2]}{str(c[3])[-5:]}")
def test_chain_candidates_equal_whole_row(case, cuda_device):
    B, gamma, V, dk, temps, zipf = case
    probs = dk == "probs"
    for seed in range(2):
        inp = wl.chain_inputs(B, gamma, V, seed=9100 + seed, device="cuda", draft_dtype=torch.float32 if probs else dk,
                              draft_is_probs=probs, zipf=zipf, temperatures=temps, stride=-(-V // 8) * 8,
                              dstride=-(-V // (4 if probs else 8)) * (4 if probs else 8))
        tk, tp = _params(B, seed)
        for kw in (dict(), dict(with_diag=False), dict(lazy=True)):
            rows = _ab(lambda: parity.gpu_chain_filtered(inp, tk, tp, **kw))
            if not kw:
                assert rows[0] > 0, rows                  # the candidates resolved rows


TREE = [
    # B, V, parents kind, temperature, zipf
    (16, 151936, None, 0.8, True),
    (12, 20000, "random", 1.0, True),
    (8, 4099, "random", 0.5, False),
]


@pytest.mark.parametrize("case", TREE, ids=lambda c: f"B{c[0]}V{c[1]}{c[2]}")
def test_tree_candidates_equal_whole_row(case, cuda_device):
    B, V, kind, T, zipf = case
    pf = (lambda g: wl.random_tree(20, 4, g)) if kind == "random" else None
    for seed in range(2):
        inp = wl.tree_sample_inputs(B, V, seed=9200 + seed, device="cuda", parents_fn=pf, temperature=T, zipf=zipf,
                                    stride=-(-V // 8) * 8)
        tk, tp = _params(B, 10 + seed)
        for kw in (dict(), dict(with_diag=False), dict(lazy=True)):
            rows = _ab(lambda: parity.gpu_sample(inp, top_k=tk, top_p=tp, **kw))
            assert rows[0] > 0, (kw, rows)


def _flat(inp_rows, V, sigma, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = inp_rows.shape[:-1] + (V,)
    inp_rows[..., :V] = (torch.randn(shape, generator=g, device="cuda") * sigma).to(inp_rows.dtype)


def test_hard_rows_agree_with_the_oracle(cuda_device):
    """Rows the first cut cannot resolve: a nearly flat row (its top-p crossing
    far below the maximum, among values spread around zero), a top_k beyond
    the first cut's values, a top_p so close to 1 that the first cut's mass
    falls short.  The deeper cut or the whole-row path takes them; the outputs
    equal the whole-row-only run and the oracle's."""
    B, gamma, V = 6, 3, 120000
    inp = wl.chain_inputs(B, gamma, V, seed=9300, device="cuda", zipf=True, temperatures=(1.0,))
    _flat(inp.target[0:2], V, 0.05, 1)                  # sequences 0-1: nearly flat target rows
    tk = torch.tensor([0, 40, 30000, 0, 2000, 50], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.9, 1.0, 1.0, 0.99999, 1.0, 0.9], dtype=torch.float32, device="cuda")
    rows = _ab(lambda: parity.gpu_chain_filtered(inp, tk, tp))
    assert rows[0] > 0 and rows[1] + rows[2] > 0, rows
    g = parity.gpu_chain_filtered(inp, tk, tp)
    o = parity.oracle_chain_filtered(inp, tk, tp)
    nflag, nbad, det = parity.compare_chain(g, o, gamma)
    assert nbad == 0, det


def test_tree_hard_rows(cuda_device):
    """The same kinds of rows on the tree paths (dense filter, the on-demand
    walk, the lazy walk)."""
    B, V = 6, 60000
    inp = wl.tree_sample_inputs(B, V, seed=9400, device="cuda", stride=V)
    _flat(inp.target[0:3], V, 0.05, 2)
    tk = torch.tensor([0, 30, 0, 5000, 20, 0], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.95, 1.0, 0.5, 1.0, 0.9, 0.99999], dtype=torch.float32, device="cuda")
    for kw in (dict(), dict(with_diag=False), dict(lazy=True)):
        rows = _ab(lambda: parity.gpu_sample(inp, top_k=tk, top_p=tp, **kw))
        assert rows[1] + rows[2] > 0, (kw, rows)
    g = parity.gpu_sample(inp, top_k=tk, top_p=tp)
    o = parity.oracle_sample(inp, top_k=tk, top_p=tp)
    nflag, nbad, det = parity.compare_tree(g, o, sample=True)
    assert nbad == 0, det


def test_tiny_values_around_the_crossing(cuda_device):
    """Rows whose values cluster around zero: the window counts the values
    |v| < 2^-10 only together (with their exact mass), so a top-k crossing
    among them is left to the whole-row path, while crossings above or below
    them stay with the candidates; every record equals the whole-row one."""
    B, gamma, V = 8, 2, 30000
    inp = wl.chain_inputs(B, gamma, V, seed=9600, device="cuda", temperatures=(1.0,))
    g = torch.Generator(device="cuda").manual_seed(5)
    rows = inp.target[:, :, :V]
    tiny = (torch.rand(rows.shape, generator=g, device="cuda") - 0.5) * 2e-3       # |v| < 2^-10
    neg = -torch.rand(rows.shape, generator=g, device="cuda") * 8.0
    pick = torch.rand(rows.shape, generator=g, device="cuda")
    vals = torch.where(pick < 0.05, tiny, neg)
    vals[..., :20] = 4.0 + torch.rand(rows.shape[:-1] + (20,), generator=g, device="cuda")
    rows.copy_(vals.to(rows.dtype))
    # top_k 500 lands among the ~1500 tiny values; 10 above them; 3000 below them
    tk = torch.tensor([500, 10, 3000, 0, 500, 10, 3000, 0], dtype=torch.int32, device="cuda")
    tp = torch.tensor([1.0, 1.0, 1.0, 0.9, 0.9, 0.5, 0.99, 0.999], dtype=torch.float32, device="cuda")
    r = _ab(lambda: parity.gpu_chain_filtered(inp, tk, tp))
    assert r[0] > 0 and r[1] > 0, r
    out = parity.gpu_chain_filtered(inp, tk, tp)
    o = parity.oracle_chain_filtered(inp, tk, tp)
    nflag, nbad, det = parity.compare_chain(out, o, gamma)
    assert nbad == 0, det


def _spread(rows, V, seed):
    """bf16 values sign * 2^u, u uniform in [-60, 3]: every 1/8-binade bucket
    of both signs is populated."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    shape = rows.shape[:-1] + (V,)
    u = torch.rand(shape, generator=g, device="cuda") * 63.0 - 60.0
    sign = torch.where(torch.rand(shape, generator=g, device="cuda") < 0.5, -1.0, 1.0)
    rows[..., :V] = (sign * torch.exp2(u)).to(rows.dtype)


def test_windowed_filter_segments(cuda_device):
    """The windowed filter counts a window of more than WF_SLOTS keys in
    segments.  Values spread over 63 binades of both signs make such a window;
    top_k = 70000 puts the top-k key in the second segment while top_p = 0.5
    puts the top-p key in the first, so the top-p search must go back to the
    segments above.  The whole-row-only run (the windowed filter in every row)
    equals the oracle and the default run."""
    B, gamma, V = 4, 2, 131072
    inp = wl.chain_inputs(B, gamma, V, seed=9700, device="cuda", temperatures=(1.0,))
    _spread(inp.target, V, 11)
    _spread(inp.draft, V, 12)
    tk = torch.tensor([70000, 70000, 0, 40000], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.5, 0.9, 0.5, 1.0], dtype=torch.float32, device="cuda")
    d, rd = _run(0, lambda: parity.gpu_chain_filtered(inp, tk, tp))
    w, rw = _run(1, lambda: parity.gpu_chain_filtered(inp, tk, tp))
    _same(d, w)
    o = parity.oracle_chain_filtered(inp, tk, tp)
    for out in (d, w):
        nflag, nbad, det = parity.compare_chain(out, o, gamma)
        assert nbad == 0, det


def test_topk_cut_from_the_statistics(cuda_device):
    """A top-k row whose top_k is at most its number of statistics entries
    (one per warp of each 16 KB chunk: 52 for V = 100000) is first cut at the
    K-th largest entry, which surely holds the crossing: no row needs a
    deeper cut or the whole-row path, also where a cut at a fixed depth holds
    too few values or where thousands of values tie at the crossing (nearly
    flat rows; rows of four repeated levels).  The records equal the
    whole-row ones and the outputs equal the oracle's."""
    B, gamma, V = 8, 2, 100000
    inp = wl.chain_inputs(B, gamma, V, seed=9800, device="cuda", zipf=True, temperatures=(1.0,))
    g = torch.Generator(device="cuda").manual_seed(7)
    rows = inp.target[..., :V]
    flat = 5.0 + torch.randn(rows.shape, generator=g, device="cuda") * 0.05
    levels = torch.tensor([6.0, 5.5, 5.0, 4.5], device="cuda")
    lv = levels[torch.randint(0, 4, rows.shape, generator=g, device="cuda")]
    rows[0:2] = flat[0:2].to(rows.dtype)              # sequences 0-1: nearly flat around 5
    rows[2:4] = lv[2:4].to(rows.dtype)                # sequences 2-3: four repeated levels
    tk = torch.tensor([1, 20, 52, 7, 1, 20, 52, 7], dtype=torch.int32, device="cuda")
    tp = torch.ones(B, dtype=torch.float32, device="cuda")
    rd = _ab(lambda: parity.gpu_chain_filtered(inp, tk, tp))
    assert rd[0] == B * (2 * gamma + 1) and rd[1] == 0 and rd[2] == 0, rd
    out = parity.gpu_chain_filtered(inp, tk, tp)
    o = parity.oracle_chain_filtered(inp, tk, tp)
    nflag, nbad, det = parity.compare_chain(out, o, gamma)
    assert nbad == 0, det


def test_counting_off_by_default(cuda_device):
    """Mode -1 (the state at load) counts nothing."""
    sv.spec_debug_filter_path(-1, read=True)
    inp = wl.chain_inputs(4, 2, 5000, seed=9500, device="cuda", zipf=True)
    tk, tp = _params(4, 3)
    parity.gpu_chain_filtered(inp, tk, tp)
    assert sv.spec_debug_filter_path(-1, read=True) == (0, 0, 0)
