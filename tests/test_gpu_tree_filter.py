"""GPU parity of spec_verify_tree_sample_filtered (target-only tree sampling on
top-k / top-p filtered node rows) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import parity
import pins
from speculative_decoding_verify_temperature_b200 import workloads as wl
from speculative_decoding_verify_temperature_b200 import spec_verify as sv

pytestmark = pytest.mark.gpu


def _params(B, V, seed):
    g = np.random.default_rng(seed)
    ks = np.array([0, 1, 2, 5, 50, max(1, V - 1), V, V + 10], np.int32)
    ps = np.array([1.0, 0.95, 0.8, 0.5, 1e-3, 0.3], np.float32)
    tk = torch.from_numpy(g.choice(ks, B).astype(np.int32)).cuda()
    tp = torch.from_numpy(g.choice(ps, B).astype(np.float32)).cuda()
    return tk, tp


def _check(inp, tk, tp, rows=None, max_flag_frac=0.2, **th):
    g = parity.gpu_sample(inp, top_k=tk, top_p=tp, **th)
    o = parity.oracle_sample(inp, rows, top_k=tk, top_p=tp, **th)
    nflag, nbad, det = parity.compare_tree(g, o, rows, sample=True)
    n = len(o["num_accepted"])
    assert nbad == 0, f"{nbad} unflagged mismatches of {n}: {det}"
    assert nflag <= max_flag_frac * n + 1, f"too many near-ties: {nflag}/{n}"
    # without diagnostics (bf16 rows) the walk filters only the rows it
    # visits: the same records, so the same walk and tokens
    d = parity.gpu_sample(inp, top_k=tk, top_p=tp, with_diag=False, **th)
    for key in ("num_accepted", "tokens", "accept_index"):
        np.testing.assert_array_equal(d[key], g[key])
    return g, o


def _q(dt):
    return 16 // (2 if dt == torch.bfloat16 else 4)


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


CASES = [
    # B, V, dtype, parents kind, draft_probs, temperature, pad
    (8, 1003, torch.bfloat16, "level", None, 0.8, 5),
    (8, 20000, torch.bfloat16, "random", "zeros", 1.0, 0),
    (8, 20000, torch.bfloat16, "random", "random", 1.0, 0),
    (6, 8192 * 2 + 3, torch.float32, "chain", None, 0.6, 1),
    (4, 9, torch.bfloat16, "root", None, 1.0, 0),
    (4, 300, torch.bfloat16, "big", None, 1.7, 4),
    (4, 300, torch.float32, "big", "random", 1.0, 4),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}V{c[1]}{str(c[2])[-4:]}{c[3]}{c[4]}")
def test_tree_filtered_parity(case, cuda_device):
    B, V, dt, kind, dp, T, pad = case
    for seed in range(3):
        stride = -(-(V + pad) // _q(dt)) * _q(dt)
        inp = wl.tree_sample_inputs(B, V, seed=8300 + seed, device="cuda", parents_fn=_parents_fn(kind),
                                    target_dtype=dt, stride=stride, temperature=T, draft_probs=dp,
                                    zipf=V > 100)
        tk, tp = _params(B, V, seed)
        _check(inp, tk, tp)
        _check(inp, tk, None)
        _check(inp, None, tp)


def test_tree_filtered_thresholds(cuda_device):
    inp = wl.tree_sample_inputs(6, 5000, seed=8310, device="cuda")
    tk, tp = _params(6, 5000, 4)
    for ts, ta in [(0.05, 1.0), (1.0, 0.5)]:
        _check(inp, tk, tp, threshold_single=ts, threshold_acc=ta)


def test_tree_filtered_filters_off_equal_unfiltered(cuda_device):
    """top_k 0 and top_p 1 everywhere: the filtered entry point emits what the
    unfiltered one does, bit for bit (diagnostics included)."""
    inp = wl.tree_sample_inputs(8, 20000, seed=8320, device="cuda", draft_probs="random")
    tk = torch.zeros(8, dtype=torch.int32, device="cuda")
    tp = torch.ones(8, dtype=torch.float32, device="cuda")
    a = parity.gpu_sample(inp)
    b = parity.gpu_sample(inp, top_k=tk, top_p=tp)
    for key in ("accept_index", "tokens", "num_accepted"):
        np.testing.assert_array_equal(a[key], b[key])
    np.testing.assert_array_equal(a["pchild"], b["pchild"])


def test_tree_filtered_topk1_is_greedy_on_gpu(cuda_device):
    """top_k = 1 on tie-free rows: filtered sampling walks exactly as greedy
    verification (both on the GPU)."""
    B, V = 32, 3000
    inp = wl.tree_sample_inputs(B, V, seed=8330, device="cuda", target_dtype=torch.float32, zipf=False,
                                parents_fn=lambda g: wl.random_tree(16, 4, g))
    am = inp.target[:, :, :V].argmax(dim=2)
    par = inp.parents.long()
    hit = torch.rand((B, inp.N), device="cuda") < 0.6
    tok = inp.tokens.clone()
    for n in range(1, inp.N):
        want = am[torch.arange(B, device="cuda"), par[:, n]].to(torch.int32)
        tok[:, n] = torch.where(hit[:, n], want, tok[:, n])
    inp.tokens = tok
    s = parity.gpu_sample(inp, top_k=torch.ones(B, dtype=torch.int32, device="cuda"))
    g = parity.gpu_greedy(inp)
    np.testing.assert_array_equal(s["num_accepted"], g["num_accepted"])
    np.testing.assert_array_equal(s["accept_index"], g["accept_index"])
    np.testing.assert_array_equal(s["tokens"], g["tokens"])


@pytest.mark.parametrize("kw", [
    dict(top_k=2, top_p=None),
    dict(top_k=None, top_p=0.7),
    dict(top_k=3, top_p=0.8, V=4, K=2, seed=3, parents=(-1, 0, 0, 1, 2)),
    dict(top_k=2, top_p=0.9, T=0.7, seed=8, draft_probs_zero=True),
])
def test_tree_filtered_lossless_through_gpu(kw, cuda_device):
    r = pins.tree_bruteforce(runner=parity.gpu_tree_sample_runner, **kw)
    assert r["ok"], (kw, r)


def test_tree_filtered_invalid_parameters(cuda_device):
    inp = wl.tree_sample_inputs(5, 3000, seed=8340, device="cuda")
    tk = torch.tensor([20, -1, 20, 20, 0], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.9, 0.9, 0.0, 1.5, 0.9], dtype=torch.float32, device="cuda")
    g, o = _check(inp, tk, tp)
    assert list(o["num_accepted"][1:4]) == [-1, -1, -1]
    assert list(g["num_accepted"][1:4]) == [-1, -1, -1]
    with pytest.raises(ValueError):
        sv.spec_verify_tree_sample_filtered(inp.target, inp.tokens, inp.parents, inp.temperature, inp.coins,
                                            inp.final_u, inp.max_depth)


def test_tree_filtered_workload3_shapes(cuda_device):
    """B=128, 32-node trees, V=151936 bf16, T=0.8, per-sequence top-k / top-p;
    launched at full size, the oracle checks 16 sequences one by one."""
    inp = wl.tree_config3(0, "cuda")
    tk, tp = _params(inp.B, inp.V, 9)
    _check(inp, tk, tp, rows=np.arange(0, 128, 8))


# ----------------------------------------------------------------------------- the lazy walk

def _lazy_same(inp, tk, tp):
    """Lazy == dense on tokens, accept indices and counts; child probabilities
    equal where the lazy walk evaluated them (children of visited nodes), NaN
    elsewhere; the final residual mass equal."""
    d = parity.gpu_sample(inp, top_k=tk, top_p=tp)
    z = parity.gpu_sample(inp, top_k=tk, top_p=tp, lazy=True)
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
        assert z["S"][b] == d["S"][b]
    return z


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}V{c[1]}{str(c[2])[-4:]}{c[3]}{c[4]}")
def test_tree_filtered_lazy_equals_dense(case, cuda_device):
    B, V, dt, kind, dp, T, pad = case
    for seed in range(2):
        stride = -(-(V + pad) // _q(dt)) * _q(dt)
        inp = wl.tree_sample_inputs(B, V, seed=8400 + seed, device="cuda", parents_fn=_parents_fn(kind),
                                    target_dtype=dt, stride=stride, temperature=T, draft_probs=dp,
                                    zipf=V > 100)
        tk, tp = _params(B, V, 10 + seed)
        _lazy_same(inp, tk, tp)
        _lazy_same(inp, tk, None)


def test_tree_filtered_lazy_workload3_shapes(cuda_device):
    inp = wl.tree_config3(0, "cuda")
    tk, tp = _params(inp.B, inp.V, 11)
    _lazy_same(inp, tk, tp)


@pytest.mark.parametrize("kw", [dict(top_k=2, top_p=None), dict(top_k=3, top_p=0.8, V=4, K=2, seed=3,
                                                                 parents=(-1, 0, 0, 1, 2))])
def test_tree_filtered_lazy_lossless_through_gpu(kw, cuda_device):
    import functools
    r = pins.tree_bruteforce(runner=functools.partial(parity.gpu_tree_sample_runner, lazy=True), **kw)
    assert r["ok"], (kw, r)
