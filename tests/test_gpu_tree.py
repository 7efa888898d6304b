"""GPU parity of spec_verify_tree_greedy / spec_verify_tree_sample against the fp64 oracle."""
import numpy as np
import pytest
import torch

import parity
import pins
from speculative_decoding_verify_temperature_b200 import workloads as wl
from speculative_decoding_verify_temperature_b200 import spec_verify as sv

pytestmark = pytest.mark.gpu


def _greedy(inp, rows=None):
    g = parity.gpu_greedy(inp)
    o = parity.oracle_greedy(inp, rows)
    nflag, nbad, det = parity.compare_tree(g, o, rows)
    assert nbad == 0, det
    return g, o


def _sample(inp, rows=None, max_flag_frac=0.2, **th):
    g = parity.gpu_sample(inp, **th)
    o = parity.oracle_sample(inp, rows, **th)
    nflag, nbad, det = parity.compare_tree(g, o, rows, sample=True)
    n = len(o["num_accepted"])
    assert nbad == 0, f"{nbad} unflagged mismatches of {n}: {det}"
    assert nflag <= max_flag_frac * n + 1
    return g, o


def _q(dt):
    return 16 // (2 if dt == torch.bfloat16 else 4)


GREEDY = [
    # B, V, dtype, parents kind, int_logits (ties), pad
    (4, 1003, torch.bfloat16, "level", None, 5),
    (6, 20000, torch.bfloat16, "random", 3, 0),
    (5, 8192 * 2 + 1, torch.bfloat16, "chain", None, 7),
    (3, 5000, torch.float32, "random", 2, 1),
    (2, 9, torch.bfloat16, "root", None, 0),
    (8, 300, torch.bfloat16, "big", 2, 4),
]


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


@pytest.mark.parametrize("case", GREEDY, ids=lambda c: f"B{c[0]}V{c[1]}{c[3]}")
def test_greedy_parity(case, cuda_device):
    B, V, dt, kind, ties, pad = case
    for seed in range(3):
        stride = -(-(V + pad) // _q(dt)) * _q(dt)
        inp = wl.tree_greedy_inputs(B, V, seed=200 + seed, device="cuda", parents_fn=_parents_fn(kind),
                                    target_dtype=dt, stride=stride, int_logits=ties, p_match=0.8)
        _greedy(inp)


def test_greedy_workload2(cuda_device):
    """B=32, 64-node trees, V=128256 bf16: every sequence, 2 rounds."""
    for r in range(2):
        g, o = _greedy(wl.tree_config2(r, "cuda"))
        assert (o["num_accepted"] >= 0).all()


def test_greedy_equals_argmax_decoding_through_gpu(cuda_device):
    r = pins.greedy_equivalence(steps=4000, runner=parity.gpu_tree_greedy_runner)
    assert r["ok"], r


def test_greedy_invalid(cuda_device):
    inp = wl.tree_greedy_inputs(5, 4000, seed=9, device="cuda", parents_fn=lambda g: wl.random_tree(10, 3, g))
    inp.target[1, 4, 7] = float("nan")
    inp.parents[2, 5] = 7                          # parent after child
    inp.tokens[3, 2] = -3                          # token out of range
    inp.parents[4, 0] = 0                          # root must have parent -1
    g, o = _greedy(inp)
    assert list(g["num_accepted"][1:]) == [-1] * 4


SAMPLE = [
    # B, V, dtype, parents kind, draft_probs, temperature, pad
    (4, 1003, torch.bfloat16, "level", None, 0.8, 5),
    (5, 20000, torch.bfloat16, "random", "zeros", 1.0, 0),
    (5, 20000, torch.bfloat16, "random", "random", 1.0, 0),
    (3, 8192 * 2 + 3, torch.float32, "chain", None, 0.6, 1),
    (2, 9, torch.bfloat16, "root", None, 1.0, 0),
    (4, 300, torch.bfloat16, "big", None, 1.7, 4),
    (4, 300, torch.float32, "big", "random", 1.0, 4),
]


@pytest.mark.parametrize("case", SAMPLE, ids=lambda c: f"B{c[0]}V{c[1]}{c[3]}{c[4]}")
def test_sample_parity(case, cuda_device):
    B, V, dt, kind, dp, T, pad = case
    for seed in range(3):
        stride = -(-(V + pad) // _q(dt)) * _q(dt)
        inp = wl.tree_sample_inputs(B, V, seed=300 + seed, device="cuda", parents_fn=_parents_fn(kind),
                                    target_dtype=dt, stride=stride, temperature=T, draft_probs=dp,
                                    zipf=V > 100)
        _sample(inp)


def test_sample_thresholds(cuda_device):
    inp = wl.tree_sample_inputs(6, 5000, seed=77, device="cuda")
    for ts, ta in [(0.05, 1.0), (1.0, 0.5), (0.3, 0.7)]:
        _sample(inp, threshold_single=ts, threshold_acc=ta)


def test_sample_workload3_sampled(cuda_device):
    """B=128, 32-node trees, V=151936 bf16, T=0.8, draft_probs NULL, launched at full
    size; the oracle checks 32 sequences one by one.  The explicit zero buffer gives
    the same outputs."""
    inp = wl.tree_config3(0, "cuda")
    rows = np.arange(0, 128, 4)
    g, o = _sample(inp, rows=rows)
    inp.draft_probs = torch.zeros((inp.B, inp.N, inp.V), dtype=torch.float32, device="cuda")
    g2 = parity.gpu_sample(inp)
    assert (g["tokens"] == g2["tokens"]).all() and (g["num_accepted"] == g2["num_accepted"]).all()


def test_sample_lossless_through_gpu_bruteforce(cuda_device):
    for kw in [dict(), dict(draft_probs_zero=True, seed=8, T=0.8), dict(parents=(-1, 0, 1, 2), V=4, K=2, seed=15)]:
        r = pins.tree_bruteforce(runner=parity.gpu_tree_sample_runner, **kw)
        assert r["ok"], (kw, r)


def test_sample_chisquare_through_gpu(cuda_device):
    r = pins.tree_chisquare(rounds=1_000_000, seed=6, runner=parity.gpu_tree_sample_runner)
    assert r["ok"], r


def test_sample_chain_tree_equals_chain_onehot_on_gpu(cuda_device):
    """Target-only tree on a chain-shaped tree == chain verify with one-hot draft
    probabilities, both on the GPU, same uniforms."""
    B, gamma, V = 16, 5, 7000
    g = torch.Generator(device="cuda").manual_seed(5)
    t = (torch.randn((B, gamma + 1, V), generator=g, device="cuda") * 2).to(torch.bfloat16)
    x = torch.randint(0, V, (B, gamma), generator=g, device="cuda", dtype=torch.int32)
    q = torch.zeros((B, gamma, V), device="cuda")
    q.scatter_(2, x.long().unsqueeze(-1), 1.0)
    coins = wl.uniforms((B, gamma), g, "cuda") * 0.05
    fu = wl.uniforms((B,), g, "cuda")
    T = torch.full((B,), 0.9, device="cuda")
    stride = -(-V // 8) * 8
    tp = torch.zeros((B, gamma + 1, stride), dtype=torch.bfloat16, device="cuda")
    tp[:, :, :V] = t
    qp = torch.zeros((B, gamma, stride), device="cuda")
    qp[:, :, :V] = q
    ct, ck = sv.spec_verify_chain(tp, qp, x, T, coins, fu, draft_is_probs=True, V=V)
    tokens = torch.cat([torch.zeros((B, 1), dtype=torch.int32, device="cuda"), x], 1).contiguous()
    parents = torch.arange(-1, gamma, dtype=torch.int32, device="cuda").expand(B, -1).contiguous()
    tc = torch.cat([coins, torch.full((B, 1), 0.5, device="cuda")], 1).contiguous()
    ai, tt, tk = sv.spec_verify_tree_sample(tp, tokens, parents, T, tc, fu, gamma, V=V)
    assert (ck == tk).all()
    for b in range(B):
        k = int(ck[b])
        assert (ct[b, :k + 1] == tt[b, :k + 1]).all()
