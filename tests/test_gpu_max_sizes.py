"""GPU parity at the limits the C ABI accepts: V = 2^20 (the largest vocabulary) for
every entry point, dense and lazy, gamma = 16 at that V, 256-node trees, and a
depth-64 chain-shaped tree.  Inputs are seeded and synthetic; the oracle checks
every sequence."""
import numpy as np
import pytest
import torch

import parity
import test_gpu_lazy as lazy_checks
import test_gpu_mss as mss_checks
from speculative_decoding_verify_temperature_b200 import workloads as wl

pytestmark = pytest.mark.gpu

V_MAX = 1 << 20                 # SPEC_MAX_V in include/spec_verify.h
GAMMA_MAX = 16                  # SPEC_MAX_GAMMA
NODES_MAX = 256                 # SPEC_MAX_NODES
DEPTH_MAX = 64                  # SPEC_MAX_DEPTH


def _chain(inp, lazy=False, tk=None, tp=None):
    """Dense: parity with the oracle.  Lazy: the lazy checks (equal to the dense
    path, diagnostics only where evaluated, and parity with the oracle)."""
    if lazy:
        lazy_checks._chain_same(inp)
        lazy_checks._chain_vs_oracle(inp)
        return None, None
    if tk is not None or tp is not None:
        g = parity.gpu_chain_filtered(inp, tk, tp)
        o = parity.oracle_chain_filtered(inp, tk, tp)
    else:
        g = parity.gpu_chain(inp)
        o = parity.oracle_chain(inp)
    nflag, nbad, det = parity.compare_chain(g, o, inp.gamma)
    assert nbad == 0, det
    assert nflag <= 1
    return g, o


@pytest.mark.parametrize("lazy", [False, True])
def test_chain_max_vocab(lazy, cuda_device):
    for seed, probs in [(0, False), (1, True)]:
        inp = wl.chain_inputs(2, 3, V_MAX, seed=9100 + seed, device="cuda", draft_is_probs=probs,
                              draft_dtype=torch.float32 if probs else torch.bfloat16, zipf=True,
                              temperatures=(0.6, 1.0))
        _chain(inp, lazy=lazy)


def test_chain_max_gamma_max_vocab(cuda_device):
    inp = wl.chain_inputs(1, GAMMA_MAX, V_MAX, seed=9110, device="cuda", zipf=True, draft_noise=0.3,
                          temperatures=(1.0,))
    g, o = _chain(inp)
    assert o["num_accepted"][0] >= 0


def test_chain_filtered_max_vocab(cuda_device):
    inp = wl.chain_inputs(3, 2, V_MAX, seed=9120, device="cuda", zipf=True, temperatures=(0.6, 1.0))
    tk = torch.tensor([50, 0, V_MAX - 1], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.9, 0.95, 0.5], dtype=torch.float32, device="cuda")
    _chain(inp, tk=tk, tp=tp)


@pytest.mark.parametrize("lazy", [False, True])
def test_greedy_max_vocab(lazy, cuda_device):
    inp = wl.tree_greedy_inputs(2, V_MAX, seed=9130, device="cuda",
                                parents_fn=lambda g: wl.random_tree(12, 4, g), p_match=0.8)
    g = parity.gpu_greedy(inp, lazy=lazy)
    o = parity.oracle_greedy(inp)
    nflag, nbad, det = parity.compare_tree(g, o)
    assert nbad == 0, det
    if lazy:
        d = parity.gpu_greedy(inp)
        for key in ("accept_index", "tokens", "num_accepted"):
            np.testing.assert_array_equal(g[key], d[key])


@pytest.mark.parametrize("lazy", [False, True])
def test_sample_max_vocab(lazy, cuda_device):
    inp = wl.tree_sample_inputs(2, V_MAX, seed=9140, device="cuda",
                                parents_fn=lambda g: wl.random_tree(10, 3, g))
    inp.coins = inp.coins * 0.2                  # still uniforms in [0, 1); the walks go deeper
    if lazy:
        lazy_checks._sample_same(inp)            # equal to the dense path, checked below
    g = parity.gpu_sample(inp)
    o = parity.oracle_sample(inp)
    nflag, nbad, det = parity.compare_tree(g, o, sample=True)
    assert nbad == 0, det
    assert nflag <= 1


@pytest.mark.parametrize("lazy", [False, True])
def test_mss_max_vocab(lazy, cuda_device):
    inp = wl.tree_mss_inputs(2, V_MAX, seed=9150, device="cuda",
                             parents_fn=lambda g: [-1, 0, 0, 0, 1, 1, 4, 4], draft_noise=2.0)
    if lazy:
        mss_checks._lazy_same(inp)               # equal to the dense path, checked below
    g = parity.gpu_mss(inp)
    o = parity.oracle_mss(inp)
    nflag, nbad, det = parity.compare_mss(g, o)
    assert nbad == 0, det
    assert nflag <= 1


def test_sample_max_nodes(cuda_device):
    inp = wl.tree_sample_inputs(3, 1 << 16, seed=9160, device="cuda",
                                parents_fn=lambda g: wl.random_tree(NODES_MAX, 6, g, max_depth=DEPTH_MAX))
    assert inp.N == NODES_MAX
    g = parity.gpu_sample(inp)
    o = parity.oracle_sample(inp)
    nflag, nbad, det = parity.compare_tree(g, o, sample=True)
    assert nbad == 0, det


def test_max_depth_chain_shaped_trees(cuda_device):
    """A chain-shaped tree of depth 64 (65 nodes): sampling with drafts that the
    target mostly accepts walks deep; greedy with matching tokens walks to the end."""
    parents = wl.chain_tree(DEPTH_MAX + 1)
    s = wl.tree_sample_inputs(2, 3000, seed=9170, device="cuda", parents_fn=lambda g: parents,
                              temperature=1.0, token_noise=0.05)
    s.coins = s.coins * 1e-4                     # nearly every test accepts
    assert s.max_depth == DEPTH_MAX
    g = parity.gpu_sample(s)
    o = parity.oracle_sample(s)
    nflag, nbad, det = parity.compare_tree(g, o, sample=True)
    assert nbad == 0, det
    assert (o["num_accepted"] == DEPTH_MAX).all()
    gr = wl.tree_greedy_inputs(2, 3000, seed=9171, device="cuda", parents_fn=lambda g: parents, p_match=1.0)
    g = parity.gpu_greedy(gr)
    o = parity.oracle_greedy(gr)
    nflag, nbad, det = parity.compare_tree(g, o)
    assert nbad == 0, det
    assert (o["num_accepted"] == DEPTH_MAX).all()
