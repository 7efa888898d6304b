"""GPU parity of spec_verify_tree_mss (tree verification with a draft distribution,
SpecInfer multi-step speculative sampling) against the fp64 oracle, through the C ABI."""
import functools

import numpy as np
import pytest
import torch

import parity
import pins
from speculative_decoding_verify_temperature_b200 import workloads as wl
from speculative_decoding_verify_temperature_b200 import spec_verify as sv

pytestmark = pytest.mark.gpu


def _mss(inp, rows=None, max_flag_frac=0.2):
    g = parity.gpu_mss(inp)
    o = parity.oracle_mss(inp, rows)
    nflag, nbad, det = parity.compare_mss(g, o, rows)
    n = len(o["num_accepted"])
    assert nbad == 0, f"{nbad} unflagged mismatches of {n}: {det}"
    assert nflag <= max_flag_frac * n + 1
    return g, o


def _parents_fn(kind):
    if kind == "random":
        return lambda g: wl.random_tree(20, 4, g)
    if kind == "chain":
        return lambda g: wl.chain_tree(9)
    if kind == "root":
        return lambda g: [-1]
    if kind == "big":
        return lambda g: wl.random_tree(256, 6, g, max_depth=64)
    if kind == "wide":
        return lambda g: [-1] + [0] * 12 + [1] * 4
    return None


CASES = [
    # B, V, target dtype, tree kind, temperature, pad, draft noise
    (4, 1003, torch.bfloat16, "level", 0.8, 5, 1.0),
    (6, 20000, torch.bfloat16, "random", 1.0, 0, 2.0),
    (5, 8192 * 2 + 1, torch.bfloat16, "wide", 1.0, 7, 3.0),      # many rejections at the root
    (3, 4096 * 3 + 3, torch.float32, "chain", 0.6, 1, 1.0),
    (2, 9, torch.bfloat16, "root", 1.0, 0, 1.0),
    (4, 300, torch.bfloat16, "big", 1.7, 4, 1.5),
    (3, 300, torch.float32, "wide", 1.0, 4, 4.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}V{c[1]}{str(c[2])[-4:]}{c[3]}")
def test_mss_parity(case, cuda_device):
    B, V, dt, kind, T, pad, noise = case
    q = 16 // (2 if dt == torch.bfloat16 else 4)
    for seed in range(3):
        inp = wl.tree_mss_inputs(B, V, seed=500 + seed, device="cuda", parents_fn=_parents_fn(kind),
                                 target_dtype=dt, stride=-(-(V + pad) // q) * q, temperature=T,
                                 draft_noise=noise, zipf=V > 100)
        _mss(inp)


def test_mss_workload5_sampled(cuda_device):
    """B=128, 32-node trees, V=151936 bf16 + f32 draft distributions, launched at
    full size; the oracle checks 16 sequences one by one."""
    inp = wl.tree_config5(0, "cuda")
    g, o = _mss(inp, rows=np.arange(0, 128, 8))
    assert (g["num_accepted"] >= 0).all()


def test_mss_lossless_through_gpu_bruteforce(cuda_device):
    for kw in [dict(), dict(V=4, K=2, seed=3, parents=(-1, 0, 0, 0, 1, 1)), dict(V=3, K=2, seed=7,
                                                                            parents=(-1, 0, 0, 1, 2, 2), T=0.7)]:
        r = pins.tree_mss_bruteforce(runner=parity.gpu_tree_mss_runner, **kw)
        assert r["ok"], (kw, r)


def test_mss_chisquare_through_gpu(cuda_device):
    r = pins.tree_mss_chisquare(rounds=1_000_000, seed=16, runner=parity.gpu_tree_mss_runner)
    assert r["ok"], r


def test_mss_chain_tree_equals_chain_on_gpu(cuda_device):
    """Multi-step sampling on a chain-shaped tree == chain verify with draft
    probabilities, both on the GPU, same uniforms."""
    B, gamma, V = 32, 5, 7000
    g = torch.Generator(device="cuda").manual_seed(9)
    stride = -(-V // 8) * 8
    t = torch.zeros((B, gamma + 1, stride), dtype=torch.bfloat16, device="cuda")
    t[:, :, :V] = (torch.randn((B, gamma + 1, V), generator=g, device="cuda") * 2).to(torch.bfloat16)
    q = torch.zeros((B, gamma + 1, stride), device="cuda")
    q[:, :, :V] = torch.softmax(t[:, :, :V].float() + torch.randn((B, gamma + 1, V), generator=g, device="cuda"), -1)
    x = torch.multinomial(q[:, :gamma, :V].reshape(-1, V), 1, generator=g).view(B, gamma).to(torch.int32)
    coins = wl.uniforms((B, gamma), g, "cuda")
    fu = wl.uniforms((B,), g, "cuda")
    T = torch.ones(B, device="cuda")
    ct, ck = sv.spec_verify_chain(t, q[:, :gamma].contiguous(), x, T, coins, fu, draft_is_probs=True, V=V)
    tokens = torch.cat([torch.zeros((B, 1), dtype=torch.int32, device="cuda"), x], 1)
    parents = torch.arange(-1, gamma, dtype=torch.int32, device="cuda").expand(B, -1).contiguous()
    tc = torch.cat([torch.full((B, 1), 0.5, device="cuda"), coins], 1)
    ai, tt, tk = sv.spec_verify_tree_mss(t, tokens, parents, T, tc, fu, gamma, q, V=V)
    torch.cuda.synchronize()
    assert torch.equal(ck, tk)
    assert torch.equal(ct, tt)


def test_mss_invalid_and_deterministic(cuda_device):
    inp = wl.tree_mss_inputs(5, 3000, seed=12, device="cuda")
    inp.temperature[1] = 0.0
    inp.parents[2, 3] = 9
    inp.target[3, 0, 11] = float("nan")
    c = int(torch.nonzero(inp.parents[4] == 0)[0])       # first child of the root
    inp.draft_probs[4, 0, int(inp.tokens[4, c])] = -1.0   # its q(x) < 0
    ws = sv.Workspace("cuda")
    buf = ws.get(sv.SPEC_ENTRY_TREE_MSS, inp.B, inp.N, inp.V)
    g = parity.gpu_mss(inp, workspace=buf)
    assert list(g["num_accepted"][1:]) == [-1] * 4
    assert (g["tokens"][1:] == -1).all() and np.isnan(g["ptest"][1:]).all()
    assert g["num_accepted"][0] >= 0
    assert sv.spec_read_device_status(buf) & (1 << sv.SPEC_ERR_DEVICE_INPUT)
    o = parity.oracle_mss(inp)
    assert list(o["num_accepted"][1:]) == [-1] * 4
    for _ in range(3):
        h = parity.gpu_mss(inp, workspace=buf)
        for key in ("tokens", "accept_index", "num_accepted"):
            assert (h[key] == g[key]).all()
        np.testing.assert_array_equal(h["ptest"], g["ptest"])


# ----------------------------------------------------------------------------- lazy walk

def _lazy_same(inp):
    d = parity.gpu_mss(inp)
    z = parity.gpu_mss(inp, lazy=True)
    for key in ("accept_index", "tokens", "num_accepted"):
        np.testing.assert_array_equal(z[key], d[key])
    valid = d["num_accepted"] >= 0
    np.testing.assert_array_equal(z["ptest"][valid], d["ptest"][valid])     # NaN where untested, both
    np.testing.assert_array_equal(z["S"][valid], d["S"][valid])
    return z


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}V{c[1]}{str(c[2])[-4:]}{c[3]}")
def test_mss_lazy_equals_dense(case, cuda_device):
    B, V, dt, kind, T, pad, noise = case
    q = 16 // (2 if dt == torch.bfloat16 else 4)
    for seed in range(3):
        inp = wl.tree_mss_inputs(B, V, seed=600 + seed, device="cuda", parents_fn=_parents_fn(kind),
                                 target_dtype=dt, stride=-(-(V + pad) // q) * q, temperature=T,
                                 draft_noise=noise, zipf=V > 100)
        z = _lazy_same(inp)
        nflag, nbad, det = parity.compare_mss(z, parity.oracle_mss(inp))
        assert nbad == 0, det


def test_mss_lazy_workload5(cuda_device):
    inp = wl.tree_config5(1, "cuda")
    z = _lazy_same(inp)
    rows = np.arange(3, 128, 16)
    nflag, nbad, det = parity.compare_mss(z, parity.oracle_mss(inp, rows), rows)
    assert nbad == 0, det


def test_mss_lazy_through_pins(cuda_device):
    run = functools.partial(parity.gpu_tree_mss_runner, lazy=True)
    for kw in [dict(), dict(V=4, K=2, seed=3, parents=(-1, 0, 0, 0, 1, 1))]:
        r = pins.tree_mss_bruteforce(runner=run, **kw)
        assert r["ok"], (kw, r)
    r = pins.tree_mss_chisquare(rounds=1_000_000, seed=17, runner=run)
    assert r["ok"], r


def test_mss_lazy_validation(cuda_device):
    """Tree structure and temperature are always checked; a NaN in the row of a
    node the walk never visits invalidates only the dense call."""
    inp = wl.tree_mss_inputs(4, 3000, seed=21, device="cuda")
    inp.temperature[1] = float("inf")
    inp.parents[2, 5] = 30
    d0 = parity.gpu_mss(inp)
    last = inp.N - 1
    planted = last not in set(d0["accept_index"][3].tolist())
    if planted:
        inp.target[3, last, 7] = float("nan")
    z = parity.gpu_mss(inp, lazy=True)
    assert list(z["num_accepted"][1:3]) == [-1, -1]
    assert z["num_accepted"][3] == d0["num_accepted"][3] and (z["tokens"][3] == d0["tokens"][3]).all()
    if planted:
        assert parity.gpu_mss(inp)["num_accepted"][3] == -1
