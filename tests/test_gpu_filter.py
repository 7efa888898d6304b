"""GPU parity of spec_verify_chain_filtered (chain verify under top-k / top-p
filtered temperature sampling) against the fp64 oracle, through the C ABI."""
import functools

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


def _check(inp, tk, tp, rows=None, max_flag_frac=0.2):
    g = parity.gpu_chain_filtered(inp, tk, tp)
    o = parity.oracle_chain_filtered(inp, tk, tp, rows)
    nflag, nbad, det = parity.compare_chain(g, o, inp.gamma, rows)
    n = len(o["num_accepted"])
    assert nbad == 0, f"{nbad} unflagged mismatches of {n}: {det}"
    assert nflag <= max_flag_frac * n + 1, f"too many near-ties: {nflag}/{n}"
    # without diagnostics (bf16 rows) only the rows the decision reaches are
    # filtered: the same records there, so the same decisions and tokens
    d = parity.gpu_chain_filtered(inp, tk, tp, with_diag=False)
    np.testing.assert_array_equal(d["num_accepted"], g["num_accepted"])
    np.testing.assert_array_equal(d["tokens"], g["tokens"])
    # the row-on-demand walk: the same records for the rows it reaches, the
    # same outputs; diagnostics where it evaluated them, NaN after
    z = parity.gpu_chain_filtered(inp, tk, tp, lazy=True)
    np.testing.assert_array_equal(z["num_accepted"], g["num_accepted"])
    np.testing.assert_array_equal(z["tokens"], g["tokens"])
    for b, k in enumerate(g["num_accepted"]):
        if k < 0:
            continue
        ev = min(k + 1, inp.gamma)
        np.testing.assert_array_equal(z["px"][b, :ev], g["px"][b, :ev])
        np.testing.assert_array_equal(z["qx"][b, :ev], g["qx"][b, :ev])
        assert np.isnan(z["px"][b, ev:]).all()
        assert z["S"][b] == g["S"][b]
    return g, o


CASES = [
    # B, gamma, V, tdt, draft (dtype or "probs"), stride pad, temperatures
    (8, 3, 1003, torch.bfloat16, torch.bfloat16, 5, (1.0,)),
    (8, 4, 8193, torch.bfloat16, torch.bfloat16, 7, (0.6, 1.0)),
    (6, 2, 20000, torch.bfloat16, torch.float32, 0, (1.3,)),
    (6, 3, 4096 * 3 + 5, torch.float32, torch.float32, 3, (0.8,)),
    (6, 5, 30001, torch.bfloat16, "probs", 3, (1.0,)),
    (4, 2, 5000, torch.float32, "probs", 0, (0.7,)),
    (3, 1, 1, torch.float32, torch.float32, 3, (1.0,)),
    (5, 2, 7, torch.bfloat16, torch.bfloat16, 1, (1.0,)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}g{c[1]}V{c[2]}{str(c[3])[-4:]}{str(c[4])[-5:]}")
def test_filtered_parity(case, cuda_device):
    B, gamma, V, tdt, dk, pad, temps = case
    probs = dk == "probs"
    ddt = torch.float32 if probs else dk
    for seed in range(3):
        q = 16 // (2 if tdt == torch.bfloat16 else 4)
        qd = 16 // (2 if ddt == torch.bfloat16 else 4)
        inp = wl.chain_inputs(B, gamma, V, seed=7000 + seed, device="cuda", target_dtype=tdt, draft_dtype=ddt,
                              draft_is_probs=probs, zipf=V > 100, temperatures=temps,
                              stride=-(-(V + pad) // q) * q, dstride=-(-(V + pad) // qd) * qd)
        tk, tp = _params(B, V, seed)
        _check(inp, tk, tp)
        _check(inp, tk, None)
        _check(inp, None, tp)


def test_filtered_ties_and_signed_zero(cuda_device):
    """Integer-valued logits (many ties, including -0 and +0): top-k keeps every
    token tied with the k-th largest value, exactly as the oracle."""
    B, gamma, V = 16, 3, 777
    inp = wl.chain_inputs(B, gamma, V, seed=42, device="cuda", target_dtype=torch.bfloat16,
                          stride=784, dstride=784)
    g = torch.Generator(device="cuda").manual_seed(3)
    ints = torch.randint(-4, 5, (B, gamma + 1, V), generator=g, device="cuda").float()
    neg = torch.rand(ints.shape, generator=g, device="cuda") < 0.5
    ints = torch.where((ints == 0) & neg, torch.full_like(ints, -0.0), ints)          # -0 and +0 both present
    inp.target[:, :, :V] = ints.to(torch.bfloat16)
    inp.draft[:, :, :V] = (ints[:, :gamma] + torch.randint(-1, 2, (B, gamma, V), generator=g, device="cuda")).to(torch.bfloat16)
    tk = torch.tensor([1, 2, 3, 10, 100, 0, 7, 1] * 2, dtype=torch.int32, device="cuda")
    tp = torch.tensor([1.0, 0.9, 0.6, 1.0, 0.4, 0.7, 1.0, 0.25] * 2, dtype=torch.float32, device="cuda")
    _check(inp, tk, tp)


def test_filtered_workload1_shape(cuda_device):
    """B=64, gamma=5, V=32000 bf16 logits with serving-style filters."""
    for r in range(2):
        inp = wl.chain_config1(r, "cuda")
        tk, tp = _params(inp.B, inp.V, 100 + r)
        _check(inp, tk, tp)


@pytest.mark.parametrize("lazy", [False, True])
def test_filtered_lossless_through_gpu(lazy, cuda_device):
    run = functools.partial(parity.gpu_chain_runner, lazy=lazy)
    for kw in [dict(), dict(V=4, gamma=2, seed=5, T=0.7, top_k=0, top_p=0.61),
               dict(V=3, gamma=3, K=3, seed=8, top_k=2, top_p=0.77),
               dict(draft_kind="probs", seed=2, top_k=2, top_p=0.9, tol=1e-7)]:
        r = pins.chain_filtered_bruteforce(runner=run, **kw)
        assert r["ok"], (kw, r)


def test_filtered_invalid_parameters(cuda_device):
    B, gamma, V = 6, 2, 3000
    inp = wl.chain_inputs(B, gamma, V, seed=9, device="cuda")
    tk = torch.tensor([0, -1, 5, 0, 3, 0], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.9, 0.9, 0.0, float("nan"), 1.5, 1.0], dtype=torch.float32, device="cuda")
    ws = sv.Workspace("cuda")
    buf = ws.get(sv.SPEC_ENTRY_CHAIN, B, gamma, V)
    g = parity.gpu_chain_filtered(inp, tk, tp, workspace=buf)
    assert list(g["num_accepted"][1:5]) == [-1] * 4
    assert g["num_accepted"][0] >= 0 and g["num_accepted"][5] >= 0
    assert sv.spec_read_device_status(buf) & (1 << sv.SPEC_ERR_DEVICE_INPUT)
    o = parity.oracle_chain_filtered(inp, tk, tp)
    assert list(o["num_accepted"][1:5]) == [-1] * 4
    z = parity.gpu_chain_filtered(inp, tk, tp, lazy=True)
    assert list(z["num_accepted"][1:5]) == [-1] * 4 and z["num_accepted"][0] >= 0
    with pytest.raises(ValueError):
        sv.spec_verify_chain_filtered(inp.target, inp.draft, inp.draft_tokens, inp.temperature, inp.coins,
                                      inp.final_u)


def test_filtered_value_repeated_beyond_16_bits(cuda_device):
    """bf16 rows longer than 65535 where one value repeats more than 65535 times
    (the window's counters are 32-bit); results match the oracle.  Also a long
    row without repeats."""
    B, gamma, V = 3, 2, 70000
    inp = wl.chain_inputs(B, gamma, V, seed=77, device="cuda", zipf=True, stride=70000, dstride=70000)
    inp.target[0, :, :V - 40] = 0.0                     # value 0 repeated 69960 times per row
    inp.draft[0, :, :V - 40] = 0.0
    tk = torch.tensor([5, 0, 100], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.9, 0.8, 1.0], dtype=torch.float32, device="cuda")
    _check(inp, tk, tp)


def test_filtered_thresholds_far_below_the_maximum(cuda_device):
    """Flat rows (logits spread over [-40, 40], T = 30, so bf16 values of both
    signs and every magnitude carry mass) where the top-p threshold and a top_k
    close to V lie far below the row's maximum: the windowed histogram has to
    move its window down (and count the row again) before it finds them."""
    B, gamma, V = 12, 2, 40000
    inp = wl.chain_inputs(B, gamma, V, seed=78, device="cuda", temperatures=(30.0,))
    g = torch.Generator(device="cuda").manual_seed(5)
    flat = (torch.rand((B, gamma + 1, V), generator=g, device="cuda") * 80.0 - 40.0)
    inp.target[:, :, :V] = flat.to(torch.bfloat16)
    inp.draft[:, :, :V] = (flat[:, :gamma] + torch.randn((B, gamma, V), generator=g, device="cuda")).to(torch.bfloat16)
    tk = torch.tensor([0, V - 3, 30000, 0, 0, 25000, 1, 0, V - 1, 0, 12000, 0], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.99, 1.0, 0.9, 0.5, 0.999, 1.0, 0.9, 0.2, 0.95, 0.75, 1.0, 0.97], dtype=torch.float32,
                      device="cuda")
    _check(inp, tk, tp)
