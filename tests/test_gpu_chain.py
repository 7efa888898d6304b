"""GPU parity of spec_verify_chain against the fp64 oracle (run through the C ABI)."""
import numpy as np
import pytest
import torch

import parity
import pins
from speculative_decoding_verify_temperature_b200 import workloads as wl
from speculative_decoding_verify_temperature_b200 import spec_verify as sv

pytestmark = pytest.mark.gpu


def _check(inp, rows=None, max_flag_frac=0.2):
    g = parity.gpu_chain(inp)
    o = parity.oracle_chain(inp, rows)
    nflag, nbad, det = parity.compare_chain(g, o, inp.gamma, rows)
    n = len(o["num_accepted"])
    assert nbad == 0, f"{nbad} unflagged mismatches of {n}: {det}"
    assert nflag <= max_flag_frac * n + 1, f"too many near-ties: {nflag}/{n}"
    return g, o, nflag


CASES = [
    # B, gamma, V, tdt, draft (dtype or "probs"), stride pad, temperatures
    (3, 1, 1003, torch.bfloat16, torch.bfloat16, 5, (1.0,)),
    (4, 4, 8192, torch.bfloat16, torch.bfloat16, 0, (0.6, 1.0)),
    (4, 4, 8193, torch.bfloat16, torch.bfloat16, 7, (0.6, 1.0)),
    (2, 16, 20000, torch.bfloat16, torch.bfloat16, 0, (1.3,)),
    (5, 3, 4096 * 3 + 5, torch.float32, torch.float32, 3, (0.8,)),
    (3, 2, 9000, torch.bfloat16, torch.float32, 0, (1.0,)),
    (3, 2, 9000, torch.float32, torch.bfloat16, 0, (1.0,)),
    (6, 5, 30001, torch.bfloat16, "probs", 3, (1.0,)),
    (2, 3, 5000, torch.float32, "probs", 0, (0.7,)),
    (1, 1, 1, torch.float32, torch.float32, 3, (1.0,)),
    (3, 2, 7, torch.bfloat16, torch.bfloat16, 1, (1.0,)),
    (64, 5, 32000, torch.bfloat16, torch.bfloat16, 0, (0.6, 1.0)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}g{c[1]}V{c[2]}{str(c[3])[-4:]}{str(c[4])[-5:]}p{c[5]}")
def test_chain_parity(case, cuda_device):
    B, gamma, V, tdt, dk, pad, temps = case
    probs = dk == "probs"
    for seed in range(3):
        q = 16 // (2 if tdt == torch.bfloat16 else 4)
        stride = -(-(V + pad) // q) * q
        ddt = torch.float32 if probs else dk
        qd = 16 // (2 if ddt == torch.bfloat16 else 4)
        dstride = -(-(V + pad) // qd) * qd
        inp = wl.chain_inputs(B, gamma, V, seed=1000 + seed, device="cuda", target_dtype=tdt,
                              draft_dtype=ddt, draft_is_probs=probs, zipf=True, draft_noise=1.0,
                              temperatures=temps, stride=stride, dstride=dstride)
        _check(inp)


def test_chain_workload0_1000_rounds(cuda_device):
    """Small chain workload: B=1, gamma=4, V=1000 f32 logits, fixed logits, 1000 rounds
    of fresh draft tokens and uniforms."""
    target, draft = wl.chain_config0_logits("cuda")
    nflag = 0
    ks = []
    for r in range(1000):
        inp = wl.chain_config0_round(r, target, draft, "cuda")
        _, o, f = _check(inp, max_flag_frac=1.0)
        nflag += f
        ks.append(int(o["num_accepted"][0]))
    assert nflag <= 20
    assert 0 < np.mean(ks) < 4


def test_chain_workload1(cuda_device):
    """B=64, gamma=5, V=32000 bf16 logits, T in {0.6, 1.0}: every sequence, 3 rounds."""
    for r in range(3):
        inp = wl.chain_config1(r, "cuda")
        _check(inp)


def test_chain_workload4_sampled(cuda_device):
    """B=512, gamma=7, V=129280 bf16 target + f32 draft probabilities, launched at
    full size; the oracle checks a sample of 48 sequences one by one."""
    inp = wl.chain_config4(0, "cuda")
    rows = np.arange(0, 512, 512 // 48)[:48]
    _check(inp, rows=rows)


def test_chain_lossless_through_gpu_bruteforce(cuda_device):
    for kw in [dict(), dict(draft_kind="logits", seed=11, T=0.7), dict(V=4, gamma=3, K=2, seed=21, T=0.6)]:
        r = pins.chain_bruteforce(runner=parity.gpu_chain_runner, **kw)
        assert r["ok"], (kw, r)


def test_chain_closed_form_through_gpu(cuda_device):
    r = pins.chain_closed_form_exact(runner=parity.gpu_chain_runner)
    assert r["ok"], r
    r = pins.chain_closed_form_mc(runner=parity.gpu_chain_runner)
    assert r["ok"], r


@pytest.mark.parametrize("seed,kind", [(3, "probs"), (13, "logits")])
def test_chain_chisquare_through_gpu(seed, kind, cuda_device):
    r = pins.chain_chisquare(rounds=1_000_000, seed=seed, draft_kind=kind, runner=parity.gpu_chain_runner)
    assert r["ok"], r


def test_chain_invalid_inputs(cuda_device):
    B, gamma, V = 6, 3, 3000
    inp = wl.chain_inputs(B, gamma, V, seed=5, device="cuda")
    inp.draft_tokens[1, 2] = V                    # token out of range
    inp.temperature[2] = 0.0                      # bad temperature
    inp.target[3, 3, 17] = float("nan")           # NaN in the bonus row
    inp.draft[4, 0, :V] = float("-inf")           # all -inf draft row
    inp.target[5, 1, 5] = float("inf")            # +inf logit
    ws = sv.Workspace("cuda")
    buf = ws.get(sv.SPEC_ENTRY_CHAIN, B, gamma, V)
    g = parity.gpu_chain(inp, workspace=buf)
    assert list(g["num_accepted"][1:]) == [-1] * 5
    assert (g["tokens"][1:] == -1).all()
    assert g["num_accepted"][0] >= 0
    st = sv.spec_read_device_status(buf)
    assert st & (1 << sv.SPEC_ERR_DEVICE_INPUT)
    assert sv.spec_read_device_status(buf) == 0           # read clears
    o = parity.oracle_chain(inp)
    assert list(o["num_accepted"][1:]) == [-1] * 5


def test_chain_deterministic_and_workspace_reuse(cuda_device):
    inp = wl.chain_config1(7, "cuda")
    ws = sv.Workspace("cuda")
    buf = ws.get(sv.SPEC_ENTRY_CHAIN, inp.B, inp.gamma, inp.V)
    a = parity.gpu_chain(inp, workspace=buf)
    for _ in range(5):
        b = parity.gpu_chain(inp, workspace=buf)
        assert (a["tokens"] == b["tokens"]).all() and (a["num_accepted"] == b["num_accepted"]).all()
        np.testing.assert_array_equal(a["px"], b["px"])


def test_chain_empty_batch(cuda_device):
    inp = wl.chain_inputs(1, 2, 100, seed=1, device="cuda", stride=104, dstride=104)
    toks = torch.empty((0, 3), dtype=torch.int32, device="cuda")
    na = torch.empty((0,), dtype=torch.int32, device="cuda")
    st = sv.lib().spec_verify_chain(0, 2, 100, None, 1, 104, None, 1, 0, 104, None, None, None, None,
                                    None, None, None, None, 0, None)
    assert st == sv.SPEC_OK
    del toks, na, inp
