"""The fused chain kernel: chain verification with draft logits of the
target's dtype whose rows span at most 8 chunks runs as one launch (a cluster
of one CTA per 16 KB chunk for each position), and must give what the oracle
gives; every other chain shape keeps the two-kernel path."""
import numpy as np
import pytest
import torch

import parity
from speculative_decoding_verify_temperature_b200 import spec_verify as sv
from speculative_decoding_verify_temperature_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _launches(inp):
    n0 = sv.spec_launch_count()
    parity.gpu_chain(inp)
    return sv.spec_launch_count() - n0


def _check(inp, rows=None):
    g = parity.gpu_chain(inp)
    o = parity.oracle_chain(inp, rows)
    nflag, nbad, det = parity.compare_chain(g, o, inp.gamma, rows)
    n = len(o["num_accepted"])
    assert nbad == 0, f"{nbad} unflagged mismatches of {n}: {det}"
    assert nflag <= 0.2 * n + 1
    return g, o


@pytest.mark.parametrize("V,dt,launches", [
    (32000, torch.bfloat16, 1), (65536, torch.bfloat16, 1), (65537, torch.bfloat16, 2),
    (1000, torch.float32, 1), (32768, torch.float32, 1), (32769, torch.float32, 2)])
def test_dispatch(V, dt, launches, cuda_device):
    inp = wl.chain_inputs(3, 2, V, seed=81, device="cuda", target_dtype=dt, draft_dtype=dt)
    assert _launches(inp) == launches


def test_other_draft_kinds_keep_two_kernels(cuda_device):
    a = wl.chain_inputs(3, 2, 9000, seed=82, device="cuda", target_dtype=torch.bfloat16,
                        draft_dtype=torch.float32)
    b = wl.chain_inputs(3, 2, 9000, seed=83, device="cuda", draft_is_probs=True)
    assert _launches(a) == 2 and _launches(b) == 2


@pytest.mark.parametrize("case", [
    # B, gamma, V, dtype, temperatures: one to eight chunks per row, ragged tails,
    # gamma at its limit, many more clusters than fit the GPU at once
    (5, 4, 65536, torch.bfloat16, (0.6, 1.0)),
    (7, 3, 65535, torch.bfloat16, (1.0,)),
    (3, 16, 40000, torch.bfloat16, (0.8,)),
    (300, 4, 24000, torch.bfloat16, (0.6, 1.0)),
    (4, 5, 32768, torch.float32, (1.0,)),
    (6, 2, 4097, torch.float32, (0.7,)),
    (2, 1, 8, torch.bfloat16, (1.0,)),
])
def test_fused_parity(case, cuda_device):
    B, gamma, V, dt, temps = case
    for seed in range(2):
        inp = wl.chain_inputs(B, gamma, V, seed=8400 + seed, device="cuda", target_dtype=dt, draft_dtype=dt,
                              zipf=True, temperatures=temps)
        assert _launches(inp) == 1
        _check(inp, rows=None if B <= 64 else np.arange(0, B, 7))


def test_fused_equal_rows_take_the_target_draw(cuda_device):
    """Draft logits equal to the target's: every residual is empty (S = 0), so
    each position's record holds a draw from p_i (the empty-residual rule); all
    drafts are accepted and the bonus comes from p_gamma."""
    inp = wl.chain_inputs(6, 3, 20000, seed=85, device="cuda", zipf=True, temperatures=(0.6, 1.0))
    inp.draft.copy_(inp.target[:, :inp.gamma])
    g, o = _check(inp)
    assert (g["num_accepted"] == inp.gamma).all()
    np.testing.assert_array_equal(g["S"], 1.0)


def test_fused_workload0_and_1(cuda_device):
    """Workload 1 in full, and 200 rounds of workload 0 (B=1, gamma=4, V=1000 f32)."""
    inp = wl.chain_config1(5, "cuda")
    assert _launches(inp) == 1
    _check(inp)
    target, draft = wl.chain_config0_logits("cuda")
    flagged = 0
    for r in range(200):
        g = parity.gpu_chain(wl.chain_config0_round(r, target, draft, "cuda"))
        o = parity.oracle_chain(wl.chain_config0_round(r, target, draft, "cuda"))
        f, bad, _ = parity.compare_chain(g, o, 4)
        assert bad == 0
        flagged += f
    assert flagged <= 10


def test_fused_counters_rest_between_calls(cuda_device):
    """The per-sequence arrival counters return to zero after each call: calls
    on one workspace, including a smaller batch in between, stay identical."""
    inp = wl.chain_config1(6, "cuda")
    ws = sv.Workspace("cuda").get(sv.SPEC_ENTRY_CHAIN, inp.B, inp.gamma, inp.V)
    a = parity.gpu_chain(inp, workspace=ws)
    small = wl.chain_inputs(5, inp.gamma, inp.V, seed=86, device="cuda", zipf=True)
    parity.gpu_chain(small, workspace=ws)
    for _ in range(3):
        b = parity.gpu_chain(inp, workspace=ws)
        np.testing.assert_array_equal(a["tokens"], b["tokens"])
        np.testing.assert_array_equal(a["S"], b["S"])
    assert sv.spec_read_device_status(ws) == 0
    cnt = ws[256:256 + 4 * inp.B].view(torch.int32)
    assert int(cnt.abs().sum()) == 0
