"""How far the CUDA path's probabilities are from the fp64 oracle's.

Accepted lengths and tokens are compared bit for bit except on sequences the
oracle flags as near-ties: a decision whose coin lies within 1e-6 of its
ratio (chain: p(x)/q(x); tree: prob_acc/theta).  That rule is sound only if
the GPU's ratio never errs by as much as the flag width.  The kernels sum
2^(x - m) in f32 with the exp2 unit's approximation and combine chunks in
fp64, so p(x) carries a small relative error; these tests measure it on the
benchmark workloads and at the largest vocabulary the library accepts, and
require the ratio error to stay below a fraction of the flag width."""
import numpy as np
import pytest

import parity
from speculative_decoding_verify_temperature_b200 import workloads as wl

pytestmark = pytest.mark.gpu

P_BOUND = 4e-7        # relative error of one probability (f32 diagnostic rounding included)
RATIO_BOUND = 6e-7    # relative error of p(x)/q(x): well inside the 1e-6 flag width


def _rel(g, o):
    m = np.isfinite(o) & (o > 0) & np.isfinite(g)
    if not m.any():
        return 0.0
    return float(np.max(np.abs(g[m] - o[m]) / o[m]))


def _chain_errors(inp, rows=None):
    g = parity.gpu_chain(inp)
    o = parity.oracle_chain(inp, rows)
    sel = parity._rows_np(rows)
    ok = (o["num_accepted"] >= 0) & (g["num_accepted"][sel] >= 0)
    gp, gq = g["px"][sel][ok], g["qx"][sel][ok]
    op, oq = o["px"][ok], o["qx"][ok]
    m = (op > 0) & (oq > 0)
    ratio = float(np.max(np.abs((gp[m] / gq[m]) / (op[m] / oq[m]) - 1.0))) if m.any() else 0.0
    return _rel(gp, op), _rel(gq, oq), ratio


def _report(name, *errs):
    print(f"{name}: " + ", ".join(f"{e:.3e}" for e in errs))


def test_chain_probability_error_workload1(cuda_device):
    ep, eq, er = _chain_errors(wl.chain_config1(0, "cuda"))
    _report("chain B64 g5 V32000 bf16 (p, q, p/q)", ep, eq, er)
    assert ep <= P_BOUND and eq <= P_BOUND and er <= RATIO_BOUND


def test_chain_probability_error_workload4(cuda_device):
    inp = wl.chain_config4(0, "cuda")
    ep, eq, er = _chain_errors(inp, rows=np.arange(0, inp.B, 16))
    _report("chain B512 g7 V129280 bf16 + f32 q (p, q as given, p/q)", ep, eq, er)
    assert ep <= P_BOUND and eq <= 1e-7 and er <= RATIO_BOUND


def test_chain_probability_error_max_vocabulary(cuda_device):
    for tdt, zipf in [("bf16", True), ("f32", False)]:
        import torch
        dt = torch.bfloat16 if tdt == "bf16" else torch.float32
        inp = wl.chain_inputs(4, 3, 1 << 20, seed=91, device="cuda", target_dtype=dt, draft_dtype=dt, zipf=zipf,
                              temperatures=(0.7, 1.0))
        ep, eq, er = _chain_errors(inp)
        _report(f"chain B4 g3 V=2^20 {tdt} (p, q, p/q)", ep, eq, er)
        assert ep <= P_BOUND and eq <= P_BOUND and er <= RATIO_BOUND


def test_tree_probability_error_workload3(cuda_device):
    inp = wl.tree_config3(0, "cuda")
    rows = np.arange(0, inp.B, 16)
    g = parity.gpu_sample(inp)
    o = parity.oracle_sample(inp, rows)
    ok = (o["num_accepted"] >= 0) & (g["num_accepted"][rows] >= 0)
    e = _rel(g["pchild"][rows][ok], o["pchild"][ok])
    _report("tree sample B128 N32 V151936 bf16 (p_parent(tok))", e)
    assert e <= P_BOUND


def test_tree_probability_error_max_vocabulary(cuda_device):
    inp = wl.tree_sample_inputs(3, 1 << 20, seed=92, device="cuda")
    g = parity.gpu_sample(inp)
    o = parity.oracle_sample(inp)
    ok = (o["num_accepted"] >= 0) & (g["num_accepted"] >= 0)
    e = _rel(g["pchild"][ok], o["pchild"][ok])
    _report("tree sample B3 V=2^20 bf16 (p_parent(tok))", e)
    assert e <= P_BOUND
