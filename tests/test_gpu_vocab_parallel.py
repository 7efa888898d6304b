"""Vocabulary-parallel chain verify on one GPU: the ranks of a tensor-parallel
group are emulated by running each shard's kernels in turn (no kernel waits on
another) and performing the exchanges (all-gather, all-reduce max) on the
host side; the result must equal the fp64 oracle on the whole rows."""
import numpy as np
import pytest
import torch

import parity
from speculative_decoding_verify_temperature_b200 import workloads as wl
from speculative_decoding_verify_temperature_b200 import spec_verify as sv

pytestmark = pytest.mark.gpu


def _shard(x, a, b):
    """Columns [a, b) of every row, in storage whose row stride is a multiple of 16 bytes."""
    q = 16 // x.element_size()
    w = b - a
    out = torch.zeros((x.shape[0], x.shape[1], -(-w // q) * q), dtype=x.dtype, device=x.device)
    out[:, :, :w] = x[:, :, a:b]
    return out


def _vp_round(inp, cuts):
    world = len(cuts) - 1
    B, g = inp.B, inp.gamma
    probs = inp.draft_is_probs
    shards, wss, recs = [], [], []
    for r in range(world):
        a, b = cuts[r], cuts[r + 1]
        t, d = _shard(inp.target, a, b), _shard(inp.draft, a, b)
        ws = sv.Workspace("cuda").get(sv.SPEC_ENTRY_CHAIN, B, g, b - a)
        shards.append((t, d, a, b - a))
        wss.append(ws)
        recs.append(sv.spec_vp_chain_stats(t, d, inp.draft_tokens, inp.temperature, vocab_offset=a,
                                           draft_is_probs=probs, V_shard=b - a, workspace=ws))
    rec_all = torch.stack(recs)                                   # the first all-gather
    outs, diags = [], []
    for r, (t, d, a, vs) in enumerate(shards):
        diag = torch.full((B, 2 * g + 1), float("nan"), device="cuda")
        outs.append(sv.spec_vp_chain_decide(rec_all, inp.draft_tokens, inp.temperature, inp.coins, V=inp.V,
                                            V_shard=vs, draft_is_probs=probs, diag=diag, workspace=wss[r]))
        diags.append(diag)
    mass_all = torch.stack([sv.spec_vp_chain_residual(t, d, rec_all, rank=r, draft_is_probs=probs, V_shard=vs,
                                                      workspace=wss[r])
                            for r, (t, d, a, vs) in enumerate(shards)])   # the second all-gather
    toks = [sv.spec_vp_chain_sample(t, d, inp.final_u, rec_all, mass_all, vocab_offset=a, rank=r,
                                    draft_is_probs=probs, V_shard=vs, diag=diags[r], workspace=wss[r])
            for r, (t, d, a, vs) in enumerate(shards)]
    tok = torch.stack(toks).max(dim=0).values                      # the all-reduce
    for r, (t, d, a, vs) in enumerate(shards):
        sv.spec_vp_chain_finish(tok, outs[r][0], V_shard=vs, workspace=wss[r])
    torch.cuda.synchronize()
    for r in range(1, world):                                      # every rank ends with the same round
        assert torch.equal(outs[r][0], outs[0][0]) and torch.equal(outs[r][1], outs[0][1])
    d = diags[0].cpu().numpy().astype(np.float64)
    return dict(tokens=outs[0][0].cpu().numpy(), num_accepted=outs[0][1].cpu().numpy(),
                px=d[:, :g], qx=d[:, g:2 * g], S=d[:, 2 * g]), toks


def _check(inp, cuts):
    g, per_rank = _vp_round(inp, cuts)
    o = parity.oracle_chain(inp)
    nflag, nbad, det = parity.compare_chain(g, o, inp.gamma)
    assert nbad == 0, det
    # exactly one shard owns each valid sequence's last token
    owners = (torch.stack(per_rank) >= 0).sum(dim=0).cpu().numpy()
    assert (owners[o["num_accepted"] >= 0] == 1).all()
    return g, o


@pytest.mark.parametrize("world", [1, 2, 4])
def test_vp_workload1_shape(world, cuda_device):
    """B=64, gamma=5, V=32000 bf16 logits split over 1, 2 or 4 uneven shards."""
    inp = wl.chain_config1(0, "cuda")
    cuts = [0] + sorted(np.random.default_rng(world).choice(np.arange(1, 32000), world - 1, replace=False).tolist()) + [32000]
    _check(inp, cuts)


@pytest.mark.parametrize("case", [
    (8, 3, 9001, torch.float32, torch.float32, False, [0, 3000, 6001, 9001]),
    (8, 4, 20000, torch.bfloat16, "probs", True, [0, 12345, 20000]),
    (6, 2, 40, torch.bfloat16, torch.bfloat16, False, [0, 9, 17, 33, 40]),
    (4, 2, 5000, torch.bfloat16, torch.float32, False, [0, 1, 5000]),
], ids=["f32x3", "bf16probs2", "tiny4", "oneelem"])
def test_vp_cases(case, cuda_device):
    B, g, V, tdt, dk, probs, cuts = case
    ddt = torch.float32 if probs else dk
    for seed in range(3):
        inp = wl.chain_inputs(B, g, V, seed=9100 + seed, device="cuda", target_dtype=tdt, draft_dtype=ddt,
                              draft_is_probs=probs, zipf=V > 100, temperatures=(0.6, 1.0))
        _check(inp, cuts)


def test_vp_invalid_and_workload4_sampled(cuda_device):
    inp = wl.chain_inputs(6, 3, 3000, seed=31, device="cuda")
    inp.temperature[1] = 0.0
    inp.target[2, 1, 2500] = float("nan")                    # NaN inside the second shard
    g, o = _check(inp, [0, 1500, 3000])
    assert list(g["num_accepted"][1:3]) == [-1, -1] and list(o["num_accepted"][1:3]) == [-1, -1]
    # the large chain workload (f32 draft probabilities) over 4 shards, a sample of sequences
    inp = wl.chain_config4(0, "cuda")
    rows = np.arange(0, 512, 64)
    g, per_rank = _vp_round(inp, [0, 40000, 64000, 100000, 129280])
    o = parity.oracle_chain(inp, rows)
    nflag, nbad, det = parity.compare_chain({k: v[rows] for k, v in g.items()}, o, inp.gamma)
    assert nbad == 0, det
