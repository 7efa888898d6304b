"""The device-side timeout path, driven without making any copy late.

The finalize kernels stage data in shared memory with bulk copies and wait for
each copy with a bounded poll.  spec_debug_wait_budget(0) makes every first
wait give up at once while the copies land normally, so the path a real
timeout takes runs on the GPU: the status word gets SPEC_ERR_TIMEOUT (and not
SPEC_ERR_COPY_IN_FLIGHT: the second, full-budget wait lets each copy land
before its CTA goes on), statistics are read from global memory instead of
the stage (the results stay correct), a sequence whose staged row pair was
lost reads -1, and the next call on the same workspace is clean."""
import numpy as np
import pytest
import torch

import parity
from speculative_decoding_verify_temperature_b200 import spec_verify as sv
from speculative_decoding_verify_temperature_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TIMEOUT = 1 << sv.SPEC_ERR_TIMEOUT
IN_FLIGHT = 1 << sv.SPEC_ERR_COPY_IN_FLIGHT


def _zero_budget(fn):
    sv.spec_debug_wait_budget(0)
    try:
        return fn()
    finally:
        sv.spec_debug_wait_budget(-1)


def test_chain_row_pair_timeout(cuda_device):
    """Chain with draft probabilities on a batch that fits one wave: the pair
    kernel stages the statistics and each half of the rejected row pair."""
    inp = wl.chain_inputs(24, 4, 40000, seed=71, device="cuda", draft_is_probs=True, draft_noise=0.5,
                          zipf=True)
    ws = sv.Workspace("cuda").get(sv.SPEC_ENTRY_CHAIN, inp.B, inp.gamma, inp.V)
    ref = parity.gpu_chain(inp, workspace=ws)
    assert sv.spec_read_device_status(ws) == 0
    k = ref["num_accepted"]
    assert (k < inp.gamma).any() and (k == inp.gamma).any()        # both paths are exercised

    out = _zero_budget(lambda: parity.gpu_chain(inp, workspace=ws))
    st = sv.spec_read_device_status(ws)
    assert st & TIMEOUT and not st & IN_FLIGHT, st
    rej = k < inp.gamma
    # a rejection needs the staged row pair, which the timeout gave up on
    assert (out["num_accepted"][rej] == -1).all()
    assert (out["tokens"][rej] == -1).all()
    # a bonus draw reads the statistics from global memory: unchanged
    np.testing.assert_array_equal(out["num_accepted"][~rej], k[~rej])
    np.testing.assert_array_equal(out["tokens"][~rej], ref["tokens"][~rej])

    again = parity.gpu_chain(inp, workspace=ws)
    assert sv.spec_read_device_status(ws) == 0
    np.testing.assert_array_equal(again["num_accepted"], k)
    np.testing.assert_array_equal(again["tokens"], ref["tokens"])


def test_chain_sliced_statistics_timeout(cuda_device):
    """More sequences than SMs: the sliced kernel stages only the statistics;
    after the timeout it reads them from global memory and stays exact."""
    inp = wl.chain_inputs(300, 2, 9000, seed=72, device="cuda", draft_is_probs=True, zipf=True)
    ws = sv.Workspace("cuda").get(sv.SPEC_ENTRY_CHAIN, inp.B, inp.gamma, inp.V)
    ref = parity.gpu_chain(inp, workspace=ws)
    assert sv.spec_read_device_status(ws) == 0
    out = _zero_budget(lambda: parity.gpu_chain(inp, workspace=ws))
    st = sv.spec_read_device_status(ws)
    assert st & TIMEOUT and not st & IN_FLIGHT, st
    np.testing.assert_array_equal(out["num_accepted"], ref["num_accepted"])
    np.testing.assert_array_equal(out["tokens"], ref["tokens"])
    again = parity.gpu_chain(inp, workspace=ws)
    assert sv.spec_read_device_status(ws) == 0
    np.testing.assert_array_equal(again["tokens"], ref["tokens"])


def test_tree_statistics_timeout(cuda_device):
    """Tree finalisation stages each sequence's statistics block."""
    for mk, run in [(wl.tree_sample_inputs, parity.gpu_sample), (wl.tree_greedy_inputs, parity.gpu_greedy)]:
        inp = mk(6, 20000, seed=73, device="cuda")
        entry = sv.SPEC_ENTRY_TREE_SAMPLE if run is parity.gpu_sample else sv.SPEC_ENTRY_TREE_GREEDY
        ws = sv.Workspace("cuda").get(entry, inp.B, inp.N, inp.V)
        ref = run(inp, workspace=ws)
        assert sv.spec_read_device_status(ws) == 0
        out = _zero_budget(lambda: run(inp, workspace=ws))
        st = sv.spec_read_device_status(ws)
        assert st & TIMEOUT and not st & IN_FLIGHT, st
        for key in ("tokens", "num_accepted"):
            np.testing.assert_array_equal(out[key], ref[key])
        again = run(inp, workspace=ws)
        assert sv.spec_read_device_status(ws) == 0
        np.testing.assert_array_equal(again["tokens"], ref["tokens"])


def test_budget_hook_restores_the_default(cuda_device):
    """A negative budget restores the default: a normal call sets no status bit."""
    sv.spec_debug_wait_budget(0)
    sv.spec_debug_wait_budget(-1)
    inp = wl.chain_inputs(4, 3, 20000, seed=74, device="cuda", draft_is_probs=True)
    ws = sv.Workspace("cuda").get(sv.SPEC_ENTRY_CHAIN, inp.B, inp.gamma, inp.V)
    parity.gpu_chain(inp, workspace=ws)
    assert sv.spec_read_device_status(ws) == 0
    torch.cuda.synchronize()
