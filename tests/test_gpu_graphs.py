"""Every entry point inside a CUDA graph, replayed with new inputs copied into the
captured buffers, gives what eager calls give; repeated eager calls on one
workspace give bit-identical results (no state leaks between calls)."""
import numpy as np
import pytest
import torch

import parity
from speculative_decoding_verify_temperature_b200 import workloads as wl
from speculative_decoding_verify_temperature_b200 import spec_verify as sv

pytestmark = pytest.mark.gpu


def _graph_equals_eager(make_sets, call):
    """make_sets() -> list of input dicts of equal shapes; call(inputs) -> tuple of outputs."""
    sets = make_sets()
    eager = [tuple(t.clone() for t in call(s)) for s in sets]
    torch.cuda.synchronize()
    static = {k: v.clone() for k, v in sets[0].items()}
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call(static)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        outs = call(static)
    for _ in range(2):
        for i, st in enumerate(sets):
            for k, v in st.items():
                static[k].copy_(v)
            g.replay()
            torch.cuda.synchronize()
            for a, b in zip(outs, eager[i]):
                assert torch.equal(a, b)


def test_graph_filtered_chain(cuda_device):
    def make():
        out = []
        for r in range(3):
            x = wl.chain_config6(r, "cuda")
            out.append(dict(t=x.target, d=x.draft, x=x.draft_tokens, T=x.temperature, c=x.coins, u=x.final_u,
                            k=x.meta["top_k"], p=x.meta["top_p"]))
        return out
    ws = sv.Workspace("cuda").get(sv.SPEC_ENTRY_CHAIN, 64, 5, 32000)
    toks = torch.empty((64, 6), dtype=torch.int32, device="cuda")
    na = torch.empty((64,), dtype=torch.int32, device="cuda")

    def call(s):
        return sv.spec_verify_chain_filtered(s["t"], s["d"], s["x"], s["T"], s["c"], s["u"], s["k"], s["p"],
                                             out_tokens=toks, out_num_accepted=na, workspace=ws)
    _graph_equals_eager(make, call)


def test_graph_mss_dense_and_lazy(cuda_device):
    def make():
        out = []
        for r in range(2):
            x = wl.tree_mss_inputs(16, 20000, seed=800 + r, device="cuda")
            out.append(dict(t=x.target, tok=x.tokens, par=x.parents, T=x.temperature, c=x.coins, u=x.final_u,
                            q=x.draft_probs))
        return out
    md = wl.tree_depth(make()[0]["par"][0].tolist())
    for lazy in (False, True):
        ws = sv.Workspace("cuda").get(sv.SPEC_ENTRY_TREE_MSS, 16, 32, 20000)
        ai = torch.empty((16, md + 1), dtype=torch.int32, device="cuda")
        ot = torch.empty_like(ai)
        na = torch.empty((16,), dtype=torch.int32, device="cuda")
        fn = sv.spec_verify_tree_mss_lazy if lazy else sv.spec_verify_tree_mss

        def call(s):
            return fn(s["t"], s["tok"], s["par"], s["T"], s["c"], s["u"], md, s["q"], out_accept_index=ai,
                      out_tokens=ot, out_num_accepted=na, workspace=ws)
        _graph_equals_eager(make, call)


def test_repeated_calls_are_bit_identical(cuda_device):
    """Same inputs, same workspace, interleaved entry points: identical outputs."""
    c = wl.chain_config1(3, "cuda")
    f = wl.chain_config6(3, "cuda")
    m = wl.tree_mss_inputs(8, 9000, seed=5, device="cuda")
    ws = sv.Workspace("cuda").get(sv.SPEC_ENTRY_CHAIN, 64, 5, 32000)
    first = None
    for it in range(3):
        a = parity.gpu_chain(c, workspace=ws)
        b = parity.gpu_chain_filtered(f, f.meta["top_k"], f.meta["top_p"], workspace=ws)
        z = parity.gpu_chain(c, workspace=ws, lazy=True)
        e = parity.gpu_mss(m)
        got = (a["tokens"], a["px"], b["tokens"], b["px"], z["tokens"], e["tokens"], e["ptest"])
        if first is None:
            first = got
        else:
            for x, y in zip(got, first):
                np.testing.assert_array_equal(x, y)
