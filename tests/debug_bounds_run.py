"""Run by tests/test_gpu_debug_bounds.py in a child process whose
SPEC_VERIFY_LIB names the bounds-checked library: every entry point on small
inputs (valid and invalid), compared with the oracle, then the device-side
bounds counter must read zero."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import torch  # noqa: E402

import parity  # noqa: E402
from speculative_decoding_verify_temperature_b200 import spec_verify as sv  # noqa: E402
from speculative_decoding_verify_temperature_b200 import workloads as wl  # noqa: E402


def main():
    assert sv.LIB_PATH.endswith("libspecverify_debug.so"), sv.LIB_PATH
    assert sv.spec_debug_bounds_hits() == 0
    bad = 0
    # chain: draft logits, draft probabilities, f32 rows over 8 chunks; then lazy and filtered
    for inp in [wl.chain_inputs(8, 4, 20000, seed=1, device="cuda", zipf=True, temperatures=(0.6, 1.0)),
                wl.chain_inputs(6, 3, 30000, seed=2, device="cuda", draft_is_probs=True),
                wl.chain_inputs(4, 2, 40000, seed=3, device="cuda", target_dtype=torch.float32,
                                draft_dtype=torch.float32)]:
        o = parity.oracle_chain(inp)
        d = parity.gpu_chain(inp)
        bad += parity.compare_chain(d, o, inp.gamma)[1]
        z = parity.gpu_chain(inp, lazy=True)             # diagnostics only where evaluated: compare tokens
        bad += int((z["tokens"] != d["tokens"]).any(axis=1).sum() + (z["num_accepted"] != d["num_accepted"]).sum())
    inp = wl.chain_inputs(6, 3, 5000, seed=4, device="cuda", zipf=True)
    tk = torch.tensor([0, 20, 50, 0, 20, 50], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.9, 1.0, 0.95, 0.9, 1.0, 0.95], dtype=torch.float32, device="cuda")
    d = parity.gpu_chain_filtered(inp, tk, tp)
    bad += parity.compare_chain(d, parity.oracle_chain_filtered(inp, tk, tp), inp.gamma)[1]
    z = parity.gpu_chain_filtered(inp, tk, tp, lazy=True)
    bad += int((z["tokens"] != d["tokens"]).any(axis=1).sum())
    # trees: greedy, target-only sampling (dense and lazy, filtered), multi-step sampling
    inp = wl.tree_greedy_inputs(4, 3000, seed=5, device="cuda")
    bad += parity.compare_tree(parity.gpu_greedy(inp), parity.oracle_greedy(inp))[1]
    inp = wl.tree_sample_inputs(4, 3000, seed=6, device="cuda")
    o = parity.oracle_sample(inp)
    d = parity.gpu_sample(inp)
    bad += parity.compare_tree(d, o, sample=True)[1]
    z = parity.gpu_sample(inp, lazy=True)
    bad += int((z["tokens"] != d["tokens"]).any(axis=1).sum() + (z["num_accepted"] != d["num_accepted"]).sum())
    tk = torch.tensor([0, 20, 50, 5], dtype=torch.int32, device="cuda")
    tp = torch.tensor([0.9, 1.0, 0.95, 0.5], dtype=torch.float32, device="cuda")
    bad += parity.compare_tree(parity.gpu_sample(inp, top_k=tk, top_p=tp),
                               parity.oracle_sample(inp, top_k=tk, top_p=tp), sample=True)[1]
    inp = wl.tree_mss_inputs(4, 3000, seed=7, device="cuda")
    bad += parity.compare_mss(parity.gpu_mss(inp), parity.oracle_mss(inp))[1]
    # invalid inputs are caught by validation before any gather
    inp = wl.chain_inputs(4, 3, 3000, seed=8, device="cuda")
    inp.draft_tokens[1, 2] = 3000
    inp.draft_tokens[2, 0] = -5
    g = parity.gpu_chain(inp)
    assert list(g["num_accepted"][1:3]) == [-1, -1]
    inp = wl.tree_sample_inputs(3, 3000, seed=9, device="cuda")
    inp.tokens[0, 3] = 1 << 20
    inp.parents[1, 4] = 7
    g = parity.gpu_sample(inp)
    assert list(g["num_accepted"][:2]) == [-1, -1]
    hits = sv.spec_debug_bounds_hits()
    print(f"mismatches={bad} bounds_hits={hits}")
    assert bad == 0 and hits == 0


if __name__ == "__main__":
    main()
