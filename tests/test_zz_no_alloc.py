"""spec_verify_chain_noalloc: the chain entry point for callers that cannot allocate
device memory where they verify (an engine plugin whose host allocator owns the
GPU, or a decode loop that cannot take cudaMalloc's implicit synchronisation).
It must give the same results as spec_verify_chain with a caller workspace, call
after call, although every call reuses the same built-in scratch array.

This file is collected last on purpose and also passes on its own in a fresh
process."""
import ctypes

import numpy as np
import pytest
import torch

from speculative_decoding_verify_temperature_b200 import spec_verify as sv
from speculative_decoding_verify_temperature_b200 import workloads as wl

RTOL = 1e-5          # the diagnostics tolerance of the parity tests


def _noalloc(L):
    f = L.spec_verify_chain_noalloc
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f.restype = i32
    f.argtypes = [i32, i32, i32, P, i32, i64, P, i32, i32, i64, P, P, P, P, P, P, P, P]
    return f


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(f, inp, toks, na, diag):
    B, g = inp.B, inp.gamma
    st = f(B, g, inp.V, _ptr(inp.target), sv._dtype(inp.target), sv._rows(inp.target, "target"),
           _ptr(inp.draft), sv.SPEC_F32 if inp.draft_is_probs else sv._dtype(inp.draft),
           int(inp.draft_is_probs), sv._rows(inp.draft, "draft"), _ptr(inp.draft_tokens),
           _ptr(inp.temperature), _ptr(inp.coins), _ptr(inp.final_u), _ptr(toks), _ptr(na),
           _ptr(diag), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point(cuda_device):
    L = sv.lib()
    f = _noalloc(L)
    cases = [
        wl.chain_config1(11, "cuda"),                                       # B=64 gamma=5 V=32000 bf16 logits
        wl.chain_inputs(24, 7, 40000, seed=5, device="cuda", draft_is_probs=True,
                        draft_noise=1.5, stride=40000, dstride=40000),      # f32 draft probabilities
        wl.chain_inputs(3, 2, 1003, seed=6, device="cuda", target_dtype=torch.float32,
                        draft_dtype=torch.float32, stride=1004, dstride=1004),  # one chunk per row
    ]
    for inp in cases:
        B, g = inp.B, inp.gamma
        ref_diag = torch.full((B, 2 * g + 1), float("nan"), device="cuda")
        ref_t, ref_k = sv.spec_verify_chain(inp.target, inp.draft, inp.draft_tokens, inp.temperature,
                                            inp.coins, inp.final_u, draft_is_probs=inp.draft_is_probs,
                                            V=inp.V, diag=ref_diag)
        torch.cuda.synchronize()
        for _ in range(2):                                                   # two calls in a row
            toks = torch.full((B, g + 1), -7, dtype=torch.int32, device="cuda")
            na = torch.full((B,), -7, dtype=torch.int32, device="cuda")
            diag = torch.full((B, 2 * g + 1), float("nan"), device="cuda")
            assert _call_noalloc(f, inp, toks, na, diag) == sv.SPEC_OK, L.spec_last_error_detail()
            torch.cuda.synchronize()
            assert torch.equal(toks, ref_t)
            assert torch.equal(na, ref_k)
            np.testing.assert_allclose(diag.cpu().numpy(), ref_diag.cpu().numpy(), rtol=RTOL, atol=1e-30)


@pytest.mark.gpu
def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    L = sv.lib()
    f = _noalloc(L)
    B, g, V = 4096, 16, 1 << 20                         # needs far more than 16 MiB of scratch
    assert sv.spec_workspace_bytes(sv.SPEC_ENTRY_CHAIN, B, g, V) > (16 << 20)
    fake = ctypes.c_void_p(1 << 20)                      # never dereferenced: rejected on the host
    st = f(B, g, V, fake, sv.SPEC_BF16, V, fake, sv.SPEC_BF16, 0, V, fake, fake, fake, fake, fake, fake,
           None, None)
    assert st == sv.SPEC_ERR_WORKSPACE
    assert b"scratch" in L.spec_last_error_detail()
