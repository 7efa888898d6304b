"""The C-ABI library loads, exports every symbol its header declares, and rejects
bad arguments on the host before touching the GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spec_verify.h")


@pytest.fixture(scope="module")
def L():
    from speculative_decoding_verify_temperature_b200 import build, spec_verify
    build.build()
    return spec_verify.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(spec_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["spec_verify_chain", "spec_verify_tree_greedy", "spec_verify_tree_sample",
              "spec_workspace_bytes", "spec_workspace_init", "spec_read_device_status",
              "spec_status_string", "spec_last_error_detail"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), f"{n} declared in spec_verify.h but not exported"


def test_bounds_checks_only_in_the_debug_build(L):
    """The release library reports that it has no bounds checks; the debug
    library exports every declared symbol too."""
    from speculative_decoding_verify_temperature_b200 import build, spec_verify as sv
    v = ctypes.c_ulonglong(7)
    L.spec_debug_bounds_hits.restype = ctypes.c_int
    assert L.spec_debug_bounds_hits(ctypes.byref(v)) == sv.SPEC_ERR_UNSUPPORTED and v.value == 0
    D = ctypes.CDLL(build.OUT_DEBUG)
    for n in declared_functions():
        assert hasattr(D, n), f"{n} missing from the debug library"


def test_status_strings(L):
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    for s in range(8):
        assert L.spec_status_string(s)
        assert L.spec_status_string(s) != b"unknown status"
    assert L.spec_status_string(sv.SPEC_OK) == b"ok"


def test_workspace_bytes(L):
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    a = sv.spec_workspace_bytes(sv.SPEC_ENTRY_CHAIN, 64, 5, 32000)
    b = sv.spec_workspace_bytes(sv.SPEC_ENTRY_CHAIN, 128, 5, 32000)
    assert 0 < a < b and a % 256 == 0
    assert sv.spec_workspace_bytes(sv.SPEC_ENTRY_TREE_SAMPLE, 128, 32, 151936) > 0
    assert sv.spec_workspace_bytes(sv.SPEC_ENTRY_CHAIN, 1, 0, 100) == 0           # gamma 0
    assert sv.spec_workspace_bytes(sv.SPEC_ENTRY_CHAIN, 1, 17, 100) == 0          # gamma > 16
    assert sv.spec_workspace_bytes(sv.SPEC_ENTRY_TREE_GREEDY, 1, 257, 100) == 0   # N > 256
    assert sv.spec_workspace_bytes(sv.SPEC_ENTRY_TREE_GREEDY, 1, 8, 0) == 0       # V = 0
    assert sv.spec_workspace_bytes(sv.SPEC_ENTRY_TREE_GREEDY, 1, 8, (1 << 20) + 1) == 0
    assert sv.spec_workspace_bytes(7, 1, 8, 100) == 0


FAKE = 1 << 20          # a 16-byte-aligned, never dereferenced address


def _chain(L, **kw):
    a = dict(B=2, gamma=3, V=1000, t=FAKE, tdt=1, ts=1000, d=FAKE, ddt=1, probs=0, ds=1000,
             x=FAKE, T=FAKE, coins=FAKE, fu=FAKE, ot=FAKE, na=FAKE, diag=None, ws=1 << 24,
             wsb=1 << 30, stream=None)
    a.update(kw)
    return L.spec_verify_chain(a["B"], a["gamma"], a["V"], a["t"], a["tdt"], a["ts"], a["d"], a["ddt"],
                               a["probs"], a["ds"], a["x"], a["T"], a["coins"], a["fu"], a["ot"],
                               a["na"], a["diag"], a["ws"], a["wsb"], a["stream"])


def test_chain_argument_errors_on_host(L):
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    E = sv.SPEC_ERR_INVALID_ARG
    assert _chain(L, B=0, t=None, d=None) == sv.SPEC_OK               # empty batch: nothing to do
    assert _chain(L, B=-1) == E
    assert _chain(L, gamma=0) == E
    assert _chain(L, gamma=17) == E
    assert _chain(L, V=0) == E
    assert _chain(L, V=(1 << 20) + 1) == E
    assert _chain(L, t=None) == E
    assert _chain(L, x=None) == E
    assert _chain(L, tdt=5) == E
    assert _chain(L, ts=999) == E                                     # stride < V
    assert _chain(L, ts=1004) == E                                    # 2008 bytes: not 16-aligned
    assert _chain(L, t=FAKE + 2) == E                                 # misaligned base
    assert _chain(L, probs=1, ddt=1) == E                             # probabilities must be f32
    assert b"16" in L.spec_last_error_detail() or L.spec_last_error_detail()
    assert _chain(L, ws=None) == sv.SPEC_ERR_WORKSPACE
    assert _chain(L, ws=(1 << 24) + 64) == sv.SPEC_ERR_WORKSPACE      # not 256-aligned
    assert _chain(L, wsb=100) == sv.SPEC_ERR_WORKSPACE                 # too small


def test_noalloc_rejects_arguments_before_any_cuda_call(L):
    """The no-allocation chain entry point checks every argument before it
    touches the device: here, with no GPU, a check that ran after a CUDA call
    would come back as SPEC_ERR_CUDA instead (on a GPU it would already have
    enqueued a clear of the shared scratch array)."""
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    f = L.spec_verify_chain_noalloc
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f.restype = i32
    f.argtypes = [i32, i32, i32, P, i32, i64, P, i32, i32, i64, P, P, P, P, P, P, P, P]

    def call(t=FAKE, tdt=1, ts=1000, d=FAKE, ddt=1, probs=0, ds=1000, x=FAKE, na=FAKE):
        return f(2, 3, 1000, t, tdt, ts, d, ddt, probs, ds, x, FAKE, FAKE, FAKE, FAKE, na, None, None)

    E = sv.SPEC_ERR_INVALID_ARG
    assert call(t=None) == E
    assert call(d=None) == E
    assert call(x=None) == E
    assert call(na=None) == E
    assert call(tdt=5) == E
    assert call(ts=1004) == E
    assert call(d=FAKE + 2) == E
    assert call(probs=1, ddt=1) == E


def test_tree_argument_errors_on_host(L):
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    E = sv.SPEC_ERR_INVALID_ARG

    def greedy(B=2, N=8, V=1000, md=4, t=FAKE, ts=1000, ws=1 << 24, wsb=1 << 30):
        return L.spec_verify_tree_greedy(B, N, V, md, t, 1, ts, FAKE, FAKE, FAKE, FAKE, FAKE, ws, wsb, None)

    def sample(th_s=1.0, th_a=1.0, dp=None, dps=0, T=FAKE):
        return L.spec_verify_tree_sample(2, 8, 1000, 4, FAKE, 1, 1000, FAKE, FAKE, T, FAKE, FAKE, dp, dps,
                                         th_s, th_a, FAKE, FAKE, FAKE, None, 1 << 24, 1 << 30, None)

    assert greedy(B=0, t=None) == sv.SPEC_OK
    assert greedy(N=0) == E
    assert greedy(N=257) == E
    assert greedy(md=-1) == E
    assert greedy(md=65) == E
    assert greedy(t=None) == E
    assert greedy(ts=1001) == E
    assert greedy(wsb=10) == sv.SPEC_ERR_WORKSPACE
    assert sample(th_s=0.0) == E
    assert sample(th_a=-1.0) == E
    assert sample(T=None) == E
    assert sample(dp=FAKE, dps=999) == E


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    monkeypatch.setattr(sv, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(sv, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        sv.lib()
