"""Benchmark of the speculative-decoding verify step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload {0..8}] [--impl {ours,reference}]

One step = one verify round (one C-ABI call) over the workload's whole batch.
Default workload 1: chain speculative sampling, B=64, gamma=5, V=32000, bf16
target + draft logits, T in {0.6, 1.0} per sequence.  With N > 1 (torchrun)
every rank verifies its own batch of the same shape (the batch axis shards
with no exchange): weak scaling, time = max over ranks.

Rank 0 prints ONE JSON line.  ``value`` is whole-job verify rounds/s with the
inputs already in HBM (CUDA-graph replays, CUDA events); L2 is kept cold by
rotating several input sets whose total exceeds the 126 MB L2 (workloads 0-1)
or by inputs larger than L2 (workloads 2-4).  ``e2e`` is the same metric through
the Python binding with pinned host buffers copied in and results copied out
every step.  ``roofline`` reports the row kernel (the dominant one) against
the measured HBM copy bandwidth; ``cpu_baseline`` times the fp64 oracle on a
bounded sample on the host cores.  The default run also measures each of the
five benchmark configurations (workloads 0-4) the same way under
``per_config``.  ``--impl reference`` runs that oracle alone as the reference
arm.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", type=int, default=1, choices=[0, 1, 2, 3, 4, 5, 6, 7, 8])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lazy-steps", type=int, default=400,
                    help="steps of the row-on-demand (lazy) entry point timed beside the dense one (0: skip)")
    ap.add_argument("--configs", default=None,
                    help="comma-separated workloads measured under per_config (default: 0,1,2,3,4 when "
                         "--workload is 1, none otherwise; 'none' skips)")
    ap.add_argument("--config-cpu-seconds", type=float, default=3.0,
                    help="oracle seconds per configuration under per_config")
    ap.add_argument("--with-diag", action="store_true",
                    help="pass diagnostics buffers (the filtered workloads then filter every row up front)")
    return ap.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ----------------------------------------------------------------------------- ranks

def reduce_max_ms(ms: float, world: int, device=None) -> float:
    """Max over ranks of a per-rank duration (the job ends when the slowest rank does)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(steps: int, world: int, max_ms: float) -> float:
    """Whole-job verify rounds/s: every rank verifies one round per step."""
    return world * steps / (max_ms / 1e3)


# ----------------------------------------------------------------------------- workloads

def make_inputs(wid: int, rnd: int, device, rank: int = 0):
    from speculative_decoding_verify_temperature_b200 import workloads as wl
    r = rnd + 100 * rank
    if wid == 0:
        t, d = wl.chain_config0_logits(device)
        return wl.chain_config0_round(r, t, d, device)
    if wid == 1:
        return wl.chain_config1(r, device)
    if wid == 2:
        return wl.tree_config2(r, device)
    if wid == 3:
        return wl.tree_config3(r, device)
    if wid == 5:
        return wl.tree_config5(r, device)
    if wid == 6:
        return wl.chain_config6(r, device)
    if wid == 8:
        return wl.tree_config8(r, device)
    if wid == 7:
        return wl.chain_config4(r, device)
    return wl.chain_config4(r, device)


def input_bytes(inp) -> int:
    n = 0
    for v in vars(inp).values():
        if hasattr(v, "element_size") and hasattr(v, "numel"):
            n += v.numel() * v.element_size()
    return n


VP_WORLD = 8          # vocabulary shards of the vocabulary-parallel workload


def vp_cuts(V: int, world: int = VP_WORLD):
    return [V * r // world for r in range(world + 1)]


def describe(wid: int, inp) -> dict:
    from speculative_decoding_verify_temperature_b200 import workloads as wl
    if wid == 7:
        return {"workload": f"vocabulary-parallel chain: {wl.WORKLOADS[4]}, split over {VP_WORLD} vocabulary shards; "
                            "timed: one rank's five device steps (shard 0); the three exchanges are prepared "
                            "once and not timed (one GPU)",
                "global_batch": inp.B, "gamma": inp.gamma, "V": inp.V, "shards": VP_WORLD,
                "V_shard": vp_cuts(inp.V)[1], "target_dtype": "bfloat16", "draft": "f32 probabilities"}
    d = {"workload": wl.WORKLOADS[wid], "global_batch": inp.B}
    if wid in (0, 1, 4, 6, 7):
        d.update(gamma=inp.gamma, V=inp.V, target_dtype=str(inp.target.dtype).split(".")[-1],
                 draft="f32 probabilities" if inp.draft_is_probs else str(inp.draft.dtype).split(".")[-1] + " logits")
    else:
        d.update(nodes=inp.N, V=inp.V, max_depth=inp.max_depth, target_dtype=str(inp.target.dtype).split(".")[-1])
    return d


class Runner:
    """Calls the verify entry point of a workload through the Python binding."""

    def __init__(self, wid, inp, ws, lazy=False, diag=False):
        self.wid, self.inp, self.ws, self.sfx = wid, inp, ws, "_lazy" if lazy else ""
        if wid == 7:
            self._vp_setup()
        import torch
        B = inp.B
        dev = inp.target.device
        self.diag = None
        if diag and wid == 6:
            self.diag = torch.empty((B, 2 * inp.gamma + 1), dtype=torch.float32, device=dev)
        if diag and wid == 8:
            self.diag = torch.empty((B, inp.N + 1), dtype=torch.float32, device=dev)
        if wid in (0, 1, 4, 6, 7):
            self.out = (torch.empty((B, inp.gamma + 1), dtype=torch.int32, device=dev),
                        torch.empty((B,), dtype=torch.int32, device=dev))
        else:
            W = inp.max_depth + 1
            self.out = (torch.empty((B, W), dtype=torch.int32, device=dev),
                        torch.empty((B, W), dtype=torch.int32, device=dev),
                        torch.empty((B,), dtype=torch.int32, device=dev))

    def _vp_setup(self):
        """Shard 0's columns of every row, and the exchanged buffers of a round
        over all shards (computed once, as the other ranks would have)."""
        import torch
        from speculative_decoding_verify_temperature_b200 import spec_verify as sv
        i = self.inp
        cuts = vp_cuts(i.V)

        def shard(x, a, b):
            q = 16 // x.element_size()
            out = torch.zeros((x.shape[0], x.shape[1], -(-(b - a) // q) * q), dtype=x.dtype, device=x.device)
            out[:, :, :b - a] = x[:, :, a:b]
            return out

        shards = [(shard(i.target, cuts[r], cuts[r + 1]), shard(i.draft, cuts[r], cuts[r + 1]), cuts[r],
                   cuts[r + 1] - cuts[r]) for r in range(VP_WORLD)]
        wss = [sv.Workspace(i.target.device).get(sv.SPEC_ENTRY_CHAIN, i.B, i.gamma, vs) for (_, _, _, vs) in shards]
        recs = [sv.spec_vp_chain_stats(t, d, i.draft_tokens, i.temperature, vocab_offset=a, draft_is_probs=True,
                                       V_shard=vs, workspace=wss[r]) for r, (t, d, a, vs) in enumerate(shards)]
        self.rec_all = torch.stack(recs)
        for r, (t, d, a, vs) in enumerate(shards):
            sv.spec_vp_chain_decide(self.rec_all, i.draft_tokens, i.temperature, i.coins, V=i.V, V_shard=vs,
                                    draft_is_probs=True, workspace=wss[r])
        self.mass_all = torch.stack([sv.spec_vp_chain_residual(t, d, self.rec_all, rank=r, draft_is_probs=True,
                                                               V_shard=vs, workspace=wss[r])
                                     for r, (t, d, a, vs) in enumerate(shards)])
        toks = [sv.spec_vp_chain_sample(t, d, i.final_u, self.rec_all, self.mass_all, vocab_offset=a, rank=r,
                                        draft_is_probs=True, V_shard=vs, workspace=wss[r])
                for r, (t, d, a, vs) in enumerate(shards)]
        self.tok = torch.stack(toks).max(dim=0).values
        self.t0, self.d0, _, self.vs0 = shards[0]
        self.ws = wss[0]
        self.rec0 = torch.empty_like(recs[0])
        self.mass0 = torch.empty_like(self.mass_all[0])
        self.tok0 = torch.empty_like(self.tok)
        del shards, recs, toks

    def __call__(self):
        from speculative_decoding_verify_temperature_b200 import spec_verify as sv
        i = self.inp
        if self.wid == 7:
            # rank 0 of the vocabulary-parallel round; exchanged buffers from the setup
            sv.spec_vp_chain_stats(self.t0, self.d0, i.draft_tokens, i.temperature, vocab_offset=0, draft_is_probs=True,
                                   V_shard=self.vs0, rec_out=self.rec0, workspace=self.ws)
            sv.spec_vp_chain_decide(self.rec_all, i.draft_tokens, i.temperature, i.coins, V=i.V, V_shard=self.vs0,
                                    draft_is_probs=True, out_tokens=self.out[0], out_num_accepted=self.out[1],
                                    workspace=self.ws)
            sv.spec_vp_chain_residual(self.t0, self.d0, self.rec_all, rank=0, draft_is_probs=True, V_shard=self.vs0,
                                      mass_out=self.mass0, workspace=self.ws)
            sv.spec_vp_chain_sample(self.t0, self.d0, i.final_u, self.rec_all, self.mass_all, vocab_offset=0, rank=0,
                                    draft_is_probs=True, V_shard=self.vs0, tok_out=self.tok0, workspace=self.ws)
            sv.spec_vp_chain_finish(self.tok, self.out[0], V_shard=self.vs0, workspace=self.ws)
        elif self.wid == 8:
            getattr(sv, "spec_verify_tree_sample_filtered" + self.sfx)(i.target, i.tokens, i.parents, i.temperature, i.coins, i.final_u,
                                                i.max_depth, i.meta["top_k"], i.meta["top_p"],
                                                draft_probs=i.draft_probs, V=i.V, out_accept_index=self.out[0],
                                                out_tokens=self.out[1], out_num_accepted=self.out[2],
                                                diag=self.diag, workspace=self.ws)
        elif self.wid == 6:
            sv.spec_verify_chain_filtered(i.target, i.draft, i.draft_tokens, i.temperature, i.coins, i.final_u,
                                          i.meta["top_k"], i.meta["top_p"], draft_is_probs=i.draft_is_probs, V=i.V,
                                          out_tokens=self.out[0], out_num_accepted=self.out[1], diag=self.diag,
                                          workspace=self.ws)
        elif self.wid in (0, 1, 4):
            getattr(sv, "spec_verify_chain" + self.sfx)(i.target, i.draft, i.draft_tokens, i.temperature, i.coins, i.final_u,
                                 draft_is_probs=i.draft_is_probs, V=i.V, out_tokens=self.out[0],
                                 out_num_accepted=self.out[1], workspace=self.ws)
        elif self.wid == 5:
            getattr(sv, "spec_verify_tree_mss" + self.sfx)(i.target, i.tokens, i.parents, i.temperature, i.coins, i.final_u, i.max_depth,
                                    i.draft_probs, V=i.V, out_accept_index=self.out[0], out_tokens=self.out[1],
                                    out_num_accepted=self.out[2], workspace=self.ws)
        elif self.wid == 2:
            getattr(sv, "spec_verify_tree_greedy" + self.sfx)(i.target, i.tokens, i.parents, i.max_depth, V=i.V,
                                       out_accept_index=self.out[0], out_tokens=self.out[1],
                                       out_num_accepted=self.out[2], workspace=self.ws)
        else:
            getattr(sv, "spec_verify_tree_sample" + self.sfx)(i.target, i.tokens, i.parents, i.temperature, i.coins, i.final_u,
                                       i.max_depth, draft_probs=i.draft_probs, V=i.V,
                                       out_accept_index=self.out[0], out_tokens=self.out[1],
                                       out_num_accepted=self.out[2], workspace=self.ws)

    def num_accepted(self):
        return self.out[-1]


def lazy_bytes_read(wid, inp, num_accepted) -> int:
    """Logit bytes the lazy walk streams for one round with these outcomes: chain
    target rows 0..k (row gamma after a full accept) plus draft-logit rows 0..k
    below gamma; trees the row of every node on the accepted path (read twice by
    the filtered walk: statistics and filter)."""
    k = num_accepted.clamp_min(0).long()
    row_t = inp.V * inp.target.element_size()
    if wid in (0, 1, 4):
        n = int((k + 1).sum()) * row_t
        if not inp.draft_is_probs:
            n += int((k + 1).clamp_max(inp.gamma).sum()) * inp.V * inp.draft.element_size()
        return n
    if wid == 8:                              # each visited row is read by the statistics and by the filter
        return 2 * int((k + 1).sum()) * row_t
    return int((k + 1).sum()) * row_t


def workspace_for(wid, inp):
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    ws = sv.Workspace(inp.target.device)
    if wid in (0, 1, 4, 6):
        return ws.get(sv.SPEC_ENTRY_CHAIN, inp.B, inp.gamma, inp.V)
    if wid == 7:
        return None                           # each rank's workspace is set up by the runner
    e = {2: sv.SPEC_ENTRY_TREE_GREEDY, 3: sv.SPEC_ENTRY_TREE_SAMPLE, 5: sv.SPEC_ENTRY_TREE_MSS,
         8: sv.SPEC_ENTRY_TREE_SAMPLE}[wid]
    return ws.get(e, inp.B, inp.N, inp.V)


def algorithmic_bytes(wid, inp) -> int:
    """Bytes of logits / probabilities the row kernel must read once per round."""
    if wid == 7:                              # rank 0's shard of the target rows
        return inp.B * (inp.gamma + 1) * vp_cuts(inp.V)[1] * inp.target.element_size()
    b = inp.target[:, :, :inp.V].numel() * inp.target.element_size()
    if wid in (0, 1, 6):
        b += inp.draft[:, :, :inp.V].numel() * inp.draft.element_size()
    return b


def round_bytes(wid, inp, num_accepted) -> int:
    """Algorithmic bytes of one whole round with these outcomes: the row
    kernel's bytes, plus, for a chain with draft probabilities, the gathered
    q(x) of every drafted token and the full q row of every sequence that
    rejects (the residual norm(max(0, p - q)) reads it once)."""
    b = algorithmic_bytes(wid, inp)
    if wid in (4, 7) and inp.draft_is_probs:
        k = num_accepted
        rejecting = int(((k >= 0) & (k < inp.gamma)).sum())
        V = vp_cuts(inp.V)[1] if wid == 7 else inp.V
        b += inp.B * inp.gamma * 4 + rejecting * V * 4
    return b


def accept_histogram(wid, inp, num_accepted) -> dict:
    """Counts of the accepted lengths (draft tokens accepted per sequence and
    round; -1 = invalid sequence) over the measured rounds."""
    top = inp.gamma if wid in (0, 1, 4, 6, 7) else inp.max_depth
    k = num_accepted.long().cpu()
    h = {str(v): int((k == v).sum()) for v in range(-1, top + 1)}
    return {key: n for key, n in h.items() if n or key != "-1"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """NVML sampling of SM clock and throttle reasons in a background thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self.stop_ev = threading.Event()
        self.mark = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:          # NVML missing: report it rather than guess
            self.nv = None
            self.err = repr(e)
            self.max_mhz = None

    def run(self):
        while not self.stop_ev.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((self.mark, mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self.run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self.stop_ev.set()
        if self.nv:
            self.t.join()

    def summary(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        timed = [s for s in self.samples if s[0]]
        window = "timed region"
        if len(timed) < 3:
            timed = self.samples
            window = "warm-up + timed region (timed region shorter than the sampling period)"
        mhz = [s[1] for s in timed]
        mask = 0
        for s in timed:
            mask |= s[2]
        reasons = [n for b, n in self.REASONS.items() if mask & b and b != 0x1]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(timed), "window": window}


# ----------------------------------------------------------------------------- oracle baseline

def cpu_baseline(wid, inp, seconds, nthreads=None):
    """Time the fp64 oracle, as it stands, on whole rounds of the same inputs until
    ``seconds`` have elapsed (at least one round).  Returns rounds/s."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import parity
    import oracle
    oracle.build()
    cores = nthreads or len(os.sched_getaffinity(0))
    # Copy the inputs to host once; the oracle reads the same bytes the GPU reads.
    n = 0
    fn = {0: parity.oracle_chain, 1: parity.oracle_chain, 4: parity.oracle_chain, 7: parity.oracle_chain,
          2: parity.oracle_greedy, 3: parity.oracle_sample, 5: parity.oracle_mss,
          8: lambda i, r, nthreads: parity.oracle_sample(i, r, nthreads=nthreads, top_k=i.meta["top_k"],
                                                        top_p=i.meta["top_p"]),
          6: lambda i, r, nthreads: parity.oracle_chain_filtered(i, i.meta["top_k"], i.meta["top_p"], r,
                                                                 nthreads=nthreads)}[wid]
    B = inp.B
    # Large workloads: a bounded sample of whole sequences per "round" of work,
    # scaled to full rounds below.
    per = B if wid in (0, 1, 6) else max(1, min(B, {2: 8, 3: 4, 4: 16, 5: 4, 7: 16, 8: 4}[wid]))
    rows = None if per == B else list(range(per))
    elapsed = 0.0
    out = None
    while n == 0 or elapsed < seconds:
        t1 = time.perf_counter()
        out = fn(inp, rows, nthreads=cores)
        elapsed += time.perf_counter() - t1
        n += 1
    rounds = n * per / B
    res = {"value": rounds / elapsed, "unit": "rounds/s", "cores": cores, "kind": "oracle",
           "sample": f"{n} x {per} of {B} sequences of one round (whole sequences), fp64 C oracle, "
                     f"OpenMP over sequences, {elapsed:.1f} s of CPU time; rounds/s scaled by {per}/{B}"}
    return res, out, rows


def sample_parity(wid, inp, o, rows, ws):
    """The CUDA path's result on the sequences the oracle baseline computed
    (the same bytes): identical accepted lengths and tokens except on the
    sequences the oracle flags as near-ties, diagnostics within 1e-5."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import parity
    if wid == 7:
        return {"checked": False, "why": "one rank of a vocabulary-parallel round; parity of the sharded path "
                                         "is in the GPU tests (all shards emulated on one GPU)"}
    n = inp.B if rows is None else len(rows)
    try:
        if wid in (0, 1, 4):
            fl, bad, _ = parity.compare_chain(parity.gpu_chain(inp, workspace=ws), o, inp.gamma, rows)
        elif wid == 6:
            g = parity.gpu_chain_filtered(inp, inp.meta["top_k"], inp.meta["top_p"], workspace=ws)
            fl, bad, _ = parity.compare_chain(g, o, inp.gamma, rows)
        elif wid == 2:
            fl, bad, _ = parity.compare_tree(parity.gpu_greedy(inp, workspace=ws), o, rows)
        elif wid == 3:
            fl, bad, _ = parity.compare_tree(parity.gpu_sample(inp, workspace=ws), o, rows, sample=True)
        elif wid == 8:
            g = parity.gpu_sample(inp, workspace=ws, top_k=inp.meta["top_k"], top_p=inp.meta["top_p"])
            fl, bad, _ = parity.compare_tree(g, o, rows, sample=True)
        else:
            fl, bad, _ = parity.compare_mss(parity.gpu_mss(inp, workspace=ws), o, rows)
        diag = True
    except AssertionError as e:
        return {"checked": True, "sequences": n, "diagnostics_within_tolerance": False, "error": str(e)[:200]}
    return {"checked": True, "sequences": n, "identical_or_flagged": n - bad, "flagged_near_ties": fl,
            "mismatches": bad, "diagnostics_within_tolerance": diag}


# ----------------------------------------------------------------------------- main

def kernel_source_hash(text: str) -> str:
    """First 16 hex digits of the SHA-256 of the kernel source with its comments
    and white space removed (a change to the code changes it, a change to a
    comment does not)."""
    code = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    code = re.sub(r"//[^\n]*", "", code)
    code = re.sub(r"\s+", "", code)
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def profile_traffic(wid):
    """Per-launch DRAM traffic of the row kernel from a committed ncu summary,
    valid only while the kernel source's code is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "speculative_decoding_verify_temperature_b200", "csrc", "spec_verify.cu")
    try:
        rec = json.load(open(path)).get(str(wid))
        h = kernel_source_hash(open(src, encoding="utf-8").read())
        if rec and rec.get("source_sha256_16") == h:
            return rec.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0}, "fallback"


def input_sets(wid, dev, rank=0):
    """The workload's rotating input sets: enough of them that their total
    exceeds twice the L2 (one set when a set alone is that large)."""
    first = make_inputs(wid, 0, dev, rank)
    nbytes = input_bytes(first)
    nsets = 1 if nbytes > 2 * L2_BYTES else min(16, -(-2 * L2_BYTES // nbytes))
    return [first] + [make_inputs(wid, r, dev, rank) for r in range(1, nsets)], nbytes


def bench_config(wid, first, nsets, nbytes, world) -> dict:
    """The `config` object of a bench line (the same for both arms)."""
    cfg = describe(wid, first)
    cfg.update(parallelism=f"batch-sharded x{world} (no collective)" if world > 1 else "single GPU",
               l2=(f"{nsets} rotating input sets of {nbytes / 1e6:.1f} MB ({nsets * nbytes / 1e6:.0f} MB > 126 MB L2)"
                   if nsets > 1 else f"inputs {nbytes / 1e6:.0f} MB > 126 MB L2"))
    return cfg


CONFIG_STEPS = {0: 2000, 1: 2000, 2: 500, 3: 250, 4: 250}


def measure(wid, dev, world, steps, warmup, local, rank=0, diag=False):
    """Time one workload: CUDA-graph replays of its rotating input sets (CUDA
    events, max over ranks), the row kernel's own duration, the launches per
    call, and the accepted lengths of the measured rounds."""
    import torch
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    sets, nbytes = input_sets(wid, dev, rank)
    first, nsets = sets[0], len(sets)
    ws = workspace_for(wid, first)
    runners = [Runner(wid, s, ws, diag=diag) for s in sets]
    stream = torch.cuda.current_stream()
    for i in range(max(3, warmup)):
        runners[i % nsets]()
    torch.cuda.synchronize()

    # --- one CUDA graph per rotation of the input sets; the library counts the
    # kernels it adds to the graph
    n0 = sv.spec_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for r in runners:
            r()
    kps = (sv.spec_launch_count() - n0) // nsets
    torch.cuda.synchronize()
    singles = []
    for r in runners:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            r()
        singles.append(g)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()

    K = steps
    sampler = ClockSampler(local)
    with sampler:
        time.sleep(0.02)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler.mark = True
        e0.record(stream)
        full, rem = divmod(K, nsets)
        for _ in range(full):
            graph.replay()
        for i in range(rem):
            singles[i].replay()
        e1.record(stream)
        torch.cuda.synchronize()
        sampler.mark = False
        if world > 1:
            torch.distributed.barrier()
    ms = e0.elapsed_time(e1)
    ms_max = reduce_max_ms(ms, world, dev)
    value = job_value(K, world, ms_max)
    del graph, singles

    # --- dominant kernel duration: the library records an event pair around its
    # row kernel; the calls are captured in a CUDA graph so that host launch
    # latency never shows up between the two events.
    nk = max(nsets, min(256, K))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
    for a, b in evs:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    pg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pg):
        for i in range(nk):
            sv.spec_profile_events(*evs[i])
            runners[i % nsets]()
        sv.spec_profile_events()
    kms = []
    for _ in range(3):
        pg.replay()
        torch.cuda.synchronize()
        kms += [a.elapsed_time(b) for a, b in evs]
    del pg
    k_avg_ms = sum(kms) / len(kms)

    # --- acceptance statistics and whole-round bytes of the benchmarked rounds
    torch.cuda.synchronize()
    acc, rb = [], 0
    for r, st in zip(runners, sets):
        r()
        k = r.num_accepted()
        acc.append(k.clone())
        rb += round_bytes(wid, st, k)
    acc = torch.cat(acc)
    # --- filtered workloads: how many rows each filter path resolved (one
    # untimed call per input set with the library's row counters on)
    filt = None
    if wid in (6, 8):
        sv.spec_debug_filter_path(0, read=True)
        for r in runners:
            r()
        a, b, c = sv.spec_debug_filter_path(-1, read=True)
        filt = {"rows_by_candidates": a, "rows_by_candidates_deeper_cut": c, "rows_by_whole_row_path": b,
                "calls": nsets}
    return dict(wid=wid, sets=sets, first=first, nsets=nsets, nbytes=nbytes, ws=ws, runners=runners, K=K,
                ms_max=ms_max, value=value, kps=kps, k_avg_ms=k_avg_ms, clocks=sampler.summary(),
                alg=algorithmic_bytes(wid, first), round_bytes=rb / nsets,
                mean_tau=float((acc.float() + 1).mean()), hist=accept_histogram(wid, first, acc), filt=filt)


ROW_KERNEL = "k_stats (streams every logit row once)"


def roofline_of(m, peaks, peak_kind):
    achieved = m["alg"] / (m["k_avg_ms"] / 1e3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": profile_traffic(m["wid"]),
            "kernel": ROW_KERNEL, "kernel_ms": round(m["k_avg_ms"], 5),
            "algorithmic_bytes_per_launch": m["alg"],
            "peak_source": ("measured (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)" if peak_kind == "measured"
                            else "fallback (MEASURED_PEAKS.json absent: 6650 GB/s, an earlier copy measurement on B200)"),
            "frac_of_nominal_8000_gbs": round(achieved / 8000.0, 4)}


def config_summary(m, peaks, peak_kind, cpu=None) -> dict:
    """The per_config entry of one measured workload."""
    step_s = m["ms_max"] / m["K"] / 1e3
    d = {"workload": describe(m["wid"], m["first"])["workload"], "steps": m["K"],
         "rounds_per_s": round(m["value"], 2), "step_us": round(step_s * 1e6, 3),
         "gpu_launches_per_step": m["kps"],
         "row_kernel": roofline_of(m, peaks, peak_kind),
         "round_algorithmic_bytes": int(m["round_bytes"]),
         "round_hbm_gbs": round(m["round_bytes"] / step_s / 1e9, 1),
         "round_frac": round(m["round_bytes"] / step_s / 1e9 / peaks["hbm_gbs"], 4),
         "mean_tau": round(m["mean_tau"], 4), "accept_length_histogram": m["hist"],
         "clocks": m["clocks"]}
    if cpu is not None:
        d["cpu_baseline"] = cpu
    return d


def run_reference(args, ws_, rank):
    import torch
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    sets, nbytes = input_sets(args.workload, dev)
    inp = sets[0]
    steps = max(1, args.steps)
    # each step is a bounded sample of the workload (see cpu_baseline)
    cb, _, _ = cpu_baseline(args.workload, inp, seconds=min(60.0, max(5.0, 0.02 * steps)))
    cfg = bench_config(args.workload, inp, len(sets), nbytes, ws_)
    line = {"impl": "reference", "metric": "verify rounds/s", "value": cb["value"], "unit": "rounds/s",
            "n_gpus": ws_, "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 / cb["value"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": cfg, "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "rounds/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_list(args):
    if args.configs is None:
        return [0, 1, 2, 3, 4] if args.workload == 1 else []
    if args.configs.strip().lower() in ("", "none"):
        return []
    return [int(c) for c in args.configs.split(",")]


def main():
    args = parse()
    ws_, rank, local = dist_env()
    import torch
    import torch.distributed as dist
    if ws_ > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if args.impl == "reference":
        run_reference(args, ws_, rank)
        if ws_ > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wid = args.workload

    m = measure(wid, dev, ws_, args.steps, args.warmup, local, rank, diag=args.with_diag)
    first, sets, ws, K = m["first"], m["sets"], m["ws"], m["K"]
    peaks, peak_kind = measured_peaks()
    roofline = roofline_of(m, peaks, peak_kind)
    value, ms_max = m["value"], m["ms_max"]
    B = first.B
    draft_per_round = B * (first.gamma if wid in (0, 1, 4, 6, 7) else first.N - 1)

    # --- end to end through the binding with host buffers
    e2e = run_e2e(wid, first, ws, args.e2e_steps, dev, ws_) if wid != 7 else {
        "value": None, "unit": "rounds/s", "note": "one rank of a vocabulary-parallel round: no single-GPU host path"}

    # --- the row-on-demand entry point on the same input sets
    # (the filtered chain has no row-on-demand variant)
    lazy = run_lazy(wid, sets, ws, args.lazy_steps, m["alg"], ws_, dev) \
        if args.lazy_steps > 0 and wid in (0, 1, 2, 3, 4, 5, 8) else None

    cfg = bench_config(wid, first, m["nsets"], m["nbytes"], ws_)
    if args.with_diag:
        cfg["diagnostics"] = "requested"
    line = {
        "metric": "verify rounds/s", "value": round(value, 2), "unit": "rounds/s", "n_gpus": ws_,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_max / K, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg,
        "timing": "CUDA-graph replays, CUDA events, max over ranks",
        "roofline": roofline,
        "round_hbm_gbs": round(m["round_bytes"] / (ms_max / K / 1e3) / 1e9, 1),
        "draft_tokens_verified_per_s": round(value * draft_per_round, 1),
        "accepted_tokens_per_s": round(value * B * m["mean_tau"], 1), "mean_tau": round(m["mean_tau"], 4),
        "accept_length_histogram": m["hist"],
        "e2e": e2e, "gpu_launches": K * m["kps"], "clocks": m["clocks"], "lazy": lazy,
    }
    if m["filt"] is not None:
        line["filter_rows"] = m["filt"]
    cpu_here = rank == 0 and ws_ == 1 and not args.no_cpu_baseline
    if cpu_here:
        cb, o, rows = cpu_baseline(wid, first, args.cpu_seconds)
        one, _, _ = cpu_baseline(wid, first, args.cpu_seconds / 4, nthreads=1)
        cb["value_1thread"] = one["value"]
        cb["parity"] = sample_parity(wid, first, o, rows, ws)
        line["cpu_baseline"] = cb
    elif rank == 0:
        line["cpu_baseline"] = None

    # --- every benchmark configuration, measured the same way
    per = {}
    for c in config_list(args):
        if c == wid:
            per[str(c)] = config_summary(m, peaks, peak_kind, line.get("cpu_baseline"))
            continue
        mc = measure(c, dev, ws_, CONFIG_STEPS.get(c, 200), 10, local, rank)
        cpu = None
        if cpu_here:
            cpu, o, rows = cpu_baseline(c, mc["first"], args.config_cpu_seconds)
            cpu["parity"] = sample_parity(c, mc["first"], o, rows, mc["ws"])
        per[str(c)] = config_summary(mc, peaks, peak_kind, cpu)
        del mc
        torch.cuda.empty_cache()
    if per:
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws_ > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_lazy(wid, sets, ws, steps, alg, world, dev):
    """Time the lazy entry point (whole rotations of the input sets in one CUDA
    graph, CUDA events, max over ranks) and count the logit bytes it reads."""
    import torch
    runners = [Runner(wid, s, ws, lazy=True) for s in sets]
    for _ in range(3):
        for r in runners:
            r()
    torch.cuda.synchronize()
    read = 0
    for r, s in zip(runners, sets):
        read += lazy_bytes_read(wid, s, r.num_accepted())
    read /= len(sets)
    from speculative_decoding_verify_temperature_b200 import spec_verify as sv
    n0 = sv.spec_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for r in runners:
            r()
    launches = (sv.spec_launch_count() - n0) // len(runners)
    reps = max(1, steps // len(runners))
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max_ms(e0.elapsed_time(e1), world, dev)
    n = reps * len(runners)
    del graph
    return {"entry": "spec_verify_*_lazy (row-on-demand level walk)", "steps": n,
            "ms_per_step": round(ms / n, 6), "value": round(job_value(n, world, ms), 2), "unit": "rounds/s",
            "gpu_launches_per_step": launches,
            "logit_bytes_read_per_step": int(read), "fraction_of_dense_bytes": round(read / alg, 4),
            "achieved_gbs_on_bytes_read": round(read / (ms / n / 1e3) / 1e9, 1)}


def run_e2e(wid, inp, ws, steps, dev, world=1):
    """Same metric through the binding: every step copies this round's inputs from
    pinned host memory, verifies, and copies the outputs back.  With several
    ranks, the whole job's rounds/s over the slowest rank's time, and the bytes
    all ranks copy per step."""
    import torch
    host = {k: v.detach().cpu().pin_memory() for k, v in vars(inp).items() if isinstance(v, torch.Tensor)}
    meta = getattr(inp, "meta", None) or {}
    host.update({"meta." + k: v.detach().cpu().pin_memory() for k, v in meta.items() if isinstance(v, torch.Tensor)})
    dev_bufs = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    import copy
    dinp = copy.copy(inp)
    if meta:
        dinp.meta = dict(meta)
    for k, v in dev_bufs.items():
        if k.startswith("meta."):
            dinp.meta[k[5:]] = v
        else:
            setattr(dinp, k, v)
    runner = Runner(wid, dinp, ws)
    out_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in runner.out]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(o.numel() * o.element_size() for o in out_host)
    stream = torch.cuda.current_stream()

    def step():
        for k, v in host.items():
            dev_bufs[k].copy_(v, non_blocking=True)
        runner()
        for o, h in zip(runner.out, out_host):
            h.copy_(o, non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max_ms(e0.elapsed_time(e1), world, dev)
    return {"value": round(job_value(steps, world, ms), 2), "unit": "rounds/s", "h2d_bytes_per_step": h2d * world,
            "d2h_bytes_per_step": d2h * world, "steps": steps}


if __name__ == "__main__":
    main()
