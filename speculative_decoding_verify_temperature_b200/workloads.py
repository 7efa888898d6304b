"""Seeded synthetic inputs for the verify/accept step.

This module is the one piece of code that both the CUDA path (tests, bench)
and the fp64 oracle consume: it makes the bytes both sides read.  It holds no
verify arithmetic.  What it does compute is the *input side* of a
speculative-decoding round, which the pages place outside the verify step:

* target logits (Gaussian, optionally with a log-Zipf rank bias),
* a stand-in drafter: draft logits = target + noise, draft tokens drawn from
  the draft distribution by the Gumbel-max trick (or by ``torch.multinomial``
  when the draft is given as probabilities), top-k style tree tokens,
* seeded uniforms ``u = k * 2**-24`` with ``k`` uniform in ``[0, 2**24)``
  (exactly representable in f32 and fp64).

Shapes, dtypes and value distributions follow the five serving-shaped
workloads of the verify benchmark (chain B1/gamma4/V1000 f32; chain
B64/gamma5/V32000 bf16; greedy tree B32/N64/V128256 bf16; target-only tree
B128/N32/V151936 bf16; chain B512/gamma7/V129280 bf16 + f32 draft
probabilities).  Everything is generated with ``torch.Generator`` seeded per
round: ``seed = 0x5EED0000 + 1000 * workload_id + round``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

SEED_BASE = 0x5EED0000
_U24 = 2.0 ** -24


def round_seed(workload_id: int, rnd: int) -> int:
    return SEED_BASE + 1000 * int(workload_id) + int(rnd)


def make_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def uniforms(shape, gen: torch.Generator, device) -> torch.Tensor:
    """f32 uniforms in [0, 1) on the 2**-24 grid (exact in f32 and fp64)."""
    k = torch.randint(0, 1 << 24, tuple(shape), generator=gen, device=device, dtype=torch.int64)
    return k.to(torch.float32) * _U24


def zipf_bias(V: int, gen: torch.Generator, device, s: float = 1.1) -> torch.Tensor:
    """Log-Zipf rank prior b_v = -s * ln(1 + rank(v)), rank = a seeded vocab permutation."""
    rank = torch.randperm(V, generator=gen, device=device)
    return -s * torch.log1p(rank.to(torch.float32))


def padded(shape_bvs, V: int, stride: int | None, dtype, device) -> torch.Tensor:
    """Allocate ``[B, R, stride]`` storage (zero padding past V) and return it."""
    B, R = shape_bvs
    stride = V if stride is None else int(stride)
    assert stride >= V
    return torch.zeros((B, R, stride), dtype=dtype, device=device)


def gumbel_argmax(logits_f32: torch.Tensor, inv_temp: torch.Tensor, gen: torch.Generator) -> torch.Tensor:
    """Stand-in drafter: a draw from softmax(logits/T) via the Gumbel-max trick.

    ``logits_f32`` is ``[B, R, V]``; ``inv_temp`` is ``[B]``.  Returns int32 ``[B, R]``.
    """
    u = torch.rand(logits_f32.shape, generator=gen, device=logits_f32.device, dtype=torch.float32)
    u = u.clamp_min_(1e-12)
    g = -torch.log(-torch.log(u))
    scores = logits_f32 * inv_temp.view(-1, 1, 1) + g
    return scores.argmax(dim=-1).to(torch.int32)


# ----------------------------------------------------------------------------- chain


@dataclass
class ChainInputs:
    target: torch.Tensor          # [B, gamma+1, stride] bf16 or f32
    draft: torch.Tensor           # [B, gamma, dstride] logits (bf16/f32) or f32 probs
    draft_is_probs: bool
    draft_tokens: torch.Tensor    # [B, gamma] int32
    temperature: torch.Tensor     # [B] f32
    coins: torch.Tensor           # [B, gamma] f32
    final_u: torch.Tensor         # [B] f32
    V: int
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.target.shape[0]

    @property
    def gamma(self):
        return self.target.shape[1] - 1


def chain_inputs(B: int, gamma: int, V: int, *, seed: int, device="cpu",
                 target_dtype=torch.bfloat16, draft_dtype=torch.bfloat16,
                 draft_is_probs: bool = False, target_sigma: float = 3.0,
                 zipf: bool = False, draft_noise: float = 1.0,
                 temperatures=(1.0,), stride: int | None = None,
                 dstride: int | None = None) -> ChainInputs:
    """One round of chain inputs.

    target = N(0, sigma^2) [+ log-Zipf bias]; draft logits = target (as stored,
    widened to f32) + N(0, draft_noise^2), stored in ``draft_dtype``; or, with
    ``draft_is_probs``, draft = softmax(target + N(0, draft_noise^2)) in f32 at
    T = 1.  Draft tokens are drawn from the draft distribution at the
    sequence's temperature (probabilities: as given).  Temperatures are drawn
    uniformly from ``temperatures`` per sequence.
    """
    g = make_gen(seed, device)
    R = gamma + 1
    tgt = torch.randn((B, R, V), generator=g, device=device, dtype=torch.float32) * target_sigma
    if zipf:
        tgt += zipf_bias(V, g, device).view(1, 1, V)
    target = padded((B, R), V, stride, target_dtype, device)
    target[:, :, :V] = tgt.to(target_dtype)
    tgt_stored = target[:, :, :V].to(torch.float32)
    del tgt
    temps = torch.tensor(list(temperatures), dtype=torch.float32, device=device)
    if len(temperatures) > 1:
        idx = torch.randint(0, len(temperatures), (B,), generator=g, device=device)
        temperature = temps[idx].contiguous()
    else:
        temperature = temps.expand(B).contiguous()
    if draft_is_probs:
        draft = padded((B, gamma), V, dstride, torch.float32, device)
        toks = torch.empty((B, gamma), dtype=torch.int32, device=device)
        # Chunk over sequences to bound the temporaries at large B*V.
        step = max(1, (1 << 27) // max(1, gamma * V))
        for b0 in range(0, B, step):
            b1 = min(B, b0 + step)
            noisy = tgt_stored[b0:b1, :gamma] + draft_noise * torch.randn(
                (b1 - b0, gamma, V), generator=g, device=device, dtype=torch.float32)
            q = torch.softmax(noisy, dim=-1)
            draft[b0:b1, :, :V] = q
            toks[b0:b1] = torch.multinomial(q.view(-1, V), 1, generator=g).view(b1 - b0, gamma).to(torch.int32)
            del noisy, q
    else:
        dl = tgt_stored[:, :gamma] + draft_noise * torch.randn(
            (B, gamma, V), generator=g, device=device, dtype=torch.float32)
        draft = padded((B, gamma), V, dstride, draft_dtype, device)
        draft[:, :, :V] = dl.to(draft_dtype)
        toks = gumbel_argmax(draft[:, :, :V].to(torch.float32), 1.0 / temperature, g)
        del dl
    coins = uniforms((B, gamma), g, device)
    final_u = uniforms((B,), g, device)
    return ChainInputs(target, draft, draft_is_probs, toks.contiguous(), temperature, coins,
                       final_u, V)


def chain_config0_logits(device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """Fixed logits of the small chain workload: B=1, gamma=4, V=1000, f32,
    target ~ N(0, 2^2), draft = target + N(0, 0.5^2)."""
    g = make_gen(round_seed(0, 0), device)
    target = torch.randn((1, 5, 1000), generator=g, device=device) * 2.0
    draft = target[:, :4] + 0.5 * torch.randn((1, 4, 1000), generator=g, device=device)
    return target.contiguous(), draft.contiguous()


def chain_config0_round(rnd: int, target: torch.Tensor, draft: torch.Tensor,
                        device="cpu") -> ChainInputs:
    """Round ``rnd`` of the small chain workload: fresh draft tokens and uniforms
    over the fixed logits, T = 1."""
    g = make_gen(round_seed(0, 1 + rnd), device)
    temperature = torch.ones(1, dtype=torch.float32, device=device)
    toks = gumbel_argmax(draft.to(torch.float32), 1.0 / temperature, g)
    coins = uniforms((1, 4), g, device)
    final_u = uniforms((1,), g, device)
    return ChainInputs(target, draft, False, toks, temperature, coins, final_u, 1000)


def chain_config1(rnd: int = 0, device="cpu") -> ChainInputs:
    """B=64, gamma=5, V=32000, bf16 target N(0, 3^2) + log-Zipf(1.1) bias, bf16
    draft logits = target + N(0, 1), T in {0.6, 1.0} per sequence."""
    return chain_inputs(64, 5, 32000, seed=round_seed(1, rnd), device=device, zipf=True,
                        target_sigma=3.0, draft_noise=1.0, temperatures=(0.6, 1.0))


def chain_config6(rnd: int = 0, device="cpu") -> ChainInputs:
    """The B=64, gamma=5, V=32000 chain workload under serving-style filters:
    per sequence top_k drawn from {0 (off), 20, 50} and top_p from {1 (off), 0.9,
    0.95}, in ``meta["top_k"]`` (int32 [B]) and ``meta["top_p"]`` (f32 [B])."""
    inp = chain_config1(rnd, device)
    g = make_gen(round_seed(6, rnd), device)
    ks = torch.tensor([0, 20, 50], dtype=torch.int32, device=device)
    ps = torch.tensor([1.0, 0.9, 0.95], dtype=torch.float32, device=device)
    inp.meta["top_k"] = ks[torch.randint(0, 3, (inp.B,), generator=g, device=device)].contiguous()
    inp.meta["top_p"] = ps[torch.randint(0, 3, (inp.B,), generator=g, device=device)].contiguous()
    return inp


def chain_config4(rnd: int = 0, device="cpu") -> ChainInputs:
    """B=512, gamma=7, V=129280, bf16 target N(0, 3^2), f32 draft probabilities
    softmax(target + N(0, 1.5^2)) at T = 1, T = 1."""
    return chain_inputs(512, 7, 129280, seed=round_seed(4, rnd), device=device,
                        draft_is_probs=True, target_sigma=3.0, draft_noise=1.5,
                        temperatures=(1.0,))


# ----------------------------------------------------------------------------- trees


def level_tree(level_sizes, max_children: int, gen: torch.Generator) -> list[int]:
    """Parent array of a tree built level by level: node 0 is the root; every
    node of level d picks its parent uniformly among the nodes of level d-1
    that still have fewer than ``max_children`` children.  Nodes of a level are
    numbered in order of their parent, so ancestors precede descendants."""
    parents = [-1]
    prev = [0]
    nchild = {0: 0}
    for size in level_sizes:
        picks = []
        for _ in range(size):
            open_ = [n for n in prev if nchild[n] < max_children]
            if not open_:
                raise ValueError("level too wide for max_children")
            j = int(torch.randint(0, len(open_), (1,), generator=gen).item())
            nchild[open_[j]] += 1
            picks.append(open_[j])
        picks.sort()
        cur = []
        for pa in picks:
            parents.append(pa)
            cur.append(len(parents) - 1)
            nchild[len(parents) - 1] = 0
        prev = cur
    return parents


def random_tree(N: int, max_children: int, gen: torch.Generator, max_depth: int | None = None) -> list[int]:
    """Random tree with N nodes: node n >= 1 picks its parent uniformly among
    earlier nodes with spare capacity (and depth < max_depth when given)."""
    parents = [-1]
    depth = [0]
    nchild = [0]
    for n in range(1, N):
        open_ = [m for m in range(n) if nchild[m] < max_children and
                 (max_depth is None or depth[m] < max_depth)]
        j = int(torch.randint(0, len(open_), (1,), generator=gen).item())
        pa = open_[j]
        parents.append(pa)
        depth.append(depth[pa] + 1)
        nchild[pa] += 1
        nchild.append(0)
    return parents


def chain_tree(N: int) -> list[int]:
    return [-1] + list(range(N - 1))


def tree_depth(parents) -> int:
    d = [0] * len(parents)
    for n in range(1, len(parents)):
        d[n] = d[parents[n]] + 1
    return max(d)


@dataclass
class TreeInputs:
    target: torch.Tensor          # [B, N, stride]
    tokens: torch.Tensor          # [B, N] int32 (tokens[:, 0] = root, not read)
    parents: torch.Tensor         # [B, N] int32
    temperature: torch.Tensor     # [B] f32
    coins: torch.Tensor           # [B, N] f32
    final_u: torch.Tensor         # [B] f32
    max_depth: int
    V: int
    draft_probs: torch.Tensor | None = None
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.target.shape[0]

    @property
    def N(self):
        return self.target.shape[1]


def tree_greedy_inputs(B: int, V: int, *, seed: int, device="cpu", parents_fn=None,
                       level_sizes=(8, 11, 11, 11, 11, 11), max_children: int = 8,
                       p_match: float = 0.7, target_sigma: float = 3.0,
                       target_dtype=torch.bfloat16, stride: int | None = None,
                       max_depth: int | None = None, int_logits: int | None = None) -> TreeInputs:
    """Greedy-tree inputs: per sequence a tree (``level_tree`` by default),
    logits N(0, sigma^2) (or, with ``int_logits=k``, integers in [0, k) to force
    many ties), and each draft token equal to the argmax of its parent's logits
    with probability ``p_match``, else uniform in [0, V)."""
    g = make_gen(seed, device)
    gc = make_gen(seed ^ 0x7EE, "cpu")
    par = [parents_fn(gc) if parents_fn else level_tree(level_sizes, max_children, gc) for _ in range(B)]
    N = len(par[0])
    assert all(len(p) == N for p in par)
    md = max(tree_depth(p) for p in par) if max_depth is None else max_depth
    if int_logits:
        lg = torch.randint(0, int_logits, (B, N, V), generator=g, device=device).to(torch.float32)
    else:
        lg = torch.randn((B, N, V), generator=g, device=device, dtype=torch.float32) * target_sigma
    target = padded((B, N), V, stride, target_dtype, device)
    target[:, :, :V] = lg.to(target_dtype)
    del lg
    parents = torch.tensor(par, dtype=torch.int32, device=device)
    amax = target[:, :, :V].to(torch.float32).argmax(dim=-1)            # [B, N]
    pa = parents.clamp_min(0).to(torch.int64)
    parent_amax = torch.gather(amax, 1, pa)
    rnd = torch.randint(0, V, (B, N), generator=g, device=device)
    use = torch.rand((B, N), generator=g, device=device) < p_match
    tokens = torch.where(use, parent_amax, rnd).to(torch.int32)
    tokens[:, 0] = 0
    temperature = torch.ones(B, dtype=torch.float32, device=device)
    coins = uniforms((B, N), g, device)
    final_u = uniforms((B,), g, device)
    return TreeInputs(target, tokens.contiguous(), parents, temperature, coins, final_u, md, V)


def tree_sample_inputs(B: int, V: int, *, seed: int, device="cpu", parents_fn=None,
                       level_sizes=(4, 8, 8, 6, 5), max_children: int = 4,
                       target_sigma: float = 3.0, zipf: bool = True, temperature: float = 0.8,
                       token_noise: float = 1.0, target_dtype=torch.bfloat16,
                       stride: int | None = None, max_depth: int | None = None,
                       draft_probs: str | None = None) -> TreeInputs:
    """Target-only tree inputs: logits N(0, sigma^2) [+ log-Zipf bias]; the
    children of each node carry the distinct top-c tokens of (the node's
    logits + N(0, token_noise^2)), c = its number of children, in rank order
    (a stand-in for a top-k drafter).  ``draft_probs``: None (NULL), "zeros"
    (explicit zero buffer) or "random" (a random distribution per row)."""
    g = make_gen(seed, device)
    gc = make_gen(seed ^ 0x7EE, "cpu")
    par = [parents_fn(gc) if parents_fn else level_tree(level_sizes, max_children, gc) for _ in range(B)]
    N = len(par[0])
    assert all(len(p) == N for p in par)
    md = max(tree_depth(p) for p in par) if max_depth is None else max_depth
    lg = torch.randn((B, N, V), generator=g, device=device, dtype=torch.float32) * target_sigma
    if zipf:
        lg += zipf_bias(V, g, device).view(1, 1, V)
    target = padded((B, N), V, stride, target_dtype, device)
    target[:, :, :V] = lg.to(target_dtype)
    del lg
    parents = torch.tensor(par, dtype=torch.int32, device=device)
    tokens = torch.zeros((B, N), dtype=torch.int32, device=device)
    for b in range(B):
        children = {}
        for n in range(1, N):
            children.setdefault(par[b][n], []).append(n)
        if not children:
            continue
        nodes = sorted(children)
        rows = target[b, nodes, :V].to(torch.float32)
        rows = rows + token_noise * torch.randn(rows.shape, generator=g, device=device)
        k = min(V, max(len(children[n]) for n in nodes))
        top = rows.topk(k, dim=-1).indices.to(torch.int32)
        for i, n in enumerate(nodes):
            for r, c in enumerate(children[n]):
                tokens[b, c] = top[i, r]
    temp = torch.full((B,), float(temperature), dtype=torch.float32, device=device)
    coins = uniforms((B, N), g, device)
    final_u = uniforms((B,), g, device)
    dp = None
    if draft_probs == "zeros":
        dp = torch.zeros((B, N, V), dtype=torch.float32, device=device)
    elif draft_probs == "random":
        dp = torch.softmax(torch.randn((B, N, V), generator=g, device=device) * 2.0, dim=-1)
    elif draft_probs is not None:
        raise ValueError(draft_probs)
    return TreeInputs(target, tokens, parents, temp, coins, final_u, md, V, dp)


def tree_mss_inputs(B: int, V: int, *, seed: int, device="cpu", parents_fn=None,
                    level_sizes=(4, 8, 8, 6, 5), max_children: int = 4,
                    target_sigma: float = 3.0, zipf: bool = True, temperature: float = 0.8,
                    draft_noise: float = 1.0, target_dtype=torch.bfloat16,
                    stride: int | None = None, max_depth: int | None = None) -> TreeInputs:
    """Inputs of tree verification with a draft distribution: logits
    N(0, sigma^2) [+ log-Zipf bias]; the draft distribution of every node is
    q_n = softmax((logits_n + N(0, draft_noise^2)) / T) in f32 (a drafter that
    samples at the target's temperature), and the children of node n carry
    tokens drawn independently from q_n, with replacement (duplicate siblings
    possible), as multi-step speculative sampling assumes."""
    g = make_gen(seed, device)
    gc = make_gen(seed ^ 0x7EE, "cpu")
    par = [parents_fn(gc) if parents_fn else level_tree(level_sizes, max_children, gc) for _ in range(B)]
    N = len(par[0])
    assert all(len(p) == N for p in par)
    md = max(tree_depth(p) for p in par) if max_depth is None else max_depth
    lg = torch.randn((B, N, V), generator=g, device=device, dtype=torch.float32) * target_sigma
    if zipf:
        lg += zipf_bias(V, g, device).view(1, 1, V)
    target = padded((B, N), V, stride, target_dtype, device)
    target[:, :, :V] = lg.to(target_dtype)
    del lg
    dp = padded((B, N), V, -(-V // 4) * 4, torch.float32, device)        # 16-byte aligned f32 rows
    step = max(1, (1 << 26) // max(1, N * V))
    for b0 in range(0, B, step):
        b1 = min(B, b0 + step)
        noisy = target[b0:b1, :, :V].to(torch.float32) + draft_noise * torch.randn(
            (b1 - b0, N, V), generator=g, device=device, dtype=torch.float32)
        dp[b0:b1, :, :V] = torch.softmax(noisy / temperature, dim=-1)
        del noisy
    parents = torch.tensor(par, dtype=torch.int32, device=device)
    tokens = torch.zeros((B, N), dtype=torch.int32, device=device)
    for b in range(B):
        children = {}
        for n in range(1, N):
            children.setdefault(par[b][n], []).append(n)
        for n, ch in children.items():
            draw = torch.multinomial(dp[b, n, :V], len(ch), replacement=True, generator=g)
            tokens[b, ch] = draw.to(torch.int32)
    temp = torch.full((B,), float(temperature), dtype=torch.float32, device=device)
    coins = uniforms((B, N), g, device)
    final_u = uniforms((B,), g, device)
    return TreeInputs(target, tokens, parents, temp, coins, final_u, md, V, dp)


def tree_config5(rnd: int = 0, device="cpu") -> TreeInputs:
    """Tree verification with a draft distribution (multi-step speculative
    sampling): the tree and target of the B=128, 32-node, V=151936 workload
    (bf16 logits N(0, 3^2) + log-Zipf(1.1), T = 0.8) plus f32 draft
    distributions softmax((logits + N(0, 1)) / T) per node, children drawn from
    them."""
    return tree_mss_inputs(128, 151936, seed=round_seed(5, rnd), device=device)


def tree_config2(rnd: int = 0, device="cpu") -> TreeInputs:
    """Greedy tree: B=32, 64 nodes (root + levels 8,11,11,11,11,11; at most 8
    children), V=128256, bf16 logits N(0, 3^2), draft token = parent argmax
    w.p. 0.7 else uniform."""
    return tree_greedy_inputs(32, 128256, seed=round_seed(2, rnd), device=device)


def tree_config3(rnd: int = 0, device="cpu") -> TreeInputs:
    """Target-only tree: B=128, 32 nodes (root + levels 4,8,8,6,5; at most 4
    children), V=151936, bf16 logits N(0, 3^2) + log-Zipf(1.1), T = 0.8,
    draft probabilities NULL (zeros)."""
    return tree_sample_inputs(128, 151936, seed=round_seed(3, rnd), device=device)


def tree_config8(rnd: int = 0, device="cpu") -> TreeInputs:
    """The B=128, 32-node, V=151936 target-only tree workload under serving-style
    filters: per sequence top_k drawn from {0 (off), 20, 50} and top_p from
    {1 (off), 0.9, 0.95}, in ``meta["top_k"]`` (int32 [B]) and ``meta["top_p"]``
    (f32 [B])."""
    inp = tree_config3(rnd, device)
    g = make_gen(round_seed(8, rnd), device)
    ks = torch.tensor([0, 20, 50], dtype=torch.int32, device=device)
    ps = torch.tensor([1.0, 0.9, 0.95], dtype=torch.float32, device=device)
    inp.meta["top_k"] = ks[torch.randint(0, 3, (inp.B,), generator=g, device=device)].contiguous()
    inp.meta["top_p"] = ps[torch.randint(0, 3, (inp.B,), generator=g, device=device)].contiguous()
    return inp


WORKLOADS = {
    0: "chain B=1 gamma=4 V=1000 f32 logits (1000 rounds)",
    1: "chain B=64 gamma=5 V=32000 bf16 target+draft logits, T in {0.6,1.0}",
    2: "greedy tree B=32 N=64 V=128256 bf16",
    3: "target-only tree B=128 N=32 V=151936 bf16, T=0.8, draft_probs NULL",
    4: "chain B=512 gamma=7 V=129280 bf16 target + f32 draft probs, T=1",
    5: "multi-step speculative sampling tree B=128 N=32 V=151936 bf16 + f32 draft distributions, T=0.8",
    6: "chain B=64 gamma=5 V=32000 bf16 target+draft logits, T in {0.6,1.0}, top-k in {0,20,50}, top-p in {1,0.9,0.95}",
    8: "target-only tree B=128 N=32 V=151936 bf16, T=0.8, draft_probs NULL, top-k in {0,20,50}, top-p in {1,0.9,0.95}",
}


def algorithmic_bytes(workload_id: int) -> int:
    """Logit/probability bytes one round must read from HBM (the roofline numerator,
    without the data-dependent residual rows of workload 4)."""
    if workload_id == 0:
        return (5 + 4) * 1000 * 4
    if workload_id == 1:
        return 64 * (6 + 5) * 32000 * 2
    if workload_id == 2:
        return 32 * 64 * 128256 * 2
    if workload_id == 3:
        return 128 * 32 * 151936 * 2
    if workload_id == 4:
        return 512 * 8 * 129280 * 2
    if workload_id == 5:
        return 128 * 32 * 151936 * 2
    if workload_id == 6:
        return 64 * (6 + 5) * 32000 * 2
    if workload_id == 8:
        return 128 * 32 * 151936 * 2
    raise ValueError(workload_id)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("annotations", "math", "torch")]
