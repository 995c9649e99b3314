"""Seeded synthetic inputs for the verify step.

This module only draws random numbers and lays them out in the buffers the
verify step reads. It holds none of the verify arithmetic (no attention, no
target softmax, no accept test, no resampling), so the CUDA path and the CPU
oracle can both be fed from it without sharing method code.

The workloads stand in for the long-tail rollout phase the source pages
describe (few active sequences with long contexts, a shrinking batch, γ from 2
to 10, EfficientRollout "Problem background"; TLT "2. When SD wins"; History
Tree Dynamic RL §5 results table with ~6k-token average responses). No dataset
is read: every tensor is drawn from a seeded torch CPU generator.

Recipe (all configurations):
  * q, K, V ~ N(0, 1) rounded to bf16 (round-to-nearest-even).
  * Paged KV pool ``[num_blocks][Hkv][16][D]``; every sequence's logical pages
    map to a random permutation of the physical pages.
  * Slots past ``ctx_len`` in a sequence's last page, and one guard page that
    every unused block-table entry points at, are filled with bf16 NaN: a
    kernel that reads a key it must not see poisons its output.
  * Target logits ~ N(0, sigma_l^2) in fp32.
  * Draft distribution for draft node c: q_c = softmax((l_parent(c) + sigma_q*eps_c)/T)
    with eps_c ~ N(0, 1) drawn per node; this models a drafter that is a
    perturbed copy of the target (EfficientRollout "Key modules" 1: a quantised
    self-drafter). sigma_q was fixed so the mean per-token acceptance
    sum_x min(p, q) is about 0.7 (0.75 at V~152k, T=1; 0.6 at V=128256, T=0.7).
  * Draft tokens d_c ~ q_c (inverse CDF of a generator uniform); at T=0 the
    drafter is greedy: d_c = argmax(l_parent(c) + sigma_q*eps_c).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import torch

BLOCK_SIZE = 16
BF16_NAN = 0x7FC0

# Tree used by the tree-verify workload: parents of nodes 0..10 (node 0 is the
# root row, i.e. the last accepted token). Root fans out 3; node 1 -> 2
# children; node 4 -> 2; node 7 -> 1 (the 3-2-2-1 spine), plus node 6 under
# node 2 and node 10 under node 5. Depths of nodes 1..10: 1,1,1,2,2,2,3,3,4,3.
TREE_PARENTS_3221 = [-1, 0, 0, 0, 1, 1, 2, 4, 4, 7, 5]


def chain_parents(num_rows: int) -> List[int]:
    """Parent array of a chain of ``num_rows`` rows: row c's parent is c-1."""
    return [-1] + list(range(num_rows - 1))


def ancestor_masks(parents: Sequence[int]) -> np.ndarray:
    """uint64 mask per row: bit j set iff node j is the row itself or one of its ancestors."""
    n = len(parents)
    if n > 64:
        raise ValueError("at most 64 rows fit a uint64 ancestor mask")
    masks = np.zeros(n, dtype=np.uint64)
    for i in range(n):
        m = 0
        j = i
        while j >= 0:
            m |= 1 << j
            j = parents[j]
        masks[i] = np.uint64(m)
    return masks


@dataclasses.dataclass
class AttnInputs:
    num_seqs: int
    num_q_rows: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    max_blocks_per_seq: int
    num_blocks: int
    q: torch.Tensor            # bf16 [B][N][Hq][D]
    k_pool: torch.Tensor       # bf16 [num_blocks][Hkv][bs][D]
    v_pool: torch.Tensor       # bf16 [num_blocks][Hkv][bs][D]
    block_table: torch.Tensor  # int32 [B][max_blocks_per_seq]
    ctx_lens: torch.Tensor     # int32 [B] (includes the N new positions)
    draft_mask: Optional[torch.Tensor]  # int64 view of uint64 [B][N], or None for a chain
    guard_block: int
    # groups of consecutive sequences sharing prefix pages (None: no groups):
    # group g = sequences [group_offsets[g], group_offsets[g+1]), prefix_lens[g] shared keys
    group_offsets: Optional[List[int]] = None
    prefix_lens: Optional[List[int]] = None

    def kv_bytes_unique(self) -> int:
        """Bytes of K and V pages that hold at least one visible key (shared pages once)."""
        tbl = self.block_table.numpy()
        seen = set()
        for b, c in enumerate(self.ctx_lens.tolist()):
            nb = (c + self.block_size - 1) // self.block_size
            seen.update(tbl[b, :nb].tolist())
        per_block = 2 * self.num_kv_heads * self.block_size * self.head_dim * 2
        return len(seen) * per_block

    def kv_bytes_logical(self) -> int:
        """Bytes of K and V for every sequence's visible keys, counted per sequence."""
        return int(sum(self.ctx_lens.tolist())) * 2 * self.num_kv_heads * self.head_dim * 2


@dataclasses.dataclass
class AcceptInputs:
    num_seqs: int
    num_rows: int
    vocab: int
    tree_parents: Optional[List[int]]  # None = chain
    target_logits: torch.Tensor  # fp32 [B][N][V]
    draft_probs: torch.Tensor    # fp32 [B][N-1][V]
    draft_tokens: torch.Tensor   # int32 [B][N-1]
    temperature: float


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def make_ctx_lens(kind: str, num_seqs: int, num_q_rows: int, seed: int, **kw) -> List[int]:
    """Context lengths (including the num_q_rows new positions).

    kind: 'fixed' (kw: length), 'uniform' (kw: lo, hi; inclusive),
    'lognormal' (kw: median, sigma, lo, hi: clamp bounds).
    """
    rng = np.random.default_rng(seed)
    if kind == "fixed":
        out = [int(kw["length"])] * num_seqs
    elif kind == "uniform":
        out = rng.integers(kw["lo"], kw["hi"] + 1, size=num_seqs).tolist()
    elif kind == "lognormal":
        x = rng.lognormal(math.log(kw["median"]), kw["sigma"], size=num_seqs)
        out = np.clip(np.rint(x), kw["lo"], kw["hi"]).astype(np.int64).tolist()
    else:
        raise ValueError(kind)
    return [max(int(c), num_q_rows) for c in out]


def make_attention_inputs(num_q_rows: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                          ctx_lens: Sequence[int], seed: int,
                          parents: Optional[Sequence[int]] = None,
                          shared_prefix_groups: int = 0, shared_prefix_tokens: int = 0,
                          explicit_chain_mask: bool = False,
                          max_blocks_per_seq: Optional[int] = None,
                          extra_blocks: int = 0) -> AttnInputs:
    """Paged-KV verify-attention inputs.

    ``shared_prefix_groups`` > 0 splits the sequences into that many equal
    groups whose first ``shared_prefix_tokens`` (a multiple of 16) map to the
    same physical pages (GRPO rollouts of one prompt sharing its KV).
    ``parents`` gives a draft tree (ancestor masks are produced); None means a
    chain, passed as a NULL mask unless ``explicit_chain_mask``.
    """
    bs = BLOCK_SIZE
    B = len(ctx_lens)
    N = num_q_rows
    g = _gen(seed)
    rng = np.random.default_rng(seed + 7919)

    nblk = [(c + bs - 1) // bs for c in ctx_lens]
    mb = max(nblk) if max_blocks_per_seq is None else int(max_blocks_per_seq)
    if max(nblk) > mb:
        raise ValueError("a context does not fit max_blocks_per_seq")

    shared_pages = 0
    if shared_prefix_groups:
        if shared_prefix_tokens % bs or B % shared_prefix_groups:
            raise ValueError("shared prefix must be whole pages and groups equal-sized")
        shared_pages = shared_prefix_tokens // bs
        for c in ctx_lens:
            if c < shared_prefix_tokens + N:
                raise ValueError("context shorter than the shared prefix plus the new rows")
    # logical page -> slot in a list of unique pages
    unique = 0
    logical = []
    group_size = B // shared_prefix_groups if shared_prefix_groups else 0
    group_base = {}
    for b in range(B):
        row = []
        for j in range(nblk[b]):
            if shared_prefix_groups and j < shared_pages:
                key = (b // group_size, j)
                if key not in group_base:
                    group_base[key] = unique
                    unique += 1
                row.append(group_base[key])
            else:
                row.append(unique)
                unique += 1
        logical.append(row)
    num_blocks = unique + 1 + int(extra_blocks)  # + guard page (+ spares)
    perm = rng.permutation(num_blocks)
    guard = int(perm[unique])

    table = np.full((B, mb), guard, dtype=np.int32)
    for b in range(B):
        for j, u in enumerate(logical[b]):
            table[b, j] = perm[u]

    shape = (num_blocks, num_kv_heads, bs, head_dim)
    k_pool = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v_pool = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    q = torch.randn((B, N, num_q_heads, head_dim), generator=g, dtype=torch.float32).to(torch.bfloat16)

    kv16 = k_pool.view(torch.int16)
    vv16 = v_pool.view(torch.int16)
    nan16 = np.int16(np.uint16(BF16_NAN).view(np.int16))
    kv16[guard] = int(nan16)
    vv16[guard] = int(nan16)
    for b in range(B):
        c = ctx_lens[b]
        last = c // bs
        if c % bs:
            pid = int(table[b, last])
            kv16[pid, :, c % bs:, :] = int(nan16)
            vv16[pid, :, c % bs:, :] = int(nan16)

    mask = None
    if parents is not None or explicit_chain_mask:
        par = list(parents) if parents is not None else chain_parents(N)
        if len(par) != N:
            raise ValueError("parents must have one entry per query row")
        m = ancestor_masks(par)
        mask = torch.from_numpy(np.tile(m, (B, 1)).view(np.int64).copy())

    offsets = prefix = None
    if shared_prefix_groups:
        offsets = [g * group_size for g in range(shared_prefix_groups + 1)]
        prefix = [int(shared_prefix_tokens)] * shared_prefix_groups
    return AttnInputs(B, N, num_q_heads, num_kv_heads, head_dim, bs, mb, num_blocks,
                      q.contiguous(), k_pool.contiguous(), v_pool.contiguous(),
                      torch.from_numpy(table), torch.tensor(list(ctx_lens), dtype=torch.int32),
                      mask, guard, offsets, prefix)


def make_accept_inputs(num_seqs: int, num_rows: int, vocab: int, seed: int, *,
                       logit_std: float, draft_noise: float, temperature: float,
                       parents: Optional[Sequence[int]] = None,
                       draft_temperature: Optional[float] = None) -> AcceptInputs:
    """Target logits, per-node draft distributions and drafted tokens.

    ``draft_temperature`` defaults to ``temperature`` (1.0 for a greedy run).
    """
    B, N, V = num_seqs, num_rows, vocab
    par = list(parents) if parents is not None else chain_parents(N)
    g = _gen(seed)
    logits = torch.randn((B, N, V), generator=g, dtype=torch.float32) * float(logit_std)
    Tq = draft_temperature if draft_temperature is not None else (temperature if temperature > 0 else 1.0)
    q = torch.empty((B, max(N - 1, 0), V), dtype=torch.float32)
    d = torch.empty((B, max(N - 1, 0)), dtype=torch.int32)
    for c in range(1, N):
        lp = logits[:, par[c], :].double()
        noisy = lp + torch.randn((B, V), generator=g, dtype=torch.float64) * float(draft_noise)
        z = noisy / Tq
        z = z - z.max(dim=1, keepdim=True).values
        e = torch.exp(z)
        qc = (e / e.sum(dim=1, keepdim=True)).float()
        q[:, c - 1, :] = qc
        if temperature > 0:
            u = torch.rand((B, 1), generator=g, dtype=torch.float64)
            cdf = torch.cumsum(qc.double(), dim=1)
            cdf = cdf / cdf[:, -1:]
            tok = torch.searchsorted(cdf, u).clamp_(max=V - 1)
            d[:, c - 1] = tok[:, 0].to(torch.int32)
        else:
            d[:, c - 1] = torch.argmax(noisy, dim=1).to(torch.int32)
    return AcceptInputs(B, N, V, None if parents is None else par, logits.contiguous(),
                        q.contiguous(), d.contiguous(), float(temperature))


def make_accept_paths(num_q_rows: int, parents: Optional[Sequence[int]], num_seqs: int, seed: int,
                      max_len: Optional[int] = None):
    """Seeded accepted paths of the shape the accept call returns: per sequence a
    random walk from the root down the draft tree (a chain when parents is None),
    stopping at a random depth. Returns (accept_len int32 [B], accept_path int32
    [B][N-1], -1 after the end)."""
    N = num_q_rows
    par = list(parents) if parents is not None else [-1] + list(range(N - 1))
    children = [[c for c in range(1, N) if par[c] == v] for v in range(N)]
    rng = np.random.default_rng(seed)
    alen = np.zeros(num_seqs, dtype=np.int32)
    path = np.full((num_seqs, max(N - 1, 1)), -1, dtype=np.int32)
    for b in range(num_seqs):
        v, depth = 0, 0
        target = int(rng.integers(0, N)) if max_len is None else int(max_len)
        while depth < target and children[v]:
            v = int(rng.choice(children[v]))
            path[b, depth] = v
            depth += 1
        alen[b] = depth
    return torch.from_numpy(alen), torch.from_numpy(path)


# ---------------------------------------------------------------------------
# The five workloads. Layer counts come from the public model configs of the
# named model shapes and turn one layer's attention time into a verify step.
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    num_layers: int
    attn: dict
    accept: dict


def workload(name: str, **over) -> Workload:
    """Return the recipe of a named workload; keyword overrides replace fields."""
    if name == "tiny_chain":
        N = 5
        attn = dict(num_q_rows=N, num_q_heads=4, num_kv_heads=1, head_dim=64,
                    ctx=dict(kind="fixed", length=128), num_seqs=2, seed=1001)
        acc = dict(num_seqs=2, num_rows=N, vocab=1000, seed=2001, logit_std=2.0,
                   draft_noise=0.5, temperature=1.0)
        w = Workload(name, 1, attn, acc)
    elif name == "qwen7b_longtail":
        N = 5
        attn = dict(num_q_rows=N, num_q_heads=28, num_kv_heads=4, head_dim=128,
                    ctx=dict(kind="uniform", lo=4096, hi=16384), num_seqs=8, seed=1002)
        acc = dict(num_seqs=8, num_rows=N, vocab=152064, seed=2002, logit_std=3.0,
                   draft_noise=0.75, temperature=1.0)
        w = Workload(name, 28, attn, acc)
    elif name == "qwen32b_sweep":
        B = over.pop("num_seqs", 16)
        gamma = over.pop("gamma", 4)
        N = gamma + 1
        attn = dict(num_q_rows=N, num_q_heads=40, num_kv_heads=8, head_dim=128,
                    ctx=dict(kind="lognormal", median=6144, sigma=0.75, lo=512, hi=32768),
                    num_seqs=B, seed=1003)
        acc = dict(num_seqs=B, num_rows=N, vocab=152064, seed=2003, logit_std=3.0,
                   draft_noise=0.75, temperature=1.0)
        w = Workload(f"{name}_B{B}_g{gamma}", 64, attn, acc)
    elif name == "tree_qwen3_30b":
        N = len(TREE_PARENTS_3221)
        attn = dict(num_q_rows=N, num_q_heads=32, num_kv_heads=4, head_dim=128,
                    ctx=dict(kind="fixed", length=24576), num_seqs=16, seed=1004,
                    parents=TREE_PARENTS_3221)
        acc = dict(num_seqs=16, num_rows=N, vocab=151936, seed=2004, logit_std=3.0,
                   draft_noise=0.75, temperature=1.0, parents=TREE_PARENTS_3221)
        w = Workload(name, 48, attn, acc)
    elif name == "grpo_shared_prefix":
        N = 7
        T = over.pop("temperature", 0.0)
        attn = dict(num_q_rows=N, num_q_heads=32, num_kv_heads=8, head_dim=128,
                    ctx=dict(kind="uniform", lo=1024 + 2048, hi=1024 + 12288), num_seqs=64,
                    seed=1005, shared_prefix_groups=4, shared_prefix_tokens=1024)
        acc = dict(num_seqs=64, num_rows=N, vocab=128256, seed=2005, logit_std=3.0,
                   draft_noise=0.6, temperature=T, draft_temperature=0.7)
        w = Workload(f"{name}_T{T:g}", 32, attn, acc)
    elif name == "grpo_long_prompt":
        # the same group shape with long prompts: 8 groups of 16 rollouts whose
        # 8192 shared prompt tokens are most of each context (the shared pages,
        # 268 MB a layer, no longer fit in L2)
        N = 7
        T = over.pop("temperature", 0.0)
        attn = dict(num_q_rows=N, num_q_heads=32, num_kv_heads=8, head_dim=128,
                    ctx=dict(kind="uniform", lo=8192 + 512, hi=8192 + 4096), num_seqs=128,
                    seed=1006, shared_prefix_groups=8, shared_prefix_tokens=8192)
        acc = dict(num_seqs=128, num_rows=N, vocab=128256, seed=2006, logit_std=3.0,
                   draft_noise=0.6, temperature=T, draft_temperature=0.7)
        w = Workload(f"{name}_T{T:g}", 32, attn, acc)
    else:
        raise ValueError(f"unknown workload {name}")
    for k, v in over.items():
        if k in w.attn:
            w.attn[k] = v
        elif k in w.accept:
            w.accept[k] = v
        else:
            raise KeyError(k)
    return w


def build_attention(w: Workload, seed_offset: int = 0) -> AttnInputs:
    a = dict(w.attn)
    ctx = a.pop("ctx")
    B = a.pop("num_seqs")
    seed = a.pop("seed") + seed_offset
    lens = make_ctx_lens(ctx["kind"], B, a["num_q_rows"], seed,
                         **{k: v for k, v in ctx.items() if k != "kind"})
    return make_attention_inputs(ctx_lens=lens, seed=seed, **a)


def build_accept(w: Workload, seed_offset: int = 0) -> AcceptInputs:
    a = dict(w.accept)
    a["seed"] = a["seed"] + seed_offset
    return make_accept_inputs(**a)
