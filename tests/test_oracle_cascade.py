"""Pins for the oracle's cascade (shared-prefix) verify attention (no GPU).

The operation is plain verify attention over each member's whole context,
with the group's prefix keys read from the group's first member's pages (SRT
review, "Tree-Structured KV Cache": a shared node is stored once). Pinned by:
a numpy brute force that gathers every key by hand; reduction to the plain
attention oracle when the members' own tables already hold the shared pages and
when the prefix is empty; the invalid-member rules; and the exact log-sum-exp
merge of a prefix-only and a suffix-only softmax, which is how the CUDA path
splits the work.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_rl_b200 import workloads as W


def _grouped(seed, N=3, Hq=4, Hkv=2, D=32, lens=(70, 53, 96, 48, 81), groups=(0, 3, 5),
             prefix=(32, 16), parents=None):
    a = W.make_attention_inputs(N, Hq, Hkv, D, list(lens), seed=seed, parents=parents, extra_blocks=6)
    return a, list(groups), list(prefix)


def _scramble_member_prefixes(a, offsets, prefix, seed):
    """Point every non-first member's prefix entries at other (valid) pages."""
    rng = np.random.default_rng(seed)
    tbl = a.block_table.numpy().copy()
    for g in range(len(prefix)):
        for b in range(offsets[g] + 1, offsets[g + 1]):
            for j in range(prefix[g] // 16):
                tbl[b, j] = rng.integers(0, a.num_blocks)
    a.block_table = torch.from_numpy(tbl)
    return a


def _brute(a, offsets, prefix):
    """Every key gathered by hand: the group's first member's page for t < P, the member's own after."""
    B, N, Hq, Hkv, D = a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads, a.head_dim
    G = Hq // Hkv
    tbl = a.block_table.numpy()
    k = a.k_pool.double().numpy()
    v = a.v_pool.double().numpy()
    q = a.q.double().numpy()
    out = np.zeros((B, N, Hq, D))
    for g in range(len(prefix)):
        for b in range(offsets[g], offsets[g + 1]):
            C = int(a.ctx_lens[b])
            P = prefix[g]
            keys = np.zeros((C, Hkv, D))
            vals = np.zeros((C, Hkv, D))
            for t in range(C):
                src = offsets[g] if t < P else b
                blk = tbl[src, t // 16]
                keys[t] = k[blk, :, t % 16, :]
                vals[t] = v[blk, :, t % 16, :]
            for i in range(N):
                vis = np.ones(C, dtype=bool)
                for j in range(N):
                    if a.draft_mask is None:
                        vis[C - N + j] = j <= i
                    else:
                        vis[C - N + j] = bool((int(a.draft_mask[b, i].item()) >> j) & 1)
                for hq in range(Hq):
                    s = keys[:, hq // G, :] @ q[b, i, hq] / np.sqrt(D)
                    s = np.where(vis, s, -np.inf)
                    w = np.exp(s - s.max())
                    out[b, i, hq] = (w[:, None] * vals[:, hq // G, :]).sum(0) / w.sum()
    return out


@pytest.mark.parametrize("parents", [None, [-1, 0, 0]])
def test_matches_brute_force_with_foreign_member_prefix_pages(parents):
    a, off, pre = _grouped(17, parents=parents)
    a = _scramble_member_prefixes(a, off, pre, seed=4)
    got, flags = oracle.cascade_attention(a, off, pre)
    assert not flags.any()
    np.testing.assert_allclose(got, _brute(a, off, pre), rtol=1e-10, atol=1e-12)


def test_reduces_to_plain_attention_when_pages_are_shared():
    # the members' own tables already map the prefix to the group's pages
    a = W.make_attention_inputs(5, 8, 2, 64, [120, 80, 99, 140], seed=21,
                                shared_prefix_groups=2, shared_prefix_tokens=64)
    plain, pf = oracle.attention(a)
    got, flags = oracle.cascade_attention(a, a.group_offsets, a.prefix_lens)
    np.testing.assert_array_equal(flags, pf)
    np.testing.assert_array_equal(got, plain)


def test_empty_prefix_is_plain_attention_on_own_tables():
    a, off, _ = _grouped(23)
    plain, _ = oracle.attention(a)
    got, flags = oracle.cascade_attention(a, off, [0, 0])
    assert not flags.any()
    np.testing.assert_array_equal(got, plain)


def test_lse_merge_of_prefix_and_suffix_is_exact():
    """softmax over all keys == merge of prefix-only and suffix-only partials by log-sum-exp."""
    a, off, pre = _grouped(29, D=16)
    a = _scramble_member_prefixes(a, off, pre, seed=9)
    want, _ = oracle.cascade_attention(a, off, pre)
    B, N, Hq, Hkv, D = a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads, a.head_dim
    G = Hq // Hkv
    tbl = a.block_table.numpy()
    k, v, q = a.k_pool.double().numpy(), a.v_pool.double().numpy(), a.q.double().numpy()
    for g in range(len(pre)):
        P = pre[g]
        for b in range(off[g], off[g + 1]):
            C = int(a.ctx_lens[b])
            for i in range(N):
                for hq in range(Hq):
                    h = hq // G
                    parts = []
                    for lo, hi, src in ((0, P, off[g]), (P, C, b)):
                        t = np.arange(lo, hi)
                        blk = tbl[src, t // 16]
                        s = k[blk, h, t % 16, :] @ q[b, i, hq] / np.sqrt(D)
                        vis = (t < C - N) | ((t - (C - N)) <= i)
                        s = np.where(vis, s, -np.inf)
                        m = s.max() if s.size and np.isfinite(s).any() else -np.inf
                        w = np.exp(s - m) if np.isfinite(m) else np.zeros_like(s)
                        parts.append((m, w.sum(), (w[:, None] * v[blk, h, t % 16, :]).sum(0)))
                    M = max(p[0] for p in parts)
                    L = sum(np.exp(p[0] - M) * p[1] for p in parts if np.isfinite(p[0]))
                    O = sum(np.exp(p[0] - M) * p[2] for p in parts if np.isfinite(p[0]))
                    np.testing.assert_allclose(O / L, want[b, i, hq], rtol=1e-10, atol=1e-12)


def test_invalid_members():
    a, off, pre = _grouped(31, lens=(70, 53, 96, 48, 81))
    # prefix not a whole number of pages: the whole group is invalid
    out, flags = oracle.cascade_attention(a, off, [24, 16])
    assert flags.tolist() == [1, 1, 1, 0, 0]
    assert not out[:3].any()
    # prefix longer than one member's context minus its new rows: that member only
    out, flags = oracle.cascade_attention(a, off, [64, 16])   # member 1 has 53 < 64 + 3
    assert flags.tolist() == [0, 1, 0, 0, 0]
    assert not out[1].any() and out[0].any() and out[2].any()
    # a bad page in the group's prefix: every member of that group
    tbl = a.block_table.numpy().copy()
    tbl[3, 0] = a.num_blocks + 5
    a.block_table = torch.from_numpy(tbl)
    _, flags = oracle.cascade_attention(a, off, [32, 16])
    assert flags.tolist() == [0, 0, 0, 1, 1]


def test_rows_match_full_and_bad_groups_rejected():
    a, off, pre = _grouped(37)
    a = _scramble_member_prefixes(a, off, pre, seed=2)
    full, _ = oracle.cascade_attention(a, off, pre)
    rows = np.array([[0, 0, 0], [1, 2, 3], [4, 1, 2], [3, 0, 1]], dtype=np.int32)
    part = oracle.cascade_attention(a, off, pre, rows=rows)
    for r, (b, i, hq) in enumerate(rows):
        np.testing.assert_array_equal(part[r], full[b, i, hq])
    with pytest.raises(ValueError):
        oracle.cascade_attention(a, [0, 3, 4], pre)     # does not end at B
    with pytest.raises(ValueError):
        oracle.cascade_attention(a, [0, 4, 3, 5], [0, 0, 0])  # decreasing
