"""Pins of the oracle's KV commit after accept (keep the root and the accepted
draft nodes, compacted behind the root in path order; a chain moves nothing).

The main pin is independent of the gather itself: a query attending over the
committed cache must equal the attention oracle over the original cache with
an explicit mask that leaves visible exactly the prefix, the root and the
accepted nodes (softmax attention does not depend on the order of its keys;
positions are already in K).
"""
import types

import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_rl_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore")


def _pools(a):
    k = a.k_pool.view(torch.int16).numpy().view(np.uint16).copy()
    v = a.v_pool.view(torch.int16).numpy().view(np.uint16).copy()
    return k, v


def _with(a, **kw):
    d = dict(a.__dict__)
    d.update(kw)
    return types.SimpleNamespace(**d)


def _bf16(x_u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x_u16.view(np.int16).copy()).view(torch.bfloat16)


@pytest.mark.parametrize("parents", [None, W.TREE_PARENTS_3221, [-1, 0, 0, 1, 2, 2, 5]])
def test_commit_then_attend_equals_masked_attention(parents):
    N = 5 if parents is None else len(parents)
    lens = [N + 3, 40, 131, 300]
    a = W.make_attention_inputs(N, 6, 2, 64, lens, seed=41, parents=parents)
    alen, path = W.make_accept_paths(N, parents, len(lens), seed=42)
    k, v = _pools(a)
    new_lens, flags = oracle.kv_commit([(k, v)], a.block_table.numpy(), a.ctx_lens.numpy(), alen.numpy(),
                                       path.numpy(), N)
    assert not flags.any()
    C = a.ctx_lens.numpy()
    assert (new_lens == C - N + 1 + alen.numpy()).all()
    # probe query: row 0 of a fresh set of queries
    probe = torch.randn(a.num_seqs, N, a.num_q_heads, a.head_dim, generator=torch.Generator().manual_seed(7))
    probe = probe.to(torch.bfloat16)
    # committed cache, one query row that sees every kept key
    after = _with(a, q=probe[:, :1].contiguous(), num_q_rows=1, k_pool=_bf16(k), v_pool=_bf16(v),
                  ctx_lens=torch.from_numpy(new_lens), draft_mask=None)
    got, f1 = oracle.attention(after)
    # original cache, the same query as row 0 of N rows whose mask keeps root + accepted nodes
    masks = np.zeros((a.num_seqs, N), dtype=np.uint64)
    for b in range(a.num_seqs):
        m = 1
        for kk in range(int(alen[b])):
            m |= 1 << int(path[b, kk])
        masks[b, :] = np.uint64(m)
    before = _with(a, q=probe, draft_mask=torch.from_numpy(masks.view(np.int64)))
    want, f2 = oracle.attention(before)
    assert not f1.any() and not f2.any()
    np.testing.assert_allclose(got[:, 0], want[:, 0], rtol=1e-12, atol=1e-12)


def test_chain_commit_moves_nothing_and_accept_len_zero_keeps_the_root():
    N = 6
    a = W.make_attention_inputs(N, 4, 2, 64, [50, 17, 200], seed=43)
    k, v = _pools(a)
    k0, v0 = k.copy(), v.copy()
    alen, path = W.make_accept_paths(N, None, 3, seed=44)
    alen[1] = 0
    path[1, :] = -1
    new_lens, flags = oracle.kv_commit([(k, v)], a.block_table.numpy(), a.ctx_lens.numpy(), alen.numpy(),
                                       path.numpy(), N)
    assert not flags.any()
    assert (new_lens == a.ctx_lens.numpy() - N + 1 + alen.numpy()).all()
    assert new_lens[1] == 17 - N + 1
    np.testing.assert_array_equal(k, k0)
    np.testing.assert_array_equal(v, v0)


def test_tree_commit_moves_rows_of_every_layer_and_head_and_nothing_else():
    N = len(W.TREE_PARENTS_3221)
    a = W.make_attention_inputs(N, 8, 4, 64, [N + 20, 129], seed=45, parents=W.TREE_PARENTS_3221)
    layers = []
    rng = np.random.default_rng(3)
    for _ in range(3):
        k = rng.integers(0, 1 << 15, size=a.k_pool.shape, dtype=np.uint16)
        layers.append((k, k ^ np.uint16(0x5555)))
    before = [(k.copy(), v.copy()) for k, v in layers]
    alen = np.array([3, 2], dtype=np.int32)
    path = np.full((2, N - 1), -1, dtype=np.int32)
    path[0, :3] = [1, 4, 7]       # root -> 1 -> 4 -> 7
    path[1, :2] = [2, 6]          # root -> 2 -> 6
    tbl, C = a.block_table.numpy(), a.ctx_lens.numpy()
    new_lens, flags = oracle.kv_commit(layers, tbl, C, alen, path, N)
    assert not flags.any()
    bs = 16
    changed = np.zeros(a.k_pool.shape[:1] + (a.k_pool.shape[2],), dtype=bool)
    for b in range(2):
        for kk in range(int(alen[b])):
            src, dst = C[b] - N + path[b, kk], C[b] - N + 1 + kk
            sb, db = tbl[b, src // bs], tbl[b, dst // bs]
            for (k, v), (k0, v0) in zip(layers, before):
                np.testing.assert_array_equal(k[db, :, dst % bs], k0[sb, :, src % bs])
                np.testing.assert_array_equal(v[db, :, dst % bs], v0[sb, :, src % bs])
            changed[db, dst % bs] = True
    for (k, v), (k0, v0) in zip(layers, before):
        keep = ~changed
        np.testing.assert_array_equal(k.transpose(0, 2, 1, 3)[keep], k0.transpose(0, 2, 1, 3)[keep])
        np.testing.assert_array_equal(v.transpose(0, 2, 1, 3)[keep], v0.transpose(0, 2, 1, 3)[keep])


def test_commit_flags_leave_bad_sequences_untouched():
    N = 5
    a = W.make_attention_inputs(N, 4, 2, 64, [40, 40, 40, 40, 40], seed=46)
    k, v = _pools(a)
    k0 = k.copy()
    tbl = a.block_table.numpy().copy()
    C = a.ctx_lens.numpy().copy()
    alen = np.array([2, 2, 5, 2, 1], dtype=np.int32)
    path = np.array([[1, 2, -1, -1], [2, 2, -1, -1], [1, 2, 3, 4], [1, 3, -1, -1], [1, -1, -1, -1]], dtype=np.int32)
    C[3] = 2                       # shorter than N
    tbl[4, (40 - 1) // 16] = a.num_blocks + 3   # a new position's page outside the pool
    new_lens, flags = oracle.kv_commit([(k, v)], tbl, C, alen, path, N)
    assert flags.tolist() == [0, 32, 32, 2, 8]
    assert new_lens.tolist() == [40 - N + 3, 40, 40, 2, 40]
    np.testing.assert_array_equal(k, k0)   # the valid one is a chain: nothing moves
