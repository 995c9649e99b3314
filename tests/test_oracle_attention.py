"""Pins for the oracle's verify attention (no GPU).

The oracle is checked against torch's scaled_dot_product_attention in fp64 on
dense-gathered K/V with an explicit boolean mask (a library routine), and
against invariants that hold for the plain definition: page permutation,
closed forms for equal keys and for a single key, chain mask == tree mask with
chain parents, GQA head sharing, and invalid-sequence handling.
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_rl_b200 import workloads as W


def _sdpa_reference(a) -> np.ndarray:
    """fp64 SDPA on K/V gathered through the block table, with the visibility mask."""
    B, N, Hq, Hkv, D = a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads, a.head_dim
    G = Hq // Hkv
    out = np.zeros((B, N, Hq, D))
    tbl = a.block_table.numpy()
    for b in range(B):
        C = int(a.ctx_lens[b])
        t = np.arange(C)
        blocks = tbl[b, t // 16]
        k = a.k_pool.double()[blocks, :, t % 16, :]  # [C][Hkv][D]
        v = a.v_pool.double()[blocks, :, t % 16, :]
        q = a.q[b].double()  # [N][Hq][D]
        vis = np.zeros((N, C), dtype=bool)
        vis[:, : C - N] = True
        for i in range(N):
            for j in range(N):
                if a.draft_mask is None:
                    ok = j <= i
                else:
                    ok = (int(a.draft_mask[b, i].item()) >> j) & 1
                vis[i, C - N + j] = bool(ok)
        for hq in range(Hq):
            h = hq // G
            o = torch.nn.functional.scaled_dot_product_attention(
                q[:, hq, :][None, None], k[:, h, :][None, None], v[:, h, :][None, None],
                attn_mask=torch.from_numpy(vis)[None, None])
            out[b, :, hq, :] = o[0, 0].numpy()
    return out


@pytest.mark.parametrize("D,Hq,Hkv,N,parents,lens", [
    (64, 4, 1, 5, None, [128, 128]),
    (128, 8, 2, 5, None, [37, 200, 16]),
    (128, 8, 4, 11, W.TREE_PARENTS_3221, [64, 130]),
    (64, 6, 3, 3, [-1, 0, 0], [20, 33]),
    (128, 4, 4, 1, None, [1, 17]),
])
def test_matches_fp64_sdpa(D, Hq, Hkv, N, parents, lens):
    a = W.make_attention_inputs(N, Hq, Hkv, D, lens, seed=11 + D + N, parents=parents)
    got, flags = oracle.attention(a)
    assert not flags.any()
    want = _sdpa_reference(a)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_attention_rows_match_full():
    a = W.make_attention_inputs(5, 8, 2, 64, [50, 77, 140], seed=3)
    full, _ = oracle.attention(a)
    rows = np.array([[0, 0, 0], [1, 4, 7], [2, 2, 3], [2, 4, 5]], dtype=np.int32)
    part = oracle.attention_rows(a, rows)
    for r, (b, i, hq) in enumerate(rows):
        np.testing.assert_array_equal(part[r], full[b, i, hq])


def test_page_permutation_invariance():
    a = W.make_attention_inputs(5, 4, 2, 64, [100, 61], seed=5)
    base, _ = oracle.attention(a)
    rng = np.random.default_rng(0)
    perm = rng.permutation(a.num_blocks)  # new id of old block x is perm[x]
    inv = np.argsort(perm)
    a.k_pool = a.k_pool[torch.from_numpy(inv)].contiguous()
    a.v_pool = a.v_pool[torch.from_numpy(inv)].contiguous()
    a.block_table = torch.from_numpy(perm[a.block_table.numpy()].astype(np.int32))
    moved, _ = oracle.attention(a)
    np.testing.assert_array_equal(base, moved)


def test_equal_keys_give_mean_of_visible_values():
    a = W.make_attention_inputs(5, 4, 1, 64, [48, 70], seed=9)
    a.k_pool[:] = a.k_pool[0, 0, 0]  # every key identical -> uniform weights
    out, _ = oracle.attention(a)
    tbl = a.block_table.numpy()
    for b in range(2):
        C = int(a.ctx_lens[b])
        t = np.arange(C)
        v = a.v_pool.double()[tbl[b, t // 16], 0, t % 16, :].numpy()
        for i in range(5):
            nvis = C - 5 + i + 1
            np.testing.assert_allclose(out[b, i, 0], v[:nvis].mean(axis=0), rtol=1e-12, atol=1e-14)


def test_single_key_returns_its_value():
    a = W.make_attention_inputs(1, 2, 1, 128, [1], seed=4)
    out, _ = oracle.attention(a)
    blk = int(a.block_table[0, 0])
    want = a.v_pool[blk, 0, 0].double().numpy()
    np.testing.assert_array_equal(out[0, 0, 0], want)
    np.testing.assert_array_equal(out[0, 0, 1], want)


def test_chain_mask_equals_null_mask():
    a = W.make_attention_inputs(6, 4, 2, 64, [90, 33], seed=21)
    b = W.make_attention_inputs(6, 4, 2, 64, [90, 33], seed=21, explicit_chain_mask=True)
    assert b.draft_mask is not None and a.draft_mask is None
    np.testing.assert_array_equal(oracle.attention(a)[0], oracle.attention(b)[0])


def test_gqa_heads_with_equal_queries_agree():
    a = W.make_attention_inputs(5, 8, 2, 64, [77], seed=13)
    a.q[:, :, 1] = a.q[:, :, 0]
    a.q[:, :, 6] = a.q[:, :, 4]
    out, _ = oracle.attention(a)
    np.testing.assert_array_equal(out[:, :, 0], out[:, :, 1])
    np.testing.assert_array_equal(out[:, :, 4], out[:, :, 6])
    assert not np.array_equal(out[:, :, 0], out[:, :, 4])  # different KV head


def test_tree_rows_ignore_non_ancestor_keys():
    # Perturbing the K/V of a new position that is not an ancestor of row i
    # must not change row i (here row 1's key for row 2, siblings under the root).
    par = [-1, 0, 0, 1]
    a = W.make_attention_inputs(4, 2, 1, 64, [40], seed=17, parents=par)
    out0, _ = oracle.attention(a)
    C = 40
    t = C - 4 + 1  # new key of node 1
    blk = int(a.block_table[0, t // 16])
    a.v_pool[blk, 0, t % 16] += 3.0
    a.k_pool[blk, 0, t % 16] -= 1.0
    out1, _ = oracle.attention(a)
    np.testing.assert_array_equal(out0[0, 2], out1[0, 2])  # node 2 does not see node 1
    np.testing.assert_array_equal(out0[0, 0], out1[0, 0])  # root does not see node 1
    assert not np.array_equal(out0[0, 1], out1[0, 1])      # node 1 sees itself
    assert not np.array_equal(out0[0, 3], out1[0, 3])      # node 3 sees its parent


def test_invalid_sequences_are_flagged_and_zero():
    a = W.make_attention_inputs(5, 4, 1, 64, [40, 40, 40], seed=2)
    a.ctx_lens[0] = 3                      # shorter than the N new rows
    a.block_table[1, 1] = a.num_blocks     # block id out of range
    out, flags = oracle.attention(a)
    assert flags.tolist() == [1, 1, 0]
    assert not out[0].any() and not out[1].any() and out[2].any()
