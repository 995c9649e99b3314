"""GPU parity of sv_kv_commit against the oracle (B200): pure data movement, so
the pools, the new lengths and the flags must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_rl_b200 as sv
from speculative_decoding_rl_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _random_tree(n, seed):
    rng = np.random.default_rng(seed)
    return [-1] + [int(rng.integers(0, c)) for c in range(1, n)]


def _run(a, layers_u16, alen, path, tbl=None, ctx=None):
    """layers_u16: list of (k, v) uint16 numpy pools. Returns GPU and oracle results."""
    tbl = a.block_table if tbl is None else tbl
    ctx = a.ctx_lens if ctx is None else ctx
    dev = [(torch.from_numpy(k.view(np.int16).copy()).cuda(), torch.from_numpy(v.view(np.int16).copy()).cuda())
           for k, v in layers_u16]
    desc = sv.SvAttnDesc(a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads, a.head_dim, 16,
                         a.max_blocks_per_seq, a.num_blocks)
    new_ctx = torch.full((a.num_seqs,), -7, dtype=torch.int32, device="cuda")
    st = torch.full((a.num_seqs,), -7, dtype=torch.int32, device="cuda")
    sv.sv_kv_commit(desc, dev, tbl.cuda(), ctx.cuda(), alen.cuda(), path.cuda(), new_ctx, st)
    torch.cuda.synchronize()
    ref = [(k.copy(), v.copy()) for k, v in layers_u16]
    want_ctx, want_flags = oracle.kv_commit(ref, tbl.numpy(), ctx.numpy(), alen.numpy(), path.numpy(),
                                            a.num_q_rows)
    return dev, new_ctx.cpu().numpy(), st.cpu().numpy(), ref, want_ctx, want_flags


def _assert_same(dev, got_ctx, got_flags, ref, want_ctx, want_flags):
    np.testing.assert_array_equal(got_ctx, want_ctx)
    np.testing.assert_array_equal(got_flags, want_flags)
    for (dk, dv), (rk, rv) in zip(dev, ref):
        np.testing.assert_array_equal(dk.cpu().numpy().view(np.uint16), rk)
        np.testing.assert_array_equal(dv.cpu().numpy().view(np.uint16), rv)


@pytest.mark.parametrize("parents,D", [(None, 128), (W.TREE_PARENTS_3221, 128), (W.TREE_PARENTS_3221, 64),
                                       ("random64", 128), ([-1, 0, 0, 1, 2, 2, 5], 64)])
def test_kv_commit_matches_oracle(parents, D):
    if parents == "random64":
        parents = _random_tree(64, 5)
    N = 5 if parents is None else len(parents)
    lens = [N, N + 1, N + 16, N + 17, N + 130, N + 1000, 4095, N + 333]
    a = W.make_attention_inputs(N, 8, 4, D, lens, seed=51)
    rng = np.random.default_rng(52)
    layers = [(rng.integers(0, 1 << 16, size=a.k_pool.shape, dtype=np.uint16),
               rng.integers(0, 1 << 16, size=a.v_pool.shape, dtype=np.uint16)) for _ in range(3)]
    alen, path = W.make_accept_paths(N, parents, len(lens), seed=53)
    alen[0] = 0
    path[0, :] = -1
    res = _run(a, layers, alen, path)
    _assert_same(*res)
    assert not res[2].any()


def test_kv_commit_flags_match_oracle():
    N = len(W.TREE_PARENTS_3221)
    a = W.make_attention_inputs(N, 8, 4, 128, [200] * 6, seed=54)
    rng = np.random.default_rng(55)
    layers = [(rng.integers(0, 1 << 16, size=a.k_pool.shape, dtype=np.uint16),
               rng.integers(0, 1 << 16, size=a.v_pool.shape, dtype=np.uint16))]
    alen, path = W.make_accept_paths(N, W.TREE_PARENTS_3221, 6, seed=56, max_len=3)
    ctx = a.ctx_lens.clone()
    tbl = a.block_table.clone()
    ctx[0] = N - 1                      # shorter than N
    tbl[1, (200 - 1) // 16] = a.num_blocks + 9
    alen[2] = N                         # too long
    alen[3] = 2
    path[3, :2] = torch.tensor([1, 1])  # not increasing
    alen[4] = 1
    path[4, 0] = 0                      # the root is not a draft node
    alen[5] = 2
    path[5, :] = -1
    path[5, :2] = torch.tensor([1, 4])  # root -> 1 -> 4
    dev, got_ctx, got_flags, ref, want_ctx, want_flags = _run(a, layers, alen, path, tbl=tbl, ctx=ctx)
    _assert_same(dev, got_ctx, got_flags, ref, want_ctx, want_flags)
    assert got_flags.tolist()[:5] == [2, 8, 32, 32, 32] and got_flags[5] == 0


def test_kv_commit_tree_full_context_rows():
    # the tree-verify shape at its full 24k context on two layers: the kept rows
    # land behind the root and every other row of the pools is untouched
    w = W.workload("tree_qwen3_30b")
    a = W.build_attention(w)
    N = a.num_q_rows
    alen, path = W.make_accept_paths(N, W.TREE_PARENTS_3221, a.num_seqs, seed=57)
    pools = [(a.k_pool.cuda(), a.v_pool.cuda()), (torch.randn_like(a.k_pool.float()).to(torch.bfloat16).cuda(),
                                                  torch.randn_like(a.v_pool.float()).to(torch.bfloat16).cuda())]
    before = [(k.clone(), v.clone()) for k, v in pools]
    desc = sv.SvAttnDesc(a.num_seqs, N, a.num_q_heads, a.num_kv_heads, a.head_dim, 16, a.max_blocks_per_seq,
                         a.num_blocks)
    new_ctx = torch.empty(a.num_seqs, dtype=torch.int32, device="cuda")
    st = torch.empty(a.num_seqs, dtype=torch.int32, device="cuda")
    sv.sv_kv_commit(desc, pools, a.block_table.cuda(), a.ctx_lens.cuda(), alen.cuda(), path.cuda(), new_ctx, st)
    torch.cuda.synchronize()
    assert (st.cpu() == 0).all()
    C = a.ctx_lens.numpy()
    assert (new_ctx.cpu().numpy() == C - N + 1 + alen.numpy()).all()
    tbl = a.block_table.numpy()
    touched = torch.zeros(a.k_pool.shape[0], 16, dtype=torch.bool)
    for (k, v), (k0, v0) in zip(pools, before):
        # bit patterns: the pools hold NaN in guard pages and past each context
        k, v, k0, v0 = (x.view(torch.int16) for x in (k, v, k0, v0))
        for b in range(a.num_seqs):
            for kk in range(int(alen[b])):
                src, dst = C[b] - N + int(path[b, kk]), C[b] - N + 1 + kk
                assert torch.equal(k[tbl[b, dst // 16], :, dst % 16], k0[tbl[b, src // 16], :, src % 16])
                assert torch.equal(v[tbl[b, dst // 16], :, dst % 16], v0[tbl[b, src // 16], :, src % 16])
                touched[tbl[b, dst // 16], dst % 16] = True
        keep = (~touched).cuda()
        assert torch.equal(k.transpose(1, 2)[keep], k0.transpose(1, 2)[keep])
        assert torch.equal(v.transpose(1, 2)[keep], v0.transpose(1, 2)[keep])
