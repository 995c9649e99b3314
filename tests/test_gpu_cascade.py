"""GPU parity of sv_cascade_verify_attention against the fp64 oracle (B200).

The shared prefix is read once per group and KV head for every member's rows
and merged with each member's own suffix by log-sum-exp. Covered: several
groups of unequal sizes (one empty, one of a single member), ragged row chunks
and a ragged last prefix tile, empty prefixes, prefix splits (with empty
splits), tree masks, head_dim 64, members whose own prefix entries point
elsewhere (they must not be read), invalid members and bad prefix pages,
garbage workspace, determinism, and the GRPO group at full size on sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_attention_close
from speculative_decoding_rl_b200 import workloads as W
from speculative_decoding_rl_b200.session import AttentionCall, CascadeCall

pytestmark = pytest.mark.gpu


def run(a, off, pre, scramble_ws=False):
    call = CascadeCall(a, off, pre)
    if scramble_ws:
        g = torch.Generator().manual_seed(9)
        call.workspace.copy_(torch.randint(0, 256, tuple(call.workspace.shape), dtype=torch.uint8, generator=g))
    out = call.run()
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), call.status.cpu().numpy()


def foreign_member_prefixes(a, off, pre, invalid=False, seed=3):
    """Non-first members' prefix entries point at other pages (or outside the pool)."""
    rng = np.random.default_rng(seed)
    tbl = a.block_table.numpy().copy()
    for g in range(len(pre)):
        for b in range(off[g] + 1, off[g + 1]):
            for j in range(pre[g] // 16):
                tbl[b, j] = a.num_blocks + 7 if invalid else rng.integers(0, a.num_blocks)
    a.block_table = torch.from_numpy(tbl)
    return a


def check(a, off, pre, what, scramble_ws=False):
    got, st = run(a, off, pre, scramble_ws)
    want, flags = oracle.cascade_attention(a, off, pre)
    assert (st == 0).all() and not flags.any(), (st, flags)
    return assert_attention_close(got, want, what)


def test_grpo_groups_match_oracle():
    lens = W.make_ctx_lens("uniform", 16, 7, 5, lo=256 + 50, hi=256 + 600)
    a = W.make_attention_inputs(7, 32, 8, 128, lens, seed=41, shared_prefix_groups=4, shared_prefix_tokens=256)
    max_abs, mean_rel = check(a, a.group_offsets, a.prefix_lens, "grpo small")
    print(f"grpo small: max_abs {max_abs:.2e} mean_rel {mean_rel:.2e}")


@pytest.mark.parametrize("invalid", [False, True])
def test_members_own_prefix_entries_are_not_read(invalid):
    lens = [400, 333, 612, 90, 251, 700, 200]
    off, pre = [0, 3, 3, 4, 7], [80, 48, 16, 128]   # an empty group, a group of one, ragged tiles
    a = W.make_attention_inputs(5, 16, 4, 128, lens, seed=42, extra_blocks=8)
    a = foreign_member_prefixes(a, off, pre, invalid=invalid)
    check(a, off, pre, f"foreign member prefixes (invalid ids: {invalid})")


@pytest.mark.parametrize("pre", [[0, 0], [0, 64], [1024, 336]])
def test_prefix_lengths_and_splits(pre):
    # two small groups on one KV head: few (group, head, chunk) items, so the
    # prefix is split over several CTAs (some splits empty for the short prefix)
    lens = [1100, 1300, 1090, 700]
    off = [0, 2, 4]
    a = W.make_attention_inputs(5, 4, 1, 128, lens, seed=43, extra_blocks=4)
    a = foreign_member_prefixes(a, off, pre, seed=5)
    check(a, off, pre, f"prefix {pre}")


def test_tree_masks_and_head_dim_64():
    lens = [300, 181, 222, 97]
    off, pre = [0, 4], [64]
    a = W.make_attention_inputs(6, 6, 6, 64, lens, seed=44, parents=[-1, 0, 0, 1, 1, 2])
    a = foreign_member_prefixes(a, off, pre, seed=6)
    check(a, off, pre, "tree, D=64, G=1")


def test_garbage_workspace_and_determinism():
    lens = W.make_ctx_lens("uniform", 8, 7, 7, lo=600, hi=2400)
    a = W.make_attention_inputs(7, 32, 8, 128, lens, seed=45, shared_prefix_groups=2, shared_prefix_tokens=512)
    g1, s1 = run(a, a.group_offsets, a.prefix_lens, scramble_ws=True)
    g2, s2 = run(a, a.group_offsets, a.prefix_lens)
    np.testing.assert_array_equal(g1, g2)
    want, flags = oracle.cascade_attention(a, a.group_offsets, a.prefix_lens)
    assert (s1 == 0).all() and not flags.any()
    assert_attention_close(g1, want, "garbage workspace")


def test_cascade_agrees_with_the_plain_call_on_shared_pages():
    lens = W.make_ctx_lens("uniform", 8, 7, 8, lo=1100, hi=3000)
    a = W.make_attention_inputs(7, 32, 8, 128, lens, seed=46, shared_prefix_groups=2, shared_prefix_tokens=1024)
    got, st = run(a, a.group_offsets, a.prefix_lens)
    plain = AttentionCall(a).run()
    torch.cuda.synchronize()
    plain = plain.float().cpu().numpy().astype(np.float64)
    assert (st == 0).all()
    assert_attention_close(got, plain, "cascade vs plain call")


def test_invalid_members_and_bad_prefix_pages():
    lens = [300, 300, 300, 300, 300, 300]
    off, pre = [0, 3, 6], [64, 32]
    a = W.make_attention_inputs(5, 8, 2, 128, lens, seed=47, extra_blocks=4)
    a.ctx_lens[1] = 64 + 4                       # shorter than its prefix plus its 5 rows
    a.ctx_lens[2] = 3                            # shorter than N
    tbl = a.block_table.numpy().copy()
    tbl[3, 1] = a.num_blocks + 3                 # a bad page among group 1's prefix pages
    a.block_table = torch.from_numpy(tbl)
    got, st = run(a, off, pre)
    want, flags = oracle.cascade_attention(a, off, pre)
    assert flags.tolist() == [0, 1, 1, 1, 1, 1]
    assert st[0] == 0 and st[1] == 2 and st[2] == 2
    assert all(int(x) & 8 for x in st[3:6]), st
    assert not got[1].any() and not got[2].any()
    assert_attention_close(got[0], want[0], "valid member beside invalid ones")


@pytest.mark.parametrize("name", ["grpo_shared_prefix", "grpo_long_prompt"])
def test_grpo_full_size_sampled_rows(name):
    w = W.workload(name)
    a = W.build_attention(w)
    got, st = run(a, a.group_offsets, a.prefix_lens)
    assert (st == 0).all()
    rng = np.random.default_rng(77)
    rows = np.stack([rng.integers(0, a.num_seqs, 64), rng.integers(0, a.num_q_rows, 64),
                     rng.integers(0, a.num_q_heads, 64)], axis=1).astype(np.int32)
    want = oracle.cascade_attention(a, a.group_offsets, a.prefix_lens, rows=rows)
    sel = got[rows[:, 0], rows[:, 1], rows[:, 2]]
    max_abs, mean_rel = assert_attention_close(sel, want, f"{name} full size, sampled rows")
    print(f"{name} full size: max_abs {max_abs:.2e} mean_rel {mean_rel:.2e}")
