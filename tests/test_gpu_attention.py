"""GPU parity of sv_verify_attention against the fp64 oracle (B200).

Full-output comparison at sizes the oracle finishes in seconds (several tiles,
ragged tails, all five workload shapes); at full size, every output row of the
7B long-tail and the tree layers, every point of the 32B batch-shrink sweep
(all rows up to 4 sequences, else sampled rows plus the longest sequence) and
sampled rows of the GRPO group; and edge cases: single key, tile-boundary
lengths, >128 query rows per KV head, explicit vs implicit chain masks,
invalid contexts and block ids.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import all_rows, assert_attention_close, oracle_rows_parallel
from speculative_decoding_rl_b200 import workloads as W
from speculative_decoding_rl_b200.session import AttentionCall

pytestmark = pytest.mark.gpu


def run(a):
    call = AttentionCall(a)
    out = call.run()
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), call.status.cpu().numpy()


def check_full(a, what):
    got, st = run(a)
    want, flags = oracle.attention(a)
    assert (st == 0).all() and not flags.any(), (st, flags)
    return assert_attention_close(got, want, what)


@pytest.mark.parametrize("case", [
    "tiny_chain", "qwen7b_small", "qwen32b_small_g8", "qwen32b_small_g2", "tree_small", "grpo_small",
])
def test_attention_matches_oracle(case):
    if case == "tiny_chain":
        a = W.build_attention(W.workload("tiny_chain"))
    elif case == "qwen7b_small":
        lens = W.make_ctx_lens("uniform", 8, 5, 2, lo=200, hi=1500)
        a = W.make_attention_inputs(5, 28, 4, 128, lens, seed=21)
    elif case == "qwen32b_small_g8":
        lens = W.make_ctx_lens("lognormal", 16, 9, 3, median=600, sigma=0.75, lo=9, hi=3000)
        a = W.make_attention_inputs(9, 40, 8, 128, lens, seed=22)
    elif case == "qwen32b_small_g2":
        lens = W.make_ctx_lens("lognormal", 5, 3, 4, median=900, sigma=0.75, lo=3, hi=3000)
        a = W.make_attention_inputs(3, 40, 8, 128, lens, seed=23)
    elif case == "tree_small":
        a = W.make_attention_inputs(11, 32, 4, 128, [700, 1031, 11, 256], seed=24,
                                    parents=W.TREE_PARENTS_3221)
    elif case == "grpo_small":
        lens = W.make_ctx_lens("uniform", 16, 7, 5, lo=256 + 50, hi=256 + 600)
        a = W.make_attention_inputs(7, 32, 8, 128, lens, seed=25, shared_prefix_groups=4,
                                    shared_prefix_tokens=256)
    max_abs, mean_rel = check_full(a, case)
    print(f"{case}: max_abs {max_abs:.2e} mean_rel {mean_rel:.2e}")


@pytest.mark.parametrize("lens", [[1], [5, 16, 17, 127, 128, 129, 255, 256, 257, 1000]])
def test_attention_tile_edges(lens):
    N = 1 if lens == [1] else 5
    a = W.make_attention_inputs(N, 8, 2, 128, lens, seed=31)
    check_full(a, f"lens {lens}")


def test_attention_head_dim_64_and_no_gqa():
    a = W.make_attention_inputs(4, 6, 6, 64, [300, 77, 512], seed=32)
    check_full(a, "D=64, G=1")


@pytest.mark.parametrize("D", [128, 64])
def test_attention_80_rows_per_unit(D):
    # N=16 x G=5 = 80 rows per KV head: one row chunk, padded to the 96-row kernel
    a = W.make_attention_inputs(16, 10, 2, D, [700, 1500, 40, 2049], seed=38)
    check_full(a, f"N=16, G=5, D={D}")


def test_attention_many_rows_per_kv_head():
    # N=64 rows x G=4 -> 256 rows per KV head: two row chunks per unit
    a = W.make_attention_inputs(64, 8, 2, 128, [400, 64, 1200], seed=33, explicit_chain_mask=True)
    check_full(a, "N=64, G=4")


def test_explicit_chain_mask_equals_null_mask():
    a = W.make_attention_inputs(6, 16, 4, 128, [900, 333], seed=34)
    b = W.make_attention_inputs(6, 16, 4, 128, [900, 333], seed=34, explicit_chain_mask=True)
    ga, _ = run(a)
    gb, _ = run(b)
    np.testing.assert_array_equal(ga, gb)


def test_attention_is_deterministic():
    a = W.make_attention_inputs(5, 28, 4, 128, [3000, 5000, 100], seed=35)
    g1, _ = run(a)
    g2, _ = run(a)
    np.testing.assert_array_equal(g1, g2)


def test_attention_flags_invalid_sequences():
    a = W.make_attention_inputs(5, 8, 2, 128, [300, 300, 300, 300], seed=36)
    a.ctx_lens[0] = 4                                  # shorter than N
    a.ctx_lens[1] = a.max_blocks_per_seq * 16 + 1      # longer than the table
    a.block_table[2, 3] = a.num_blocks + 5             # out-of-range block id
    got, st = run(a)
    want, flags = oracle.attention(a)
    assert st[0] == 2 and st[1] == 2 and st[2] == 8 and st[3] == 0
    assert not got[0].any() and not got[1].any()
    assert_attention_close(got[3], want[3], "valid sequence next to invalid ones")


def test_split_units_need_no_workspace_initialisation():
    # A 40k-token sequence next to a short one: its units are split over dozens
    # of CTAs and merged by the last to arrive. The workspace starts as random
    # bytes (arrival counters from no call), then all ones; every call must give
    # the oracle's result and the same bits.
    a = W.make_attention_inputs(5, 16, 2, 128, [40000, 300], seed=37)
    call = AttentionCall(a)
    g = torch.Generator().manual_seed(5)
    call.workspace.copy_(torch.randint(0, 256, tuple(call.workspace.shape), dtype=torch.uint8, generator=g))
    first = call.run().clone()
    second = call.run().clone()
    call.workspace.fill_(255)
    third = call.run().clone()
    torch.cuda.synchronize()
    assert (call.status.cpu().numpy() == 0).all()
    want, flags = oracle.attention(a)
    assert not flags.any()
    got = first.float().cpu().numpy().astype(np.float64)
    assert_attention_close(got, want, "split units, random workspace")
    assert torch.equal(first, second) and torch.equal(first, third)


@pytest.mark.parametrize("name,over,nrows", [
    ("grpo_shared_prefix", {}, 256),
])
def test_full_size_sampled_rows_other_shapes(name, over, nrows):
    # the GRPO group with its shared prompt pages, at full size; the oracle
    # computes sampled rows
    w = W.workload(name, **over)
    a = W.build_attention(w)
    got, st = run(a)
    assert (st == 0).all()
    rng = np.random.default_rng(sum(map(ord, name)) + len(over))
    rows = np.stack([rng.integers(0, a.num_seqs, nrows), rng.integers(0, a.num_q_rows, nrows),
                     rng.integers(0, a.num_q_heads, nrows)], axis=1).astype(np.int32)
    want = oracle_rows_parallel(a, rows)
    sel = got[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_attention_close(sel, want, f"{name} {over} full size, sampled rows")


@pytest.mark.parametrize("name", ["qwen7b_longtail", "tree_qwen3_30b"])
def test_full_size_full_output(name):
    # every output row of the full-size layer against the oracle (rows spread over host threads)
    a = W.build_attention(W.workload(name))
    got, st = run(a)
    assert (st == 0).all()
    rows = all_rows(a)
    want = oracle_rows_parallel(a, rows)
    max_abs, mean_rel = assert_attention_close(got[rows[:, 0], rows[:, 1], rows[:, 2]], want,
                                               f"{name} full size, every row")
    print(f"{name} full output ({len(rows)} rows): max_abs {max_abs:.2e} mean_rel {mean_rel:.2e}")


@pytest.mark.parametrize("B", [256, 64, 16, 4, 1])
@pytest.mark.parametrize("gamma", [2, 4, 8])
def test_32b_sweep_every_point(B, gamma):
    # each point of the Qwen2.5-32B batch-shrink sweep at full size: every row
    # up to 4 sequences, else 64 seeded rows plus every row of the longest sequence
    a = W.build_attention(W.workload("qwen32b_sweep", num_seqs=B, gamma=gamma))
    got, st = run(a)
    assert (st == 0).all()
    if B <= 4:
        rows = all_rows(a)
    else:
        rng = np.random.default_rng(1000 * B + gamma)
        samp = np.stack([rng.integers(0, B, 64), rng.integers(0, a.num_q_rows, 64),
                         rng.integers(0, a.num_q_heads, 64)], axis=1).astype(np.int32)
        longest = int(np.argmax(a.ctx_lens.numpy()))
        whole = all_rows(a)
        rows = np.concatenate([samp, whole[whole[:, 0] == longest]])
    want = oracle_rows_parallel(a, rows)
    max_abs, mean_rel = assert_attention_close(got[rows[:, 0], rows[:, 1], rows[:, 2]], want,
                                               f"32B sweep B={B} gamma={gamma}")
    print(f"32B sweep B={B} gamma={gamma} ({len(rows)} rows): max_abs {max_abs:.2e} mean_rel {mean_rel:.2e}")
