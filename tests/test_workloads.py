"""Seeded input generator: determinism, layout and recipe checks (no GPU)."""
import numpy as np
import torch

from speculative_decoding_rl_b200 import workloads as W


def test_attention_inputs_are_deterministic_and_well_formed():
    a = W.make_attention_inputs(5, 8, 2, 64, [37, 200, 16], seed=4)
    b = W.make_attention_inputs(5, 8, 2, 64, [37, 200, 16], seed=4)
    for name in ("q", "k_pool", "v_pool", "block_table", "ctx_lens"):
        assert torch.equal(getattr(a, name).view(torch.int16) if getattr(a, name).dtype == torch.bfloat16
                           else getattr(a, name),
                           getattr(b, name).view(torch.int16) if getattr(b, name).dtype == torch.bfloat16
                           else getattr(b, name))
    tbl = a.block_table.numpy()
    used = []
    for bb, c in enumerate(a.ctx_lens.tolist()):
        nb = (c + 15) // 16
        used += tbl[bb, :nb].tolist()
        assert (tbl[bb, nb:] == a.guard_block).all()
    assert len(set(used)) == len(used)  # private pages are distinct
    assert a.guard_block not in used
    assert torch.isnan(a.k_pool[a.guard_block].float()).all()
    # slots past ctx_len in a last page are NaN, visible slots are finite
    c = 37
    last = int(tbl[0, c // 16])
    assert torch.isnan(a.v_pool[last, :, c % 16:].float()).all()
    assert torch.isfinite(a.v_pool[last, :, :c % 16].float()).all()


def test_shared_prefix_pages():
    w = W.workload("grpo_shared_prefix", temperature=0.0)
    a = W.build_attention(w)
    tbl = a.block_table.numpy()
    assert a.num_seqs == 64
    for g in range(4):
        rows = tbl[g * 16:(g + 1) * 16, :64]
        assert (rows == rows[0]).all()
    assert len(set(tbl[0:16, :64].ravel()) & set(tbl[16:32, :64].ravel())) == 0
    assert a.kv_bytes_unique() < a.kv_bytes_logical()


def test_ctx_len_recipes():
    lens = W.make_ctx_lens("uniform", 1000, 5, 1, lo=4096, hi=16384)
    assert min(lens) >= 4096 and max(lens) <= 16384
    lens = W.make_ctx_lens("lognormal", 2000, 9, 1, median=6144, sigma=0.75, lo=512, hi=32768)
    assert min(lens) >= 512 and max(lens) <= 32768
    assert 5000 < np.median(lens) < 7500


def test_tree_masks():
    m = W.ancestor_masks(W.TREE_PARENTS_3221)
    assert int(m[0]) == 1
    assert int(m[9]) == (1 << 9) | (1 << 7) | (1 << 4) | (1 << 1) | 1
    assert int(m[10]) == (1 << 10) | (1 << 5) | (1 << 1) | 1
    chain = W.ancestor_masks(W.chain_parents(5))
    assert [int(x) for x in chain] == [1, 3, 7, 15, 31]


def test_draft_recipe_gives_about_seventy_percent_acceptance():
    a = W.build_accept(W.workload("qwen7b_longtail"))
    l = a.target_logits.double()
    p = torch.softmax(l[:, :-1], dim=-1)
    beta = torch.minimum(p, a.draft_probs.double()).sum(-1)
    assert 0.6 < float(beta.mean()) < 0.8
    # drafts are valid tokens drawn from q
    assert int(a.draft_tokens.min()) >= 0 and int(a.draft_tokens.max()) < a.vocab


def test_long_prompt_groups_share_their_prompt_pages():
    w = W.workload("grpo_long_prompt")
    a = W.build_attention(w)
    tbl = a.block_table.numpy()
    assert a.num_seqs == 128 and list(a.group_offsets) == list(range(0, 129, 16))
    assert list(a.prefix_lens) == [8192] * 8
    npg = 8192 // 16
    for g in range(8):
        rows = tbl[g * 16:(g + 1) * 16, :npg]
        assert (rows == rows[0]).all()
        # each member's own pages follow the prompt and are its alone
        own = [set(tbl[b, npg:(int(a.ctx_lens[b]) + 15) // 16]) for b in range(g * 16, (g + 1) * 16)]
        assert all(len(x & y) == 0 for i, x in enumerate(own) for y in own[i + 1:])
    lens = a.ctx_lens.numpy()
    assert lens.min() >= 8192 + 512 and lens.max() <= 8192 + 4096
