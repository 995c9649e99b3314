"""GPU parity of sv_accept against the fp64 oracle (B200).

Greedy: bit-exact accept lengths, paths and tokens. Sampling: bit-exact except
near ties flagged by the oracle (counted). Inputs are the seeded workloads of
the verify step at their full vocabulary sizes, plus edge cases.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import compare_accept
from speculative_decoding_rl_b200 import workloads as W
from speculative_decoding_rl_b200.session import AcceptCall

pytestmark = pytest.mark.gpu


def run_both(a, seed, temperature=None):
    T = a.temperature if temperature is None else temperature
    call = AcceptCall(a, seed=seed, temperature=T)
    call.run()
    torch.cuda.synchronize()
    orc = oracle.accept(a.target_logits, a.draft_probs, a.draft_tokens, T, seed, parents=a.tree_parents)
    bad, exempt = compare_accept(call.accept_len.cpu().numpy(), call.next_token.cpu().numpy(),
                                 call.path.cpu().numpy(), call.status.cpu().numpy(), orc, greedy=(T == 0))
    return bad, exempt, orc, call


@pytest.mark.parametrize("name,over,T", [
    ("tiny_chain", {}, 1.0),
    ("tiny_chain", {}, 0.0),
    ("qwen7b_longtail", {}, 1.0),
    ("qwen32b_sweep", dict(num_seqs=16, gamma=8), 1.0),
    ("qwen32b_sweep", dict(num_seqs=4, gamma=2), 1.0),
    ("tree_qwen3_30b", {}, 1.0),
    ("grpo_shared_prefix", dict(temperature=0.0), 0.0),
    ("grpo_shared_prefix", dict(temperature=0.7), 0.7),
])
def test_accept_matches_oracle(name, over, T):
    w = W.workload(name, **over)
    a = W.build_accept(w)
    total_exempt = 0
    for seed in (0, 1, 12345678901):
        bad, exempt, orc, _ = run_both(a, seed, T)
        assert not bad, f"{name} seed {seed}: {bad[:5]}"
        total_exempt += exempt
    print(f"{name} T={T}: {a.num_seqs * 3} sequences, {total_exempt} near-tie exemptions")


def test_accept_many_small_problems():
    # many sequences, small vocab, chain and tree, several seeds
    for parents in (None, W.TREE_PARENTS_3221, [-1, 0, 0, 1, 1, 2]):
        N = 5 if parents is None else len(parents)
        a = W.make_accept_inputs(512, N, 37, seed=9, logit_std=1.0, draft_noise=0.8, temperature=1.0,
                                 parents=parents)
        for seed in range(4):
            bad, _, _, _ = run_both(a, seed)
            assert not bad, bad[:5]
        bad, _, _, _ = run_both(a, 0, temperature=0.0)
        assert not bad, bad[:5]


def test_accept_gamma_zero_and_vocab_edges():
    for V in (1, 3, 8, 1001, 4099):
        a = W.make_accept_inputs(64, 1, V, seed=V, logit_std=2.0, draft_noise=0.5, temperature=1.0)
        bad, _, _, _ = run_both(a, 7)
        assert not bad, (V, bad[:5])
        bad, _, _, _ = run_both(a, 7, temperature=0.0)
        assert not bad, (V, bad[:5])


def test_accept_flags_nonfinite_and_bad_tokens():
    a = W.make_accept_inputs(6, 5, 300, seed=3, logit_std=1.0, draft_noise=0.5, temperature=1.0)
    a.target_logits[0, 3, 17] = float("nan")
    a.target_logits[1, 0, 5] = float("inf")
    a.target_logits[2, 2, :] = float("-inf")
    a.draft_tokens[3, 0] = -1
    a.draft_tokens[4, 1] = 300
    for T in (1.0, 0.0):
        bad, _, orc, call = run_both(a, 5, T)
        assert not bad, bad
        st = call.status.cpu().numpy()
        assert st[0] == 1 and st[1] == 1 and st[2] == 1
        assert st[3] & 4 and st[5] == 0


def test_accept_draft_equal_to_target_accepts_everything():
    a = W.make_accept_inputs(32, 6, 5000, seed=4, logit_std=2.0, draft_noise=0.5, temperature=1.0)
    p = torch.softmax(a.target_logits[:, :-1].double(), dim=-1).float()
    a.draft_probs.copy_(p)
    call = AcceptCall(a, seed=3)
    call.run()
    torch.cuda.synchronize()
    assert (call.accept_len.cpu() == 5).all()


def test_accept_is_deterministic_and_seed_sensitive():
    a = W.build_accept(W.workload("qwen7b_longtail"))
    c1 = AcceptCall(a, seed=42)
    c1.run()
    c2 = AcceptCall(a, seed=42)
    c2.run()
    c3 = AcceptCall(a, seed=43)
    c3.run()
    torch.cuda.synchronize()
    assert torch.equal(c1.accept_len, c2.accept_len) and torch.equal(c1.next_token, c2.next_token)
    assert not (torch.equal(c1.accept_len, c3.accept_len) and torch.equal(c1.next_token, c3.next_token))
