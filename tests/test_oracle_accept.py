"""Pins for the oracle's accept/resample rule (no GPU).

What fixes the rule without an implementation to compare against:
  * losslessness (Accelerating RL Post-Training Rollouts via System-Integrated
    Speculative Decoding, Abstract): with drafts redrawn per trial, the token
    emitted at every position, given the walk reached it, follows the target
    p of that position -- checked by chi-square over 10^6 seeded trials at
    V = 8, for a chain and for the 3-2-2-1 draft tree;
  * the standard closed form of this rule: P(accept | reached) = sum_x min(p, q),
    so the accept-length histogram is a product of those rates;
  * special cases: gamma = 0 is plain sampling from p; q = p always accepts;
    a one-hot q at d accepts with probability p(d) and then resamples p with d
    removed; T = 0 accepts exactly up to the first mismatch with argmax; a tree
    in which every node has at most one child equals the chain;
  * the inverse CDF equals numpy's searchsorted on the cumulative sum;
  * work on top of a rejected draft is discarded (TLT reading notes, "1. RL and
    SD"): nothing after the first rejection changes the result.
"""
import numpy as np
import pytest
from scipy import stats

import oracle
from speculative_decoding_rl_b200 import workloads as W

TRIALS = 1_000_000
CHUNK = 100_000


def softmax(l, T=1.0):
    z = (np.asarray(l, dtype=np.float64)) / T
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def draw(rng, probs, n):
    """n draws from one distribution (generator-side inverse CDF)."""
    cdf = np.cumsum(probs.astype(np.float64))
    cdf /= cdf[-1]
    return np.minimum(np.searchsorted(cdf, rng.random(n), side="right"), len(probs) - 1).astype(np.int32)


def run_trials(logits, q, parents, T, trials=TRIALS, seed0=0):
    """Replicate one (logits, q) problem over many trials, redrawing drafts per trial."""
    N, V = logits.shape
    par = W.chain_parents(N) if parents is None else parents
    rng = np.random.default_rng(12345 + N)
    out = []
    for k in range(trials // CHUNK):
        L = np.broadcast_to(logits, (CHUNK, N, V)).copy()
        Q = np.broadcast_to(q, (CHUNK, N - 1, V)).copy()
        D = np.stack([draw(rng, q[c - 1], CHUNK) for c in range(1, N)], axis=1) if N > 1 \
            else np.zeros((CHUNK, 0), np.int32)
        r = oracle.accept(L, Q, D, T, seed=seed0 + k, parents=parents)
        out.append((D, r))
    D = np.concatenate([d for d, _ in out])
    res = {name: np.concatenate([getattr(r, name) for _, r in out])
           for name in ("accept_len", "accept_path", "next_token", "tie_depth", "tie_draw", "flags")}
    assert not res["flags"].any()
    return D, res, par


def chi2_pvalue(samples, p):
    counts = np.bincount(samples, minlength=len(p))
    exp = p * counts.sum()
    assert exp.min() >= 5, "expected cell count below 5"
    return stats.chisquare(counts, exp).pvalue


def test_gamma_zero_is_plain_sampling():
    rng = np.random.default_rng(1)
    l = rng.normal(0, 1.0, size=(1, 8)).astype(np.float32)
    p = softmax(l[0].astype(np.float64))
    _, res, _ = run_trials(l, np.zeros((0, 8), np.float32), None, 1.0)
    assert (res["accept_len"] == 0).all()
    assert chi2_pvalue(res["next_token"], p) > 0.01


def _chain_problem(seed, V=8, gamma=4, T=1.0, noise=0.8):
    rng = np.random.default_rng(seed)
    l = rng.normal(0, 0.8, size=(gamma + 1, V)).astype(np.float32)
    q = np.stack([softmax((l[i].astype(np.float64) + rng.normal(0, noise, V)) / T) for i in range(gamma)])
    return l, q.astype(np.float32)


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_chain_output_distribution_matches_target(T):
    l, q = _chain_problem(7, T=T)
    gamma = l.shape[0] - 1
    D, res, _ = run_trials(l, q, None, T)
    a = res["accept_len"]
    p = softmax(l.astype(np.float64), T)
    for i in range(gamma + 1):
        reached = a >= i
        tok = np.where(a[reached] > i, D[reached][:, min(i, gamma - 1)] if i < gamma else 0,
                       res["next_token"][reached])
        assert chi2_pvalue(tok, p[i]) > 0.01, f"position {i}"


def test_chain_accept_length_matches_closed_form():
    T = 1.0
    l, q = _chain_problem(8, T=T)
    gamma = l.shape[0] - 1
    _, res, _ = run_trials(l, q, None, T)
    p = softmax(l.astype(np.float64), T)
    beta = np.minimum(p[:gamma], q.astype(np.float64)).sum(axis=1)
    probs = np.array([np.prod(beta[:k]) * (1 - beta[k]) for k in range(gamma)] + [np.prod(beta)])
    counts = np.bincount(res["accept_len"], minlength=gamma + 1)
    assert stats.chisquare(counts, probs * counts.sum()).pvalue > 0.01


def test_draft_equal_to_target_always_accepts():
    rng = np.random.default_rng(3)
    l = rng.normal(0, 2.0, size=(5, 50)).astype(np.float32)
    q = softmax(l[:4].astype(np.float64)).astype(np.float32)
    B = 2000
    L = np.broadcast_to(l, (B, 5, 50)).copy()
    Q = np.broadcast_to(q, (B, 4, 50)).copy()
    D = np.stack([draw(rng, q[c], B) for c in range(4)], axis=1)
    r = oracle.accept(L, Q, D, 1.0, seed=99)
    assert (r.accept_len == 4).all()


def test_one_hot_draft():
    # q = delta at d: accept with probability p(d); on rejection the residual
    # max(0, p - q) is p with d removed, renormalised.
    rng = np.random.default_rng(4)
    V = 8
    l = rng.normal(0, 0.6, size=(2, V)).astype(np.float32)
    p0 = softmax(l[0].astype(np.float64))
    d = 3
    q = np.zeros((1, V), np.float32)
    q[0, d] = 1.0
    B = TRIALS
    acc, nxt = [], []
    for k in range(B // CHUNK):
        L = np.broadcast_to(l, (CHUNK, 2, V)).copy()
        Q = np.broadcast_to(q, (CHUNK, 1, V)).copy()
        D = np.full((CHUNK, 1), d, np.int32)
        r = oracle.accept(L, Q, D, 1.0, seed=500 + k)
        acc.append(r.accept_len)
        nxt.append(r.next_token)
    acc = np.concatenate(acc)
    nxt = np.concatenate(nxt)
    assert stats.binomtest(int((acc == 1).sum()), B, p0[d]).pvalue > 0.01
    rej = nxt[acc == 0]
    assert not (rej == d).any()
    resid = p0.copy()
    resid[d] = 0.0
    resid /= resid.sum()
    keep = np.arange(V) != d
    counts = np.bincount(rej, minlength=V)[keep]
    assert stats.chisquare(counts, resid[keep] * counts.sum()).pvalue > 0.01


def test_greedy_accepts_up_to_first_argmax_mismatch():
    rng = np.random.default_rng(5)
    B, N, V = 400, 6, 40
    l = rng.normal(0, 1.0, size=(B, N, V)).astype(np.float32)
    am = l.argmax(axis=2)
    D = am[:, :N - 1].astype(np.int32).copy()
    # corrupt a random position (or none) per sequence
    cut = rng.integers(0, N, size=B)
    for b in range(B):
        if cut[b] < N - 1:
            D[b, cut[b]] = (D[b, cut[b]] + 1 + rng.integers(0, V - 1)) % V
    q = rng.random((B, N - 1, V)).astype(np.float32)  # ignored at T = 0
    r = oracle.accept(l, q, D, 0.0, seed=0)
    np.testing.assert_array_equal(r.accept_len, np.minimum(cut, N - 1))
    np.testing.assert_array_equal(r.next_token, am[np.arange(B), r.accept_len])
    assert (r.tie_depth == -1).all() and (r.tie_draw == 0).all()
    for b in range(B):
        k = r.accept_len[b]
        assert r.accept_path[b, :k].tolist() == list(range(1, k + 1))
        assert (r.accept_path[b, k:] == -1).all()


@pytest.mark.parametrize("T", [1.0, 0.7, 0.0])
def test_outputs_ignore_everything_after_the_first_rejection(T):
    """Work on top of a rejected draft is discarded (TLT reading notes, "1. RL and SD"):
    replacing every later draft token, draft row and target row changes nothing."""
    N, V = 7, 200
    a = W.make_accept_inputs(256, N, V, seed=41, logit_std=2.0, draft_noise=1.5, temperature=T)
    l, q, d = a.target_logits.numpy(), a.draft_probs.numpy(), a.draft_tokens.numpy()
    r = oracle.accept(l, q, d, T, seed=5)
    rng = np.random.default_rng(6)
    l2, q2, d2 = l.copy(), q.copy(), d.copy()
    rejected = 0
    for b in range(l.shape[0]):
        k = int(r.accept_len[b])  # drafts 1..k accepted, draft k+1 (column k) rejected
        if k == N - 1:
            continue
        rejected += 1
        l2[b, k + 1:] = rng.normal(0, 3, size=l2[b, k + 1:].shape)       # target rows after node k
        q2[b, k + 1:] = rng.dirichlet(np.ones(V), size=N - 2 - k)         # drafts k+2 .. N-1
        d2[b, k + 1:] = rng.integers(0, V, size=N - 2 - k)
    r2 = oracle.accept(l2, q2, d2, T, seed=5)
    assert rejected > 50
    for name in ("accept_len", "accept_path", "next_token", "tie_depth", "tie_draw", "flags"):
        np.testing.assert_array_equal(getattr(r, name), getattr(r2, name))


def test_greedy_lowest_index_on_ties():
    l = np.zeros((1, 2, 10), np.float32)
    l[0, 0, [2, 5, 7]] = 3.0
    l[0, 1, [4, 9]] = 1.0
    r = oracle.accept(l, np.zeros((1, 1, 10), np.float32), np.array([[2]], np.int32), 0.0, 0)
    assert r.accept_len[0] == 1 and r.next_token[0] == 4
    r = oracle.accept(l, np.zeros((1, 1, 10), np.float32), np.array([[5]], np.int32), 0.0, 0)
    assert r.accept_len[0] == 0 and r.next_token[0] == 2


def test_tree_of_single_children_equals_chain():
    a = W.make_accept_inputs(64, 6, 300, seed=31, logit_std=2.0, draft_noise=0.7, temperature=1.0)
    r1 = oracle.accept(a.target_logits, a.draft_probs, a.draft_tokens, 1.0, seed=77)
    r2 = oracle.accept(a.target_logits, a.draft_probs, a.draft_tokens, 1.0, seed=77,
                       parents=W.chain_parents(6))
    for name in ("accept_len", "accept_path", "next_token", "tie_depth", "tie_draw"):
        np.testing.assert_array_equal(getattr(r1, name), getattr(r2, name))


def test_tree_output_distribution_matches_target():
    par = W.TREE_PARENTS_3221
    N, V, T = len(par), 8, 1.0
    rng = np.random.default_rng(21)
    l = rng.normal(0, 0.6, size=(N, V)).astype(np.float32)
    q = np.stack([softmax(l[par[c]].astype(np.float64) + rng.normal(0, 0.9, V)) for c in range(1, N)])
    q = q.astype(np.float32)
    D, res, _ = run_trials(l, q, par, T)
    p = softmax(l.astype(np.float64), T)
    path = res["accept_path"]
    a = res["accept_len"]
    B = len(a)
    checked = 0
    for v in range(N):
        if v == 0:
            reached = np.ones(B, bool)
            depth = 0
        else:
            depth = 0
            x = v
            while x != 0:
                depth += 1
                x = par[x]
            reached = path[:, depth - 1] == v
        if reached.sum() < 20000:
            continue
        cont = a[reached] > depth
        child = path[reached][:, depth] if depth < N - 1 else np.full(reached.sum(), -1)
        tok = np.where(cont, D[reached][np.arange(reached.sum()), np.maximum(child, 1) - 1],
                       res["next_token"][reached])
        assert chi2_pvalue(tok, p[v]) > 0.01, f"node {v}"
        checked += 1
    assert checked >= 8


def test_inv_cdf_matches_searchsorted():
    rng = np.random.default_rng(6)
    for _ in range(300):
        V = int(rng.integers(1, 60))
        w = rng.random(V) * (rng.random(V) < 0.7)
        if w.sum() == 0:
            w[rng.integers(0, V)] = 1.0
        u = float(rng.random())
        x, gap = oracle.inv_cdf(w, u)
        c = np.cumsum(w)
        want = int(np.searchsorted(c, u * c[-1], side="right"))
        assert x == min(want, V - 1) or (want == V and w[x] > 0)
        assert w[x] > 0
        assert gap >= 0


def test_flags_for_bad_inputs():
    a = W.make_accept_inputs(3, 4, 50, seed=1, logit_std=1.0, draft_noise=0.5, temperature=1.0)
    l = a.target_logits.numpy().copy()
    d = a.draft_tokens.numpy().copy()
    l[0, 2, 7] = np.nan
    d[1, 0] = 50  # out of range
    r = oracle.accept(l, a.draft_probs, d, 1.0, seed=3)
    assert r.flags.tolist()[0] == 1 and r.accept_len[0] == 0 and r.next_token[0] == 0
    assert r.flags[1] & 4 and r.accept_len[1] == 0
    assert r.flags[2] == 0


def test_draw_band_brackets_the_drawn_token():
    a = W.make_accept_inputs(200, 5, 3000, seed=12, logit_std=3.0, draft_noise=0.75, temperature=1.0)
    r = oracle.accept(a.target_logits, a.draft_probs, a.draft_tokens, 1.0, seed=4)
    assert (r.draw_lo <= r.next_token).all() and (r.next_token <= r.draw_hi).all()
    # the band is a single token unless the draw is a near tie
    narrow = r.draw_lo == r.draw_hi
    assert (narrow | (r.tie_draw > 0) | (r.tie_depth >= 0)).all()
