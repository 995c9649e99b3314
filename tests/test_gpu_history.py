"""GPU parity of sv_history_draft against the oracle (B200): drafts, lengths and
one-hot rows must match exactly. A small alphabet makes short keys recur, so
reward ties, first positions and the cross-group fallback are all exercised."""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_rl_b200 as sv

pytestmark = pytest.mark.gpu


def _inputs(seed, H=48, B=40, alphabet=50, hmax=2000, smax=300, groups=4):
    rng = np.random.default_rng(seed)
    hl = rng.integers(1, hmax, size=H).astype(np.int32)
    ht = rng.integers(0, alphabet, size=(H, hmax)).astype(np.int32)
    hr = np.round(rng.random(H), 1).astype(np.float32)          # ties on purpose
    hg = rng.integers(0, groups, size=H).astype(np.int32)
    sl = rng.integers(0, smax, size=B).astype(np.int32)
    st = rng.integers(0, alphabet, size=(B, smax)).astype(np.int32)
    sg = rng.integers(0, groups + 2, size=B).astype(np.int32)   # two groups without history
    # plant a few keys taken from the history so that long keys match too
    for b in range(0, B, 3):
        h = int(rng.integers(0, H))
        if hl[h] > 20 and sl[b] > 12:
            p = int(rng.integers(0, hl[h] - 12))
            st[b, sl[b] - 10:sl[b]] = ht[h, p:p + 10]
    return ht, hl, hr, hg, st, sl, sg


def _gpu(ht, hl, hr, hg, st, sl, sg, K, gamma, vocab):
    B, H = st.shape[0], ht.shape[0]
    d = sv.SvHistoryDesc(B, H, ht.shape[1], st.shape[1], K, gamma, vocab)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    drafts = torch.full((B, gamma), -9, dtype=torch.int32, device="cuda")
    dlen = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    probs = torch.full((B, gamma, vocab), 7.0, dtype=torch.float32, device="cuda") if vocab else None
    sv.sv_history_draft(d, t(ht), t(hl), t(hr), t(hg), t(st), t(sl), t(sg), drafts, dlen, probs)
    torch.cuda.synchronize()
    return drafts.cpu().numpy(), dlen.cpu().numpy(), None if probs is None else probs.cpu().numpy()


@pytest.mark.parametrize("K,gamma,vocab,seed", [(1, 4, 0, 1), (3, 4, 50, 2), (3, 7, 0, 3), (8, 5, 50, 4),
                                                 (10, 6, 0, 5), (2, 63, 50, 6)])
def test_history_draft_matches_oracle(K, gamma, vocab, seed):
    args = _inputs(seed)
    got = _gpu(*args, K, gamma, vocab)
    want = oracle.history_draft(*args, K, gamma, vocab)
    np.testing.assert_array_equal(got[0], want[0])
    np.testing.assert_array_equal(got[1], want[1])
    if vocab:
        np.testing.assert_array_equal(got[2], want[2])
    assert (want[1] > 0).any()   # misses are pinned in the oracle tests


def test_history_draft_rollout_scale():
    # 64 earlier responses of 8k tokens, 64 sequences, the 7-token chain drafts of the GRPO shape
    args = _inputs(9, H=64, B=64, alphabet=2000, hmax=8192, smax=4096, groups=4)
    got = _gpu(*args, 4, 6, 0)
    want = oracle.history_draft(*args, 4, 6, 0)
    np.testing.assert_array_equal(got[0], want[0])
    np.testing.assert_array_equal(got[1], want[1])
