"""Host speculative-decoding controller (sv_ctl_*): policy behaviour on
simulated steps, no GPU. Costs follow a 7B-shaped target on one B200: 15 GB of
weights (memory-bound at small token counts), 1.4e10 flops per token."""
import numpy as np
import pytest

import speculative_decoding_rl_b200 as sv

BUCKETS = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512]


def verify_table(gmax=8, scale=0.002):
    return np.array([[0.02 + scale * b * (g + 1) for g in range(gmax + 1)] for b in BUCKETS])


def make(**kw):
    c = sv.default_ctl_config()
    c.target_weight_bytes = 15e9
    c.target_flops_per_token = 1.4e10
    c.hbm_gbs = 6537.0
    c.tensor_tflops = 1600.0
    c.model_draft_ms = 0.2
    c.history_draft_ms = 0.02
    c.use_model_drafter = 0
    for k, v in kw.pop("cfg", {}).items():
        setattr(c, k, v)
    return sv.SdController(c, kw.pop("buckets", BUCKETS), kw.pop("verify", verify_table()))


def chain_step(rng, batch, gamma, beta):
    """accept lengths of a chain with per-token acceptance beta, truncated at gamma"""
    a = np.minimum(rng.geometric(1 - beta, size=batch) - 1, gamma)
    return int(a.sum()), int((a < gamma).sum())


def test_default_config_carries_the_timing_guard_defaults():
    c = sv.default_ctl_config()
    assert (c.history_upper_batch, c.model_max_batch, c.model_probe_max_batch) == (64, 8, 2)
    assert (c.history_warmup_records, c.model_cold_start_guard) == (1, 1)
    assert (c.compare_after_steps, c.model_probe_steps) == (64, 8)
    assert (c.score_ema_alpha, c.switch_margin, c.bad_step_ratio) == (0.3, 1.02, 0.98)
    assert (c.cooldown_steps, c.max_cooldown_steps, c.cooldown_growth) == (8192, 65536, 4.0)


def test_roofline_toggle_turns_speculation_off_once_the_target_is_compute_bound():
    ctl = make()
    on = [ctl.decide(b).speculate for b in (1, 2, 4, 8, 16, 32)]
    off = [ctl.decide(b).speculate for b in (128, 256, 384, 512)]
    assert all(on) and not any(off)
    # once off it stays off as the batch grows (same acceptance)
    seq = [ctl.decide(b).speculate for b in range(1, 513)]
    first_off = seq.index(0)
    assert not any(seq[first_off:])


def test_elastic_enable_waits_for_the_batch_to_shrink():
    ctl = make(cfg=dict(elastic_max_batch=16))
    assert ctl.decide(17).speculate == 0 and ctl.decide(64).speculate == 0
    assert ctl.decide(16).speculate == 1 and ctl.decide(3).speculate == 1


def test_acceptance_estimate_tracks_a_simulated_drafter_and_gamma_follows_it():
    chosen = []
    for beta in (0.3, 0.6, 0.9):
        ctl = make(cfg=dict(accept_decay=0.99))
        rng = np.random.default_rng(int(beta * 100))
        for _ in range(400):
            d = ctl.decide(8)
            g = d.gamma if d.speculate else 4
            acc, rej = chain_step(rng, 8, g, beta)
            ctl.observe(8, g, sv.SV_DRAFTER_HISTORY, acc, rej, 3.0)
        assert abs(ctl.acceptance() - beta) < 0.05, (beta, ctl.acceptance())
        chosen.append(ctl.decide(8).gamma)
    assert chosen[0] <= chosen[1] <= chosen[2] and chosen[0] < chosen[2], chosen


def test_beg_mab_tries_every_draft_length_then_settles_on_the_best_median():
    ctl = make(cfg=dict(gamma_policy=sv.SV_CTL_GAMMA_MAB, mab_window=16, mab_explore=0.05, seed=3))
    rng = np.random.default_rng(0)
    best = {1: 1.0, 2: 1.3, 3: 1.6, 4: 1.4, 5: 1.2, 6: 1.0, 7: 0.9, 8: 0.8}
    picks = []
    for step in range(400):
        d = ctl.decide(8)
        assert d.speculate
        g = d.gamma
        picks.append(g)
        rate = best[g] * (1 + 0.1 * rng.standard_normal())
        acc, rej = 8 * g // 2, 4
        ctl.observe(8, g, sv.SV_DRAFTER_HISTORY, acc, rej, (8 + acc) / max(rate, 1e-3))
    assert picks[:8] == list(range(1, 9))
    tail = np.array(picks[100:])
    assert (tail == 3).mean() > 0.85, np.bincount(tail)


def _guard_ctl(**kw):
    cfg = dict(use_model_drafter=1)
    cfg.update(kw)
    # memory-bound target and tiny verify costs: speculation always pays here
    return make(cfg=cfg, verify=verify_table(scale=1e-6))


def _feed(ctl, batch, drafter, rate, n):
    for _ in range(n):
        ctl.observe(batch, 4, drafter, 2 * batch, batch // 2, (batch + 2 * batch) / rate)


def test_timing_guard_uses_history_at_large_batch_and_nothing_at_or_above_its_limit():
    ctl = _guard_ctl()
    assert ctl.decide(16, 5).drafter == sv.SV_DRAFTER_HISTORY
    d = ctl.decide(64, 5)
    assert d.speculate == 0 and d.drafter == sv.SV_DRAFTER_NONE
    assert ctl.decide(2, 0).drafter == sv.SV_DRAFTER_HISTORY     # cold start guard


def test_timing_guard_probes_after_64_history_steps_and_switches_on_a_better_score():
    ctl = _guard_ctl()
    for _ in range(64):
        assert ctl.decide(2, 5).drafter == sv.SV_DRAFTER_HISTORY
        _feed(ctl, 2, sv.SV_DRAFTER_HISTORY, 1.0, 1)
    for _ in range(8):                                            # the probe
        assert ctl.decide(2, 5).drafter == sv.SV_DRAFTER_MODEL
        _feed(ctl, 2, sv.SV_DRAFTER_MODEL, 1.5, 1)
    for _ in range(20):
        assert ctl.decide(2, 5).drafter == sv.SV_DRAFTER_MODEL
        _feed(ctl, 2, sv.SV_DRAFTER_MODEL, 1.5, 1)
    # the model drafter degrades below history x 0.98: back to history
    _feed(ctl, 2, sv.SV_DRAFTER_MODEL, 0.5, 5)
    assert ctl.decide(2, 5).drafter == sv.SV_DRAFTER_HISTORY


def test_timing_guard_cooldown_grows_fourfold_after_bad_probes_up_to_its_cap():
    ctl = _guard_ctl()
    _feed(ctl, 2, sv.SV_DRAFTER_HISTORY, 1.0, 64)
    gaps = []
    for _ in range(4):
        for _ in range(8):                                        # a bad probe
            assert ctl.decide(2, 5).drafter == sv.SV_DRAFTER_MODEL
            _feed(ctl, 2, sv.SV_DRAFTER_MODEL, 0.8, 1)
        n = 0
        while ctl.decide(2, 5).drafter == sv.SV_DRAFTER_HISTORY:
            _feed(ctl, 2, sv.SV_DRAFTER_HISTORY, 1.0, 1)
            n += 1
            assert n <= 70000
        gaps.append(n)
    assert gaps == [8192, 32768, 65536, 65536], gaps


def test_probe_only_at_small_batch():
    ctl = _guard_ctl()
    _feed(ctl, 4, sv.SV_DRAFTER_HISTORY, 1.0, 200)   # batch 4: bucket of 4, above the probe limit of 2
    assert all(ctl.decide(4, 5).drafter == sv.SV_DRAFTER_HISTORY for _ in range(10))


@pytest.mark.parametrize("field,value", [
    ("num_buckets", 0), ("gamma_max", 0), ("gamma_max", 64), ("hbm_gbs", 0.0), ("accept_prior", 1.0),
    ("accept_decay", 1.0), ("mab_window", 0), ("mab_explore", 1.5), ("gamma_policy", 7),
    ("score_ema_alpha", 0.0), ("cooldown_growth", 0.5), ("model_probe_steps", 0),
])
def test_invalid_configs_are_refused(field, value):
    c = sv.default_ctl_config()
    c.target_weight_bytes, c.target_flops_per_token = 15e9, 1.4e10
    setattr(c, field, value)
    table = verify_table()
    if field == "gamma_max":
        with pytest.raises(sv.SvError):
            c2 = sv.default_ctl_config()
            c2.gamma_max = value
            table2 = np.zeros((len(BUCKETS), max(value, 0) + 1))
            sv.SdController(c2, BUCKETS, table2 if value > 0 else np.zeros((len(BUCKETS), 1)))
        return
    with pytest.raises(sv.SvError):
        sv.SdController(c, BUCKETS if field != "num_buckets" else [], table if field != "num_buckets"
                        else np.zeros((0, 9)))


def test_observe_rejects_inconsistent_steps():
    ctl = make()
    for args in [(0, 4, 1, 0, 0, 1.0), (8, 4, 1, 33, 0, 1.0), (8, 4, 1, 4, 9, 1.0), (8, 4, 1, 4, 1, 0.0),
                 (8, 99, 1, 0, 0, 1.0), (8, 4, 3, 0, 0, 1.0)]:
        with pytest.raises(sv.SvError):
            ctl.observe(*args)
