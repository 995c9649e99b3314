// Host speculative-decoding controller: per decode step, whether to speculate,
// how many drafts and which drafter, from measured costs and observed
// acceptance. No GPU work. Policies (see include/specverify.h):
//  - elastic enable (TLT reading notes, "Elastic enable");
//  - roofline toggle (EfficientRollout, "System-aware SD toggle policy");
//  - acceptance-aware draft length (EfficientRollout, "Acceptance-aware
//    draft-length adaptation") or BEG-MAB (TLT reading notes, "BEG-MAB");
//  - timing_guard drafter switch (History Tree PR, dynamic_rl timing_guard).
// Readings where the pages stop short: acceptance is a censored geometric
// estimate per drafter (each sequence contributes its accepted drafts and one
// rejection if it stopped before gamma), decayed per step, with a prior of
// four pseudo-counts; a model-drafter probe is bad when most of its steps are
// bad or its score does not beat the history score by the switch margin; after
// a good probe the model drafter stays until its score drops below the history
// score times the bad-step ratio, which starts a cooldown like a bad probe.
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <deque>
#include <new>
#include <vector>

#include "../../include/specverify.h"

namespace sv {
void record_error(const char *msg);
}

namespace {

constexpr double PRIOR_COUNTS = 4.0;

struct Guard {  // timing_guard state of one batch bucket
    double hist_score = 0.0, model_score = 0.0;
    bool hist_has = false, model_has = false;
    int64_t hist_steps = 0;
    int probe_left = 0, probe_bad = 0, probe_len = 0;
    bool on_model = false;
    int64_t cooldown_until = 0;
    double cooldown_len = 0.0;
};

}  // namespace

struct sv_ctl {
    sv_ctl_config cfg;
    std::vector<double> verify;            // [bucket][gamma]
    double acc_a[3] = {0, 0, 0};           // decayed accepted drafts, per drafter
    double acc_r[3] = {0, 0, 0};           // decayed rejections, per drafter
    int64_t steps = 0;
    uint64_t rng = 0;
    std::vector<Guard> guard;              // per bucket
    std::vector<std::vector<std::deque<double>>> mab;  // [bucket][gamma] recent tokens/ms

    int bucket_of(int batch) const {
        for (int i = 0; i < cfg.num_buckets; ++i)
            if (batch <= cfg.bucket_max_batch[i]) return i;
        return cfg.num_buckets - 1;
    }
    double beta(int drafter) const {
        const double p = cfg.accept_prior;
        return (acc_a[drafter] + PRIOR_COUNTS * p) / (acc_a[drafter] + acc_r[drafter] + PRIOR_COUNTS);
    }
    // expected tokens one sequence advances per verify step: sum_{k=0..gamma} beta^k
    static double expected_tokens(double b, int gamma) {
        double e = 0.0, t = 1.0;
        for (int k = 0; k <= gamma; ++k) { e += t; t *= b; }
        return e;
    }
    double target_ms(double tokens) const {
        const double mem = cfg.target_weight_bytes / (cfg.hbm_gbs * 1e9);
        const double cmp = tokens * cfg.target_flops_per_token / (cfg.tensor_tflops * 1e12);
        return 1e3 * std::max(mem, cmp);
    }
    double step_ms(int bucket, int batch, int gamma, int drafter) const {
        const double v = verify[(size_t)bucket * (cfg.gamma_max + 1) + gamma];
        if (gamma == 0) return target_ms(batch) + v;
        const double draft = drafter == SV_DRAFTER_MODEL ? gamma * cfg.model_draft_ms : cfg.history_draft_ms;
        return target_ms((double)batch * (gamma + 1)) + draft + v;
    }
    double rate(int bucket, int batch, int gamma, int drafter) const {
        const double tok = gamma == 0 ? batch : batch * expected_tokens(beta(drafter), gamma);
        return tok / step_ms(bucket, batch, gamma, drafter);
    }
    uint64_t next_rand() {  // splitmix64
        uint64_t z = (rng += 0x9E3779B97F4A7C15ull);
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    }
    double uniform() { return (double)(next_rand() >> 11) * (1.0 / 9007199254740992.0); }

    int choose_drafter(int bucket, int batch, int hist_records) {
        const bool hist_ok = batch < cfg.history_upper_batch;
        const bool model_ok = cfg.use_model_drafter && batch <= cfg.model_max_batch &&
                              !(cfg.model_cold_start_guard && hist_records < cfg.history_warmup_records);
        if (!model_ok) return hist_ok ? SV_DRAFTER_HISTORY : SV_DRAFTER_NONE;
        Guard &g = guard[bucket];
        if (g.probe_left > 0 || g.on_model) return SV_DRAFTER_MODEL;
        if (steps < g.cooldown_until) return hist_ok ? SV_DRAFTER_HISTORY : SV_DRAFTER_NONE;
        if (g.hist_steps >= cfg.compare_after_steps && batch <= cfg.model_probe_max_batch) {
            g.probe_left = cfg.model_probe_steps;  // probe the model drafter
            g.probe_len = cfg.model_probe_steps;
            g.probe_bad = 0;
            return SV_DRAFTER_MODEL;
        }
        return hist_ok ? SV_DRAFTER_HISTORY : SV_DRAFTER_MODEL;
    }

    void start_cooldown(Guard &g) {
        g.on_model = false;
        if (g.cooldown_len <= 0.0) g.cooldown_len = cfg.cooldown_steps;
        g.cooldown_until = steps + 1 + (int64_t)g.cooldown_len;  // called while observing step `steps`
        g.cooldown_len = std::min(g.cooldown_len * cfg.cooldown_growth, (double)cfg.max_cooldown_steps);
    }
};

static bool bad(const char *msg) {
    sv::record_error(msg);
    return false;
}

static bool check_config(const sv_ctl_config *c) {
    if (!c) return bad("config is NULL");
    if (c->num_buckets < 1 || c->num_buckets > SV_CTL_MAX_BUCKETS) return bad("num_buckets must be in [1, 64]");
    for (int i = 0; i < c->num_buckets; ++i)
        if (c->bucket_max_batch[i] < 1 || (i > 0 && c->bucket_max_batch[i] <= c->bucket_max_batch[i - 1]))
            return bad("bucket_max_batch must be positive and increasing");
    if (c->gamma_max < 1 || c->gamma_max > SV_CTL_MAX_GAMMA) return bad("gamma_max must be in [1, 63]");
    if (!c->verify_ms) return bad("verify_ms is NULL");
    for (int i = 0; i < c->num_buckets * (c->gamma_max + 1); ++i)
        if (!(c->verify_ms[i] >= 0.0) || isinf(c->verify_ms[i])) return bad("verify_ms entries must be finite and >= 0");
    if (!(c->hbm_gbs > 0.0) || !(c->tensor_tflops > 0.0)) return bad("hbm_gbs and tensor_tflops must be positive");
    if (!(c->target_weight_bytes >= 0.0) || !(c->target_flops_per_token >= 0.0) || !(c->model_draft_ms >= 0.0) ||
        !(c->history_draft_ms >= 0.0))
        return bad("target costs and draft costs must be >= 0");
    if (c->elastic_max_batch < 0) return bad("elastic_max_batch < 0");
    if (c->gamma_policy != SV_CTL_GAMMA_ACCEPTANCE && c->gamma_policy != SV_CTL_GAMMA_MAB) return bad("unknown gamma_policy");
    if (!(c->accept_prior > 0.0 && c->accept_prior < 1.0)) return bad("accept_prior must be in (0, 1)");
    if (!(c->accept_decay >= 0.0 && c->accept_decay < 1.0)) return bad("accept_decay must be in [0, 1)");
    if (c->mab_window < 1) return bad("mab_window < 1");
    if (!(c->mab_explore >= 0.0 && c->mab_explore <= 1.0)) return bad("mab_explore must be in [0, 1]");
    if (c->history_upper_batch < 0 || c->model_max_batch < 0 || c->model_probe_max_batch < 0 ||
        c->history_warmup_records < 0 || c->compare_after_steps < 0 || c->model_probe_steps < 1 ||
        c->cooldown_steps < 0 || c->max_cooldown_steps < c->cooldown_steps)
        return bad("timing_guard counts out of range");
    if (!(c->score_ema_alpha > 0.0 && c->score_ema_alpha <= 1.0)) return bad("score_ema_alpha must be in (0, 1]");
    if (!(c->switch_margin > 0.0) || !(c->cooldown_growth >= 1.0) || !(c->bad_step_ratio > 0.0))
        return bad("switch_margin, cooldown_growth or bad_step_ratio out of range");
    return true;
}

extern "C" {

void sv_ctl_default_config(sv_ctl_config *c) {
    if (!c) return;
    memset(c, 0, sizeof *c);
    c->hbm_gbs = 1.0;
    c->tensor_tflops = 1.0;
    c->gamma_max = 8;
    c->gamma_policy = SV_CTL_GAMMA_ACCEPTANCE;
    c->accept_prior = 0.7;
    c->accept_decay = 0.9;
    c->mab_window = 32;
    c->mab_explore = 0.05;
    // timing_guard: the History Tree PR's defaults
    c->use_model_drafter = 1;
    c->history_upper_batch = 64;
    c->model_max_batch = 8;
    c->model_probe_max_batch = 2;
    c->history_warmup_records = 1;
    c->model_cold_start_guard = 1;
    c->compare_after_steps = 64;
    c->model_probe_steps = 8;
    c->score_ema_alpha = 0.3;
    c->switch_margin = 1.02;
    c->cooldown_steps = 8192;
    c->max_cooldown_steps = 65536;
    c->cooldown_growth = 4.0;
    c->bad_step_ratio = 0.98;
}

sv_ctl *sv_ctl_create(const sv_ctl_config *config) {
    if (!check_config(config)) return nullptr;
    sv_ctl *c = new (std::nothrow) sv_ctl;
    if (!c) {
        sv::record_error("out of host memory");
        return nullptr;
    }
    c->cfg = *config;
    const size_t n = (size_t)config->num_buckets * (config->gamma_max + 1);
    c->verify.assign(config->verify_ms, config->verify_ms + n);
    c->cfg.verify_ms = nullptr;  // the copy is what is used
    c->rng = config->seed;
    c->guard.assign(config->num_buckets, Guard());
    c->mab.assign(config->num_buckets, std::vector<std::deque<double>>(config->gamma_max + 1));
    return c;
}

void sv_ctl_destroy(sv_ctl *ctl) { delete ctl; }

double sv_ctl_acceptance(const sv_ctl *ctl) {
    if (!ctl) return 0.0;
    // the estimate of the drafter with more evidence
    const int d = (ctl->acc_a[SV_DRAFTER_MODEL] + ctl->acc_r[SV_DRAFTER_MODEL] >
                   ctl->acc_a[SV_DRAFTER_HISTORY] + ctl->acc_r[SV_DRAFTER_HISTORY]) ? SV_DRAFTER_MODEL
                                                                                    : SV_DRAFTER_HISTORY;
    return ctl->beta(d);
}

sv_status sv_ctl_decide(sv_ctl *ctl, int32_t batch, int32_t history_records, sv_ctl_decision *out) {
    if (!ctl || !out) {
        sv::record_error("ctl or out is NULL");
        return SV_ERR_INVALID_ARG;
    }
    if (batch < 1) {
        sv::record_error("batch < 1");
        return SV_ERR_INVALID_ARG;
    }
    const sv_ctl_config &c = ctl->cfg;
    const int bucket = ctl->bucket_of(batch);
    out->bucket = bucket;
    const double plain = ctl->rate(bucket, batch, 0, SV_DRAFTER_NONE);
    out->speculate = 0;
    out->gamma = 0;
    out->drafter = SV_DRAFTER_NONE;
    out->expected_tokens_per_ms = plain;
    if (c.elastic_max_batch > 0 && batch > c.elastic_max_batch) return SV_OK;  // elastic enable
    const int drafter = ctl->choose_drafter(bucket, batch, history_records);
    if (drafter == SV_DRAFTER_NONE) return SV_OK;
    // the best draft length under the cost model (the roofline toggle's comparison)
    int best = 1;
    double best_rate = 0.0;
    for (int g = 1; g <= c.gamma_max; ++g) {
        const double r = ctl->rate(bucket, batch, g, drafter);
        if (r > best_rate) { best_rate = r; best = g; }
    }
    const bool probing = ctl->guard[bucket].probe_left > 0 && drafter == SV_DRAFTER_MODEL;
    if (best_rate <= plain && !probing) return SV_OK;  // roofline toggle: speculation does not pay
    int gamma = best;
    if (c.gamma_policy == SV_CTL_GAMMA_MAB) {
        auto &arms = ctl->mab[bucket];
        int pick = -1;
        for (int g = 1; g <= c.gamma_max && pick < 0; ++g)
            if (arms[g].empty()) pick = g;  // every arm once first
        if (pick < 0 && ctl->uniform() < c.mab_explore) pick = 1 + (int)(ctl->next_rand() % (uint64_t)c.gamma_max);
        if (pick < 0) {
            double best_med = -1.0;
            for (int g = 1; g <= c.gamma_max; ++g) {
                std::vector<double> w(arms[g].begin(), arms[g].end());
                std::nth_element(w.begin(), w.begin() + w.size() / 2, w.end());
                const double med = w[w.size() / 2];
                if (med > best_med) { best_med = med; pick = g; }
            }
        }
        gamma = pick;
    }
    out->speculate = 1;
    out->gamma = gamma;
    out->drafter = drafter;
    out->expected_tokens_per_ms = ctl->rate(bucket, batch, gamma, drafter);
    return SV_OK;
}

sv_status sv_ctl_observe(sv_ctl *ctl, const sv_ctl_step *s) {
    if (!ctl || !s) {
        sv::record_error("ctl or step is NULL");
        return SV_ERR_INVALID_ARG;
    }
    const sv_ctl_config &c = ctl->cfg;
    if (s->batch < 1 || s->gamma < 0 || s->gamma > c.gamma_max || s->drafter < 0 || s->drafter > 2 ||
        s->accepted_drafts < 0 || s->accepted_drafts > (int64_t)s->batch * s->gamma || s->rejections < 0 ||
        s->rejections > s->batch || !(s->step_ms > 0.0) || isinf(s->step_ms)) {
        sv::record_error("step out of range");
        return SV_ERR_INVALID_ARG;
    }
    const int bucket = ctl->bucket_of(s->batch);
    const double tokens = (double)s->batch + (double)s->accepted_drafts;
    const double r = tokens / s->step_ms;
    if (s->gamma > 0 && s->drafter != SV_DRAFTER_NONE) {
        for (int d = 1; d <= 2; ++d) { ctl->acc_a[d] *= c.accept_decay; ctl->acc_r[d] *= c.accept_decay; }
        ctl->acc_a[s->drafter] += (double)s->accepted_drafts;
        ctl->acc_r[s->drafter] += (double)s->rejections;
        if (c.gamma_policy == SV_CTL_GAMMA_MAB) {
            auto &w = ctl->mab[bucket][s->gamma];
            w.push_back(r);
            while ((int)w.size() > c.mab_window) w.pop_front();
        }
    }
    Guard &g = ctl->guard[bucket];
    const double a = c.score_ema_alpha;
    if (s->drafter == SV_DRAFTER_HISTORY) {
        g.hist_score = g.hist_has ? (1 - a) * g.hist_score + a * r : r;
        g.hist_has = true;
        ++g.hist_steps;
    } else if (s->drafter == SV_DRAFTER_MODEL) {
        g.model_score = g.model_has ? (1 - a) * g.model_score + a * r : r;
        g.model_has = true;
        const bool bad_step = g.hist_has && r < g.hist_score * c.bad_step_ratio;
        if (g.probe_left > 0) {
            g.probe_bad += bad_step;
            if (--g.probe_left == 0) {
                const bool good = 2 * g.probe_bad <= g.probe_len &&
                                  (!g.hist_has || g.model_score > g.hist_score * c.switch_margin);
                if (good) {
                    g.on_model = true;
                    g.cooldown_len = c.cooldown_steps;  // consecutive bad probes start over
                } else {
                    ctl->start_cooldown(g);
                }
            }
        } else if (g.on_model && g.hist_has && g.model_score < g.hist_score * c.bad_step_ratio) {
            ctl->start_cooldown(g);
        }
    }
    ++ctl->steps;
    return SV_OK;
}

}  // extern "C"
