#!/usr/bin/env python
"""Verify-step benchmark: verify-steps/s and accepted tokens/s on B200.

One step = the whole verify hot path for one batch: sv_verify_attention for
every layer of the named model shape (each layer with its own KV pool, so no
layer reads another's bytes from L2) followed by one sv_accept over the
vocabulary. The timed work per step (several GB of KV) is far larger than the
126 MB L2, so no flush is needed between steps.

Default workload: the largest single-GPU configuration, the Qwen2.5-32B-shaped
batch-shrink sweep point with B=256 active sequences and gamma=8 (40 q heads /
8 kv heads, D=128, contexts lognormal around 6k capped at 32k, vocab 152064,
T=1), 64 layers. --workload / --num-seqs / --gamma select the other
configurations (one line each).

--impl reference times the fp64 CPU oracle on the host cores instead (the
baseline arm: the pages ship no runnable implementation of this path).
Multi-GPU (torchrun): every rank runs its own replica of the workload
(sequences are independent; no data-path collective); value = all ranks'
steps / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from speculative_decoding_rl_b200 import replicas as R  # noqa: E402
from speculative_decoding_rl_b200 import workloads as W  # noqa: E402

METRIC = "verify-steps/s & accepted tok/s at 1 B200; KV+logit HBM GB/s as % of peak"
UNIT = "verify-steps/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen32b_sweep")
    ap.add_argument("--layers", type=int, default=None, help="override the layer count")
    ap.add_argument("--num-seqs", type=int, default=None, help="active sequences B (qwen32b_sweep)")
    ap.add_argument("--gamma", type=int, default=None, help="chain drafts per sequence (qwen32b_sweep)")
    ap.add_argument("--cascade", action="store_true",
                    help="read each group's shared prompt pages once (sv_cascade_verify_attention); "
                         "workloads whose sequences come in groups only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-sample-seconds", type=float, default=12.0,
                    help="oracle time per CPU leg (one core, then every core)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# the sources the attention kernels are built from (a recorded ncu traffic
# figure stays valid while these are unchanged)
ATTENTION_SOURCES = ("sv_attention.cu", "sv_tc.cuh", "sv_device.cuh", "sv_internal.h")


def _code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace runs collapsed, so that
    an edit of a comment leaves the hash of the code unchanged."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "speculative_decoding_rl_b200", "csrc")
    for name in ATTENTION_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu summary, if it
    matches the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_hash") != kernel_source_hash() or d.get("workload") != workload:
        return None
    return d.get("dram_bytes_per_call")


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self):
        sm, mx, pw, reasons = [], [], [], set()
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            try:
                pw.append(float(parts[3]))
            except ValueError:
                pass
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "power_w": statistics.median(pw) if pw else None, "samples": len(sm)}


def dist_setup():
    world, rank, local = R.env_ranks()
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world > 1:
        R.init("nccl", timeout_s=120, device=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    R.barrier(world)


def max_over_ranks(x: float, world: int) -> float:
    return R.max_over_ranks(x, world, device="cuda")


def sum_over_ranks(x: float, world: int) -> float:
    return R.sum_over_ranks(x, world, device="cuda")


# ---------------------------------------------------------------------------
# CPU oracle timing (bounded sample)
# ---------------------------------------------------------------------------

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(w: W.Workload, a0, acc, layers: int, budget_s: float, seed: int = 0, threads: int = 1):
    """Time the oracle on a bounded sample and scale to verify-steps/s.

    Attention: whole query-row sets of (sequence, KV head) units in a seeded
    random order, handed to ``threads`` host threads (the oracle is plain C and
    the binding releases the GIL, so the threads run on separate cores) until
    70% of the budget is spent; the wall time is scaled by the ratio of total to
    sampled (rows x visible keys) work. Accept: chunks of whole sequences the
    same way with the rest of the budget, scaled by sequences."""
    import threading
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    B, N, Hq, Hkv = a0.num_seqs, a0.num_q_rows, a0.num_q_heads, a0.num_kv_heads
    G = Hq // Hkv
    lens = a0.ctx_lens.numpy()
    total_work = float(lens.sum()) * N * Hq
    rng = np.random.default_rng(seed)
    units = list(rng.permutation(B * Hkv))
    lock = threading.Lock()

    def attn_worker(deadline):
        work = 0.0
        while time.perf_counter() < deadline:
            with lock:
                if not units:
                    break
                u = int(units.pop())
            b, h = divmod(u, Hkv)
            rows = np.array([[b, i, h * G + g] for i in range(N) for g in range(G)], dtype=np.int32)
            oracle.attention_rows(a0, rows)
            work += float(lens[b]) * N * G
        return work

    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        work = sum(ex.map(attn_worker, [t0 + 0.7 * budget_s] * threads))
    t_attn = time.perf_counter() - t0
    chunk = 4
    starts = list(range(0, B, chunk))[::-1]

    def acc_worker(deadline):
        done = 0
        while time.perf_counter() < deadline or done == 0:
            with lock:
                if not starts:
                    break
                b0 = starts.pop()
            b1 = min(B, b0 + chunk)
            oracle.accept(acc.target_logits[b0:b1], acc.draft_probs[b0:b1], acc.draft_tokens[b0:b1],
                          acc.temperature, seed, parents=acc.tree_parents)
            done += b1 - b0
        return done

    t1 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        seqs = sum(ex.map(acc_worker, [t1 + 0.3 * budget_s] * threads))
    t_acc = (time.perf_counter() - t1) * B / seqs
    t_attn_layer = t_attn * total_work / work
    step = layers * t_attn_layer + t_acc
    how = "single-threaded" if threads == 1 else f"{threads} host threads"
    sample = (f"oracle attention on {work / (N * G):.0f} of {lens.sum() * Hkv} (sequence, kv-head) keys "
              f"({100 * work / total_work:.1f}% of one layer, scaled by work to {layers} layers) "
              f"+ oracle accept on {seqs} of {B} sequences (scaled by sequences); fp64, {how}")
    return 1.0 / step, t_attn_layer, t_acc, sample


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def make_workload(args):
    over = {}
    if args.num_seqs is not None or args.gamma is not None:
        if args.workload != "qwen32b_sweep":
            raise SystemExit("--num-seqs / --gamma apply to the qwen32b_sweep workload")
    if args.workload == "qwen32b_sweep":
        # the sweep's largest point unless a point is named
        over["num_seqs"] = 256 if args.num_seqs is None else args.num_seqs
        over["gamma"] = 8 if args.gamma is None else args.gamma
    return W.workload(args.workload, **over)


def pool_plan(a0, layers: int):
    """Distinct KV pools kept on the device and the L2 statement of the config."""
    pool_bytes = 2 * a0.k_pool.numel() * 2
    n_pools = max(1, min(layers, POOL_BUDGET_BYTES // max(1, pool_bytes)))
    l2 = ("inputs larger than L2 (every layer has its own KV pool)" if n_pools == layers else
          f"inputs larger than L2 ({n_pools} KV pools of {pool_bytes / 1e9:.1f} GB cycled over {layers} layers)")
    return pool_bytes, n_pools, l2


def config_of(w, a0, acc_in, layers: int, cascade: bool, world: int) -> dict:
    """The workload's description, identical in both arms' lines."""
    _, _, l2 = pool_plan(a0, layers)
    return {"workload": w.name, "layers": layers, "num_seqs": a0.num_seqs, "gamma": a0.num_q_rows - 1,
            "q_heads": a0.num_q_heads, "kv_heads": a0.num_kv_heads, "head_dim": a0.head_dim,
            "ctx_tokens_total": int(a0.ctx_lens.sum()), "vocab": acc_in.vocab,
            "temperature": acc_in.temperature, "tree": acc_in.tree_parents is not None, "cascade": bool(cascade),
            "l2": l2, "parallelism": f"replicas x{world}"}


def accept_launches(acc_in) -> int:
    """Kernels one sv_accept call launches: the statistics pass and a walk, then
    a pass and a walk per possible rejection pass (T > 0): one for a chain, the
    worst walk's count for a tree (earlier siblings rejected on the way to a
    node, plus that node's children or one pass when it has none)."""
    if acc_in.temperature == 0:
        return 2
    N = acc_in.num_rows
    par = acc_in.tree_parents if acc_in.tree_parents is not None else [-1] + list(range(N - 1))
    rounds = 1
    for v in range(N):
        rej, u = 0, v
        while u > 0:
            rej += sum(1 for c in range(1, u) if par[c] == par[u])
            u = par[u]
        kids = sum(1 for c in range(v + 1, N) if par[c] == v)
        rounds = max(rounds, rej + max(kids, 1))
    return 2 + 2 * rounds


def accept_bytes(acc_in, accept_len, accept_path) -> float:
    """Algorithmic bytes of one accept call: every logit once, the draft
    probabilities at the drafts, and for the draw one logit row plus the draft
    row of each rejected child of the final node (R sequences whose final node
    has children), or the final node's logit row alone (the other B - R).
    Greedy: every logit once."""
    B, N, V = acc_in.num_seqs, acc_in.num_rows, acc_in.vocab
    base = 4.0 * V * B * N
    if acc_in.temperature == 0 or N == 1:
        return base if N > 1 or acc_in.temperature == 0 else base + 4.0 * V * B
    par = acc_in.tree_parents if acc_in.tree_parents is not None else [-1] + list(range(N - 1))
    children = [[c for c in range(1, N) if par[c] == v] for v in range(N)]
    total = base + 4.0 * B * (N - 1)
    for b in range(B):
        a = int(accept_len[b])
        v = int(accept_path[b][a - 1]) if a > 0 else 0
        k = len(children[v])
        total += 4.0 * V * (1 + k) if k else 4.0 * V
    return total


# distinct KV pools are kept within this many bytes; layers beyond cycle through
# them (each pool is then far larger than L2, so no layer finds another's pages cached)
POOL_BUDGET_BYTES = 48 << 30

def run_reference(args, world, rank):
    if rank != 0:
        return
    w = make_workload(args)
    layers = args.layers or w.num_layers
    a0 = W.build_attention(w)
    acc = W.build_accept(w)
    cores = host_cores()
    budget = max(2.0, 120.0 / max(1, args.steps + args.warmup))
    vals = []
    for k in range(args.warmup + args.steps):
        v, _, _, sample = oracle_sample(w, a0, acc, layers, budget, seed=k, threads=cores)
        if k >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, a0, acc, layers, args.cascade, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample + f"; each step a bounded sample of {budget:.1f} s, scaled"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import speculative_decoding_rl_b200 as sv
    from speculative_decoding_rl_b200.session import AcceptCall, AttentionCall, CascadeCall

    dev = torch.device("cuda", local)
    w = make_workload(args)
    layers = args.layers or w.num_layers
    a0 = W.build_attention(w)
    acc_in = W.build_accept(w)
    B, N, Hq, D = a0.num_seqs, a0.num_q_rows, a0.num_q_heads, a0.head_dim
    if args.cascade and a0.group_offsets is None:
        raise SystemExit(f"--cascade: workload {w.name} has no groups of sequences sharing a prefix")
    Call = CascadeCall if args.cascade else AttentionCall

    # Layer 0 from the seeded CPU generator; layers 1.. get their own pools and
    # queries drawn on the device (same sequences and page tables). Distinct pools
    # are capped by POOL_BUDGET_BYTES; past that, layers reuse pools cyclically.
    calls = [Call(a0, device=str(dev))]
    g = torch.Generator(device=dev)
    g.manual_seed(1234 + rank)
    pool_bytes, n_pools, _ = pool_plan(a0, layers)
    for li in range(1, layers):
        c = Call.__new__(Call)
        c.inputs = a0
        c.desc = calls[0].desc
        if args.cascade:
            c.cdesc = calls[0].cdesc
        c.block_table, c.ctx_lens, c.mask = calls[0].block_table, calls[0].ctx_lens, calls[0].mask
        if li < n_pools:
            c.k_pool = torch.randn(a0.k_pool.shape, generator=g, device=dev, dtype=torch.bfloat16)
            c.v_pool = torch.randn(a0.v_pool.shape, generator=g, device=dev, dtype=torch.bfloat16)
        else:
            c.k_pool, c.v_pool = calls[li % n_pools].k_pool, calls[li % n_pools].v_pool
        c.q = torch.randn(a0.q.shape, generator=g, device=dev, dtype=torch.bfloat16)
        c.out = torch.empty_like(c.q)
        c.status = None
        c.ws_bytes, c.workspace = calls[0].ws_bytes, calls[0].workspace
        c.kv = sv.SvPagedKV(c.k_pool.data_ptr(), c.v_pool.data_ptr())
        calls.append(c)
    acc = AcceptCall(acc_in, device=str(dev), seed=0)
    stream = torch.cuda.current_stream(dev)

    K, Wm = args.steps, args.warmup
    lens_out = torch.zeros((Wm + K, B), dtype=torch.int32, device=dev)
    paths_out = torch.zeros((Wm + K, B, max(N - 1, 1)), dtype=torch.int32, device=dev)

    def step(k):
        for c in calls:
            c.run()
        acc.seed = k
        acc.accept_len = lens_out[k]
        acc.path = paths_out[k]
        acc.run()

    def graph_of(fn):
        """A CUDA graph of fn's launches (the library calls launch on the current stream)."""
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        return gr

    def replay_ms(gr, reps=3):
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            gr.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return float(np.median(ts))

    # parity spot check before timing: sampled attention rows of layer 0 and the accept
    import oracle
    step(0)
    torch.cuda.synchronize()
    rows = np.stack([np.arange(16) % B, (np.arange(16) * 3) % N, (np.arange(16) * 7) % Hq], 1).astype(np.int32)
    ref = (oracle.cascade_attention(a0, a0.group_offsets, a0.prefix_lens, rows=rows) if args.cascade
           else oracle.attention_rows(a0, rows))
    got = calls[0].out.float().cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    parity_attn = float(np.abs(got - ref).max())
    o = oracle.accept(acc_in.target_logits, acc_in.draft_probs, acc_in.draft_tokens, acc_in.temperature, 0,
                      parents=acc_in.tree_parents)
    g_len, g_tok = lens_out[0].cpu().numpy(), acc.next_token.cpu().numpy()
    exempt = (o.tie_depth >= 0) | (o.tie_draw > 0)
    in_band = (g_tok >= o.draw_lo) & (g_tok <= o.draw_hi)
    ok = np.where(o.tie_depth >= 0, True,
                  (g_len == o.accept_len) & np.where(o.tie_draw > 0, in_band, g_tok == o.next_token))
    parity = {"attn_max_abs_sampled": parity_attn, "accept_seqs_matching": int(ok.sum()), "accept_seqs": B,
              "accept_exempt": int(exempt.sum()),
              "accept_rule": "exact, or within the oracle's near-tie band (|u - r/q| < 1e-5; draw threshold "
                             "within 1e-5 of a CDF step), counted in accept_exempt"}

    # The K timed steps (each with its own Philox seed and outputs) as one CUDA
    # graph, so that host launch overhead is not timed: W eager warm-up steps,
    # one untimed replay, then the timed replay.
    for k in range(1, Wm):
        step(k)
    torch.cuda.synchronize()
    g_steps = graph_of(lambda: [step(k) for k in range(Wm, Wm + K)])
    g_steps.replay()
    torch.cuda.synchronize()
    barrier(world)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier(world)
        start.record()
        g_steps.replay()
        end.record()
        torch.cuda.synchronize()
    barrier(world)
    elapsed = start.elapsed_time(end) / 1e3
    # per-call attention time: one step's layers back to back in a graph
    g_layers = graph_of(lambda: [c.run() for c in calls])
    g_layers.replay()
    torch.cuda.synchronize()
    t_attn = replay_ms(g_layers) / 1e3 / layers
    t_plain = None
    if args.cascade:
        # the plain call on the same inputs (its workspace is the front of the cascade's)
        g_plain = graph_of(lambda: [AttentionCall.run(c) for c in calls])
        g_plain.replay()
        torch.cuda.synchronize()
        t_plain = replay_ms(g_plain) / 1e3 / layers

    elapsed_max = max_over_ranks(elapsed, world)
    steps_total = sum_over_ranks(float(K), world)
    value = steps_total / elapsed_max
    accepted = float((lens_out[Wm:Wm + K].to(torch.int64) + 1).sum().item())
    accepted_total = sum_over_ranks(accepted, world)
    tok_s = accepted_total / elapsed_max
    # the timed steps' accept statistics (this rank): a step is "effective" when it
    # accepted at least one draft
    timed_lens = lens_out[Wm:Wm + K].to(torch.float64)
    accept_stats = {"draft_len": N - 1, "mean_accept_len": float(timed_lens.mean().item()),
                    "effective_percent": 100.0 * float((timed_lens >= 1).to(torch.float64).mean().item())}

    lens_h = lens_out[Wm:Wm + K].cpu().numpy()
    paths_h = paths_out[Wm:Wm + K].cpu().numpy()

    # accept-call timing: 5 calls back to back in a graph, into scratch outputs
    # (the timed steps' results stay as they are)
    acc.accept_len = torch.zeros(B, dtype=torch.int32, device=dev)
    acc.path = torch.zeros((B, max(N - 1, 1)), dtype=torch.int32, device=dev)

    def five_accepts():
        for k in range(5):
            acc.seed = k
            acc.run()
    g_acc = graph_of(five_accepts)
    g_acc.replay()
    torch.cuda.synchronize()
    t_acc = replay_ms(g_acc) / 5e3

    # roofline of the dominant call (attention)
    kv_bytes = a0.kv_bytes_unique()
    q_out = 2 * B * N * Hq * D * 2
    tbl = int(sum((int(c) + 15) // 16 for c in a0.ctx_lens.tolist())) * 4
    alg_bytes = kv_bytes + q_out + tbl
    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / t_attn / 1e9
    # accept: the algorithmic bytes of each timed step's outcome, averaged
    acc_bytes = float(np.mean([accept_bytes(acc_in, lens_h[k], paths_h[k]) for k in range(K)]))
    step_bytes = layers * alg_bytes + acc_bytes

    # e2e through the C-ABI with host buffers: inputs of a step copied H2D from
    # pinned memory, results D2H, inside the timed region.
    e2e = None
    if not args.no_e2e:
        host_q = [c.q.cpu().pin_memory() for c in calls]
        host_l = acc_in.target_logits.pin_memory()
        host_p = acc_in.draft_probs.pin_memory()
        host_d = acc_in.draft_tokens.pin_memory()
        host_t = a0.block_table.pin_memory()
        host_c = a0.ctx_lens.pin_memory()
        res_len = torch.empty((K, B), dtype=torch.int32).pin_memory()
        res_tok = torch.empty((K, B), dtype=torch.int32).pin_memory()
        h2d = (sum(h.numel() * h.element_size() for h in host_q) + host_l.numel() * 4 + host_p.numel() * 4
               + host_d.numel() * 4 + host_t.numel() * 4 + host_c.numel() * 4)
        d2h = 2 * B * 4

        # The copies go on their own stream, in the order the step consumes them
        # (table and lengths, each layer's q, then the accept inputs), so layer
        # l's attention waits only for its own q and the accept for the logits;
        # a copy into a buffer waits for the previous step's reader of it.
        copy_stream = torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        tbl_ready, tbl_free, in_ready, in_free = ev(), ev(), ev(), ev()
        q_ready = [ev() for _ in calls]
        q_free = [ev() for _ in calls]

        def e2e_step(k):
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(tbl_free)
                calls[0].block_table.copy_(host_t, non_blocking=True)
                calls[0].ctx_lens.copy_(host_c, non_blocking=True)
                tbl_ready.record(copy_stream)
                for li, (c, h) in enumerate(zip(calls, host_q)):
                    copy_stream.wait_event(q_free[li])
                    c.q.copy_(h, non_blocking=True)
                    q_ready[li].record(copy_stream)
                copy_stream.wait_event(in_free)
                acc.logits.copy_(host_l, non_blocking=True)
                acc.q.copy_(host_p, non_blocking=True)
                acc.drafts.copy_(host_d, non_blocking=True)
                in_ready.record(copy_stream)
            stream.wait_event(tbl_ready)
            for li, c in enumerate(calls):
                stream.wait_event(q_ready[li])
                c.run(stream)
                q_free[li].record(stream)
            tbl_free.record(stream)
            stream.wait_event(in_ready)
            acc.seed = k
            acc.run(stream)
            in_free.record(stream)
            res_len[k % K].copy_(acc.accept_len, non_blocking=True)
            res_tok[k % K].copy_(acc.next_token, non_blocking=True)

        for k in range(Wm):
            e2e_step(k)
        torch.cuda.synchronize()
        barrier(world)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        copy_stream.wait_stream(stream)  # no copy of the timed steps starts before s2
        for k in range(K):
            e2e_step(k)
        e2.record(stream)
        torch.cuda.synchronize()
        e2e_elapsed = max_over_ranks(s2.elapsed_time(e2) / 1e3, world)
        # e2e step k ran with Philox seed k on the same inputs as device step k
        e2e_same = bool(np.array_equal(res_len.numpy(), lens_out[:K].cpu().numpy()))
        e2e = {"value": steps_total / e2e_elapsed, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "accept_len_matches_device": e2e_same,
               "copied": "every layer's q, logits, draft probs, drafts, block table, ctx_lens in; accept_len, "
                         "next_token out; the KV cache is the model's resident state and is not copied",
               "overlap": "copies on a second stream, each layer waiting for its own q and the accept for "
                          "its inputs"}

    # KV commit after accept (keep the root and the accepted nodes, compacted),
    # over the distinct pools, with the last step's accept results; reported
    # beside the verify step, which stays attention + accept
    n_commit = min(layers, n_pools)
    commit_layers = [(calls[i].k_pool, calls[i].v_pool) for i in range(n_commit)]
    torch.cuda.synchronize()
    alen_c = lens_out[Wm + K - 1].clone()  # the last timed step's accept results, as a pair
    path_c = paths_out[Wm + K - 1].clone()
    from speculative_decoding_rl_b200.session import CommitCall
    cc = CommitCall(calls[0].desc, commit_layers, calls[0].block_table, calls[0].ctx_lens, alen_c, path_c,
                    device=str(dev))
    cst = cc.status

    def commit():
        cc.run(stream)

    for _ in range(2):
        commit()
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(10):
        commit()
    c1.record(stream)
    torch.cuda.synchronize()
    a_host, p_host = alen_c.cpu().numpy(), path_c.cpu().numpy()
    moved = sum(int(a_host[b]) for b in range(B)
                if any(int(p_host[b, k]) != k + 1 for k in range(int(a_host[b]))))
    commit_info = {"call_ms": c0.elapsed_time(c1) / 10, "layers": n_commit,
                   "bytes_moved": 2 * 2 * moved * a0.num_kv_heads * D * 2 * n_commit,
                   "flags_clear": bool((cst == 0).all().item())}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, ta, tc, sample = oracle_sample(w, a0, acc_in, layers, args.cpu_sample_seconds)
        cores = host_cores()
        va, taa, tca, samplea = oracle_sample(w, a0, acc_in, layers, args.cpu_sample_seconds, seed=1,
                                              threads=cores)
        cpu = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
               "oracle_attn_layer_s": ta, "oracle_accept_s": tc,
               "all_cores": {"value": va, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": samplea,
                             "oracle_attn_layer_s": taa, "oracle_accept_s": tca}}

    clocks = clk.summary()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": 1e3 * elapsed_max / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w, a0, acc_in, layers, args.cascade, world),
            "accepted_tok_s": tok_s, "accept_stats": accept_stats,
            "t_attn_call_ms": 1e3 * t_attn, "t_accept_call_ms": 1e3 * t_acc,
            "t_attn_plain_call_ms": None if t_plain is None else 1e3 * t_plain,
            "hbm_gbs_step": step_bytes / (elapsed_max / K) / 1e9,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None if args.cascade else recorded_traffic(w.name),
                         "kernel": ("sv_cascade_verify_attention call: cascade_prefix_kernel + attn_tc_kernel"
                                    " + attn_combine_kernel" if args.cascade else
                                    "sv_verify_attention call: attn_tc_kernel + attn_combine_kernel"),
                         "algorithmic_bytes_per_call": alg_bytes, "peak_source": peak_kind},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": K * ((3 if args.cascade else 2) * layers + accept_launches(acc_in)),
            "clocks": clocks, "parity": parity, "kv_commit": commit_info,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        # host-only arm: rank 0 runs the oracle, other ranks exit without work
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
