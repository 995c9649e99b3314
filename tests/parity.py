"""Comparison rules shared by the GPU parity tests.

Attention (fp32 accumulation, bf16 output) against the fp64 oracle:
    max |gpu - oracle| <= 2e-2 and sum|gpu - oracle| / sum|oracle| <= 5e-3.
Accept: greedy results must match bit for bit. With sampling, a decision may
differ only where the oracle marked a near tie (|u - r(d)/q(d)| < 1e-5 for an
accept test, or a draw threshold within 1e-5 of a CDF step); everything after
the first near tie of a sequence is then exempt, and the number of exempt
sequences is reported. An exempt draw must still pick a token inside the
oracle's band: a token the draw selects for some threshold within 1e-5 of
the total mass of the sampled one.
"""
from __future__ import annotations

import numpy as np

ATTN_MAX_ABS = 2e-2
ATTN_MEAN_REL = 5e-3


def attention_errors(gpu: np.ndarray, ref: np.ndarray):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    diff = np.abs(g - r)
    max_abs = float(diff.max()) if diff.size else 0.0
    denom = float(np.abs(r).sum())
    mean_rel = float(diff.sum() / denom) if denom > 0 else float(diff.sum())
    return max_abs, mean_rel


def assert_attention_close(gpu, ref, what=""):
    max_abs, mean_rel = attention_errors(gpu, ref)
    assert np.isfinite(np.asarray(gpu, dtype=np.float64)).all(), f"{what}: non-finite output"
    assert max_abs <= ATTN_MAX_ABS, f"{what}: max abs error {max_abs:.3e}"
    assert mean_rel <= ATTN_MEAN_REL, f"{what}: mean relative error {mean_rel:.3e}"
    return max_abs, mean_rel


def compare_accept(gpu_len, gpu_next, gpu_path, gpu_status, orc, greedy: bool):
    """Returns (mismatches: list of (b, reason), exempt_count)."""
    gpu_len = np.asarray(gpu_len)
    gpu_next = np.asarray(gpu_next)
    gpu_path = None if gpu_path is None else np.asarray(gpu_path)
    gpu_status = None if gpu_status is None else np.asarray(gpu_status)
    B = len(orc.accept_len)
    bad, exempt = [], 0
    for b in range(B):
        if gpu_status is not None and int(gpu_status[b]) != int(orc.flags[b]):
            bad.append((b, f"status {int(gpu_status[b])} != {int(orc.flags[b])}"))
            continue
        if orc.flags[b] & 1:
            if gpu_len[b] != 0 or gpu_next[b] != 0:
                bad.append((b, "non-finite sequence must return 0/0"))
            continue
        n = orc.accept_path.shape[1]
        opath = orc.accept_path[b] if n else np.zeros(0, np.int32)
        gpath = gpu_path[b, :n] if (gpu_path is not None and n) else None
        td, tw = int(orc.tie_depth[b]), int(orc.tie_draw[b])
        if greedy:
            assert td < 0 and tw == 0
        if td >= 0:
            exempt += 1
            if gpu_len[b] < td or (gpath is not None and not np.array_equal(gpath[:td], opath[:td])):
                bad.append((b, f"path before near tie at depth {td} differs"))
            continue
        if gpu_len[b] != orc.accept_len[b]:
            bad.append((b, f"accept_len {int(gpu_len[b])} != {int(orc.accept_len[b])}"))
            continue
        if gpath is not None and not np.array_equal(gpath, opath):
            bad.append((b, "accept_path differs"))
            continue
        if tw:
            exempt += 1
            if not (orc.draw_lo[b] <= gpu_next[b] <= orc.draw_hi[b]):
                bad.append((b, f"near-tie draw {int(gpu_next[b])} outside [{int(orc.draw_lo[b])}, "
                               f"{int(orc.draw_hi[b])}]"))
            continue
        if gpu_next[b] != orc.next_token[b]:
            bad.append((b, f"next_token {int(gpu_next[b])} != {int(orc.next_token[b])}"))
    return bad, exempt


def host_threads() -> int:
    import os
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def all_rows(a) -> np.ndarray:
    """Every (b, i, hq) output row of an attention input set."""
    b, i, h = np.meshgrid(np.arange(a.num_seqs), np.arange(a.num_q_rows), np.arange(a.num_q_heads), indexing="ij")
    return np.stack([b.ravel(), i.ravel(), h.ravel()], axis=1).astype(np.int32)


def oracle_rows_parallel(a, rows: np.ndarray, threads: int = 0) -> np.ndarray:
    """oracle.attention_rows over chunks of rows on several host threads (the
    oracle is reentrant C and its binding releases the GIL); same values as one
    call, in the order of ``rows``."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or host_threads()
    chunks = np.array_split(rows, max(1, min(4 * threads, len(rows))))
    with ThreadPoolExecutor(threads) as ex:
        parts = list(ex.map(lambda r: oracle.attention_rows(a, r), chunks))
    return np.concatenate(parts) if parts else np.zeros((0, a.head_dim))
