"""Python access to the fp64 CPU oracle in ``oracle.c``.

TEST INFRASTRUCTURE ONLY: tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it. It imports nothing from the CUDA library
package, and the library never imports it.

``build()`` compiles ``oracle.c`` with gcc into ``liboracle.so`` beside it;
``lib()`` loads it (building first when the shared object is missing or older
than the source).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

TIE_EPS = 1e-5


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_SO)
        P = C.c_void_p
        i32, u32, u64, f64 = C.c_int, C.c_uint32, C.c_uint64, C.c_double
        L.orc_philox4x32_10.argtypes = [P, P, P]
        L.orc_philox4x32_10.restype = None
        L.orc_philox4x32_10_many.argtypes = [C.c_long, P, P, P]
        L.orc_philox4x32_10_many.restype = None
        L.orc_uniform.argtypes = [u64, u32, u32, u32, u32]
        L.orc_uniform.restype = f64
        L.orc_attention.argtypes = [i32] * 8 + [P] * 8
        L.orc_attention.restype = i32
        L.orc_attention_rows.argtypes = [i32] * 8 + [P] * 6 + [P, i32, P]
        L.orc_attention_rows.restype = i32
        L.orc_cascade_attention.argtypes = [i32] * 9 + [P] * 8 + [P, i32, P, P]
        L.orc_cascade_attention.restype = i32
        L.orc_accept.argtypes = [i32, i32, i32, P, P, P, P, f64, u64, P, P, P, P, P, P, P, P]
        L.orc_accept.restype = i32
        L.orc_inv_cdf.argtypes = [P, i32, f64, P]
        L.orc_inv_cdf.restype = i32
        L.orc_kv_commit.argtypes = [i32] * 8 + [P] * 8
        L.orc_kv_commit.restype = i32
        L.orc_history_draft.argtypes = [i32] * 7 + [P] * 10
        L.orc_history_draft.restype = i32
        _lib = L
    return _lib


def _np(x, dtype) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor on the CPU
        x = x.detach().cpu().numpy()
    a = np.ascontiguousarray(x)
    if a.dtype != dtype:
        a = a.view(dtype) if a.dtype.itemsize == np.dtype(dtype).itemsize else a.astype(dtype)
    return a


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def philox4x32_10(ctr: Sequence[int], key: Sequence[int]) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def philox4x32_10_many(ctrs: np.ndarray, key: Sequence[int]) -> np.ndarray:
    """The block function of every row of ``ctrs`` (uint32 [n][4]) under ``key`` (two words)."""
    c = np.ascontiguousarray(ctrs, dtype=np.uint32).reshape(-1, 4)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros_like(c)
    lib().orc_philox4x32_10_many(len(c), _p(c), _p(k), _p(out))
    return out


def uniform(seed: int, c0: int, c1: int, c2: int, c3: int = 0) -> float:
    return lib().orc_uniform(seed, c0, c1, c2, c3)


def attention(a) -> np.ndarray:
    """fp64 [B][N][Hq][D] verify attention of an ``AttnInputs``-like object; also returns flags."""
    import torch
    q = _np(a.q.view(torch.int16), np.uint16)
    k = _np(a.k_pool.view(torch.int16), np.uint16)
    v = _np(a.v_pool.view(torch.int16), np.uint16)
    tbl = _np(a.block_table, np.int32)
    lens = _np(a.ctx_lens, np.int32)
    mask = _np(a.draft_mask, np.uint64) if a.draft_mask is not None else None
    out = np.zeros((a.num_seqs, a.num_q_rows, a.num_q_heads, a.head_dim), dtype=np.float64)
    flags = np.zeros(a.num_seqs, dtype=np.int32)
    rc = lib().orc_attention(a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads, a.head_dim,
                             a.block_size, a.max_blocks_per_seq, a.num_blocks, _p(q), _p(k), _p(v),
                             _p(tbl), _p(lens), _p(mask), _p(out), _p(flags))
    if rc:
        raise ValueError(f"orc_attention returned {rc}")
    return out, flags


def attention_rows(a, rows: np.ndarray) -> np.ndarray:
    """fp64 [len(rows)][D] outputs for selected (b, i, hq) triples."""
    import torch
    q = _np(a.q.view(torch.int16), np.uint16)
    k = _np(a.k_pool.view(torch.int16), np.uint16)
    v = _np(a.v_pool.view(torch.int16), np.uint16)
    tbl = _np(a.block_table, np.int32)
    lens = _np(a.ctx_lens, np.int32)
    mask = _np(a.draft_mask, np.uint64) if a.draft_mask is not None else None
    r = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    out = np.zeros((r.shape[0], a.head_dim), dtype=np.float64)
    rc = lib().orc_attention_rows(a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads,
                                  a.head_dim, a.block_size, a.max_blocks_per_seq, a.num_blocks,
                                  _p(q), _p(k), _p(v), _p(tbl), _p(lens), _p(mask), _p(r),
                                  r.shape[0], _p(out))
    if rc:
        raise ValueError(f"orc_attention_rows returned {rc}")
    return out


def cascade_attention(a, group_offsets: Sequence[int], prefix_lens: Sequence[int],
                      rows: Optional[np.ndarray] = None):
    """Cascade (shared-prefix) verify attention of an ``AttnInputs``-like object.

    Group g = sequences [group_offsets[g], group_offsets[g+1]); its first
    prefix_lens[g] keys come from the pages of its first member. Without
    ``rows``: (fp64 [B][N][Hq][D], flags [B]); with rows (b, i, hq): fp64 [nrows][D].
    """
    import torch
    q = _np(a.q.view(torch.int16), np.uint16)
    k = _np(a.k_pool.view(torch.int16), np.uint16)
    v = _np(a.v_pool.view(torch.int16), np.uint16)
    tbl = _np(a.block_table, np.int32)
    lens = _np(a.ctx_lens, np.int32)
    mask = _np(a.draft_mask, np.uint64) if a.draft_mask is not None else None
    off = np.ascontiguousarray(group_offsets, dtype=np.int32)
    pre = np.ascontiguousarray(prefix_lens, dtype=np.int32)
    G = len(pre)
    if off.shape[0] != G + 1:
        raise ValueError("group_offsets needs one entry more than prefix_lens")
    if rows is None:
        out = np.zeros((a.num_seqs, a.num_q_rows, a.num_q_heads, a.head_dim), dtype=np.float64)
        flags = np.zeros(a.num_seqs, dtype=np.int32)
        r, nr = None, 0
    else:
        r = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
        nr = r.shape[0]
        out = np.zeros((nr, a.head_dim), dtype=np.float64)
        flags = None
    rc = lib().orc_cascade_attention(a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads,
                                     a.head_dim, a.block_size, a.max_blocks_per_seq, a.num_blocks,
                                     G, _p(off), _p(pre), _p(q), _p(k), _p(v), _p(tbl), _p(lens),
                                     _p(mask), _p(r), nr, _p(out), _p(flags))
    if rc:
        raise ValueError(f"orc_cascade_attention returned {rc}")
    return out if rows is not None else (out, flags)


class AcceptResult:
    def __init__(self, B, N):
        self.accept_len = np.zeros(B, dtype=np.int32)
        self.accept_path = np.full((B, max(N - 1, 0)), -1, dtype=np.int32)
        self.next_token = np.zeros(B, dtype=np.int32)
        self.tie_depth = np.full(B, -1, dtype=np.int32)
        self.tie_draw = np.zeros(B, dtype=np.int32)
        self.draw_lo = np.zeros(B, dtype=np.int32)
        self.draw_hi = np.zeros(B, dtype=np.int32)
        self.flags = np.zeros(B, dtype=np.int32)


def accept(logits, draft_probs, draft_tokens, temperature: float, seed: int,
           parents: Optional[Sequence[int]] = None) -> AcceptResult:
    """Accept/resample of B sequences; shapes [B][N][V], [B][N-1][V], [B][N-1]."""
    l = _np(logits, np.float32)
    B, N, V = l.shape
    q = _np(draft_probs, np.float32)
    d = _np(draft_tokens, np.int32)
    if q is None or q.size == 0:
        q = np.zeros((B, max(N - 1, 0), V), dtype=np.float32)
    if d is None or d.size == 0:
        d = np.zeros((B, max(N - 1, 0)), dtype=np.int32)
    par = None if parents is None else np.ascontiguousarray(parents, dtype=np.int32)
    res = AcceptResult(B, N)
    path = res.accept_path if N > 1 else np.zeros((B, 1), dtype=np.int32)
    rc = lib().orc_accept(B, N, V, _p(par), _p(l), _p(q), _p(d), float(temperature), int(seed),
                          _p(res.accept_len), _p(path), _p(res.next_token),
                          _p(res.tie_depth), _p(res.tie_draw), _p(res.draw_lo), _p(res.draw_hi),
                          _p(res.flags))
    if rc:
        raise ValueError(f"orc_accept returned {rc}")
    return res


def inv_cdf(w: np.ndarray, u: float):
    a = np.ascontiguousarray(w, dtype=np.float64)
    gap = np.zeros(1, dtype=np.float64)
    x = lib().orc_inv_cdf(_p(a), a.size, float(u), _p(gap))
    return x, float(gap[0])


def kv_commit(pools, block_table, ctx_lens, accept_len, accept_path, num_q_rows: int):
    """KV commit after accept, in place on the numpy uint16 (bf16 bits) pools.

    pools: list of (k_pool, v_pool) arrays [num_blocks][Hkv][bs][D], one pair per
    layer. Returns (new_ctx_lens, flags)."""
    k0 = pools[0][0]
    num_blocks, Hkv, bs, D = k0.shape
    tbl = np.ascontiguousarray(block_table, dtype=np.int32)
    B, max_blocks = tbl.shape
    lens = np.ascontiguousarray(ctx_lens, dtype=np.int32)
    alen = np.ascontiguousarray(accept_len, dtype=np.int32)
    N = int(num_q_rows)
    path = np.ascontiguousarray(accept_path, dtype=np.int32).reshape(B, max(N - 1, 1)) if N > 1 else \
        np.zeros((B, 1), dtype=np.int32)
    for k, v in pools:
        assert k.dtype == np.uint16 and v.dtype == np.uint16 and k.flags.c_contiguous and v.flags.c_contiguous
    kp = (C.c_void_p * len(pools))(*[k.ctypes.data for k, _ in pools])
    vp = (C.c_void_p * len(pools))(*[v.ctypes.data for _, v in pools])
    new_lens = np.zeros(B, dtype=np.int32)
    flags = np.zeros(B, dtype=np.int32)
    rc = lib().orc_kv_commit(B, N, Hkv, D, bs, max_blocks, num_blocks, len(pools), C.cast(kp, C.c_void_p),
                             C.cast(vp, C.c_void_p), _p(tbl), _p(lens), _p(alen), _p(path), _p(new_lens),
                             _p(flags))
    if rc:
        raise ValueError(f"orc_kv_commit returned {rc}")
    return new_lens, flags


def history_draft(history_tokens, history_lens, history_reward, history_group, seq_tokens, seq_lens,
                  seq_group, key_len: int, gamma: int, vocab: int = 0):
    """Weight-free drafts from earlier responses. Returns (drafts [B][gamma],
    draft_len [B], one-hot probs [B][gamma][vocab] or None)."""
    ht = np.ascontiguousarray(history_tokens, dtype=np.int32)
    st = np.ascontiguousarray(seq_tokens, dtype=np.int32)
    H, hs = ht.shape
    B, ss = st.shape
    hl = np.ascontiguousarray(history_lens, dtype=np.int32)
    hr = np.ascontiguousarray(history_reward, dtype=np.float32)
    hg = np.ascontiguousarray(history_group, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    sg = np.ascontiguousarray(seq_group, dtype=np.int32)
    drafts = np.zeros((B, gamma), dtype=np.int32)
    dlen = np.zeros(B, dtype=np.int32)
    probs = np.zeros((B, gamma, vocab), dtype=np.float32) if vocab > 0 else None
    rc = lib().orc_history_draft(B, H, hs, ss, int(key_len), int(gamma), int(vocab), _p(ht), _p(hl), _p(hr),
                                 _p(hg), _p(st), _p(sl), _p(sg), _p(drafts), _p(dlen), _p(probs))
    if rc:
        raise ValueError(f"orc_history_draft returned {rc}")
    return drafts, dlen, probs
