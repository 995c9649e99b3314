"""Python binding of libspecverify (the speculative-decoding verify step on B200).

Argument marshalling only: every step of the verify path runs in the CUDA
kernels of ``libspecverify.so``. The functions keep the C names and argument
order of ``include/specverify.h``; tensor arguments may be torch CUDA tensors
(their ``data_ptr()`` is passed) or raw integer device addresses. There is no
CPU fallback: the first call raises ImportError if the shared library is
missing (the library is loaded lazily so that the input generator module can
be imported on machines without it).
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

__all__ = [
    "SvError", "SvAttnDesc", "SvPagedKV", "SvAcceptDesc", "SvKVLayer",
    "sv_verify_attention_workspace_size", "sv_verify_attention", "sv_verify_attention_noalloc", "sv_accept",
    "sv_accept_workspace_size",
    "SvCascadeDesc", "make_cascade_desc", "sv_cascade_attention_workspace_size", "sv_cascade_verify_attention",
    "sv_kv_commit", "make_kv_layers", "SdController", "SvCtlConfig", "SvHistoryDesc", "sv_history_draft",
    "sv_status_string", "sv_last_error", "sv_version", "library_path",
    "sv_testing_philox4x32_10", "sv_testing_verify_attention_stalled", "SV_FLAG_TIMEOUT",
    "SV_FLAG_NONFINITE", "SV_FLAG_BAD_CONTEXT", "SV_FLAG_BAD_TOKEN", "SV_FLAG_BAD_BLOCK",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libspecverify.so")

SV_OK, SV_ERR_INVALID_ARG, SV_ERR_UNSUPPORTED, SV_ERR_CUDA, SV_ERR_WORKSPACE = range(5)
SV_FLAG_NONFINITE = 1
SV_FLAG_BAD_CONTEXT = 2
SV_FLAG_BAD_TOKEN = 4
SV_FLAG_BAD_BLOCK = 8
SV_FLAG_TIMEOUT = 16
SV_FLAG_BAD_PATH = 32
SV_COMMIT_MAX_LAYERS = 128
SV_CTL_GAMMA_ACCEPTANCE, SV_CTL_GAMMA_MAB = 0, 1
SV_DRAFTER_NONE, SV_DRAFTER_HISTORY, SV_DRAFTER_MODEL = 0, 1, 2
SV_CTL_MAX_BUCKETS = 64
SV_NOALLOC_SCRATCH_BYTES = 64 << 20
SV_CASCADE_MAX_GROUPS = 128


class SvError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{sv_status_string(status)}: {detail}")
        self.status = status


class SvAttnDesc(C.Structure):
    _fields_ = [("num_seqs", C.c_int32), ("num_q_rows", C.c_int32), ("num_q_heads", C.c_int32),
                ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("block_size", C.c_int32),
                ("max_blocks_per_seq", C.c_int32), ("num_blocks", C.c_int32)]


class SvPagedKV(C.Structure):
    _fields_ = [("k_pool", C.c_void_p), ("v_pool", C.c_void_p)]


class SvCascadeDesc(C.Structure):
    _fields_ = [("num_groups", C.c_int32), ("group_offsets", C.POINTER(C.c_int32)),
                ("prefix_lens", C.POINTER(C.c_int32))]


class SvKVLayer(C.Structure):
    _fields_ = [("k_pool", C.c_void_p), ("v_pool", C.c_void_p)]


class SvCtlConfig(C.Structure):
    _fields_ = [("target_weight_bytes", C.c_double), ("target_flops_per_token", C.c_double),
                ("hbm_gbs", C.c_double), ("tensor_tflops", C.c_double), ("model_draft_ms", C.c_double),
                ("history_draft_ms", C.c_double), ("num_buckets", C.c_int32),
                ("bucket_max_batch", C.c_int32 * SV_CTL_MAX_BUCKETS), ("gamma_max", C.c_int32),
                ("verify_ms", C.POINTER(C.c_double)), ("elastic_max_batch", C.c_int32),
                ("gamma_policy", C.c_int32), ("accept_prior", C.c_double), ("accept_decay", C.c_double),
                ("mab_window", C.c_int32), ("mab_explore", C.c_double), ("seed", C.c_uint64),
                ("use_model_drafter", C.c_int32), ("history_upper_batch", C.c_int32),
                ("model_max_batch", C.c_int32), ("model_probe_max_batch", C.c_int32),
                ("history_warmup_records", C.c_int32), ("model_cold_start_guard", C.c_int32),
                ("compare_after_steps", C.c_int32), ("model_probe_steps", C.c_int32),
                ("score_ema_alpha", C.c_double), ("switch_margin", C.c_double), ("cooldown_steps", C.c_int32),
                ("max_cooldown_steps", C.c_int32), ("cooldown_growth", C.c_double),
                ("bad_step_ratio", C.c_double)]


class SvCtlDecision(C.Structure):
    _fields_ = [("speculate", C.c_int32), ("gamma", C.c_int32), ("drafter", C.c_int32), ("bucket", C.c_int32),
                ("expected_tokens_per_ms", C.c_double)]


class SvCtlStep(C.Structure):
    _fields_ = [("batch", C.c_int32), ("gamma", C.c_int32), ("drafter", C.c_int32),
                ("accepted_drafts", C.c_int64), ("rejections", C.c_int64), ("step_ms", C.c_double)]


class SvHistoryDesc(C.Structure):
    _fields_ = [("num_seqs", C.c_int32), ("num_history", C.c_int32), ("history_stride", C.c_int32),
                ("seq_stride", C.c_int32), ("key_len", C.c_int32), ("gamma", C.c_int32), ("vocab", C.c_int32)]


class SvAcceptDesc(C.Structure):
    _fields_ = [("num_seqs", C.c_int32), ("num_rows", C.c_int32), ("vocab", C.c_int32),
                ("tree_parents", C.POINTER(C.c_int32))]


def _load() -> C.CDLL:
    if not os.path.exists(_SO):
        raise ImportError(
            f"libspecverify.so not found at {_SO}; build it with "
            "`python -m speculative_decoding_rl_b200.build` (nvcc, sm_100a)")
    L = C.CDLL(_SO)
    P, i32, u64, f32, sz = C.c_void_p, C.c_int32, C.c_uint64, C.c_float, C.c_size_t
    L.sv_verify_attention_workspace_size.argtypes = [C.POINTER(SvAttnDesc)]
    L.sv_verify_attention_workspace_size.restype = sz
    L.sv_verify_attention.argtypes = [C.POINTER(SvAttnDesc), P, C.POINTER(SvPagedKV), P, P, P, P, P, sz, P, P]
    L.sv_verify_attention.restype = C.c_int
    L.sv_verify_attention_noalloc.argtypes = [C.POINTER(SvAttnDesc), P, C.POINTER(SvPagedKV), P, P, P, P, P, P]
    L.sv_verify_attention_noalloc.restype = C.c_int
    L.sv_cascade_attention_workspace_size.argtypes = [C.POINTER(SvAttnDesc), C.POINTER(SvCascadeDesc)]
    L.sv_cascade_attention_workspace_size.restype = sz
    L.sv_cascade_verify_attention.argtypes = [C.POINTER(SvAttnDesc), C.POINTER(SvCascadeDesc), P,
                                              C.POINTER(SvPagedKV), P, P, P, P, P, sz, P, P]
    L.sv_cascade_verify_attention.restype = C.c_int
    L.sv_accept_workspace_size.argtypes = [C.POINTER(SvAcceptDesc)]
    L.sv_accept_workspace_size.restype = sz
    L.sv_accept.argtypes = [C.POINTER(SvAcceptDesc), P, P, P, f32, u64, P, P, P, P, P, sz, P]
    L.sv_accept.restype = C.c_int
    L.sv_kv_commit.argtypes = [C.POINTER(SvAttnDesc), i32, C.POINTER(SvKVLayer), P, P, P, P, P, P, P]
    L.sv_kv_commit.restype = C.c_int
    L.sv_ctl_default_config.argtypes = [C.POINTER(SvCtlConfig)]
    L.sv_ctl_default_config.restype = None
    L.sv_ctl_create.argtypes = [C.POINTER(SvCtlConfig)]
    L.sv_ctl_create.restype = C.c_void_p
    L.sv_ctl_destroy.argtypes = [C.c_void_p]
    L.sv_ctl_destroy.restype = None
    L.sv_ctl_decide.argtypes = [C.c_void_p, i32, i32, C.POINTER(SvCtlDecision)]
    L.sv_ctl_decide.restype = C.c_int
    L.sv_ctl_observe.argtypes = [C.c_void_p, C.POINTER(SvCtlStep)]
    L.sv_ctl_observe.restype = C.c_int
    L.sv_ctl_acceptance.argtypes = [C.c_void_p]
    L.sv_ctl_acceptance.restype = C.c_double
    L.sv_history_draft.argtypes = [C.POINTER(SvHistoryDesc)] + [P] * 10 + [P]
    L.sv_history_draft.restype = C.c_int
    L.sv_testing_philox4x32_10.argtypes = [u64, P, P, C.c_int64, P]
    L.sv_testing_philox4x32_10.restype = C.c_int
    L.sv_testing_verify_attention_stalled.argtypes = [C.POINTER(SvAttnDesc), P, C.POINTER(SvPagedKV), P, P, P, P,
                                                      P, sz, P, u64, P]
    L.sv_testing_verify_attention_stalled.restype = C.c_int
    L.sv_status_string.argtypes = [C.c_int]
    L.sv_status_string.restype = C.c_char_p
    L.sv_last_error.argtypes = []
    L.sv_last_error.restype = C.c_char_p
    L.sv_version.argtypes = []
    L.sv_version.restype = i32
    return L


_lib_handle = None


def _L() -> C.CDLL:
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


def library_path() -> str:
    return _SO


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        if x.device.type != "cuda":
            raise ValueError("tensor arguments must live on a CUDA device")
        return x.data_ptr()
    raise TypeError(f"expected a CUDA tensor or an int address, got {type(x)}")


def _stream(s) -> Optional[int]:
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int) -> None:
    if st != SV_OK:
        raise SvError(st, sv_last_error())


def sv_status_string(status: int) -> str:
    return _L().sv_status_string(int(status)).decode()


def sv_last_error() -> str:
    return _L().sv_last_error().decode()


def sv_version() -> int:
    return int(_L().sv_version())


def sv_verify_attention_workspace_size(desc: SvAttnDesc) -> int:
    return int(_L().sv_verify_attention_workspace_size(C.byref(desc)))


def sv_verify_attention(desc: SvAttnDesc, q, paged_kv: SvPagedKV, block_table, ctx_lens, draft_mask,
                        out, workspace, workspace_bytes: int, status_flags=None, stream=None) -> None:
    _check(_L().sv_verify_attention(C.byref(desc), _ptr(q), C.byref(paged_kv), _ptr(block_table),
                                    _ptr(ctx_lens), _ptr(draft_mask), _ptr(out), _ptr(workspace),
                                    int(workspace_bytes), _ptr(status_flags), _stream(stream)))


def sv_verify_attention_noalloc(desc: SvAttnDesc, q, paged_kv: SvPagedKV, block_table, ctx_lens,
                                draft_mask, out, status_flags=None, stream=None) -> None:
    """sv_verify_attention without a workspace argument, for callers that cannot
    allocate device memory: the partials go to the library's built-in scratch
    array (SV_NOALLOC_SCRATCH_BYTES). Calls that overlap on the GPU race on it."""
    _check(_L().sv_verify_attention_noalloc(C.byref(desc), _ptr(q), C.byref(paged_kv), _ptr(block_table),
                                            _ptr(ctx_lens), _ptr(draft_mask), _ptr(out), _ptr(status_flags),
                                            _stream(stream)))


def make_cascade_desc(group_offsets: Sequence[int], prefix_lens: Sequence[int]) -> SvCascadeDesc:
    """The host-side group description of sv_cascade_verify_attention; it keeps its arrays alive."""
    n = len(prefix_lens)
    if len(group_offsets) != n + 1:
        raise ValueError("group_offsets needs one entry more than prefix_lens")
    off = (C.c_int32 * (n + 1))(*[int(x) for x in group_offsets])
    pre = (C.c_int32 * max(n, 1))(*[int(x) for x in prefix_lens])
    d = SvCascadeDesc(n, C.cast(off, C.POINTER(C.c_int32)), C.cast(pre, C.POINTER(C.c_int32)))
    d._keep = (off, pre)
    return d


def sv_cascade_attention_workspace_size(desc: SvAttnDesc, cdesc: SvCascadeDesc) -> int:
    return int(_L().sv_cascade_attention_workspace_size(C.byref(desc), C.byref(cdesc)))


def sv_cascade_verify_attention(desc: SvAttnDesc, cdesc: SvCascadeDesc, q, paged_kv: SvPagedKV, block_table,
                                ctx_lens, draft_mask, out, workspace, workspace_bytes: int, status_flags=None,
                                stream=None) -> None:
    """sv_verify_attention for groups of consecutive sequences that share their first
    prefix_lens[g] keys on the pages of the group's first member."""
    _check(_L().sv_cascade_verify_attention(C.byref(desc), C.byref(cdesc), _ptr(q), C.byref(paged_kv),
                                            _ptr(block_table), _ptr(ctx_lens), _ptr(draft_mask), _ptr(out),
                                            _ptr(workspace), int(workspace_bytes), _ptr(status_flags),
                                            _stream(stream)))


def sv_accept_workspace_size(desc: SvAcceptDesc) -> int:
    return int(_L().sv_accept_workspace_size(C.byref(desc)))


def sv_accept(desc: SvAcceptDesc, target_logits, draft_probs, draft_tokens, temperature: float,
              philox_seed: int, accept_len, next_token, accept_path=None, status_flags=None,
              workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    _check(_L().sv_accept(C.byref(desc), _ptr(target_logits), _ptr(draft_probs), _ptr(draft_tokens),
                          float(temperature), int(philox_seed) & 0xFFFFFFFFFFFFFFFF, _ptr(accept_len),
                          _ptr(next_token), _ptr(accept_path), _ptr(status_flags), _ptr(workspace),
                          int(workspace_bytes), _stream(stream)))


def sv_kv_commit(desc: SvAttnDesc, layers, block_table, ctx_lens, accept_len, accept_path, new_ctx_lens,
                 status_flags=None, stream=None) -> None:
    """layers: a sequence of (k_pool, v_pool) pairs (tensors or device addresses), one per
    layer, or an array built once with ``make_kv_layers``."""
    arr = layers if isinstance(layers, C.Array) else make_kv_layers(layers)
    _check(_L().sv_kv_commit(C.byref(desc), len(layers), arr, _ptr(block_table), _ptr(ctx_lens), _ptr(accept_len),
                             _ptr(accept_path), _ptr(new_ctx_lens), _ptr(status_flags), _stream(stream)))


def make_kv_layers(layers) -> C.Array:
    """The SvKVLayer array of sv_kv_commit, built once for repeated calls."""
    return (SvKVLayer * len(layers))(*[SvKVLayer(_ptr(k), _ptr(v)) for k, v in layers])


def sv_history_draft(desc: SvHistoryDesc, history_tokens, history_lens, history_reward, history_group,
                     seq_tokens, seq_lens, seq_group, draft_tokens, draft_len, draft_probs=None,
                     stream=None) -> None:
    _check(_L().sv_history_draft(C.byref(desc), _ptr(history_tokens), _ptr(history_lens), _ptr(history_reward),
                                 _ptr(history_group), _ptr(seq_tokens), _ptr(seq_lens), _ptr(seq_group),
                                 _ptr(draft_tokens), _ptr(draft_len), _ptr(draft_probs), _stream(stream)))


def sv_testing_philox4x32_10(key: int, counters, out, n: int, stream=None) -> None:
    """Test hook: the device Philox4x32-10 words of n counters (uint32 [n][4] each)."""
    _check(_L().sv_testing_philox4x32_10(int(key) & 0xFFFFFFFFFFFFFFFF, _ptr(counters), _ptr(out), int(n),
                                         _stream(stream)))


def sv_testing_verify_attention_stalled(desc: SvAttnDesc, q, paged_kv: SvPagedKV, block_table, ctx_lens,
                                        draft_mask, out, workspace, workspace_bytes: int, status_flags,
                                        wait_limit_ns: int, stream=None) -> None:
    """Test hook: sv_verify_attention with one wait per CTA made to run out after
    wait_limit_ns; every sequence comes back flagged SV_FLAG_TIMEOUT."""
    _check(_L().sv_testing_verify_attention_stalled(C.byref(desc), _ptr(q), C.byref(paged_kv), _ptr(block_table),
                                                    _ptr(ctx_lens), _ptr(draft_mask), _ptr(out), _ptr(workspace),
                                                    int(workspace_bytes), _ptr(status_flags), int(wait_limit_ns),
                                                    _stream(stream)))


def default_ctl_config() -> SvCtlConfig:
    c = SvCtlConfig()
    _L().sv_ctl_default_config(C.byref(c))
    return c


class SdController:
    """The host speculative-decoding controller (sv_ctl_*): decide() before a
    step, observe() after it. verify_ms: [num_buckets][gamma_max + 1] measured
    verify-path milliseconds (index 0: a plain decode step)."""

    def __init__(self, config: SvCtlConfig, bucket_max_batch: Sequence[int], verify_ms):
        import numpy as np
        v = np.ascontiguousarray(verify_ms, dtype=np.float64)
        config.num_buckets = len(bucket_max_batch)
        for i, b in enumerate(bucket_max_batch):
            config.bucket_max_batch[i] = int(b)
        config.gamma_max = v.shape[1] - 1
        config.verify_ms = v.ctypes.data_as(C.POINTER(C.c_double))
        self._h = _L().sv_ctl_create(C.byref(config))
        if not self._h:
            raise SvError(SV_ERR_INVALID_ARG, sv_last_error())

    def decide(self, batch: int, history_records: int = 1) -> SvCtlDecision:
        d = SvCtlDecision()
        _check(_L().sv_ctl_decide(self._h, int(batch), int(history_records), C.byref(d)))
        return d

    def observe(self, batch: int, gamma: int, drafter: int, accepted_drafts: int, rejections: int,
                step_ms: float) -> None:
        s = SvCtlStep(int(batch), int(gamma), int(drafter), int(accepted_drafts), int(rejections), float(step_ms))
        _check(_L().sv_ctl_observe(self._h, C.byref(s)))

    def acceptance(self) -> float:
        return _L().sv_ctl_acceptance(self._h)

    def close(self) -> None:
        if self._h:
            _L().sv_ctl_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def make_accept_desc(num_seqs: int, num_rows: int, vocab: int,
                     tree_parents: Optional[Sequence[int]] = None) -> SvAcceptDesc:
    """Build an SvAcceptDesc; the parents array is kept alive on the returned object."""
    d = SvAcceptDesc(num_seqs, num_rows, vocab, None)
    if tree_parents is not None:
        arr = (C.c_int32 * len(tree_parents))(*[int(x) for x in tree_parents])
        d.tree_parents = C.cast(arr, C.POINTER(C.c_int32))
        d._parents_keepalive = arr
    return d
