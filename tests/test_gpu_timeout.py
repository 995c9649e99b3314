"""A bounded device-side wait that runs out (B200).

Every wait of the attention kernel gives up after a limit and flags the call
instead of hanging. The test hook makes one wait per CTA wait on a barrier
that nothing arrives on, with a short limit: the call must return, flag every
sequence SV_FLAG_TIMEOUT, and leave the context usable, so that the next
ordinary call on the same stream matches the oracle. No fault, no hang: the
kernel takes its ordinary abort path (its own copies and products are let
finish, TMEM is freed)."""
import time

import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_rl_b200 as sv
from parity import assert_attention_close
from speculative_decoding_rl_b200 import workloads as W
from speculative_decoding_rl_b200.session import AttentionCall

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ms", [5, 50])
def test_stalled_wait_times_out_and_the_next_call_is_exact(limit_ms):
    a = W.make_attention_inputs(5, 16, 2, 128, [900, 2100, 37, 4000, 640], seed=31)
    call = AttentionCall(a)
    status = torch.full((a.num_seqs,), -1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    sv.sv_testing_verify_attention_stalled(call.desc, call.q, call.kv, call.block_table, call.ctx_lens, call.mask,
                                           call.out, call.workspace, call.ws_bytes, status, limit_ms * 1_000_000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    st = status.cpu().numpy()
    assert (st & sv.SV_FLAG_TIMEOUT).all(), st
    assert elapsed < 10.0, elapsed  # bounded: the wait gave up, nothing hung
    # the context is intact: an ordinary call on the same stream is exact
    out = call.run().float().cpu().numpy()
    torch.cuda.synchronize()
    ref, flags = oracle.attention(a)
    assert (call.status.cpu().numpy() == flags).all()
    assert_attention_close(out, ref, "after a timed-out call")


def test_stalled_call_rejects_limits_outside_the_range():
    a = W.make_attention_inputs(5, 8, 2, 128, [64], seed=3)
    call = AttentionCall(a)
    for lim in (0, 999_999, 2_000_000_001):
        with pytest.raises(sv.SvError) as e:
            sv.sv_testing_verify_attention_stalled(call.desc, call.q, call.kv, call.block_table, call.ctx_lens,
                                                   None, call.out, call.workspace, call.ws_bytes, None, lim)
        assert e.value.status == sv.SV_ERR_INVALID_ARG
