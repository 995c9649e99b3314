"""sv_verify_attention_noalloc: the attention entry point for callers that
cannot allocate device memory (it uses the library's built-in scratch array
instead of a workspace argument).

Checks, through the C-ABI, that two calls in a row give the same results as
sv_verify_attention with a caller-provided workspace, bit for bit (the same
kernels on the same inputs are deterministic; only where the partials live
differs), and that a request larger than the built-in scratch is refused
before anything runs. Collected last on purpose.
"""
import numpy as np
import pytest
import torch

import speculative_decoding_rl_b200 as sv
from speculative_decoding_rl_b200 import workloads as W
from speculative_decoding_rl_b200.session import AttentionCall

pytestmark = pytest.mark.gpu


def _noalloc(call: AttentionCall):
    out = torch.full_like(call.q, float("nan"))
    status = torch.full_like(call.status, -1)
    sv.sv_verify_attention_noalloc(call.desc, call.q, call.kv, call.block_table, call.ctx_lens, call.mask,
                                   out, status)
    torch.cuda.synchronize()
    return out.view(torch.int16).cpu().numpy(), status.cpu().numpy()


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [
        W.build_attention(W.workload("qwen7b_longtail")),
        W.make_attention_inputs(11, 32, 4, 128, [700, 1031, 11, 256], seed=24,
                                parents=W.TREE_PARENTS_3221),
    ]
    for a in cases:
        call = AttentionCall(a)
        ref = call.run().view(torch.int16).cpu().numpy()
        torch.cuda.synchronize()
        ref_status = call.status.cpu().numpy()
        assert sv.sv_verify_attention_workspace_size(call.desc) <= sv.SV_NOALLOC_SCRATCH_BYTES
        for _ in range(2):  # the scratch keeps the previous call's contents
            got, status = _noalloc(call)
            np.testing.assert_array_equal(status, ref_status)
            np.testing.assert_array_equal(got, ref)  # bf16 bits of every output


def test_noalloc_refuses_requests_beyond_the_scratch():
    a = W.make_attention_inputs(5, 8, 2, 128, [64], seed=3)
    call = AttentionCall(a)
    big = sv.SvAttnDesc(512, 16, 64, 8, 128, 16, 8, a.num_blocks)
    assert sv.sv_verify_attention_workspace_size(big) > sv.SV_NOALLOC_SCRATCH_BYTES
    with pytest.raises(sv.SvError) as e:
        sv.sv_verify_attention_noalloc(big, call.q, call.kv, call.block_table, call.ctx_lens, None,
                                       call.out, None)
    assert e.value.status == sv.SV_ERR_WORKSPACE
    assert "scratch" in sv.sv_last_error()
