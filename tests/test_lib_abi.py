"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before any launch (no GPU needed)."""
import ctypes as C
import os
import re
import subprocess

import pytest

import speculative_decoding_rl_b200 as sv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("specverify.h", "specverify_testing.h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        names.update(re.findall(r"SV_API\s+[\w\s\*]*?\b(sv_\w+)\s*\(", open(h).read()))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("sv_verify_attention", "sv_verify_attention_workspace_size", "sv_accept", "sv_accept_workspace_size",
              "sv_testing_philox4x32_10", "sv_testing_verify_attention_stalled",
              "sv_cascade_verify_attention", "sv_cascade_attention_workspace_size",
              "sv_status_string", "sv_last_error", "sv_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(sv.library_path())
    out = subprocess.check_output(["nm", "-D", "--defined-only", sv.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in declared_functions():
        assert hasattr(lib, n), n
        assert n in exported, n


def test_library_is_built_for_sm100a_only():
    from speculative_decoding_rl_b200 import build
    flags = build.NVCC_FLAGS
    targets = [flags[i + 1] for i, f in enumerate(flags) if f == "-gencode"]
    assert targets == ["arch=compute_100a,code=sm_100a"], targets
    assert not any(f.startswith("-arch") or f.startswith("--gpu-architecture") for f in flags)


def test_status_strings_and_version():
    assert sv.sv_status_string(0) == "SV_OK"
    assert sv.sv_status_string(4) == "SV_ERR_WORKSPACE"
    assert sv.sv_version() >= 100


def _attn_desc(**kw):
    d = dict(num_seqs=2, num_q_rows=5, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
             max_blocks_per_seq=8, num_blocks=32)
    d.update(kw)
    return sv.SvAttnDesc(**d)


@pytest.mark.parametrize("kw,status", [
    (dict(num_q_rows=0), sv.SV_ERR_INVALID_ARG),
    (dict(num_q_rows=65), sv.SV_ERR_INVALID_ARG),
    (dict(num_q_heads=6, num_kv_heads=4), sv.SV_ERR_INVALID_ARG),
    (dict(head_dim=96), sv.SV_ERR_UNSUPPORTED),
    (dict(block_size=32), sv.SV_ERR_UNSUPPORTED),
    (dict(num_seqs=-1), sv.SV_ERR_INVALID_ARG),
    (dict(num_seqs=5000), sv.SV_ERR_UNSUPPORTED),
    (dict(num_blocks=0), sv.SV_ERR_INVALID_ARG),
])
def test_attention_rejects_bad_descriptors(kw, status):
    d = _attn_desc(**kw)
    with pytest.raises(sv.SvError) as e:
        sv.sv_verify_attention(d, 16, sv.SvPagedKV(16, 16), 16, 16, None, 16, 256, 1 << 20)
    assert e.value.status == status
    assert sv.sv_verify_attention_workspace_size(d) == 0


def test_attention_rejects_null_and_misaligned_pointers():
    d = _attn_desc()
    with pytest.raises(sv.SvError) as e:
        sv.sv_verify_attention(d, None, sv.SvPagedKV(16, 16), 16, 16, None, 16, 256, 1 << 20)
    assert e.value.status == sv.SV_ERR_INVALID_ARG
    with pytest.raises(sv.SvError) as e:
        sv.sv_verify_attention(d, 8, sv.SvPagedKV(16, 16), 16, 16, None, 16, 256, 1 << 20)
    assert e.value.status == sv.SV_ERR_INVALID_ARG


def test_attention_with_no_sequences_is_a_no_op():
    sv.sv_verify_attention(_attn_desc(num_seqs=0), None, sv.SvPagedKV(None, None), None, None, None,
                           None, None, 0)


@pytest.mark.parametrize("off,pre", [
    ([0], []),                       # no groups
    ([0, 1], [16]),                  # offsets end before num_seqs
    ([1, 2], [16]),                  # offsets start after 0
    ([0, 2, 1, 2], [0, 0, 0]),       # decreasing
    ([0, 1, 2], [16, 8]),            # prefix not whole pages
    ([0, 1, 2], [-16, 0]),           # negative prefix
    ([0, 2], [16 * 9]),              # prefix past max_blocks_per_seq pages
    ([0] * 130 + [2], [0] * 130),    # more than SV_CASCADE_MAX_GROUPS
])
def test_cascade_rejects_bad_groups(off, pre):
    d = _attn_desc()
    c = sv.make_cascade_desc(off, pre)
    with pytest.raises(sv.SvError) as e:
        sv.sv_cascade_verify_attention(d, c, 16, sv.SvPagedKV(16, 16), 16, 16, None, 16, 256, 1 << 20)
    assert e.value.status == sv.SV_ERR_INVALID_ARG
    assert sv.sv_cascade_attention_workspace_size(d, c) == 0


def test_cascade_rejects_bad_descriptors_and_pointers():
    c = sv.make_cascade_desc([0, 2], [16])
    with pytest.raises(sv.SvError) as e:
        sv.sv_cascade_verify_attention(_attn_desc(head_dim=96), c, 16, sv.SvPagedKV(16, 16), 16, 16, None, 16,
                                       256, 1 << 20)
    assert e.value.status == sv.SV_ERR_UNSUPPORTED
    with pytest.raises(sv.SvError) as e:
        sv.sv_cascade_verify_attention(_attn_desc(), c, 8, sv.SvPagedKV(16, 16), 16, 16, None, 16, 256, 1 << 20)
    assert e.value.status == sv.SV_ERR_INVALID_ARG
    lib = C.CDLL(sv.library_path())
    lib.sv_cascade_verify_attention.restype = C.c_int
    st = lib.sv_cascade_verify_attention(C.byref(_attn_desc()), None, C.c_void_p(16), None, None, None, None,
                                         None, None, C.c_size_t(0), None, None)
    assert st == sv.SV_ERR_INVALID_ARG


def test_cascade_desc_needs_one_offset_per_group_boundary():
    with pytest.raises(ValueError):
        sv.make_cascade_desc([0, 1], [16, 16])
    with pytest.raises(ValueError):
        sv.make_cascade_desc([0, 1, 2, 3], [16, 16])
    d = sv.make_cascade_desc([0, 3, 5], [32, 0])
    assert d.num_groups == 2 and [d.group_offsets[i] for i in range(3)] == [0, 3, 5]
    assert [d.prefix_lens[i] for i in range(2)] == [32, 0]


def test_cascade_with_no_sequences_is_a_no_op():
    sv.sv_cascade_verify_attention(_attn_desc(num_seqs=0), sv.make_cascade_desc([0, 0], [32]), None,
                                   sv.SvPagedKV(None, None), None, None, None, None, None, 0)


@pytest.mark.parametrize("kw,parents,temp,status", [
    (dict(num_rows=0), None, 1.0, sv.SV_ERR_INVALID_ARG),
    (dict(num_rows=65), None, 1.0, sv.SV_ERR_INVALID_ARG),
    (dict(vocab=0), None, 1.0, sv.SV_ERR_INVALID_ARG),
    (dict(vocab=10_000_000), None, 1.0, sv.SV_ERR_UNSUPPORTED),
    (dict(), [-1, 0, 2, 1], 1.0, sv.SV_ERR_INVALID_ARG),   # parent not before child
    (dict(), [0, 0, 1, 2], 1.0, sv.SV_ERR_INVALID_ARG),    # root parent must be -1
    (dict(), None, -1.0, sv.SV_ERR_INVALID_ARG),
    (dict(), None, float("nan"), sv.SV_ERR_INVALID_ARG),
    (dict(), None, float("inf"), sv.SV_ERR_INVALID_ARG),
])
def test_accept_rejects_bad_arguments(kw, parents, temp, status):
    d = dict(num_seqs=2, num_rows=4, vocab=100)
    d.update(kw)
    desc = sv.make_accept_desc(d["num_seqs"], d["num_rows"], d["vocab"], parents)
    with pytest.raises(sv.SvError) as e:
        sv.sv_accept(desc, 16, 16, 16, temp, 0, 16, 16, None, None, stream=0)
    assert e.value.status == status


def test_accept_workspace_is_required_and_sized():
    desc = sv.make_accept_desc(4, 5, 1000)
    need = sv.sv_accept_workspace_size(desc)
    assert need > 0 and need % 256 == 0
    assert sv.sv_accept_workspace_size(sv.make_accept_desc(8, 5, 1000)) > need
    assert sv.sv_accept_workspace_size(sv.make_accept_desc(4, 5, 100_000)) > need
    assert sv.sv_accept_workspace_size(sv.make_accept_desc(4, 0, 1000)) == 0
    assert sv.sv_accept_workspace_size(sv.make_accept_desc(4, 5, 10_000_000)) == 0
    for ws, nbytes in [(None, need), (256, need - 1), (128, need)]:
        with pytest.raises(sv.SvError) as e:
            sv.sv_accept(desc, 16, 16, 16, 1.0, 0, 16, 16, None, None, ws, nbytes, stream=0)
        assert e.value.status == sv.SV_ERR_WORKSPACE
        assert "workspace" in sv.sv_last_error()


def test_accept_requires_outputs_and_drafts():
    desc = sv.make_accept_desc(2, 4, 100)
    with pytest.raises(sv.SvError) as e:
        sv.sv_accept(desc, 16, 16, None, 1.0, 0, 16, 16, None, None, stream=0)
    assert e.value.status == sv.SV_ERR_INVALID_ARG
    with pytest.raises(sv.SvError) as e:
        sv.sv_accept(desc, 16, None, 16, 1.0, 0, 16, 16, None, None, stream=0)
    assert e.value.status == sv.SV_ERR_INVALID_ARG
    with pytest.raises(sv.SvError) as e:
        sv.sv_accept(desc, 16, 16, 16, 1.0, 0, None, 16, None, None, stream=0)
    assert e.value.status == sv.SV_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,layers,status", [
    (dict(num_q_rows=0), 1, 1), (dict(num_q_rows=65), 1, 1), (dict(head_dim=12), 1, 2),
    (dict(head_dim=264), 1, 2), (dict(block_size=32), 1, 2), (dict(num_kv_heads=0), 1, 1),
    (dict(num_blocks=0), 1, 1), ({}, 0, 1), ({}, 129, 1),
])
def test_kv_commit_rejects_bad_arguments(kw, layers, status):
    base = dict(num_seqs=2, num_q_rows=5, num_q_heads=4, num_kv_heads=2, head_dim=128, block_size=16,
                max_blocks_per_seq=4, num_blocks=8)
    base.update(kw)
    d = sv.SvAttnDesc(*[base[k] for k in ("num_seqs", "num_q_rows", "num_q_heads", "num_kv_heads", "head_dim",
                                          "block_size", "max_blocks_per_seq", "num_blocks")])
    with pytest.raises(sv.SvError) as e:
        sv.sv_kv_commit(d, [(256, 512)] * layers, 64, 64, 64, 64, 64)
    assert e.value.status == status


def test_kv_commit_rejects_null_and_misaligned_pointers():
    d = sv.SvAttnDesc(2, 5, 4, 2, 128, 16, 4, 8)
    for layers, args in [([(256, 8)], (64, 64, 64, 64, 64)), ([(256, 512)], (0, 64, 64, 64, 64)),
                         ([(256, 512)], (64, 64, 64, 0, 64)), ([(256, 512)], (64, 66, 64, 64, 64))]:
        with pytest.raises(sv.SvError) as e:
            sv.sv_kv_commit(d, layers, *args)
        assert e.value.status == 1
    sv.sv_kv_commit(sv.SvAttnDesc(0, 5, 4, 2, 128, 16, 4, 8), [(256, 512)], 0, 0, 0, 0, 0)  # no sequences


@pytest.mark.parametrize("kw", [dict(key_len=0), dict(key_len=65), dict(gamma=0), dict(gamma=64),
                                dict(history_stride=0), dict(vocab=-1), dict(num_seqs=-1)])
def test_history_draft_rejects_bad_descriptors(kw):
    base = dict(num_seqs=2, num_history=3, history_stride=16, seq_stride=16, key_len=3, gamma=4, vocab=0)
    base.update(kw)
    d = sv.SvHistoryDesc(*[base[k] for k in ("num_seqs", "num_history", "history_stride", "seq_stride",
                                             "key_len", "gamma", "vocab")])
    with pytest.raises(sv.SvError) as e:
        sv.sv_history_draft(d, *([64] * 9))
    assert e.value.status == 1


def test_history_draft_rejects_null_and_misaligned_pointers():
    d = sv.SvHistoryDesc(2, 3, 16, 16, 3, 4, 8)
    with pytest.raises(sv.SvError):
        sv.sv_history_draft(d, 64, 64, 64, 64, 64, 64, 64, 64, 64, None)  # vocab > 0 without probs
    with pytest.raises(sv.SvError):
        sv.sv_history_draft(d, 64, 64, 66, 64, 64, 64, 64, 64, 64, 64)
    sv.sv_history_draft(sv.SvHistoryDesc(0, 3, 16, 16, 3, 4, 0), 0, 0, 0, 0, 0, 0, 0, 0, 0)


def test_kv_commit_refuses_outputs_that_alias_inputs():
    # an in-place length update (new_ctx_lens == ctx_lens) would let late CTAs
    # read the new length; it is refused on the host before any launch
    d = sv.SvAttnDesc(4, 5, 4, 2, 128, 16, 4, 8)
    base = dict(block_table=0x10000, ctx_lens=0x20000, accept_len=0x30000, accept_path=0x40000,
                new_ctx_lens=0x50000, status_flags=0x60000)
    for out_name in ("new_ctx_lens", "status_flags"):
        for in_name in ("block_table", "ctx_lens", "accept_len", "accept_path"):
            for delta in (0, 4, 12):
                args = dict(base)
                args[out_name] = base[in_name] + delta
                with pytest.raises(sv.SvError) as e:
                    sv.sv_kv_commit(d, [(256, 512)], args["block_table"], args["ctx_lens"], args["accept_len"],
                                    args["accept_path"], args["new_ctx_lens"], args["status_flags"])
                assert e.value.status == sv.SV_ERR_INVALID_ARG, (out_name, in_name, delta)
                assert "overlap" in sv.sv_last_error()
    args = dict(base)
    args["status_flags"] = base["new_ctx_lens"] + 8
    with pytest.raises(sv.SvError):
        sv.sv_kv_commit(d, [(256, 512)], *[args[k] for k in ("block_table", "ctx_lens", "accept_len", "accept_path",
                                                             "new_ctx_lens", "status_flags")])


def test_testing_hooks_reject_bad_arguments():
    with pytest.raises(sv.SvError) as e:
        sv.sv_testing_philox4x32_10(0, 16, 16, -1, stream=0)
    assert e.value.status == sv.SV_ERR_INVALID_ARG
    with pytest.raises(sv.SvError) as e:
        sv.sv_testing_philox4x32_10(0, 8, 16, 4, stream=0)
    assert e.value.status == sv.SV_ERR_INVALID_ARG
    sv.sv_testing_philox4x32_10(0, None, None, 0, stream=0)  # nothing to do
    d = _attn_desc()
    for lim in (0, 2_000_000_001):
        with pytest.raises(sv.SvError) as e:
            sv.sv_testing_verify_attention_stalled(d, 16, sv.SvPagedKV(16, 16), 16, 16, None, 16, 256, 1 << 20,
                                                   None, lim, stream=0)
        assert e.value.status == sv.SV_ERR_INVALID_ARG
    with pytest.raises(sv.SvError) as e:  # descriptor checks as for the plain call
        sv.sv_testing_verify_attention_stalled(_attn_desc(head_dim=96), 16, sv.SvPagedKV(16, 16), 16, 16, None, 16,
                                               256, 1 << 20, None, 10_000_000, stream=0)
    assert e.value.status == sv.SV_ERR_UNSUPPORTED
