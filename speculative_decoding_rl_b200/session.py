"""Device-resident call objects for the verify-step entry points and the KV commit.

Each object owns the device buffers of one call (inputs copied once with
torch, outputs, workspace) and ``run()`` makes exactly one C-ABI call on the
current torch stream. This is plumbing only: torch allocates memory and
supplies the stream, the library does all the work.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (SvAttnDesc, SvPagedKV, make_accept_desc, make_cascade_desc, make_kv_layers, sv_accept,
               sv_accept_workspace_size, sv_cascade_attention_workspace_size, sv_cascade_verify_attention,
               sv_kv_commit, sv_verify_attention, sv_verify_attention_workspace_size)


class AttentionCall:
    def __init__(self, a, device: str = "cuda", out: Optional[torch.Tensor] = None,
                 with_status: bool = True):
        dev = torch.device(device)
        self.inputs = a
        self.desc = SvAttnDesc(a.num_seqs, a.num_q_rows, a.num_q_heads, a.num_kv_heads, a.head_dim,
                               a.block_size, a.max_blocks_per_seq, a.num_blocks)
        self.q = a.q.to(dev)
        self.k_pool = a.k_pool.to(dev)
        self.v_pool = a.v_pool.to(dev)
        self.block_table = a.block_table.to(dev)
        self.ctx_lens = a.ctx_lens.to(dev)
        self.mask = a.draft_mask.to(dev) if a.draft_mask is not None else None
        self.out = out if out is not None else torch.empty_like(self.q)
        self.status = torch.full((a.num_seqs,), -1, dtype=torch.int32, device=dev) if with_status else None
        self.ws_bytes = sv_verify_attention_workspace_size(self.desc)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)
        self.kv = SvPagedKV(self.k_pool.data_ptr(), self.v_pool.data_ptr())

    def run(self, stream=None) -> torch.Tensor:
        sv_verify_attention(self.desc, self.q, self.kv, self.block_table, self.ctx_lens, self.mask,
                            self.out, self.workspace, self.ws_bytes, self.status, stream)
        return self.out

    def kv_bytes(self) -> int:
        return self.inputs.kv_bytes_unique()


class CascadeCall(AttentionCall):
    """sv_cascade_verify_attention over groups of consecutive sequences whose first
    prefix_lens[g] keys sit on the group's first member's pages (default: the
    groups recorded in the inputs)."""

    def __init__(self, a, group_offsets=None, prefix_lens=None, device: str = "cuda",
                 out: Optional[torch.Tensor] = None, with_status: bool = True):
        super().__init__(a, device=device, out=out, with_status=with_status)
        off = a.group_offsets if group_offsets is None else group_offsets
        pre = a.prefix_lens if prefix_lens is None else prefix_lens
        if off is None or pre is None:
            raise ValueError("the inputs carry no groups; pass group_offsets and prefix_lens")
        self.group_offsets, self.prefix_lens = list(off), list(pre)
        self.cdesc = make_cascade_desc(self.group_offsets, self.prefix_lens)
        self.ws_bytes = sv_cascade_attention_workspace_size(self.desc, self.cdesc)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=self.q.device)

    def run(self, stream=None) -> torch.Tensor:
        sv_cascade_verify_attention(self.desc, self.cdesc, self.q, self.kv, self.block_table, self.ctx_lens,
                                    self.mask, self.out, self.workspace, self.ws_bytes, self.status, stream)
        return self.out


class AcceptCall:
    def __init__(self, a, device: str = "cuda", seed: int = 0, with_path: bool = True,
                 with_status: bool = True, temperature: Optional[float] = None):
        dev = torch.device(device)
        self.inputs = a
        self.temperature = a.temperature if temperature is None else float(temperature)
        self.seed = int(seed)
        self.desc = make_accept_desc(a.num_seqs, a.num_rows, a.vocab, a.tree_parents)
        self.logits = a.target_logits.to(dev)
        self.q = a.draft_probs.to(dev)
        self.drafts = a.draft_tokens.to(dev)
        B, N = a.num_seqs, a.num_rows
        self.accept_len = torch.full((B,), -7, dtype=torch.int32, device=dev)
        self.next_token = torch.full((B,), -7, dtype=torch.int32, device=dev)
        self.path = torch.full((B, max(N - 1, 1)), -7, dtype=torch.int32, device=dev) if with_path else None
        self.status = torch.full((B,), -7, dtype=torch.int32, device=dev) if with_status else None
        self.ws_bytes = sv_accept_workspace_size(self.desc)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)

    def run(self, stream=None):
        sv_accept(self.desc, self.logits, self.q if self.q.numel() else None,
                  self.drafts if self.drafts.numel() else None, self.temperature, self.seed,
                  self.accept_len, self.next_token, self.path, self.status, self.workspace, self.ws_bytes,
                  stream)
        return self.accept_len, self.next_token


class CommitCall:
    """KV commit after accept over a fixed set of layers' pools (arguments prepared once)."""

    def __init__(self, desc, layers, block_table, ctx_lens, accept_len, accept_path, device: str = "cuda"):
        dev = torch.device(device)
        B = desc.num_seqs
        self.desc = desc
        self.layers = layers
        self._arr = make_kv_layers(layers)
        self.block_table, self.ctx_lens = block_table, ctx_lens
        self.accept_len, self.accept_path = accept_len, accept_path
        self.new_ctx_lens = torch.empty(B, dtype=torch.int32, device=dev)
        self.status = torch.empty(B, dtype=torch.int32, device=dev)

    def run(self, stream=None):
        sv_kv_commit(self.desc, self._arr, self.block_table, self.ctx_lens, self.accept_len, self.accept_path,
                     self.new_ctx_lens, self.status, stream)
        return self.new_ctx_lens
