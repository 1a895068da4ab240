"""PagedKVCache: one layer's paged K/V pool plus the calls a decode step makes.

A thin convenience layer over the binding: it allocates the pools with torch
(device memory is PyTorch's job here) and forwards to the C ABI.  Per step, a
caller appends each sequence's new token (``append``: slot computation and
cache write) and then runs ``decode`` (split-K paged attention + merge).
"""
from __future__ import annotations

import torch

from . import (BLOCK_SIZE, KV_BF16, KV_F32, KV_FP8_E4M3, KV_INT4, KV_INT8, KV_KIVI4,
               compute_slot_mapping, empty_pool, empty_residual, kivi_decode_attention,
               kivi_quantize_blocks,
               kv_pool_create, paged_attention_multi_query, paged_attention_workspace_bytes,
               paged_decode_attention, paged_decode_attention_append,
               paged_decode_workspace_bytes, reshape_and_cache)

_DTYPES = {"f32": KV_F32, "bf16": KV_BF16, "fp8": KV_FP8_E4M3, "int8": KV_INT8,
           "int4": KV_INT4, "kivi4": KV_KIVI4}


class PagedKVCache:
    def __init__(self, num_blocks: int, num_kv_heads: int, head_dim: int, dtype: str,
                 device="cuda", poison: bool = False):
        self.kv_dtype = dtype
        self.device = torch.device(device)
        self.desc = kv_pool_create(num_blocks, BLOCK_SIZE, num_kv_heads, head_dim, _DTYPES[dtype])
        fill = None
        if poison:
            fill = 0x7F if dtype in ("fp8", "int8", "int4", "kivi4") else float("nan")
        self.k_pool, self.v_pool, self.scales = empty_pool(self.desc, self.device, fill)
        self.dev_error = torch.zeros(1, dtype=torch.int32, device=self.device)

    # ---- a1 + a2/a3: slots and cache write ---------------------------------------
    def append(self, block_table: torch.Tensor, seq_ids: torch.Tensor, positions: torch.Tensor,
               k_new: torch.Tensor, v_new: torch.Tensor, slots: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        if slots is None:
            slots = torch.empty(seq_ids.numel(), dtype=torch.int64, device=self.device)
        compute_slot_mapping(block_table, seq_ids, positions, slots, BLOCK_SIZE, self.dev_error,
                             stream)
        reshape_and_cache(self.desc, self.k_pool, self.v_pool, self.scales, k_new, v_new, slots,
                          self.dev_error, stream)
        return slots

    # ---- a4..a10: paged split-K decode + merge --------------------------------------
    def workspace_bytes(self, batch: int, num_q_heads: int, max_context_len: int,
                        partition_tokens: int = 0) -> int:
        return paged_decode_workspace_bytes(self.desc, batch, num_q_heads, max_context_len,
                                            partition_tokens)

    def alloc_workspace(self, batch: int, num_q_heads: int, max_context_len: int,
                        partition_tokens: int = 0) -> torch.Tensor | None:
        n = self.workspace_bytes(batch, num_q_heads, max_context_len, partition_tokens)
        return torch.empty(n, dtype=torch.uint8, device=self.device) if n else None

    def decode(self, q: torch.Tensor, block_table: torch.Tensor, context_lens: torch.Tensor,
               max_context_len: int, scale: float, out: torch.Tensor | None = None,
               partition_tokens: int = 0, workspace: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty_like(q)
        if workspace is None:
            workspace = self.alloc_workspace(q.shape[0], q.shape[1], max_context_len,
                                             partition_tokens)
        return paged_decode_attention(self.desc, out, q, self.k_pool, self.v_pool, self.scales,
                                      block_table, context_lens, max_context_len,
                                      scale, partition_tokens, workspace, self.dev_error, stream)

    def decode_append(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                      block_table: torch.Tensor, context_lens: torch.Tensor,
                      max_context_len: int, scale: float, out: torch.Tensor | None = None,
                      partition_tokens: int = 0, workspace: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
        """One decode step in one launch pair: each sequence's new token (k_new/v_new
        [batch][kv_heads][head_dim]) is stored at position context_lens[b] - 1 and
        attended to with the rest of its context."""
        if out is None:
            out = torch.empty_like(q)
        if workspace is None:
            workspace = self.alloc_workspace(q.shape[0], q.shape[1], max_context_len,
                                             partition_tokens)
        return paged_decode_attention_append(self.desc, out, q, self.k_pool, self.v_pool,
                                             self.scales, k_new, v_new, block_table,
                                             context_lens, max_context_len, scale,
                                             partition_tokens, workspace, self.dev_error, stream)

    # ---- KIVI pools: full blocks quantised, the newest L mod 16 tokens in a bf16 residual
    def alloc_residual(self, batch: int, poison: bool = False):
        self.res_k, self.res_v = empty_residual(self.desc, batch, self.device,
                                                float("nan") if poison else None)
        return self.res_k, self.res_v

    def kivi_fill(self, block_ids: torch.Tensor, k_rows: torch.Tensor, v_rows: torch.Tensor,
                  stream=None) -> None:
        """Quantise full blocks (k_rows/v_rows [n][16][kv_heads][head_dim])."""
        kivi_quantize_blocks(self.desc, self.k_pool, self.v_pool, self.scales, k_rows, v_rows,
                             block_ids, self.dev_error, stream)

    def kivi_decode(self, q: torch.Tensor, block_table: torch.Tensor, context_lens: torch.Tensor,
                    max_context_len: int, scale: float, k_new: torch.Tensor | None = None,
                    v_new: torch.Tensor | None = None, out: torch.Tensor | None = None,
                    partition_tokens: int = 0, workspace: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty_like(q)
        if workspace is None:
            workspace = self.alloc_workspace(q.shape[0], q.shape[1], max_context_len,
                                             partition_tokens)
        return kivi_decode_attention(self.desc, out, q, self.k_pool, self.v_pool, self.scales,
                                     self.res_k, self.res_v, k_new, v_new, block_table,
                                     context_lens, max_context_len, scale, partition_tokens,
                                     workspace, self.dev_error, stream)

    def errors(self) -> int:
        """The device error word (KV_DEVERR_* bits); synchronises."""
        return int(self.dev_error.item())

    def clear_errors(self) -> None:
        self.dev_error.zero_()

    # ---- several query tokens per sequence (speculative verification, prefill chunk)
    def attend(self, q: torch.Tensor, block_table: torch.Tensor, context_lens: torch.Tensor,
               max_context_len: int, scale: float, out: torch.Tensor | None = None,
               partition_tokens: int = 0, workspace: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        """q: [batch][Q][num_q_heads][head_dim]; the Q tokens are the last Q of each context."""
        if out is None:
            out = torch.empty_like(q)
        if workspace is None:
            n = paged_attention_workspace_bytes(self.desc, q.shape[0], q.shape[2], q.shape[1],
                                                max_context_len, partition_tokens)
            workspace = torch.empty(n, dtype=torch.uint8, device=self.device)
        return paged_attention_multi_query(self.desc, out, q, self.k_pool, self.v_pool,
                                           self.scales, block_table, context_lens,
                                           max_context_len, scale, partition_tokens, workspace,
                                           self.dev_error, stream)
