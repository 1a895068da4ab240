"""Test plumbing: stage a generated workload on the GPU through the library,
and evaluate the oracle on the same inputs.

GPU side: the pool is filled by the library's own slot computation and cache
write (history tokens), then a step appends each sequence's new token and
decodes.  Oracle side: the contiguous per-sequence K/V the generator drew
(FP8 / INT8 / INT4: quantised by the oracle's own encoder), never the GPU's pool.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import oracle
from paged_kv_cache_401_b200.cache import PagedKVCache
from workloads import Inputs, storage_view

TOL = {  # max-abs, max-rel (relative to the output's max magnitude)
    "f32": (1e-4, 1e-4),
    "bf16": (2e-2, 1e-2),
    "fp8": (5e-2, None),
    "int8": (5e-2, None),
    "int4": (5e-2, None),
    "kivi4": (5e-2, None),
}


@dataclass
class Staged:
    inp: Inputs
    cache: PagedKVCache
    block_table: torch.Tensor
    context_lens: torch.Tensor
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    seq_ids: torch.Tensor
    positions: torch.Tensor

    @property
    def max_context_len(self) -> int:
        return self.inp.max_context_len


def stage(inp: Inputs, device="cuda", poison=True, block_table: np.ndarray | None = None,
          chunk: int = 1 << 17) -> Staged:
    spec = inp.spec
    cache = PagedKVCache(inp.num_blocks, spec.num_kv_heads, spec.head_dim, spec.kv_dtype,
                         device, poison=poison)
    table = inp.block_table if block_table is None else block_table
    bt = torch.from_numpy(np.ascontiguousarray(table)).to(device)
    n = len(inp.fill_rows)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        rows = torch.from_numpy(inp.fill_rows[c0:c1])
        cache.append(bt, torch.from_numpy(inp.fill_seq_ids[c0:c1]).to(device),
                     torch.from_numpy(inp.fill_positions[c0:c1]).to(device),
                     inp.k[rows].to(device), inp.v[rows].to(device))
    app = torch.from_numpy(inp.append_rows)
    return Staged(inp=inp, cache=cache, block_table=bt,
                  context_lens=torch.from_numpy(inp.context_lens).to(device),
                  q=inp.q.to(device), k_new=inp.k[app].to(device), v_new=inp.v[app].to(device),
                  seq_ids=torch.arange(spec.batch if inp.q.shape[0] == spec.batch
                                       else inp.q.shape[0], dtype=torch.int32, device=device),
                  positions=torch.from_numpy(inp.append_positions).to(device))


def step(st: Staged, partition_tokens: int = 0, out: torch.Tensor | None = None) -> torch.Tensor:
    """One decode step: append the new token of every sequence, then decode."""
    st.cache.append(st.block_table, st.seq_ids, st.positions, st.k_new, st.v_new)
    return st.cache.decode(st.q, st.block_table, st.context_lens, st.max_context_len,
                           st.inp.spec.scale, out=out, partition_tokens=partition_tokens)


def oracle_out(inp: Inputs, seqs=None) -> tuple[np.ndarray, np.ndarray]:
    """Oracle output for the listed sequences (all by default): (indices, out)."""
    spec = inp.spec
    seqs = np.arange(inp.q.shape[0]) if seqs is None else np.asarray(seqs)
    q = storage_view(inp.q)[seqs]
    lens = inp.context_lens[seqs]
    if spec.kv_dtype in oracle.QUANTIZED:
        ks, vs, kc, vc, offs, o = [], [], [], [], [], 0
        for s in seqs:
            a, n = int(inp.seq_offsets[s]), int(inp.context_lens[s])
            kf = inp.k[a:a + n].float().numpy()
            vf = inp.v[a:a + n].float().numpy()
            c1, s1 = oracle.quantize_rows(kf, spec.kv_dtype)
            c2, s2 = oracle.quantize_rows(vf, spec.kv_dtype)
            kc.append(c1), ks.append(s1), vc.append(c2), vs.append(s2)
            offs.append(o)
            o += n
        out = oracle.decode_attention(q, np.concatenate(kc), np.concatenate(vc),
                                      np.array(offs, np.int64), lens, spec.scale,
                                      spec.num_kv_heads, spec.kv_dtype, spec.q_dtype,
                                      k_scale=np.concatenate(ks), v_scale=np.concatenate(vs))
    else:
        out = oracle.decode_attention(q, storage_view(inp.k), storage_view(inp.v),
                                      inp.seq_offsets[seqs], lens, spec.scale, spec.num_kv_heads,
                                      spec.kv_dtype, spec.q_dtype)
    return seqs, out


def check_close(gpu: torch.Tensor, ref: np.ndarray, kv_dtype: str) -> dict:
    """Compare a GPU output (any float dtype) with the double oracle; returns stats."""
    g = gpu.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), "non-finite GPU output"
    err = np.abs(g - ref)
    max_abs = float(err.max())
    max_rel = max_abs / max(float(np.abs(ref).max()), 1e-30)
    atol, rtol = TOL[kv_dtype]
    if gpu.dtype == torch.bfloat16 and kv_dtype == "f32":
        # a bf16 output is rounded to 8 significant bits: the bf16 criterion applies
        atol, rtol = TOL["bf16"]
    assert max_abs <= atol, f"max-abs {max_abs:.3e} > {atol}"
    if rtol is not None:
        assert max_rel <= rtol, f"max-rel {max_rel:.3e} > {rtol}"
    return {"max_abs": max_abs, "max_rel": max_rel}


# ---------------------------------------------------------------- KIVI pools
@dataclass
class KiviStaged:
    inp: Inputs
    cache: PagedKVCache
    block_table: torch.Tensor
    context_lens: torch.Tensor
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor

    @property
    def max_context_len(self) -> int:
        return self.inp.max_context_len


def stage_kivi(inp: Inputs, device="cuda", chunk: int = 4096) -> KiviStaged:
    """History (positions 0 .. L-2) through the library: full blocks quantised by
    kivi_quantize_blocks, the incomplete block's rows copied into the residual."""
    from workloads import kivi_layout
    spec = inp.spec
    cache = PagedKVCache(inp.num_blocks, spec.num_kv_heads, spec.head_dim, "kivi4", device,
                         poison=True)
    res_k, res_v = cache.alloc_residual(inp.q.shape[0], poison=True)
    lay = kivi_layout(inp)
    for c0 in range(0, len(lay.block_ids), chunk):
        rows = torch.from_numpy(lay.block_rows[c0:c0 + chunk].reshape(-1))
        n = min(chunk, len(lay.block_ids) - c0)
        shape = (n, 16, spec.num_kv_heads, spec.head_dim)
        cache.kivi_fill(torch.from_numpy(lay.block_ids[c0:c0 + chunk]).to(device),
                        inp.k[rows].reshape(shape).to(device), inp.v[rows].reshape(shape).to(device))
    if len(lay.res_rows):
        rr = torch.from_numpy(lay.res_rows)
        sq, sl = torch.from_numpy(lay.res_seq).long(), torch.from_numpy(lay.res_slot).long()
        res_k[sq, :, sl] = inp.k[rr].to(device)
        res_v[sq, :, sl] = inp.v[rr].to(device)
    app = torch.from_numpy(inp.append_rows)
    return KiviStaged(inp=inp, cache=cache,
                      block_table=torch.from_numpy(np.ascontiguousarray(inp.block_table)).to(device),
                      context_lens=torch.from_numpy(inp.context_lens).to(device),
                      q=inp.q.to(device), k_new=inp.k[app].to(device), v_new=inp.v[app].to(device))


def oracle_out_kivi(inp: Inputs, seqs=None, lens=None) -> tuple[np.ndarray, np.ndarray]:
    """Oracle decode over each sequence's first lens[b] tokens (default: its
    context) as a KIVI cache holds them: full blocks quantised, the rest exact."""
    spec = inp.spec
    seqs = np.arange(inp.q.shape[0]) if seqs is None else np.asarray(seqs)
    lens = inp.context_lens if lens is None else np.asarray(lens, dtype=np.int32)
    ks, vs, offs, o = [], [], [], 0
    for b in seqs:
        a, n = int(inp.seq_offsets[b]), int(lens[b])
        k64, v64 = oracle.kivi_sequence(inp.k[a:a + n].float().numpy(),
                                        inp.v[a:a + n].float().numpy())
        ks.append(k64), vs.append(v64), offs.append(o)
        o += n
    out = oracle.decode_attention(storage_view(inp.q)[seqs], np.concatenate(ks), np.concatenate(vs),
                                  np.array(offs, np.int64), lens[seqs], spec.scale,
                                  spec.num_kv_heads, "f64", spec.q_dtype)
    return seqs, out
