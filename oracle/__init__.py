"""CPU oracle for paged GQA decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The product path (the CUDA
library and its Python binding) never imports it, and this package imports
nothing from the product.  It holds a plain, slow, obviously correct
restatement, in double precision, of every step of the decode hot path:

* ``kv_cache_bytes``      -- the KV-size formula ("KV Cache 深度解析", §二 显存账本).
* ``slot_mapping``        -- logical position -> physical slot through a block
                             table (same page, §三 PagedAttention: 16-token
                             blocks, logical-contiguous / physical-scattered;
                             "llm-inference-optimization" notes, §二 PagedKVCache:
                             write offset inside the last block).
* ``scatter_to_pool``     -- the cache write: K/V rows placed in their slots of
                             a pool laid out [block][kv_head][slot][dim].
* ``e4m3_decode`` / ``e4m3_encode`` / ``quantize_rows`` -- the FP8-E4M3 codec
                             and per-(token, kv head) absmax/448 scales
                             ("KV Cache 深度解析", §四 KV Cache 量化);
                             ``quantize_rows(x, "int8")`` the INT8 cache, symmetric
                             absmax/127 (k1-blog "KV Cache 量化", freetools
                             "KV Cache量化": INT8 halves the cache like FP8);
                             ``quantize_rows(x, "int4")`` the INT4 cache, the
                             asymmetric 4-bit routine of the
                             "llm-inference-optimization" notes §四 per row.
* ``quantize_blocks_kivi`` / ``kivi_dequantize`` -- the KIVI cache (freetools
                             "KV Cache量化": K per channel over a block, V per
                             token, newest tokens at full precision).
* ``decode_attention``    -- softmax(q·Kᵀ·scale)·V over a CONTIGUOUS per-sequence
                             copy, GQA head grouping, two passes in double
                             (C, OpenMP); "KV Cache 深度解析", §一 and §六.
* ``multi_query_attention`` -- Q query tokens per sequence, the last Q of its
                             context, each attending causally ("KV Cache 深度解析"
                             §五 chunked prefill; speculative verification).
* ``decode_attention_bruteforce`` -- the same in numpy, one (sequence, head) at
                             a time, following the page's §六 step(): tiny inputs.
* ``decode_attention_split`` -- the blockwise online-softmax update of the
                             "llm-inference-optimization" notes (§三 Flash
                             Attention), run per sequence partition, then the
                             log-sum-exp merge of partitions, in double.

Every function here is pinned by ``tests/test_oracle_*.py`` to something other
than itself (printed values, closed forms, library routines, brute force).
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build

F32, BF16, FP8_E4M3, INT8, INT4, F64 = 0, 1, 2, 3, 4, 5
_DTYPE_CODES = {"f32": F32, "bf16": BF16, "fp8": FP8_E4M3, "int8": INT8, "int4": INT4,
                "f64": F64}
QUANTIZED = ("fp8", "int8", "int4")

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_quantize_rows.restype = None
        lib.oracle_quantize_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                             ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_quantize_rows_int8.restype = None
        lib.oracle_quantize_rows_int8.argtypes = lib.oracle_quantize_rows.argtypes
        lib.oracle_quantize_rows_int4.restype = None
        lib.oracle_quantize_rows_int4.argtypes = lib.oracle_quantize_rows.argtypes
        lib.oracle_quantize_blocks_kivi.restype = None
        lib.oracle_quantize_blocks_kivi.argtypes = [ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_int64, ctypes.c_int32,
                                                    ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_decode_attention.restype = ctypes.c_int
        lib.oracle_decode_attention.argtypes = [
            ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32]
        lib.oracle_multi_query_attention.restype = ctypes.c_int
        lib.oracle_multi_query_attention.argtypes = [
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
            ctypes.c_void_p]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """OpenMP threads the C oracle's parallel loop uses."""
    return int(_load().oracle_num_threads())


# --------------------------------------------------------------------------
# KV size ("KV Cache 深度解析", §二: KV bytes = 2 x layers x kv_heads x
# head_dim x seq_len x batch x bytes_per_elem)
# --------------------------------------------------------------------------
def kv_cache_bytes(layers: int, kv_heads: int, head_dim: int, seq_len: int, batch: int,
                   bytes_per_elem: int) -> int:
    return 2 * layers * kv_heads * head_dim * seq_len * batch * bytes_per_elem


# --------------------------------------------------------------------------
# Paging: block table -> slots, and the cache write into a pool
# --------------------------------------------------------------------------
def slot_mapping(block_table: np.ndarray, seq_ids: np.ndarray, positions: np.ndarray,
                 block_size: int = 16) -> np.ndarray:
    """slot = block_table[seq][pos // block_size] * block_size + pos % block_size.

    A token at position p of a sequence lives in the sequence's logical block
    p // block_size, at offset p % block_size inside it; the block table says
    which physical block that logical block is.
    """
    out = np.empty(len(seq_ids), dtype=np.int64)
    for i, (s, p) in enumerate(zip(seq_ids.tolist(), positions.tolist())):
        phys = int(block_table[s, p // block_size])
        out[i] = phys * block_size + p % block_size
    return out


def scatter_to_pool(pool: np.ndarray, rows: np.ndarray, slots: np.ndarray,
                    block_size: int = 16) -> np.ndarray:
    """Expected pool after writing token rows into their slots.

    pool : [num_blocks][kv_heads][block_size][head_dim] (any element type,
           e.g. uint16 bf16 bits, float32, uint8 codes);
    rows : [num_tokens][kv_heads][head_dim] of the same element type;
    slots: [num_tokens] int64; a negative slot is padding and is skipped.
    Returns a modified copy; untouched slots keep their previous contents.
    """
    out = pool.copy()
    for t, slot in enumerate(slots.tolist()):
        if slot < 0:
            continue
        blk, off = divmod(int(slot), block_size)
        for h in range(rows.shape[1]):
            out[blk, h, off, :] = rows[t, h, :]
    return out


def scatter_scales_to_pool(scale_pool: np.ndarray, scales: np.ndarray, slots: np.ndarray,
                           which: int, block_size: int = 16) -> np.ndarray:
    """Expected scale pool after a write: the pool is laid out
    [num_blocks][kv_heads][2][block_size] (K row scales, then V row scales, of
    each (block, kv head)); ``which`` is 0 for K, 1 for V.  scales: [T][kv_heads].
    INT4 parameter pools carry a trailing (scale, zero) axis on both."""
    out = scale_pool.copy()
    for t, slot in enumerate(slots.tolist()):
        if slot < 0:
            continue
        blk, off = divmod(int(slot), block_size)
        out[blk, :, which, off] = scales[t, :]
    return out


# --------------------------------------------------------------------------
# FP8 E4M3 codec ("KV Cache 深度解析", §四: fp16 -> fp8 E4M3, 3 mantissa bits,
# per-token scales to hold outliers)
# --------------------------------------------------------------------------
def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(codes, dtype=np.uint8).reshape(-1)
    table = np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[flat].reshape(np.shape(codes))


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(x, dtype=np.float32).reshape(-1)
    out = np.fromiter((lib.oracle_e4m3_encode(float(v)) for v in flat), dtype=np.uint8,
                      count=flat.size)
    return out.reshape(np.shape(x))


def quantize_rows(x: np.ndarray, kind: str = "fp8") -> tuple[np.ndarray, np.ndarray]:
    """x: [..., D] float32 -> (codes [..., D], scales float32 [...]).

    kind "fp8": uint8 E4M3 codes, scale absmax/448; "int8": int8 codes,
    scale absmax/127, round to nearest (ties to even), clamp to +-127;
    "int4": uint8 codes 0..15 (one per element, unpacked) and params
    float32 [..., 2] = (scale, zero point) per row."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    d = x.shape[-1]
    rows = x.size // d
    scales = np.empty(x.shape[:-1], dtype=np.float32)
    lib = _load()
    if kind == "int8":
        codes = np.empty(x.shape, dtype=np.int8)
        lib.oracle_quantize_rows_int8(_ptr(x), rows, d, _ptr(codes), _ptr(scales))
    elif kind == "int4":
        codes = np.empty(x.shape, dtype=np.uint8)
        params = np.empty(x.shape[:-1] + (2,), dtype=np.float32)
        lib.oracle_quantize_rows_int4(_ptr(x), rows, d, _ptr(codes), _ptr(params))
        return codes, params
    elif kind == "fp8":
        codes = np.empty(x.shape, dtype=np.uint8)
        lib.oracle_quantize_rows(_ptr(x), rows, d, _ptr(codes), _ptr(scales))
    else:
        raise ValueError(f"unknown quantisation {kind!r}")
    return codes, scales


def quantize_blocks_kivi(k: np.ndarray, v: np.ndarray):
    """KIVI quantisation of full blocks of one kv head: k, v [blocks][16][D]
    float32 -> (k_codes [blocks][16][D] uint8, k_params [blocks][D][2],
    v_codes [blocks][16][D] uint8, v_params [blocks][16][2]); params are
    (scale, zero) as float32, K per channel over the block, V per token row."""
    k = np.ascontiguousarray(k, dtype=np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    nb, bs, d = k.shape
    assert bs == 16 and v.shape == k.shape
    kc = np.empty(k.shape, np.uint8)
    vc = np.empty(v.shape, np.uint8)
    kp = np.empty((nb, d, 2), np.float32)
    vp = np.empty((nb, 16, 2), np.float32)
    _load().oracle_quantize_blocks_kivi(_ptr(k), _ptr(v), nb, d, _ptr(kc), _ptr(kp), _ptr(vc),
                                        _ptr(vp))
    return kc, kp, vc, vp


def kivi_dequantize(k_codes, k_params, v_codes, v_params):
    """(code - zero) * scale in float64: K with per-channel parameters, V per row."""
    k = (k_codes.astype(np.float64) - k_params[:, None, :, 1]) * k_params[:, None, :, 0]
    v = (v_codes.astype(np.float64) - v_params[:, :, 1:2]) * v_params[:, :, 0:1]
    return k, v


def kivi_sequence(k_rows: np.ndarray, v_rows: np.ndarray):
    """One sequence's K/V [L][Hkv][D] (float32 values of the stored source rows)
    as the KIVI cache holds them, in float64: full blocks quantised (K per
    channel, V per token), the last L mod 16 tokens exact."""
    L, hkv, d = k_rows.shape
    full = L // 16
    k64 = k_rows.astype(np.float64).copy()
    v64 = v_rows.astype(np.float64).copy()
    if full:
        kb = k_rows[:full * 16].reshape(full, 16, hkv, d).transpose(0, 2, 1, 3).reshape(-1, 16, d)
        vb = v_rows[:full * 16].reshape(full, 16, hkv, d).transpose(0, 2, 1, 3).reshape(-1, 16, d)
        kd, vd = kivi_dequantize(*quantize_blocks_kivi(kb, vb))
        k64[:full * 16] = kd.reshape(full, hkv, 16, d).transpose(0, 2, 1, 3).reshape(-1, hkv, d)
        v64[:full * 16] = vd.reshape(full, hkv, 16, d).transpose(0, 2, 1, 3).reshape(-1, hkv, d)
    return k64, v64


# --------------------------------------------------------------------------
# Decode attention over contiguous per-sequence K/V
# --------------------------------------------------------------------------
def decode_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, seq_offsets: np.ndarray,
                     lens: np.ndarray, scale: float, num_kv_heads: int, kv_dtype: str,
                     q_dtype: str, k_scale: np.ndarray | None = None,
                     v_scale: np.ndarray | None = None, return_weights: bool = False):
    """Double-precision decode attention (C oracle).

    q     : [B][Hq][D]   float32 (q_dtype "f32") or uint16 bf16 bits ("bf16")
    k, v  : [T][Hkv][D]  float32 / uint16 bf16 bits / uint8 E4M3 codes / int8 codes /
                         float64 ("f64", values already dequantised)
    seq_offsets : [B] int64, first token of each sequence in k/v
    lens  : [B] int32 context lengths (>= 1)
    k_scale, v_scale : [T][Hkv] float32 for kv_dtype "fp8" / "int8";
                       [T][Hkv][2] (scale, zero) for "int4"
    (int4 codes: uint8 0..15, one per element)
    Returns out [B][Hq][D] float64 (and weights [B][Hq][max(lens)] if asked).
    """
    lib = _load()
    b, hq, d = q.shape
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    seq_offsets = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    if kv_dtype in QUANTIZED:
        k_scale = np.ascontiguousarray(k_scale, dtype=np.float32)
        v_scale = np.ascontiguousarray(v_scale, dtype=np.float32)
    out = np.empty((b, hq, d), dtype=np.float64)
    max_len = int(lens.max()) if b else 0
    weights = np.empty((b, hq, max_len), dtype=np.float64) if return_weights else None
    rc = lib.oracle_decode_attention(_DTYPE_CODES[kv_dtype], _DTYPE_CODES[q_dtype], _ptr(q),
                                     _ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale),
                                     _ptr(seq_offsets), _ptr(lens), b, hq, num_kv_heads, d,
                                     float(scale), _ptr(out), _ptr(weights), max_len)
    if rc != 0:
        raise ValueError("oracle_decode_attention: invalid arguments")
    return (out, weights) if return_weights else out


def multi_query_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, seq_offsets: np.ndarray,
                          lens: np.ndarray, scale: float, num_kv_heads: int, kv_dtype: str,
                          q_dtype: str, k_scale: np.ndarray | None = None,
                          v_scale: np.ndarray | None = None) -> np.ndarray:
    """Causal multi-query attention (C oracle): q [B][Q][Hq][D]; query token i of
    sequence b sees positions 0 .. L_b - Q + i.  Returns out [B][Q][Hq][D] float64."""
    lib = _load()
    b, nq, hq, d = q.shape
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    seq_offsets = np.ascontiguousarray(seq_offsets, dtype=np.int64)
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    if kv_dtype in QUANTIZED:
        k_scale = np.ascontiguousarray(k_scale, dtype=np.float32)
        v_scale = np.ascontiguousarray(v_scale, dtype=np.float32)
    out = np.empty((b, nq, hq, d), dtype=np.float64)
    rc = lib.oracle_multi_query_attention(_DTYPE_CODES[kv_dtype], _DTYPE_CODES[q_dtype], nq,
                                          _ptr(q), _ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale),
                                          _ptr(seq_offsets), _ptr(lens), b, hq, num_kv_heads, d,
                                          float(scale), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_multi_query_attention: invalid arguments")
    return out


def widen(x: np.ndarray, dtype: str, scales: np.ndarray | None = None) -> np.ndarray:
    """Stored values -> float64, exactly (bf16 bits shifted into binary32;
    E4M3 / INT8 codes decoded and multiplied by their row scale)."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32) \
            .astype(np.float64)
    if dtype == "int8":
        return np.asarray(x, dtype=np.int8).astype(np.float64) * \
            np.asarray(scales, dtype=np.float64)[..., None]
    if dtype == "int4":
        pz = np.asarray(scales, dtype=np.float64)
        return (np.asarray(x, dtype=np.uint8).astype(np.float64) - pz[..., 1:2]) * pz[..., 0:1]
    return e4m3_decode(x) * np.asarray(scales, dtype=np.float64)[..., None]


def decode_attention_bruteforce(q64: np.ndarray, k64: np.ndarray, v64: np.ndarray,
                                seq_offsets, lens, scale: float, num_kv_heads: int) -> np.ndarray:
    """numpy float64, one (sequence, query head) at a time, in the order of
    "KV Cache 深度解析" §六's step(): scores = q·Kᵀ·scale; subtract the max;
    exponentiate; divide by the sum; weight V.  For tiny inputs only."""
    b, hq, d = q64.shape
    group = hq // num_kv_heads
    out = np.zeros((b, hq, d))
    for s in range(b):
        t0, n = int(seq_offsets[s]), int(lens[s])
        for h in range(hq):
            kk = k64[t0:t0 + n, h // group, :]
            vv = v64[t0:t0 + n, h // group, :]
            scores = (kk @ q64[s, h]) * scale
            scores = scores - scores.max()
            attn = np.exp(scores) / np.exp(scores).sum()
            out[s, h] = attn @ vv
    return out


def decode_attention_split(q64: np.ndarray, k64: np.ndarray, v64: np.ndarray, seq_offsets,
                           lens, scale: float, num_kv_heads: int, partition_tokens: int,
                           tile_tokens: int = 16) -> np.ndarray:
    """Sequence-partitioned (split-K) decode in double.

    Inside a partition, tiles of ``tile_tokens`` keys are folded in with the
    blockwise online-softmax update of the "llm-inference-optimization" notes
    (§三 Flash Attention): running max m, running sum l, running output o,
        m' = max(m, max_t s_t);  l' = e^(m-m') l + sum_t e^(s_t-m');
        o' = e^(m-m') o + sum_t e^(s_t-m') V_t.
    Partitions are then merged by their log-sum-exp (the page's last line
    writes the log-sum-exp as l + log l, which is a misprint; the reading used
    is m + log l, equivalently the (m, l) pair):
        M = max_p m_p;  w_p = e^(m_p - M);  out = sum_p w_p o_p / sum_p w_p l_p.
    """
    b, hq, d = q64.shape
    group = hq // num_kv_heads
    out = np.zeros((b, hq, d))
    for s in range(b):
        t0, n = int(seq_offsets[s]), int(lens[s])
        for h in range(hq):
            kk = k64[t0:t0 + n, h // group, :]
            vv = v64[t0:t0 + n, h // group, :]
            parts = []
            for p0 in range(0, n, partition_tokens):
                p1 = min(p0 + partition_tokens, n)
                m, l, o = -math.inf, 0.0, np.zeros(d)
                for j in range(p0, p1, tile_tokens):
                    jj = min(j + tile_tokens, p1)
                    sc = (kk[j:jj] @ q64[s, h]) * scale
                    m_new = max(m, float(sc.max()))
                    c = math.exp(m - m_new) if m != -math.inf else 0.0
                    p = np.exp(sc - m_new)
                    l = c * l + p.sum()
                    o = c * o + p @ vv[j:jj]
                    m = m_new
                parts.append((m, l, o))
            big_m = max(pm for pm, _, _ in parts)
            num = sum(math.exp(pm - big_m) * po for pm, _, po in parts)
            den = sum(math.exp(pm - big_m) * pl for pm, pl, _ in parts)
            out[s, h] = num / den
    return out
