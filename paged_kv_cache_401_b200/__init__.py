"""Python binding of libpagedkv.so: paged GQA decode attention on B200.

Argument marshalling only.  Every step of the decode path (slot computation,
cache write, split-K decode, log-sum-exp merge, FP8 quantise/dequantise) runs
in the library's CUDA kernels; PyTorch supplies device memory and streams.
The functions carry the C ABI's names (include/paged_kv.h) and raise
``KvError`` on a non-OK status.  There is no fallback: if the compiled
library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpagedkv.so")

KV_F32, KV_BF16, KV_FP8_E4M3, KV_INT8, KV_INT4, KV_KIVI4 = 0, 1, 2, 3, 4, 5
# pools of codes with parameters: fp32 scales (8-bit), (scale, zero) pairs (4-bit)
QUANTIZED = (KV_FP8_E4M3, KV_INT8, KV_INT4, KV_KIVI4)
KV_OK, KV_ERR_INVALID_ARGUMENT, KV_ERR_UNSUPPORTED, KV_ERR_CUDA = 0, 1, 2, 3
KV_ERR_OUT_OF_BLOCKS = 4
KV_DEVERR_BAD_SLOT = 0x1
KV_DEVERR_BAD_CONTEXT_LEN = 0x2
KV_DEVERR_BAD_BLOCK_ID = 0x4
KV_DEVERR_TIMEOUT = 0x8
KV_DEVERR_BAD_POSITION = 0x10
BLOCK_SIZE = 16

EXPORTED = ("kv_pool_create", "compute_slot_mapping", "reshape_and_cache",
            "paged_decode_num_ranges", "paged_decode_workspace_bytes",
            "paged_decode_attention", "paged_decode_attention_static_workspace",
            "paged_decode_attention_append", "kivi_quantize_blocks", "kivi_decode_attention",
            "paged_attention_workspace_bytes", "paged_attention_multi_query",
            "paged_kv_copy_blocks", "kv_block_manager_create", "kv_block_manager_destroy",
            "kv_block_manager_num_free_blocks", "kv_block_manager_refcount",
            "kv_block_manager_add_sequence", "kv_block_manager_fork",
            "kv_block_manager_free_sequence", "kv_block_manager_append_slots",
            "kv_block_manager_export", "kv_status_string")
KV_STATIC_WORKSPACE_BYTES = 16 * 1024 * 1024


class KvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {kv_status_string(status)} ({status})")
        self.status = status


class KvPoolDesc(ctypes.Structure):
    """Mirror of kv_pool_desc (plain data; owns nothing)."""
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("elem_bytes", ctypes.c_int32),
                ("kv_bytes", ctypes.c_uint64), ("scale_bytes", ctypes.c_uint64),
                ("stride_block", ctypes.c_int64), ("stride_head", ctypes.c_int64),
                ("stride_slot", ctypes.c_int64)]


_lib = None
_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


def _load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m paged_kv_cache_401_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        desc_p = ctypes.POINTER(KvPoolDesc)
        sig = {
            "kv_pool_create": (_I32, [_I32, _I32, _I32, _I32, _I32, desc_p]),
            "compute_slot_mapping": (_I32, [_P, _I32, _I32, _I32, _P, _P, _I32, _P, _P, _P]),
            "reshape_and_cache": (_I32, [desc_p, _P, _P, _P, _P, _P, _I32, _P, _I32, _P, _P]),
            "paged_decode_num_ranges": (_I32, [desc_p, _I32, _I32, _I32, _I32]),
            "paged_decode_workspace_bytes": (_SZ, [desc_p, _I32, _I32, _I32, _I32]),
            "paged_decode_attention": (_I32, [desc_p, _P, _P, _I32, _P, _P, _P, _P, _I32, _P,
                                              _I32, _I32, _I32, ctypes.c_float, _I32, _P, _SZ,
                                              _P, _P]),
            "paged_decode_attention_append": (_I32, [desc_p, _P, _P, _I32, _P, _P, _P, _P, _P,
                                                     _I32, _P, _I32, _P, _I32, _I32, _I32,
                                                     ctypes.c_float, _I32, _P, _SZ, _P, _P]),
            "kivi_quantize_blocks": (_I32, [desc_p, _P, _P, _P, _P, _P, _I32, _P, _I32, _P, _P]),
            "kivi_decode_attention": (_I32, [desc_p, _P, _P, _I32, _P, _P, _P, _P, _P, _P, _P, _P,
                                             _I32, _P, _I32, _I32, _I32, ctypes.c_float, _I32,
                                             _P, _SZ, _P, _P]),
            "paged_decode_attention_static_workspace": (
                _I32, [desc_p, _P, _P, _I32, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32,
                       ctypes.c_float, _I32, _P, _P]),
            "paged_attention_workspace_bytes": (_SZ, [desc_p, _I32, _I32, _I32, _I32, _I32]),
            "paged_attention_multi_query": (_I32, [desc_p, _P, _P, _I32, _I32, _P, _P, _P, _P,
                                                   _I32, _P, _I32, _I32, _I32, ctypes.c_float,
                                                   _I32, _P, _SZ, _P, _P]),
            "paged_kv_copy_blocks": (_I32, [desc_p, _P, _P, _P, _P, _P, _I32, _P, _P]),
            "kv_block_manager_create": (_I32, [_I32, _I32, _I32, _P]),
            "kv_block_manager_destroy": (None, [_P]),
            "kv_block_manager_num_free_blocks": (_I32, [_P]),
            "kv_block_manager_refcount": (_I32, [_P, _I32]),
            "kv_block_manager_add_sequence": (_I32, [_P, _P]),
            "kv_block_manager_fork": (_I32, [_P, _I32, _P]),
            "kv_block_manager_free_sequence": (_I32, [_P, _I32]),
            "kv_block_manager_append_slots": (_I32, [_P, _P, _I32, _P, _P, _P, _P]),
            "kv_block_manager_export": (_I32, [_P, _P, _P]),
            "kv_status_string": (ctypes.c_char_p, [_I32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


def library() -> ctypes.CDLL:
    """The loaded libpagedkv.so (raises if it has not been built)."""
    return _load()


def kv_dtype_of(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KV_F32
    if t.dtype == torch.bfloat16:
        return KV_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return KV_FP8_E4M3
    if t.dtype == torch.int8:
        return KV_INT8
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libpagedkv must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, status: int) -> None:
    if status != KV_OK:
        raise KvError(fn, status)


def kv_status_string(status: int) -> str:
    return _load().kv_status_string(int(status)).decode()


def kv_pool_create(num_blocks: int, block_size: int, num_kv_heads: int, head_dim: int,
                   dtype: int) -> KvPoolDesc:
    desc = KvPoolDesc()
    _check("kv_pool_create", _load().kv_pool_create(num_blocks, block_size, num_kv_heads,
                                                    head_dim, dtype, ctypes.byref(desc)))
    return desc


def empty_pool(desc: KvPoolDesc, device, fill: float | int | None = None):
    """Allocate (k_pool, v_pool, scales) tensors for a descriptor: pools
    [num_blocks][kv_heads][16][head_dim] (INT4: [..][head_dim / 2] bytes, two
    codes each); scales [num_blocks][kv_heads][2][16] fp32 (K then V row
    scales) for FP8 / INT8, [num_blocks][kv_heads][2][16][2] (scale, zero) for
    INT4, else None.  ``fill`` poisons every element (NaN, or a byte; scales
    get NaN)."""
    four_bit = desc.dtype in (KV_INT4, KV_KIVI4)
    cols = desc.head_dim // 2 if four_bit else desc.head_dim
    shape = (desc.num_blocks, desc.num_kv_heads, desc.block_size, cols)
    dt = {KV_F32: torch.float32, KV_BF16: torch.bfloat16, KV_FP8_E4M3: torch.uint8,
          KV_INT8: torch.int8, KV_INT4: torch.uint8, KV_KIVI4: torch.uint8}[desc.dtype]
    k = torch.empty(shape, dtype=dt, device=device)
    v = torch.empty(shape, dtype=dt, device=device)
    scales = None
    if desc.dtype == KV_KIVI4:    # (scale, zero) of 128 key channels, then of 16 value rows
        scales = torch.empty((desc.num_blocks, desc.num_kv_heads, desc.head_dim + desc.block_size,
                              2), dtype=torch.float32, device=device)
    elif desc.dtype in QUANTIZED:
        extra = (2,) if desc.dtype == KV_INT4 else ()
        scales = torch.empty((desc.num_blocks, desc.num_kv_heads, 2, desc.block_size) + extra,
                             dtype=torch.float32, device=device)
    if fill is not None:
        for t in (k, v):
            t.fill_(fill)
        if scales is not None:
            scales.fill_(float("nan"))
    return k, v, scales


def compute_slot_mapping(block_table: torch.Tensor, seq_ids: torch.Tensor,
                         positions: torch.Tensor, slot_mapping: torch.Tensor,
                         block_size: int = BLOCK_SIZE, dev_error: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    batch, max_blocks = block_table.shape
    _check("compute_slot_mapping", _load().compute_slot_mapping(
        _ptr(block_table), batch, max_blocks, block_size, _ptr(seq_ids), _ptr(positions),
        seq_ids.numel(), _ptr(slot_mapping), _ptr(dev_error), _stream(stream)))
    return slot_mapping


def reshape_and_cache(pool: KvPoolDesc, k_pool: torch.Tensor, v_pool: torch.Tensor,
                      scales: torch.Tensor | None, k_new: torch.Tensor, v_new: torch.Tensor,
                      slot_mapping: torch.Tensor, dev_error: torch.Tensor | None = None,
                      stream=None) -> None:
    _check("reshape_and_cache", _load().reshape_and_cache(
        ctypes.byref(pool), _ptr(k_pool), _ptr(v_pool), _ptr(scales),
        _ptr(k_new), _ptr(v_new), kv_dtype_of(k_new), _ptr(slot_mapping), k_new.shape[0],
        _ptr(dev_error), _stream(stream)))


def paged_decode_num_ranges(pool: KvPoolDesc, batch: int, num_q_heads: int,
                            max_context_len: int, partition_tokens: int = 0) -> int:
    return int(_load().paged_decode_num_ranges(ctypes.byref(pool), batch, num_q_heads,
                                               max_context_len, partition_tokens))


def paged_decode_workspace_bytes(pool: KvPoolDesc, batch: int, num_q_heads: int,
                                 max_context_len: int, partition_tokens: int = 0) -> int:
    return int(_load().paged_decode_workspace_bytes(ctypes.byref(pool), batch, num_q_heads,
                                                    max_context_len, partition_tokens))


def paged_decode_attention(pool: KvPoolDesc, out: torch.Tensor, q: torch.Tensor,
                           k_pool: torch.Tensor, v_pool: torch.Tensor,
                           scales: torch.Tensor | None,
                           block_table: torch.Tensor, context_lens: torch.Tensor,
                           max_context_len: int, scale: float, partition_tokens: int = 0,
                           workspace: torch.Tensor | None = None,
                           dev_error: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    batch, num_q_heads, _ = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("paged_decode_attention", _load().paged_decode_attention(
        ctypes.byref(pool), _ptr(out), _ptr(q), kv_dtype_of(q), _ptr(k_pool), _ptr(v_pool),
        _ptr(scales), _ptr(block_table), block_table.shape[1],
        _ptr(context_lens), batch, num_q_heads, max_context_len, float(scale),
        partition_tokens, _ptr(workspace), ws_bytes, _ptr(dev_error), _stream(stream)))
    return out


def paged_decode_attention_append(pool: KvPoolDesc, out: torch.Tensor, q: torch.Tensor,
                                  k_pool: torch.Tensor, v_pool: torch.Tensor,
                                  scales: torch.Tensor | None, k_new: torch.Tensor,
                                  v_new: torch.Tensor, block_table: torch.Tensor,
                                  context_lens: torch.Tensor, max_context_len: int, scale: float,
                                  partition_tokens: int = 0,
                                  workspace: torch.Tensor | None = None,
                                  dev_error: torch.Tensor | None = None,
                                  stream=None) -> torch.Tensor:
    """One decode step in one call: k_new/v_new [batch][kv_heads][head_dim] are
    stored at position context_lens[b] - 1 of each sequence (as reshape_and_cache
    would) and attended to along with the rest of the context."""
    batch, num_q_heads, _ = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("paged_decode_attention_append", _load().paged_decode_attention_append(
        ctypes.byref(pool), _ptr(out), _ptr(q), kv_dtype_of(q), _ptr(k_pool), _ptr(v_pool),
        _ptr(scales), _ptr(k_new), _ptr(v_new), kv_dtype_of(k_new), _ptr(block_table),
        block_table.shape[1], _ptr(context_lens), batch, num_q_heads, max_context_len,
        float(scale), partition_tokens, _ptr(workspace), ws_bytes, _ptr(dev_error),
        _stream(stream)))
    return out


def empty_residual(desc: KvPoolDesc, batch: int, device, fill: float | None = None):
    """(res_k, res_v) bf16 [batch][kv_heads][16][head_dim]: a KIVI cache's newest
    L mod 16 tokens per sequence, kept unquantised."""
    shape = (batch, desc.num_kv_heads, desc.block_size, desc.head_dim)
    res = [torch.empty(shape, dtype=torch.bfloat16, device=device) for _ in range(2)]
    if fill is not None:
        for t in res:
            t.fill_(fill)
    return res[0], res[1]


def kivi_quantize_blocks(pool: KvPoolDesc, k_pool: torch.Tensor, v_pool: torch.Tensor,
                         params: torch.Tensor, k_rows: torch.Tensor, v_rows: torch.Tensor,
                         block_ids: torch.Tensor, dev_error: torch.Tensor | None = None,
                         stream=None) -> None:
    """k_rows, v_rows: [n][16][kv_heads][head_dim] (fp32 or bf16), full blocks that
    go to block_ids [n] of a KIVI pool."""
    _check("kivi_quantize_blocks", _load().kivi_quantize_blocks(
        ctypes.byref(pool), _ptr(k_pool), _ptr(v_pool), _ptr(params), _ptr(k_rows),
        _ptr(v_rows), kv_dtype_of(k_rows), _ptr(block_ids), block_ids.numel(), _ptr(dev_error),
        _stream(stream)))


def kivi_decode_attention(pool: KvPoolDesc, out: torch.Tensor, q: torch.Tensor,
                          k_pool: torch.Tensor, v_pool: torch.Tensor, params: torch.Tensor,
                          res_k: torch.Tensor, res_v: torch.Tensor,
                          k_new: torch.Tensor | None, v_new: torch.Tensor | None,
                          block_table: torch.Tensor, context_lens: torch.Tensor,
                          max_context_len: int, scale: float, partition_tokens: int = 0,
                          workspace: torch.Tensor | None = None,
                          dev_error: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """A decode step over a KIVI pool; k_new/v_new (bf16 [batch][kv_heads][head_dim])
    are appended at position context_lens[b] - 1 first (None: no append)."""
    batch, num_q_heads, _ = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kivi_decode_attention", _load().kivi_decode_attention(
        ctypes.byref(pool), _ptr(out), _ptr(q), kv_dtype_of(q), _ptr(k_pool), _ptr(v_pool),
        _ptr(params), _ptr(res_k), _ptr(res_v), _ptr(k_new), _ptr(v_new), _ptr(block_table),
        block_table.shape[1], _ptr(context_lens), batch, num_q_heads, max_context_len,
        float(scale), partition_tokens, _ptr(workspace), ws_bytes, _ptr(dev_error),
        _stream(stream)))
    return out


def paged_decode_attention_static_workspace(
        pool: KvPoolDesc, out: torch.Tensor, q: torch.Tensor, k_pool: torch.Tensor,
        v_pool: torch.Tensor, scales: torch.Tensor | None,
        block_table: torch.Tensor, context_lens: torch.Tensor, max_context_len: int,
        scale: float, partition_tokens: int = 0, dev_error: torch.Tensor | None = None,
        stream=None) -> torch.Tensor:
    """paged_decode_attention without a caller workspace (for callers that cannot
    allocate device memory): the partials live in the library's fixed
    KV_STATIC_WORKSPACE_BYTES device array, shared by every call on the device."""
    batch, num_q_heads, _ = q.shape
    _check("paged_decode_attention_static_workspace",
           _load().paged_decode_attention_static_workspace(
               ctypes.byref(pool), _ptr(out), _ptr(q), kv_dtype_of(q), _ptr(k_pool),
               _ptr(v_pool), _ptr(scales), _ptr(block_table),
               block_table.shape[1], _ptr(context_lens), batch, num_q_heads, max_context_len,
               float(scale), partition_tokens, _ptr(dev_error), _stream(stream)))
    return out


def paged_attention_workspace_bytes(pool: KvPoolDesc, batch: int, num_q_heads: int,
                                    num_query_tokens: int, max_context_len: int,
                                    partition_tokens: int = 0) -> int:
    return int(_load().paged_attention_workspace_bytes(ctypes.byref(pool), batch, num_q_heads,
                                                       num_query_tokens, max_context_len,
                                                       partition_tokens))


def paged_attention_multi_query(pool: KvPoolDesc, out: torch.Tensor, q: torch.Tensor,
                                k_pool: torch.Tensor, v_pool: torch.Tensor,
                                scales: torch.Tensor | None, block_table: torch.Tensor,
                                context_lens: torch.Tensor, max_context_len: int, scale: float,
                                partition_tokens: int = 0, workspace: torch.Tensor | None = None,
                                dev_error: torch.Tensor | None = None,
                                stream=None) -> torch.Tensor:
    """q, out: [batch][num_query_tokens][num_q_heads][head_dim]."""
    batch, nq, num_q_heads, _ = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("paged_attention_multi_query", _load().paged_attention_multi_query(
        ctypes.byref(pool), _ptr(out), _ptr(q), kv_dtype_of(q), nq, _ptr(k_pool), _ptr(v_pool),
        _ptr(scales), _ptr(block_table), block_table.shape[1], _ptr(context_lens), batch,
        num_q_heads, max_context_len, float(scale), partition_tokens, _ptr(workspace), ws_bytes,
        _ptr(dev_error), _stream(stream)))
    return out


# ---------------------------------------------------------------- block manager
def paged_kv_copy_blocks(pool: KvPoolDesc, k_pool: torch.Tensor, v_pool: torch.Tensor,
                         scales: torch.Tensor | None, copy_src: torch.Tensor,
                         copy_dst: torch.Tensor, dev_error: torch.Tensor | None = None,
                         stream=None) -> None:
    _check("paged_kv_copy_blocks", _load().paged_kv_copy_blocks(
        ctypes.byref(pool), _ptr(k_pool), _ptr(v_pool), _ptr(scales), _ptr(copy_src),
        _ptr(copy_dst), copy_src.numel(), _ptr(dev_error), _stream(stream)))


class BlockManager:
    """Host block manager (kv_block_manager_* in include/paged_kv.h)."""

    def __init__(self, num_blocks: int, max_seqs: int, max_blocks_per_seq: int):
        lib = _load()
        self.num_blocks, self.max_seqs, self.max_blocks_per_seq = (num_blocks, max_seqs,
                                                                   max_blocks_per_seq)
        self._h = ctypes.c_void_p()
        _check("kv_block_manager_create", lib.kv_block_manager_create(
            num_blocks, max_seqs, max_blocks_per_seq, ctypes.byref(self._h)))

    def __del__(self):
        if getattr(self, "_h", None) and self._h.value and _lib is not None:
            _lib.kv_block_manager_destroy(self._h)
            self._h = ctypes.c_void_p()

    @property
    def num_free_blocks(self) -> int:
        return int(_load().kv_block_manager_num_free_blocks(self._h))

    def refcount(self, block: int) -> int:
        return int(_load().kv_block_manager_refcount(self._h, block))

    def add_sequence(self) -> int:
        s = ctypes.c_int32()
        _check("kv_block_manager_add_sequence",
               _load().kv_block_manager_add_sequence(self._h, ctypes.byref(s)))
        return s.value

    def fork(self, parent: int) -> int:
        c = ctypes.c_int32()
        _check("kv_block_manager_fork", _load().kv_block_manager_fork(self._h, parent,
                                                                       ctypes.byref(c)))
        return c.value

    def free_sequence(self, seq: int) -> None:
        _check("kv_block_manager_free_sequence", _load().kv_block_manager_free_sequence(self._h,
                                                                                         seq))

    def append_slots(self, seq_ids):
        """-> (slots int64 [n], copies [(src, dst), ...]) as numpy / list."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        n = ids.size
        slots = np.empty(n, dtype=np.int64)
        src = np.empty(max(n, 1), dtype=np.int32)
        dst = np.empty(max(n, 1), dtype=np.int32)
        nc = ctypes.c_int32()
        _check("kv_block_manager_append_slots", _load().kv_block_manager_append_slots(
            self._h, ids.ctypes.data, n, slots.ctypes.data, src.ctypes.data, dst.ctypes.data,
            ctypes.byref(nc)))
        return slots, list(zip(src[:nc.value].tolist(), dst[:nc.value].tolist()))

    def export(self):
        """-> (block_table int32 [max_seqs][max_blocks_per_seq], context_lens int32 [max_seqs])."""
        import numpy as np
        table = np.empty((self.max_seqs, self.max_blocks_per_seq), dtype=np.int32)
        lens = np.empty(self.max_seqs, dtype=np.int32)
        _check("kv_block_manager_export", _load().kv_block_manager_export(
            self._h, table.ctypes.data, lens.ctypes.data))
        return table, lens
