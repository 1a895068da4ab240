"""Host-side checks of libpagedkv.so that need no GPU.

The library loads, exports every entry point include/paged_kv.h declares, and
its host logic (geometry, argument validation, workspace sizing, the split
into consumer ranges) behaves as documented.  No call here enqueues device work: every
call is rejected on the host before any launch, or is host-only.
"""
import ctypes
import os
import re

import pytest

import paged_kv_cache_401_b200 as pk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "paged_kv.h")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_401_b200 import build
    build.build()


def _declared():
    text = open(HEADER, encoding="utf-8").read()
    return re.findall(r"KV_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_binding_names():
    assert sorted(_declared()) == sorted(pk.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(pk.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {pk.LIB_PATH}").read().split("\n")
    text_syms = {ln.split()[-1] for ln in out if " T " in ln}
    assert text_syms == set(_declared())


def test_status_strings():
    assert pk.kv_status_string(0) == "KV_OK"
    assert pk.kv_status_string(3) == "KV_ERR_CUDA"
    assert pk.kv_status_string(99) == "KV_STATUS_UNKNOWN"


def test_pool_geometry_llama_shape():
    d = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_BF16)
    assert (d.stride_slot, d.stride_head, d.stride_block) == (128, 16 * 128, 8 * 16 * 128)
    assert d.kv_bytes == 8192 * 8 * 16 * 128 * 2 == 256 * 2**20
    assert d.scale_bytes == 0 and d.elem_bytes == 2
    f = pk.kv_pool_create(100, 16, 8, 64, pk.KV_FP8_E4M3)
    assert f.kv_bytes == 100 * 8 * 16 * 64 and f.scale_bytes == 100 * 8 * 2 * 16 * 4
    i = pk.kv_pool_create(100, 16, 8, 64, pk.KV_INT8)
    assert (i.kv_bytes, i.scale_bytes, i.elem_bytes) == (f.kv_bytes, f.scale_bytes, 1)
    n = pk.kv_pool_create(100, 16, 8, 128, pk.KV_INT4)      # 64-byte rows, (scale, zero) pairs
    assert (n.kv_bytes, n.scale_bytes, n.elem_bytes) == (100 * 8 * 16 * 64, 100 * 8 * 2 * 16 * 8, 0)
    assert n.stride_slot == 128                              # strides count codes


@pytest.mark.parametrize("args,status", [
    ((0, 16, 8, 128, pk.KV_BF16), pk.KV_ERR_INVALID_ARGUMENT),
    ((10, 32, 8, 128, pk.KV_BF16), pk.KV_ERR_UNSUPPORTED),
    ((10, 16, 8, 96, pk.KV_BF16), pk.KV_ERR_UNSUPPORTED),
    ((10, 16, 8, 128, 7), pk.KV_ERR_UNSUPPORTED),
    ((10, 16, 8, 64, pk.KV_INT4), pk.KV_ERR_UNSUPPORTED),        # 4-bit: head_dim 128 only
    ((10, 16, 0, 128, pk.KV_BF16), pk.KV_ERR_INVALID_ARGUMENT),
])
def test_pool_create_rejects(args, status):
    with pytest.raises(pk.KvError) as e:
        pk.kv_pool_create(*args)
    assert e.value.status == status


def test_workspace_bytes_and_ranges():
    d = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_BF16)
    # balanced default: one range per consumer warp of 3 CTAs x 4 warps on each of 148 SMs
    assert pk.paged_decode_num_ranges(d, 32, 32, 4096, 0) == 148 * 3 * 4
    # the range count does not depend on the group size or q dtype (the workspace
    # size must not either); group-8 fp32 kernels, one CTA per SM, run it in waves
    assert pk.paged_decode_num_ranges(d, 32, 64, 4096, 0) == 148 * 3 * 4
    # explicit partition: ranges of at most 512 tokens over 32 x 8 x 256 tiles
    assert pk.paged_decode_num_ranges(d, 32, 32, 4096, 512) == 32 * 8 * 256 // 32
    assert pk.paged_decode_num_ranges(d, 32, 32, 4096, 500) == 0
    # one-block partitions: one range per tile, more than the 65535 ranges the kernels'
    # 32-bit range arithmetic covers (they switch to 64-bit there)
    assert pk.paged_decode_num_ranges(d, 32, 32, 4096, 16) == 32 * 8 * 256
    ranges = 148 * 12
    pieces = 32 * 8 + ranges
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    want = up(4 * 33) + up(pieces * 4 * 8) + pieces * 4 * 128 * 4
    assert pk.paged_decode_workspace_bytes(d, 32, 32, 4096, 0) == want
    assert pk.paged_decode_workspace_bytes(d, 32, 30, 4096, 0) == 0


def _call_decode(desc, **kw):
    lib = pk.library()
    args = dict(out=4096, q=8192, q_dtype=pk.KV_BF16, k_pool=1 << 20, v_pool=2 << 20,
                scales=None, block_table=3 << 20, max_blocks=256,
                context_lens=4 << 20, batch=32, num_q_heads=32, max_context_len=4096,
                scale=0.088, partition=512, workspace=5 << 20, workspace_bytes=1 << 30,
                dev_error=None, stream=None)
    args.update(kw)
    return lib.paged_decode_attention(
        ctypes.byref(desc), args["out"], args["q"], args["q_dtype"], args["k_pool"],
        args["v_pool"], args["scales"], args["block_table"],
        args["max_blocks"], args["context_lens"], args["batch"], args["num_q_heads"],
        args["max_context_len"], args["scale"], args["partition"], args["workspace"],
        args["workspace_bytes"], args["dev_error"], args["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(num_q_heads=24), pk.KV_ERR_UNSUPPORTED),                 # group 3
    (dict(num_q_heads=30), pk.KV_ERR_INVALID_ARGUMENT),            # not a multiple of Hkv
    (dict(num_q_heads=128), pk.KV_ERR_UNSUPPORTED),                # group 16
    (dict(q_dtype=pk.KV_FP8_E4M3), pk.KV_ERR_UNSUPPORTED),
    (dict(q_dtype=pk.KV_INT8), pk.KV_ERR_UNSUPPORTED),
    (dict(max_context_len=4097), pk.KV_ERR_INVALID_ARGUMENT),      # beyond the table
    (dict(max_context_len=0), pk.KV_ERR_INVALID_ARGUMENT),
    (dict(partition=500), pk.KV_ERR_INVALID_ARGUMENT),             # not a multiple of 16
    (dict(max_blocks=1 << 24, max_context_len=1 << 28, batch=2048),
     pk.KV_ERR_UNSUPPORTED),                                        # tile list >= 2^31
    (dict(q=8192 + 8), pk.KV_ERR_INVALID_ARGUMENT),                # misaligned
    (dict(k_pool=None), pk.KV_ERR_INVALID_ARGUMENT),
    (dict(scales=6 << 20), pk.KV_ERR_INVALID_ARGUMENT),            # scales on a bf16 pool
    (dict(workspace_bytes=100), pk.KV_ERR_INVALID_ARGUMENT),       # too small
    (dict(workspace=None), pk.KV_ERR_INVALID_ARGUMENT),
    (dict(scale=float("nan")), pk.KV_ERR_INVALID_ARGUMENT),
])
def test_decode_host_validation(kw, status):
    d = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_BF16)
    assert _call_decode(d, **kw) == status


def _call_append(desc, **kw):
    lib = pk.library()
    args = dict(out=4096, q=8192, q_dtype=pk.KV_BF16, k_pool=1 << 20, v_pool=2 << 20,
                scales=None, k_new=7 << 20, v_new=8 << 20, src_dtype=pk.KV_BF16,
                block_table=3 << 20, max_blocks=256, context_lens=4 << 20, batch=32,
                num_q_heads=32, max_context_len=4096, scale=0.088, partition=512,
                workspace=5 << 20, workspace_bytes=1 << 30, dev_error=None, stream=None)
    args.update(kw)
    return lib.paged_decode_attention_append(
        ctypes.byref(desc), args["out"], args["q"], args["q_dtype"], args["k_pool"],
        args["v_pool"], args["scales"], args["k_new"], args["v_new"], args["src_dtype"],
        args["block_table"], args["max_blocks"], args["context_lens"], args["batch"],
        args["num_q_heads"], args["max_context_len"], args["scale"], args["partition"],
        args["workspace"], args["workspace_bytes"], args["dev_error"], args["stream"])


@pytest.mark.parametrize("pool,kw,status", [
    (pk.KV_BF16, dict(src_dtype=pk.KV_F32), pk.KV_ERR_UNSUPPORTED),      # no conversion
    (pk.KV_BF16, dict(k_new=None), pk.KV_ERR_INVALID_ARGUMENT),
    (pk.KV_BF16, dict(v_new=(8 << 20) + 4), pk.KV_ERR_INVALID_ARGUMENT),  # misaligned
    (pk.KV_BF16, dict(num_q_heads=24), pk.KV_ERR_UNSUPPORTED),          # as the decode
    (pk.KV_FP8_E4M3, dict(scales=6 << 20, src_dtype=pk.KV_INT8), pk.KV_ERR_UNSUPPORTED),
    (pk.KV_INT8, dict(scales=6 << 20, src_dtype=pk.KV_FP8_E4M3), pk.KV_ERR_UNSUPPORTED),
    (pk.KV_INT8, dict(src_dtype=pk.KV_F32), pk.KV_ERR_INVALID_ARGUMENT),  # needs scales
])
def test_decode_append_host_validation(pool, kw, status):
    d = pk.kv_pool_create(8192, 16, 8, 128, pool)
    assert _call_append(d, **kw) == status


def test_decode_int4_needs_the_tensor_core_shape():
    d = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_INT4)
    assert _call_decode(d, q_dtype=pk.KV_F32, scales=6 << 20) == pk.KV_ERR_UNSUPPORTED


@pytest.mark.parametrize("which", ["k_pool", "v_pool"])
def test_decode_4bit_pools_need_32_byte_alignment(which):
    # 4-bit pools are copied as 4-bit elements padded in shared memory, which needs
    # 32-byte aligned sources: a 16-byte aligned pool is refused on the host
    d = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_INT4)
    base = {"k_pool": 1 << 20, "v_pool": 2 << 20}[which]
    assert _call_decode(d, scales=6 << 20, **{which: base + 16}) == pk.KV_ERR_INVALID_ARGUMENT
    dk = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_KIVI4)
    lib = pk.library()
    ptrs = dict(k_pool=1 << 20, v_pool=2 << 20)
    ptrs[which] += 16
    status = lib.kivi_decode_attention(
        ctypes.byref(dk), 4096, 8192, pk.KV_BF16, ptrs["k_pool"], ptrs["v_pool"], 6 << 20,
        9 << 20, 10 << 20, None, None, 3 << 20, 256, 4 << 20, 32, 32, 4096, 0.088, 0,
        5 << 20, 1 << 30, None, None)
    assert status == pk.KV_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("dtype", [pk.KV_FP8_E4M3, pk.KV_INT8, pk.KV_INT4])
def test_decode_quantized_pool_requires_scales(dtype):
    d = pk.kv_pool_create(8192, 16, 8, 128, dtype)
    assert _call_decode(d) == pk.KV_ERR_INVALID_ARGUMENT
    assert _call_decode(d, scales=(6 << 20) + 4) == pk.KV_ERR_INVALID_ARGUMENT  # misaligned


def test_decode_needs_a_workspace_even_for_one_range():
    d = pk.kv_pool_create(64, 16, 1, 64, pk.KV_F32)
    assert _call_decode(d, q_dtype=pk.KV_F32, batch=1, num_q_heads=4, max_blocks=4,
                        max_context_len=20, workspace=None) == pk.KV_ERR_INVALID_ARGUMENT


def test_decode_empty_batch_is_a_no_op():
    d = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_BF16)
    assert _call_decode(d, batch=0) == pk.KV_OK


def test_cache_write_host_validation():
    lib = pk.library()
    d = pk.kv_pool_create(64, 16, 8, 128, pk.KV_BF16)
    f = pk.kv_pool_create(64, 16, 8, 128, pk.KV_FP8_E4M3)
    ok = dict(kp=1 << 20, vp=2 << 20, sc=None, kn=3 << 20, vn=4 << 20,
              src=pk.KV_BF16, slots=5 << 20, n=4)

    def call(desc, **kw):
        a = dict(ok)
        a.update(kw)
        return lib.reshape_and_cache(ctypes.byref(desc), a["kp"], a["vp"], a["sc"], a["kn"],
                                     a["vn"], a["src"], a["slots"], a["n"], None, None)

    assert call(d, n=0) == pk.KV_OK                                   # nothing to do
    assert call(d, src=pk.KV_F32) == pk.KV_ERR_UNSUPPORTED            # no conversion on copy
    assert call(d, kn=(3 << 20) + 4) == pk.KV_ERR_INVALID_ARGUMENT    # misaligned
    assert call(d, sc=6 << 20) == pk.KV_ERR_INVALID_ARGUMENT          # scales on a bf16 pool
    assert call(d, n=-1) == pk.KV_ERR_INVALID_ARGUMENT
    assert call(f) == pk.KV_ERR_INVALID_ARGUMENT                      # fp8 needs scales
    assert call(f, sc=6 << 20, src=pk.KV_FP8_E4M3) == pk.KV_ERR_UNSUPPORTED
    i = pk.kv_pool_create(64, 16, 8, 128, pk.KV_INT8)
    assert call(i) == pk.KV_ERR_INVALID_ARGUMENT                      # int8 needs scales
    assert call(i, sc=6 << 20, src=pk.KV_INT8) == pk.KV_ERR_UNSUPPORTED


def test_slot_mapping_host_validation():
    lib = pk.library()
    assert lib.compute_slot_mapping(1 << 20, 2, 4, 16, 2 << 20, 3 << 20, 0, 4 << 20, None,
                                    None) == pk.KV_OK
    assert lib.compute_slot_mapping(1 << 20, 2, 4, 32, 2 << 20, 3 << 20, 5, 4 << 20, None,
                                    None) == pk.KV_ERR_UNSUPPORTED
    assert lib.compute_slot_mapping(None, 2, 4, 16, 2 << 20, 3 << 20, 5, 4 << 20, None,
                                    None) == pk.KV_ERR_INVALID_ARGUMENT


def _call_mq(desc, q_tokens, **kw):
    lib = pk.library()
    a = dict(out=4096, q=8192, q_dtype=pk.KV_BF16, k_pool=1 << 20, v_pool=2 << 20, scales=None,
             block_table=3 << 20, max_blocks=256, context_lens=4 << 20, batch=4, num_q_heads=32,
             max_context_len=4096, scale=0.088, partition=0, workspace=None, workspace_bytes=0)
    a.update(kw)
    return lib.paged_attention_multi_query(
        ctypes.byref(desc), a["out"], a["q"], a["q_dtype"], q_tokens, a["k_pool"], a["v_pool"],
        a["scales"], a["block_table"], a["max_blocks"], a["context_lens"], a["batch"],
        a["num_q_heads"], a["max_context_len"], a["scale"], a["partition"], a["workspace"],
        a["workspace_bytes"], None, None)


def test_multi_query_host_validation():
    bf = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_BF16)
    f32 = pk.kv_pool_create(8192, 16, 8, 128, pk.KV_F32)
    d64 = pk.kv_pool_create(8192, 16, 8, 64, pk.KV_BF16)
    assert _call_mq(bf, 5) == pk.KV_ERR_UNSUPPORTED                  # 4 heads x 5 tokens > 16
    assert _call_mq(f32, 2) == pk.KV_ERR_UNSUPPORTED                 # fp32 KV: one token only
    assert _call_mq(d64, 2) == pk.KV_ERR_UNSUPPORTED                 # head_dim 64: one token only
    assert _call_mq(bf, 2, q_dtype=pk.KV_F32) == pk.KV_ERR_UNSUPPORTED
    assert _call_mq(bf, 0) == pk.KV_ERR_INVALID_ARGUMENT
    assert _call_mq(bf, 4, max_context_len=3) == pk.KV_ERR_INVALID_ARGUMENT
    assert _call_mq(bf, 4) == pk.KV_ERR_INVALID_ARGUMENT             # no workspace
    # one query token is the decode; 4 heads x 4 tokens = 16 rows per kv head run
    # 2 CTAs per SM (the wide tile), so 148 * 2 * 4 ranges
    w1 = pk.paged_attention_workspace_bytes(bf, 32, 32, 1, 4096, 0)
    assert w1 == pk.paged_decode_workspace_bytes(bf, 32, 32, 4096, 0)
    assert pk.paged_decode_num_ranges(bf, 32, 32, 4096, 0) == 148 * 3 * 4
    pieces, rows = 32 * 8 + 148 * 2 * 4, 16
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    want = up(4 * 33) + up(pieces * rows * 8) + pieces * rows * 128 * 4
    assert pk.paged_attention_workspace_bytes(bf, 32, 32, 4, 4096, 0) == want
