"""GPU: paged_decode_attention_static_workspace, the decode for callers that
cannot allocate device memory (an engine that reserved all of HBM for its KV
pool, a plugin whose host runtime owns the allocator, a loop that cannot take
cudaMalloc's implicit synchronisation).

It is called through the C ABI twice in a row, on two different workloads, and
each output is checked against the regular entry point's (which takes a
caller-allocated workspace) within the parity tolerances of the other tests.
The second call finds the first call's partials still in the shared array.
This file is collected last so a failure here stops a -x run only after every
other test has run; it also passes on its own in a fresh process.
"""
import ctypes
import math

import pytest
import torch

import paged_kv_cache_401_b200 as pk
from gpu_harness import TOL, stage
from workloads import Spec, make_inputs

pytestmark = pytest.mark.gpu


def _workload(kv, lens, idx):
    return make_inputs(Spec(f"noalloc-{kv}", idx, batch=len(lens), num_q_heads=32,
                            num_kv_heads=8, head_dim=128, kv_dtype=kv, q_dtype="bf16",
                            lens=("fixed", tuple(lens)), scale=1 / math.sqrt(128),
                            slack_blocks=2))


def _static_call(st, partition):
    c = st.cache
    lib = pk.library()
    out = torch.empty_like(st.q)
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    status = lib.paged_decode_attention_static_workspace(
        ctypes.byref(c.desc), out.data_ptr(), st.q.data_ptr(), pk.kv_dtype_of(st.q),
        c.k_pool.data_ptr(), c.v_pool.data_ptr(), ptr(c.scales),
        st.block_table.data_ptr(), st.block_table.shape[1], st.context_lens.data_ptr(),
        st.q.shape[0], st.q.shape[1], st.max_context_len, st.inp.spec.scale, partition,
        c.dev_error.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert status == pk.KV_OK, pk.kv_status_string(status)
    return out


def _regular_call(st, partition):
    return st.cache.decode(st.q, st.block_table, st.context_lens, st.max_context_len,
                           st.inp.spec.scale, partition_tokens=partition)


def _assert_close(a, b, kv):
    atol, rtol = TOL[kv]
    diff = (a.float() - b.float()).abs().max().item()
    assert diff <= atol
    if rtol is not None:
        assert diff <= rtol * b.float().abs().max().item()


def test_static_workspace_matches_regular_entry_two_calls():
    runs = [
        (_workload("bf16", [4096, 1, 17, 2000, 3333, 4095], 60), 256),   # 16 partitions
        (_workload("fp8", [700, 5000, 64, 129], 61), 512),               # other sizes after it
    ]
    for inp, partition in runs:
        st = stage(inp)
        st.cache.append(st.block_table, st.seq_ids, st.positions, st.k_new, st.v_new)
        assert st.cache.workspace_bytes(inp.q.shape[0], 32, inp.max_context_len, partition) > 0
        want = _regular_call(st, partition)
        got = _static_call(st, partition)
        torch.cuda.synchronize()
        assert st.cache.errors() == 0
        assert torch.isfinite(got.float()).all()
        _assert_close(got, want, inp.spec.kv_dtype)


def test_static_workspace_refuses_oversized_requests():
    desc = pk.kv_pool_create(1 << 16, 16, 8, 128, pk.KV_BF16)
    need = pk.paged_decode_workspace_bytes(desc, 64, 32, 1 << 16, 256)
    assert need > pk.KV_STATIC_WORKSPACE_BYTES
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    status = pk.library().paged_decode_attention_static_workspace(
        ctypes.byref(desc), p, p, pk.KV_BF16, p, p, None, p, 4096, p, 64, 32, 1 << 16,
        0.1, 256, None, torch.cuda.current_stream().cuda_stream)
    assert status == pk.KV_ERR_INVALID_ARGUMENT
