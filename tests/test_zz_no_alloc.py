"""GPU: paged_decode_attention_static_workspace, the decode for callers that
cannot allocate device memory (an engine that reserved all of HBM for its KV
pool, a plugin whose host runtime owns the allocator, a loop that cannot take
cudaMalloc's implicit synchronisation).

It is called through the C ABI several times in a row, on different
workloads, and each output is compared with the regular entry point's (which
takes a caller-allocated workspace).  Both run the same kernels with the same
split, and the split-K arithmetic does not depend on where the workspace
lives, so the outputs must be equal bit for bit.  Every call after the first
finds the previous call's partials still in the shared array.  One call uses
the default split (partition_tokens 0) at 256 sequences x 8 kv heads x 4 query
heads per group, the size the library's fixed array is stated to cover.
This file is collected last so a failure here stops a -x run only after every
other test has run; it also passes on its own in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_401_b200 as pk
from gpu_harness import stage
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


def test_static_workspace_matches_regular_entry_several_calls():
    lens256 = np.random.default_rng(64).integers(1, 2049, size=256).tolist()
    runs = [
        (_workload("bf16", [4096, 1, 17, 2000, 3333, 4095], 60), 256),   # 16 partitions
        (_workload("fp8", [700, 5000, 64, 129], 61), 512),               # other sizes after it
        (_workload("bf16", lens256, 62), 0),                             # default split, B256 G4
    ]
    for inp, partition in runs:
        st = stage(inp)
        st.cache.append(st.block_table, st.seq_ids, st.positions, st.k_new, st.v_new)
        need = st.cache.workspace_bytes(inp.q.shape[0], 32, inp.max_context_len, partition)
        assert 0 < need <= pk.KV_STATIC_WORKSPACE_BYTES
        want = _regular_call(st, partition)
        for _ in range(2):                          # a second call over the first's partials
            got = _static_call(st, partition)
            torch.cuda.synchronize()
            assert st.cache.errors() == 0
            assert torch.equal(got, want)


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
