"""GPU: the fused append+decode call against the separate calls it replaces.

paged_decode_attention_append must leave the pools exactly as
compute_slot_mapping + reshape_and_cache leave them (codes and scales for
8-bit pools, bit for bit) and return exactly the output of
paged_decode_attention on those pools; it is also checked against the oracle.
"""
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_401_b200 as pk
from gpu_harness import check_close, oracle_out, stage
from workloads import POISON_BLOCK, Spec, make_inputs

pytestmark = pytest.mark.gpu


def _spec(kv, q, D, G, lens, idx=110, hkv=2):
    return Spec(f"fa-{kv}-{q}-{D}-{G}", idx, batch=len(lens), num_q_heads=G * hkv,
                num_kv_heads=hkv, head_dim=D, kv_dtype=kv, q_dtype=q,
                lens=("fixed", tuple(lens)), scale=1.0 / math.sqrt(D), slack_blocks=3)


def _bits(t):
    if t is None:
        return None
    t = t.detach().clone()
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else (
        t.view(torch.int32) if t.dtype == torch.float32 else t)


def _pools(cache):
    return [_bits(t) for t in (cache.k_pool, cache.v_pool, cache.scales) if t is not None]


def _restore(cache, saved):
    for t, s in zip([t for t in (cache.k_pool, cache.v_pool, cache.scales) if t is not None],
                    saved):
        t.view(s.dtype).copy_(s)


LENS = [1, 2, 15, 16, 17, 64, 65, 300, 1025]


@pytest.mark.parametrize("kv,q", [("bf16", "bf16"), ("f32", "f32"), ("fp8", "bf16"),
                                  ("int8", "bf16"), ("bf16", "f32"), ("fp8", "f32"),
                                  ("int8", "f32"), ("int4", "bf16")])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_fused_equals_separate_calls(kv, q, D, G):
    if kv == "int4" and D != 128:
        pytest.skip("4-bit pools have head_dim 128")
    inp = make_inputs(_spec(kv, q, D, G, LENS, idx=110 + G))
    st = stage(inp)
    c = st.cache
    history = _pools(c)
    _, ref = oracle_out(inp)
    for part in (0, 16, 64):
        _restore(c, history)
        c.clear_errors()
        c.append(st.block_table, st.seq_ids, st.positions, st.k_new, st.v_new)
        want = c.decode(st.q, st.block_table, st.context_lens, st.max_context_len,
                        inp.spec.scale, partition_tokens=part).clone()
        want_pools = _pools(c)
        _restore(c, history)
        got = c.decode_append(st.q, st.k_new, st.v_new, st.block_table, st.context_lens,
                              st.max_context_len, inp.spec.scale, partition_tokens=part)
        assert c.errors() == 0
        assert torch.equal(_bits(got), _bits(want)), f"output differs (partition {part})"
        for a, b in zip(_pools(c), want_pools):
            assert torch.equal(a, b), f"pool differs (partition {part})"
        check_close(got, ref, kv)


def test_fused_steps_grow_the_context():
    # three fused steps in a row: each step's token is attended to by the next steps
    kv, D, G = "bf16", 128, 4
    lens = [40, 16, 1000]
    inp = make_inputs(_spec(kv, "bf16", D, G, [n + 2 for n in lens], idx=120))
    st = stage(inp, poison=True)
    c = st.cache
    # the staged history holds positions < L - 1; rewind two more tokens and redo them fused
    g = torch.Generator().manual_seed(9)
    for back in (2, 1, 0):
        lens_t = torch.from_numpy(inp.context_lens - back).to(st.q.device)
        k_new = torch.randn(st.k_new.shape, generator=g).to(st.k_new.dtype).cuda()
        v_new = torch.randn(st.v_new.shape, generator=g).to(st.v_new.dtype).cuda()
        before = _pools(c)
        out = c.decode_append(st.q, k_new, v_new, st.block_table, lens_t,
                              int(lens_t.max()), inp.spec.scale)
        fused_pools = _pools(c)
        _restore(c, before)
        pos = lens_t.to(torch.int32) - 1
        c.append(st.block_table, st.seq_ids, pos, k_new, v_new)
        sep = c.decode(st.q, st.block_table, lens_t, int(lens_t.max()), inp.spec.scale)
        assert torch.equal(_bits(out), _bits(sep))
        for a, b in zip(fused_pools, _pools(c)):
            assert torch.equal(a, b)
    assert c.errors() == 0


@pytest.mark.parametrize("kv", ["bf16", "fp8", "int4"])
def test_fused_bad_last_block_writes_nothing_for_that_sequence(kv):
    inp = make_inputs(_spec(kv, "bf16", 128, 4, [100, 200, 33], idx=121))
    st = stage(inp)
    c = st.cache
    before = _pools(c)
    bt = st.block_table.clone()
    bt[1, (200 - 1) // 16] = POISON_BLOCK             # the block of sequence 1's new token
    out = c.decode_append(st.q, st.k_new, st.v_new, bt, st.context_lens, 200, inp.spec.scale)
    assert c.errors() == pk.KV_DEVERR_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    # sequences 0 and 2 are written and decoded as usual
    _, ref = oracle_out(inp, [0, 2])
    check_close(out[[0, 2]], ref, kv)
    # nothing was written into sequence 1's slot (its block is unchanged)
    blk = int(inp.block_table[1, (200 - 1) // 16])
    for a, b in zip(_pools(c), before):
        assert torch.equal(a[blk], b[blk])


def test_fused_invalid_context_length_gives_zeros_and_writes_nothing():
    inp = make_inputs(_spec("int8", "bf16", 128, 2, [50, 90], idx=122))
    st = stage(inp)
    c = st.cache
    before = _pools(c)
    lens = st.context_lens.clone()
    lens[0] = 0
    out = c.decode_append(st.q, st.k_new, st.v_new, st.block_table, lens, 90, inp.spec.scale)
    assert c.errors() == pk.KV_DEVERR_BAD_CONTEXT_LEN
    assert (out[0].float() == 0).all()
    blk = int(inp.block_table[0, (50 - 1) // 16])
    for a, b in zip(_pools(c), before):
        assert torch.equal(a[blk], b[blk])
    check_close(out[[1]], oracle_out(inp, [1])[1], "int8")


def test_fused_full_size_llama():
    # the step the benchmark times, on its full workload: every sequence and head
    inp = make_inputs("llama")
    st = stage(inp)
    out = st.cache.decode_append(st.q, st.k_new, st.v_new, st.block_table, st.context_lens,
                                 st.max_context_len, inp.spec.scale)
    assert st.cache.errors() == 0
    _, ref = oracle_out(inp)
    check_close(out, ref, "bf16")


def test_decode_step_replays_in_a_cuda_graph():
    # the fused step captures into a CUDA graph (host work -- argument checks, tensor
    # maps -- happens at capture) and every replay gives the eager call's bits
    inp = make_inputs(_spec("bf16", "bf16", 128, 4, [300, 1025, 17], idx=123))
    st = stage(inp)
    c = st.cache
    out = torch.empty_like(st.q)
    ws = c.alloc_workspace(3, 8, st.max_context_len)
    s = torch.cuda.Stream()

    def call():
        c.decode_append(st.q, st.k_new, st.v_new, st.block_table, st.context_lens,
                        st.max_context_len, inp.spec.scale, out=out, workspace=ws)

    with torch.cuda.stream(s):
        call()
        torch.cuda.synchronize()
        eager = out.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            call()
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    assert c.errors() == 0
