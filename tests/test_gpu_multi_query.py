"""GPU: multi-query paged attention (Q causal query tokens per sequence) against
the oracle's causal multi-query attention.  Tolerances as for decode: bf16 KV
max-abs 2e-2 / max-rel 1e-2, FP8, INT8 and INT4 KV max-abs 5e-2."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_401_b200 as pk
from gpu_harness import check_close, stage
from workloads import Spec, make_inputs, storage_view

pytestmark = pytest.mark.gpu


def _spec(kv, G, lens, idx=70, hkv=2):
    return Spec(f"mq-{kv}-{G}", idx, batch=len(lens), num_q_heads=G * hkv, num_kv_heads=hkv,
                head_dim=128, kv_dtype=kv, q_dtype="bf16", lens=("fixed", tuple(lens)),
                scale=1.0 / math.sqrt(128), slack_blocks=3)


def _oracle(inp, qm):
    spec = inp.spec
    q = storage_view(qm)
    if spec.kv_dtype in oracle.QUANTIZED:
        kc, ks = oracle.quantize_rows(inp.k.float().numpy(), spec.kv_dtype)
        vc, vs = oracle.quantize_rows(inp.v.float().numpy(), spec.kv_dtype)
        return oracle.multi_query_attention(q, kc, vc, inp.seq_offsets, inp.context_lens,
                                           spec.scale, spec.num_kv_heads, spec.kv_dtype, "bf16",
                                           k_scale=ks, v_scale=vs)
    return oracle.multi_query_attention(q, storage_view(inp.k), storage_view(inp.v),
                                        inp.seq_offsets, inp.context_lens, spec.scale,
                                        spec.num_kv_heads, spec.kv_dtype, "bf16")


def _full_cache(inp):
    st = stage(inp)
    st.cache.append(st.block_table, st.seq_ids, st.positions, st.k_new, st.v_new)
    return st


CASES = [(g, q) for g in (1, 2, 4, 8) for q in (2, 3, 4, 5, 8, 16) if g * q <= 16]


@pytest.mark.parametrize("kv", ["bf16", "fp8", "int8", "int4"])
@pytest.mark.parametrize("G,Q", CASES)
def test_multi_query_parity(kv, G, Q):
    lens = [Q, Q + 1, 17, 33, 100, 1025, 2048 + 3]
    inp = make_inputs(_spec(kv, G, lens, idx=70 + G * 20 + Q))
    st = _full_cache(inp)
    g = torch.Generator().manual_seed(5 + Q)
    qm = torch.randn(len(lens), Q, G * 2, 128, generator=g).to(torch.bfloat16)
    ref = _oracle(inp, qm)
    for part in (0, 16, 64):
        st.cache.clear_errors()
        out = st.cache.attend(qm.cuda(), st.block_table, st.context_lens, inp.max_context_len,
                              inp.spec.scale, partition_tokens=part)
        assert st.cache.errors() == 0
        check_close(out.reshape(-1, 128), ref.reshape(-1, 128), kv)


def test_one_query_token_equals_decode_bitwise():
    inp = make_inputs(_spec("bf16", 4, [7, 300, 4097], idx=90))
    st = _full_cache(inp)
    dec = st.cache.decode(st.q, st.block_table, st.context_lens, inp.max_context_len,
                          inp.spec.scale)
    mq = st.cache.attend(st.q[:, None].contiguous(), st.block_table, st.context_lens,
                         inp.max_context_len, inp.spec.scale)
    assert torch.equal(dec, mq[:, 0])


def test_short_context_gives_zeros_and_flag():
    inp = make_inputs(_spec("bf16", 4, [50, 70], idx=91))
    st = _full_cache(inp)
    qm = torch.randn(2, 4, 8, 128).to(torch.bfloat16).cuda()
    lens = st.context_lens.clone()
    lens[1] = 3                                   # fewer tokens than query tokens
    out = st.cache.attend(qm, st.block_table, lens, inp.max_context_len, inp.spec.scale)
    assert st.cache.errors() == pk.KV_DEVERR_BAD_CONTEXT_LEN
    assert (out[1] == 0).all()
    assert torch.isfinite(out.float()).all()


def test_llama_shape_speculative_verification():
    # 32 sequences x 4096 tokens, Q = 4 draft tokens verified at once (G * Q = 16
    # rows); every sequence, query token and head against the oracle
    inp = make_inputs("llama")
    st = _full_cache(inp)
    qm = torch.randn(32, 4, 32, 128, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    out = st.cache.attend(qm.cuda(), st.block_table, st.context_lens, inp.max_context_len,
                          inp.spec.scale)
    assert st.cache.errors() == 0
    ref = oracle.multi_query_attention(storage_view(qm), storage_view(inp.k),
                                       storage_view(inp.v), inp.seq_offsets, inp.context_lens,
                                       inp.spec.scale, 8, "bf16", "bf16")
    check_close(out.reshape(-1, 128), ref.reshape(-1, 128), "bf16")
