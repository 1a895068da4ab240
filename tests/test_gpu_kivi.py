"""GPU: the KIVI cache (keys per channel over a block, values per token, the
newest L mod 16 tokens unquantised) against the oracle.

Block quantisation is compared bit for bit (codes and parameters); decode
steps, with and without the append, within max-abs 5e-2 (the budget of the
other 4-bit path: exact code widening, f16 q * scale and P * scale)."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_401_b200 as pk
from gpu_harness import check_close, oracle_out_kivi, stage_kivi
from paged_kv_cache_401_b200.cache import PagedKVCache
from workloads import POISON_BLOCK, Spec, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _spec(G, lens, idx=130, hkv=2):
    return Spec(f"kivi-{G}", idx, batch=len(lens), num_q_heads=G * hkv, num_kv_heads=hkv,
                head_dim=128, kv_dtype="kivi4", q_dtype="bf16", lens=("fixed", tuple(lens)),
                scale=1.0 / math.sqrt(128), slack_blocks=3)


def _pack(codes):
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("src", ["f32", "bf16"])
def test_kivi_quantize_blocks_bitexact(src):
    rng = np.random.default_rng(41)
    nb, hkv, n = 40, 2, 12
    x_k = (rng.standard_normal((n, 16, hkv, 128)) * rng.uniform(0.05, 30, (n, 1, hkv, 128)))
    x_v = rng.standard_normal((n, 16, hkv, 128)) * rng.uniform(0.05, 30, (n, 16, hkv, 1))
    x_k[0, :, 0, 3] = 1.25                      # constant key channel
    x_k[1, :, 1, :] = np.abs(x_k[1, :, 1, :]) + 2  # positive channels: negative zero points
    x_v[2, 5, 0, :] = -0.5                      # constant value row
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[src]
    k = torch.from_numpy(x_k.astype(np.float32)).to(tdt)
    v = torch.from_numpy(x_v.astype(np.float32)).to(tdt)
    ids = rng.permutation(nb)[:n].astype(np.int32)
    cache = PagedKVCache(nb, hkv, 128, "kivi4", DEV, poison=True)
    cache.kivi_fill(torch.from_numpy(ids).to(DEV), k.to(DEV), v.to(DEV))
    assert cache.errors() == 0
    # oracle: per (block, kv head) groups
    kb = k.float().numpy().transpose(0, 2, 1, 3).reshape(n * hkv, 16, 128)
    vb = v.float().numpy().transpose(0, 2, 1, 3).reshape(n * hkv, 16, 128)
    kc, kp, vc, vp = oracle.quantize_blocks_kivi(kb, vb)
    kpool, vpool = cache.k_pool.cpu().numpy(), cache.v_pool.cpu().numpy()
    params = cache.scales.cpu().numpy()
    for i, blk in enumerate(ids):
        for h in range(hkv):
            j = i * hkv + h
            assert (kpool[blk, h] == _pack(kc[j])).all()
            assert (vpool[blk, h] == _pack(vc[j])).all()
            assert (params[blk, h, :128].view(np.int32) == kp[j].view(np.int32)).all()
            assert (params[blk, h, 128:].view(np.int32) == vp[j].view(np.int32)).all()
    # untouched blocks keep their poison
    rest = np.setdiff1d(np.arange(nb), ids)
    assert (kpool[rest] == 0x7F).all() and np.isnan(params[rest]).all()


LENS = [1, 2, 15, 16, 17, 31, 32, 33, 300, 1024, 1025]


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_kivi_decode_append_parity(G):
    # the step stores each new token in the residual (L % 16 == 0: completing and
    # quantising its block) and attends to quantised blocks + residual
    inp = make_inputs(_spec(G, LENS, idx=130 + G))
    _, ref = oracle_out_kivi(inp)
    for part in (0, 16, 64):
        st = stage_kivi(inp)
        out = st.cache.kivi_decode(st.q, st.block_table, st.context_lens, st.max_context_len,
                                   inp.spec.scale, st.k_new, st.v_new, partition_tokens=part)
        assert st.cache.errors() == 0
        check_close(out, ref, "kivi4")


@pytest.mark.parametrize("offset", [8.0, 120.0])
def test_kivi_key_channels_with_large_offsets(offset):
    # key channels that sit far from zero relative to their spread in a block (up to
    # ~130 times the range): zero points of over a thousand codes, q times large
    # per-channel scales.  The codes minus zero stay exact in f16 (|c - zero| <= 2048);
    # what grows is the f16 rounding of q * scale, which stays well inside the budget
    inp = make_inputs(_spec(4, [300, 1024, 1025, 2047], idx=150))
    g = torch.Generator().manual_seed(7)
    off = (torch.rand(2, 128, generator=g) * 2 - 1) * offset  # per (kv head, channel)
    inp.k[:] = (inp.k.float() * 0.25 + off[None]).to(inp.k.dtype)
    _, ref = oracle_out_kivi(inp)
    st = stage_kivi(inp)
    out = st.cache.kivi_decode(st.q, st.block_table, st.context_lens, st.max_context_len,
                               inp.spec.scale, st.k_new, st.v_new)
    assert st.cache.errors() == 0
    check_close(out, ref, "kivi4")


@pytest.mark.parametrize("rising", [True, False])
def test_kivi_running_max_growth_patterns(rising):
    # keys scaled by a ramp over positions: the running max grows in nearly every
    # tile (rising) or settles early (falling)
    inp = make_inputs(_spec(4, [40, 1000, 2047, 3001], idx=139))
    for s in range(inp.q.shape[0]):
        a, n = int(inp.seq_offsets[s]), int(inp.context_lens[s])
        g = torch.linspace(0.2, 3.0, n) if rising else torch.linspace(3.0, 0.2, n)
        inp.k[a:a + n] = (inp.k[a:a + n].float() * g[:, None, None]).to(inp.k.dtype)
    _, ref = oracle_out_kivi(inp)
    st = stage_kivi(inp)
    out = st.cache.kivi_decode(st.q, st.block_table, st.context_lens, st.max_context_len,
                               inp.spec.scale, st.k_new, st.v_new)
    assert st.cache.errors() == 0
    check_close(out, ref, "kivi4")


def test_kivi_flush_writes_the_completed_block():
    lens = [16, 32, 48, 17]                     # the first three complete a block
    inp = make_inputs(_spec(4, lens, idx=140))
    st = stage_kivi(inp)
    st.cache.kivi_decode(st.q, st.block_table, st.context_lens, st.max_context_len,
                         inp.spec.scale, st.k_new, st.v_new)
    assert st.cache.errors() == 0
    kpool, params = st.cache.k_pool.cpu().numpy(), st.cache.scales.cpu().numpy()
    for b, L in enumerate(lens[:3]):
        a = int(inp.seq_offsets[b])
        last = L // 16 - 1
        rows = inp.k[a + 16 * last:a + 16 * last + 16].float().numpy()      # [16][Hkv][D]
        vrows = inp.v[a + 16 * last:a + 16 * last + 16].float().numpy()
        kc, kp, _, vp = oracle.quantize_blocks_kivi(rows.transpose(1, 0, 2), vrows.transpose(1, 0, 2))
        blk = int(inp.block_table[b, last])
        assert (kpool[blk] == _pack(kc)).all()
        assert (params[blk, :, :128].view(np.int32) == kp.view(np.int32)).all()
        assert (params[blk, :, 128:].view(np.int32) == vp.view(np.int32)).all()
    # sequence 3 (L = 17) keeps its new token in residual row 0
    res = st.cache.res_k.cpu()
    assert torch.equal(res[3, :, 0], inp.k[int(inp.seq_offsets[3]) + 16])


def test_kivi_steps_across_a_block_boundary():
    # four steps per sequence, contexts 14 -> 15 -> 16 (a block completes) -> 17, ...
    from workloads import Inputs
    inp = make_inputs(_spec(4, [17, 33, 1003], idx=141))
    start = inp.context_lens - 3                    # the cache holds positions < start - 1
    hist = Inputs(spec=inp.spec, context_lens=start.astype(np.int32), seq_offsets=inp.seq_offsets,
                  q=inp.q, k=inp.k, v=inp.v, block_table=inp.block_table,
                  num_blocks=inp.num_blocks, fill_rows=inp.fill_rows,
                  fill_seq_ids=inp.fill_seq_ids, fill_positions=inp.fill_positions)
    st = stage_kivi(hist)
    for step in range(4):
        lens = (start + step).astype(np.int32)
        rows = torch.from_numpy(inp.seq_offsets + lens - 1)     # the token this step appends
        out = st.cache.kivi_decode(st.q, st.block_table, torch.from_numpy(lens).to(DEV),
                                   int(lens.max()), inp.spec.scale, inp.k[rows].to(DEV),
                                   inp.v[rows].to(DEV))
        check_close(out, oracle_out_kivi(inp, lens=lens)[1], "kivi4")
    assert st.cache.errors() == 0


def test_kivi_decode_without_append_and_bad_inputs():
    inp = make_inputs(_spec(4, [40, 64, 7], idx=142))
    st = stage_kivi(inp)
    c = st.cache
    # no append: the history alone (context lengths L - 1)
    lens = st.context_lens - 1
    out = c.kivi_decode(st.q, st.block_table, lens, st.max_context_len, inp.spec.scale)
    check_close(out, oracle_out_kivi(inp, lens=inp.context_lens - 1)[1], "kivi4")
    # an invalid length gives zeros and the error bit
    lens[1] = 0
    out = c.kivi_decode(st.q, st.block_table, lens, st.max_context_len, inp.spec.scale)
    assert c.errors() == pk.KV_DEVERR_BAD_CONTEXT_LEN
    assert (out[1].float() == 0).all()
    c.clear_errors()
    # a bad block id of a full block is reported, never read
    bt = st.block_table.clone()
    bt[1, 1] = POISON_BLOCK
    out = c.kivi_decode(st.q, bt, st.context_lens - 1, st.max_context_len, inp.spec.scale)
    assert c.errors() == pk.KV_DEVERR_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()


def test_kivi_full_size():
    # every sequence and query head of the 64-sequence workload against the oracle
    inp = make_inputs("kivi")
    st = stage_kivi(inp)
    out = st.cache.kivi_decode(st.q, st.block_table, st.context_lens, st.max_context_len,
                               inp.spec.scale, st.k_new, st.v_new)
    assert st.cache.errors() == 0
    _, ref = oracle_out_kivi(inp)
    check_close(out, ref, "kivi4")
