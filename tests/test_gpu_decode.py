"""GPU: paged decode attention against the double-precision oracle.

Tolerances (max-abs, and max-abs relative to the output's largest magnitude):
bf16 KV 2e-2 / 1e-2 and FP8 KV 5e-2 (the stated pass criteria), INT8 KV as
FP8 (the same f16 tensor-core arithmetic on exactly widened codes); fp32 KV
1e-4 / 1e-4 (fp32 accumulation over <= a few thousand terms of |x| ~ 1).
"""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

import paged_kv_cache_401_b200 as pk
from gpu_harness import check_close, oracle_out, stage, step
from workloads import POISON_BLOCK, WORKLOADS, Spec, make_inputs

pytestmark = pytest.mark.gpu


def _spec(kv, q, D, G, lens, idx=50, hkv=2):
    return Spec(f"t-{kv}-{q}-{D}-{G}", idx, batch=len(lens), num_q_heads=G * hkv,
                num_kv_heads=hkv, head_dim=D, kv_dtype=kv, q_dtype=q,
                lens=("fixed", tuple(lens)), scale=1.0 / math.sqrt(D), slack_blocks=3)


LENS = [1, 2, 15, 16, 17, 63, 64, 65, 300, 1023, 1025]


@pytest.mark.parametrize("kv,q", [("bf16", "bf16"), ("f32", "f32"), ("fp8", "bf16"),
                                  ("bf16", "f32"), ("f32", "bf16"), ("fp8", "f32"),
                                  ("int8", "bf16"), ("int8", "f32"), ("int4", "bf16")])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_parity_shapes(kv, q, D, G):
    if kv == "int4" and D != 128:
        pytest.skip("4-bit pools have head_dim 128")
    inp = make_inputs(_spec(kv, q, D, G, LENS))
    st = stage(inp)
    _, ref = oracle_out(inp)
    for part in (0, 16, 64, 1024):
        st.cache.clear_errors()
        out = step(st, partition_tokens=part)
        check_close(out, ref, kv)
        assert st.cache.errors() == 0


@pytest.mark.parametrize("kv", ["bf16", "fp8", "int8", "int4"])
def test_decode_key_channels_with_large_offsets(kv):
    # keys far from zero relative to their spread (per-channel offsets up to 120):
    # large scores, large row scales and zero points.  The codes are the oracle's own,
    # so the comparison measures the tile arithmetic
    inp = make_inputs(_spec(kv, "bf16", 128, 4, [300, 1024, 1025, 2047], idx=152))
    g = torch.Generator().manual_seed(8)
    off = (torch.rand(2, 128, generator=g) * 2 - 1) * 120.0  # per (kv head, channel)
    inp.k[:] = (inp.k.float() * 0.25 + off[None]).to(inp.k.dtype)
    st = stage(inp)
    _, ref = oracle_out(inp)
    out = step(st)
    assert st.cache.errors() == 0
    check_close(out, ref, kv)


@pytest.mark.parametrize("part", [16, 48, 256, 1008, 1024, 1040, 4096, 8192])
def test_decode_partition_edges(part):
    # context lengths at partition size -1/0/+1 and at block boundaries
    lens = [part - 1 if part > 16 else 1, part, part + 1, 2 * part + 17, 2048, 16, 17]
    inp = make_inputs(_spec("bf16", "bf16", 128, 4, lens, idx=51))
    st = stage(inp)
    out = step(st, partition_tokens=part)
    check_close(out, oracle_out(inp)[1], "bf16")


def test_tiny_workload_step():
    inp = make_inputs("tiny")
    st = stage(inp)
    out = step(st)
    stats = check_close(out, oracle_out(inp)[1], "f32")
    assert stats["max_abs"] < 1e-4
    # the step's appends (positions 37 and 100) landed in blocks 2 and 6 of each table
    for s, pos in enumerate(inp.append_positions):
        blk = int(inp.block_table[s, pos // 16])
        got = st.cache.k_pool[blk, 0, pos % 16].cpu()
        assert torch.equal(got, inp.k[int(inp.append_rows[s]), 0])
    assert st.cache.errors() == 0


def test_length_one_returns_v_bitwise():
    for kv in ("bf16", "f32"):
        inp = make_inputs(_spec(kv, kv, 128, 4, [1, 1, 1], idx=52))
        st = stage(inp)
        out = step(st).cpu()
        for s in range(3):
            vrow = inp.v[int(inp.seq_offsets[s])]             # [Hkv][D]
            want = vrow.repeat_interleave(4, dim=0).to(out.dtype)
            assert torch.equal(out[s], want)


def test_identical_keys_give_mean_v():
    inp = make_inputs(_spec("bf16", "bf16", 128, 4, [700, 33], idx=53))
    for s in range(2):
        a, n = int(inp.seq_offsets[s]), int(inp.context_lens[s])
        inp.k[a:a + n] = inp.k[a]
    st = stage(inp)
    out = step(st).float().cpu().numpy()
    for s in range(2):
        a, n = int(inp.seq_offsets[s]), int(inp.context_lens[s])
        mean = inp.v[a:a + n].double().mean(0).numpy()          # [Hkv][D]
        want = np.repeat(mean, 4, axis=0)
        assert np.abs(out[s] - want).max() <= 2e-2


def _ramp_keys(inp, rising: bool):
    """Scale every sequence's keys by a factor ramping over its positions (0.2 -> 3 or
    3 -> 0.2): rising, a row's running max grows in nearly every tile; falling, it
    settles in the first tiles and the online softmax's corrections stay exactly 1."""
    for s in range(inp.q.shape[0]):
        a, n = int(inp.seq_offsets[s]), int(inp.context_lens[s])
        g = torch.linspace(0.2, 3.0, n) if rising else torch.linspace(3.0, 0.2, n)
        inp.k[a:a + n] = (inp.k[a:a + n].float() * g[:, None, None]).to(inp.k.dtype)


@pytest.mark.parametrize("kv", ["bf16", "fp8", "int8", "int4"])
@pytest.mark.parametrize("rising", [True, False])
def test_running_max_growth_patterns(kv, rising):
    inp = make_inputs(_spec(kv, "bf16", 128, 4, [40, 1000, 2047, 3001], idx=57))
    _ramp_keys(inp, rising)
    st = stage(inp)
    _, ref = oracle_out(inp)
    for part in (0, 256):
        out = step(st, partition_tokens=part)
        check_close(out, ref, kv)
    assert st.cache.errors() == 0


def test_permuted_pool_is_bitwise_invariant():
    inp = make_inputs(_spec("bf16", "bf16", 128, 4, [5, 400, 1500, 3000], idx=54))
    base = step(stage(inp), partition_tokens=256).cpu()
    rng = np.random.default_rng(9)
    remap = rng.permutation(inp.num_blocks).astype(np.int32)
    table = inp.block_table.copy()
    used = table != POISON_BLOCK
    table[used] = remap[table[used]]
    again = step(stage(inp, block_table=table), partition_tokens=256).cpu()
    assert torch.equal(base, again)


def test_aliased_prefix_equals_private_copies_bitwise():
    spec = replace(WORKLOADS["ragged"], index=55)
    inp = make_inputs(spec, batch=12)                 # 12 sequences, all sharing one prefix
    assert inp.block_table[0, 0] == inp.block_table[5, 0]
    shared = step(stage(inp)).cpu()
    # private copies: give every sharing sequence its own prefix blocks and write them
    from workloads import Inputs
    table = inp.block_table.copy()
    extra = inp.num_blocks
    rows, sids, poss = [], [], []
    for s in range(1, 12):
        table[s, :128] = np.arange(extra, extra + 128, dtype=np.int32)
        extra += 128
        a = int(inp.seq_offsets[s])
        rows.append(a + np.arange(2048))
        sids.append(np.full(2048, s, np.int32))
        poss.append(np.arange(2048, dtype=np.int32))
    priv = Inputs(spec=inp.spec, context_lens=inp.context_lens, seq_offsets=inp.seq_offsets,
                  q=inp.q, k=inp.k, v=inp.v, block_table=table, num_blocks=extra,
                  fill_rows=np.concatenate([inp.fill_rows] + rows),
                  fill_seq_ids=np.concatenate([inp.fill_seq_ids] + sids),
                  fill_positions=np.concatenate([inp.fill_positions] + poss))
    private = step(stage(priv)).cpu()
    assert torch.equal(shared, private)


def test_deterministic_repeat():
    inp = make_inputs(_spec("fp8", "bf16", 128, 4, [3000, 17, 900], idx=56))
    st = stage(inp)
    a = step(st, partition_tokens=512).clone()
    b = step(st, partition_tokens=512)
    assert torch.equal(a, b)


def test_bad_context_lengths_give_zeros_and_flag():
    inp = make_inputs(_spec("bf16", "bf16", 128, 4, [100, 200, 300, 50], idx=57))
    st = stage(inp)
    _, ref = oracle_out(inp)
    st.cache.append(st.block_table, st.seq_ids, st.positions, st.k_new, st.v_new)
    lens = st.context_lens.clone()
    lens[1] = 0
    lens[3] = 301                                    # above max_context_len = 300
    out = st.cache.decode(st.q, st.block_table, lens, 300, inp.spec.scale, partition_tokens=64)
    assert st.cache.errors() == pk.KV_DEVERR_BAD_CONTEXT_LEN
    o = out.cpu()
    assert (o[1] == 0).all() and (o[3] == 0).all()
    check_close(out[[0, 2]], ref[[0, 2]], "bf16")


def test_bad_block_id_is_reported_not_read():
    inp = make_inputs(_spec("bf16", "bf16", 128, 4, [100, 200], idx=58))
    st = stage(inp)
    _, ref = oracle_out(inp)
    st.cache.append(st.block_table, st.seq_ids, st.positions, st.k_new, st.v_new)
    bt = st.block_table.clone()
    bt[1, 3] = POISON_BLOCK
    bt[1, 5] = -7
    out = st.cache.decode(st.q, bt, st.context_lens, 200, inp.spec.scale, partition_tokens=64)
    assert st.cache.errors() == pk.KV_DEVERR_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    check_close(out[[0]], ref[[0]], "bf16")


# ---------------------------------------------------------------- full-size workloads
def _full_size(name, part=0):
    """One step of a full-size workload; every sequence and every query head of
    the output compared with the oracle, element by element."""
    inp = make_inputs(name)
    st = stage(inp)
    out = step(st, partition_tokens=part)
    assert st.cache.errors() == 0
    _, ref = oracle_out(inp)
    return check_close(out, ref, inp.spec.kv_dtype), inp, st


def test_llama_full_size():
    _full_size("llama")


def test_llama_full_size_more_ranges_than_32bit_shortcuts():
    # 16-token partitions over 32 x 4096 tokens x 8 kv heads: 65536 ranges, one
    # tile each -- past the 32-bit shortcuts of the range arithmetic (more than
    # 65535 ranges, tiles x ranges >= 2^32), so the 64-bit paths cut and merge
    stats, inp, st = _full_size("llama", part=16)
    assert pk.paged_decode_num_ranges(st.cache.desc, inp.q.shape[0], inp.spec.num_q_heads,
                                      inp.max_context_len, 16) == 65536


def test_ragged_full_size():
    _full_size("ragged")


def test_long_full_size():
    _full_size("long")


def _logical_slots(inp):
    """(physical block, offset in block, row of k/v) of every token 0 .. L_b - 1
    of every sequence, from the block table (a workload without shared blocks)."""
    blk, off, rows = [], [], []
    for s in range(inp.q.shape[0]):
        pos = np.arange(int(inp.context_lens[s]))
        blk.append(inp.block_table[s, pos // 16])
        off.append(pos % 16)
        rows.append(int(inp.seq_offsets[s]) + pos)
    return np.concatenate(blk), np.concatenate(off), np.concatenate(rows)


def _assert_quantised_pools_bitexact(inp, st, kind, chunk=1 << 16):
    """The whole K pool, V pool and scale pool after the step, byte for byte:
    every token's codes and row parameters from the oracle's quantiser in its
    slot, every other slot still holding the poison the pools were filled with."""
    import oracle
    blk, off, rows = _logical_slots(inp)
    got_sc = st.cache.scales.cpu().numpy()
    want_sc = np.full(got_sc.shape, np.nan, np.float32)
    for which, (pool, src) in enumerate(((st.cache.k_pool, inp.k), (st.cache.v_pool, inp.v))):
        got = pool.cpu().numpy()
        want = np.full(got.shape, 0x7F, got.dtype)
        for c0 in range(0, len(rows), chunk):
            sl = slice(c0, c0 + chunk)
            codes, sc = oracle.quantize_rows(src[torch.from_numpy(rows[sl])].float().numpy(),
                                             kind)
            if kind == "int4":
                codes = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
            want[blk[sl], :, off[sl], :] = codes
            want_sc[blk[sl], :, which, off[sl]] = sc
        assert np.array_equal(got, want), f"{'KV'[which]} pool differs"
    assert np.array_equal(got_sc.view(np.int32), want_sc.view(np.int32)), "scale pool differs"


@pytest.mark.parametrize("kind", ["fp8", "int8", "int4"])
def test_quantized_full_size_and_pools_bitexact(kind):
    stats, inp, st = _full_size(kind)
    _assert_quantised_pools_bitexact(inp, st, kind)


def test_workspace_needs_no_initialisation():
    # the workspace holds only what each call writes before reading it: garbage in
    # it must not matter, and repeated calls on one workspace give the same bits
    inp = make_inputs(_spec("bf16", "bf16", 128, 4, [3000, 17, 900, 4096], idx=59))
    st = stage(inp)
    st.cache.append(st.block_table, st.seq_ids, st.positions, st.k_new, st.v_new)
    _, ref = oracle_out(inp)
    n = st.cache.workspace_bytes(4, 8, inp.max_context_len, 64)
    for fill in (0xFF, 0x00, 0x5A):
        ws = torch.full((n,), fill, dtype=torch.uint8, device="cuda")
        outs = [st.cache.decode(st.q, st.block_table, st.context_lens, inp.max_context_len,
                                inp.spec.scale, partition_tokens=64, workspace=ws).clone()
                for _ in range(3)]
        assert st.cache.errors() == 0
        check_close(outs[0], ref, "bf16")
        assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
