"""GPU: slot computation and cache write are bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_401_b200 as pk
from paged_kv_cache_401_b200.cache import PagedKVCache

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    return t.numpy()


def test_slot_mapping_bitexact_and_bad_positions():
    rng = np.random.default_rng(1)
    B, MB = 7, 9
    table = rng.permutation(200)[:B * MB].reshape(B, MB).astype(np.int32)
    sids = rng.integers(0, B, 500).astype(np.int32)
    poss = rng.integers(0, MB * 16, 500).astype(np.int32)
    expect = oracle.slot_mapping(table, sids, poss, 16)
    bad = np.array([[0, MB * 16], [B, 3], [-1, 0], [2, -5]], dtype=np.int32)
    sids_all = np.r_[sids, bad[:, 0]]
    poss_all = np.r_[poss, bad[:, 1]]
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    slots = torch.empty(len(sids_all), dtype=torch.int64, device=DEV)
    pk.compute_slot_mapping(torch.from_numpy(table).to(DEV), torch.from_numpy(sids_all).to(DEV),
                            torch.from_numpy(poss_all).to(DEV), slots, 16, err)
    got = slots.cpu().numpy()
    assert (got[:500] == expect).all()
    assert (got[500:] == -1).all()
    assert err.item() == pk.KV_DEVERR_BAD_POSITION


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("f32", 128), ("bf16", 64), ("bf16", 128)])
def test_cache_copy_bitexact(dtype, D):
    rng = np.random.default_rng(2)
    NB, Hkv, T = 40, 3, 300
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    cache = PagedKVCache(NB, Hkv, D, dtype, DEV, poison=True)
    k = torch.randn(T, Hkv, D, dtype=torch.float32).to(tdt)
    v = torch.randn(T, Hkv, D, dtype=torch.float32).to(tdt)
    slots = rng.permutation(NB * 16)[:T].astype(np.int64)
    slots[5] = -1                       # padding
    slots[6] = NB * 16 + 3              # out of range: skipped, reported
    before = {id(cache.k_pool): _bits(cache.k_pool), id(cache.v_pool): _bits(cache.v_pool)}
    pk.reshape_and_cache(cache.desc, cache.k_pool, cache.v_pool, None, k.to(DEV),
                         v.to(DEV), torch.from_numpy(slots).to(DEV), cache.dev_error)
    slots_ok = slots.copy()
    slots_ok[6] = -1
    for pool, src in ((cache.k_pool, k), (cache.v_pool, v)):
        # expected: the pool's poisoned bits as filled, with the written rows replaced
        want = oracle.scatter_to_pool(before[id(pool)], _bits(src), slots_ok)
        assert (_bits(pool) == want).all()
    assert cache.errors() == pk.KV_DEVERR_BAD_SLOT


def _fp8_rows(rng, T, Hkv, D):
    x = rng.normal(size=(T, Hkv, D)).astype(np.float32)
    x[0] = 0.0                                   # zero rows: scale 0, codes 0
    x[1, 0, :] = 0.0
    x[1, 0, 7] = 1e-3                            # a single non-zero element
    x[2] *= 1e-4                                 # small magnitudes
    x[3, :, ::7] *= 50.0                         # outlier channels: subnormal codes elsewhere
    x[4] *= 3e4                                  # large magnitudes
    x[5, 1, :] = np.linspace(-1, 1, D)           # ties are likely on a regular grid
    x[7, 0, :] = np.abs(x[7, 0, :]) + 3.0        # all positive (INT4: negative zero point)
    x[8, 1, :] = -np.abs(x[8, 1, :]) - 3.0       # all negative (INT4: zero point above 15)
    x[9, 0, :] = 0.625                           # constant, non-zero
    return x


def _pack_int4(codes):
    """One code per element -> the pool's bytes: dim 2i low nibble, 2i+1 high."""
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("kind", ["fp8", "int8", "int4"])
@pytest.mark.parametrize("src", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
def test_cache_quant_bitexact(kind, src, D):
    if kind == "int4" and D != 128:
        pytest.skip("4-bit pools have head_dim 128")
    rng = np.random.default_rng(3 + D)
    NB, Hkv, T = 50, 2, 400
    x_k = _fp8_rows(rng, T, Hkv, D)
    x_v = rng.normal(size=(T, Hkv, D)).astype(np.float32)
    if kind == "int8":
        # scale 127/127 = 1 and exact half-integer quotients: every code is a tie
        # (the values are exact in bf16 too, so both source types see the row)
        x_k[6, 0, :] = np.arange(D) - D / 2 + 0.5
        x_k[6, 0, 0] = 127.0
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[src]
    k = torch.from_numpy(x_k.copy()).to(tdt)
    v = torch.from_numpy(x_v).to(tdt)
    if kind == "int8":
        assert k[6, 0, 1].item() == 1 - D / 2 + 0.5 and k[6, 0, 0].item() == 127.0
    slots = rng.permutation(NB * 16)[:T].astype(np.int64)
    slots[9] = -1
    cache = PagedKVCache(NB, Hkv, D, kind, DEV, poison=True)
    pk.reshape_and_cache(cache.desc, cache.k_pool, cache.v_pool, cache.scales, k.to(DEV),
                         v.to(DEV), torch.from_numpy(slots).to(DEV), cache.dev_error)
    want_scales = np.full(tuple(cache.scales.shape), np.nan, np.float32)
    for which, (pool, src_t) in enumerate(((cache.k_pool, k), (cache.v_pool, v))):
        codes, scales = oracle.quantize_rows(src_t.float().numpy(), kind)
        if kind == "int4":
            codes = _pack_int4(codes)
        want_codes = oracle.scatter_to_pool(np.full(tuple(pool.shape), 0x7F, codes.dtype), codes,
                                            slots)
        want_scales = oracle.scatter_scales_to_pool(want_scales, scales, slots, which)
        assert (pool.cpu().numpy() == want_codes).all()
    assert (_bits(cache.scales) == want_scales.view(np.int32)).all()
    assert cache.errors() == 0
