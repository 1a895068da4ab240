"""GPU: block copies, and a fork / copy-on-write decode step driven by the host
block manager, checked against the oracle on each sequence's own tokens."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_401_b200 as pk
from paged_kv_cache_401_b200.cache import PagedKVCache
from workloads import storage_view

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    return t.numpy()


@pytest.mark.parametrize("kv", ["bf16", "f32", "fp8", "int8", "int4"])
def test_copy_blocks_bitexact(kv):
    nb, hkv, d = 24, 2, 64 if kv == "f32" else 128
    cache = PagedKVCache(nb, hkv, d, kv, DEV)
    g = torch.Generator(device="cpu").manual_seed(3)
    if kv in ("fp8", "int8", "int4"):
        dt = cache.k_pool.dtype
        lo, hi = (-127, 128) if kv == "int8" else (0, 255)
        cache.k_pool.copy_(torch.randint(lo, hi, cache.k_pool.shape, generator=g, dtype=dt))
        cache.v_pool.copy_(torch.randint(lo, hi, cache.v_pool.shape, generator=g, dtype=dt))
        cache.scales.copy_(torch.rand(cache.scales.shape, generator=g))
    else:
        for t in (cache.k_pool, cache.v_pool):
            t.copy_(torch.randn(t.shape, generator=g).to(t.dtype))
    before = [_bits(t) for t in (cache.k_pool, cache.v_pool, cache.scales) if t is not None]
    src = np.array([3, 7, 7, 20], dtype=np.int32)
    dst = np.array([0, 11, 12, 5], dtype=np.int32)
    pk.paged_kv_copy_blocks(cache.desc, cache.k_pool, cache.v_pool, cache.scales,
                            torch.from_numpy(src).to(DEV), torch.from_numpy(dst).to(DEV),
                            cache.dev_error)
    after = [_bits(t) for t in (cache.k_pool, cache.v_pool, cache.scales) if t is not None]
    for b, a in zip(before, after):
        want = b.copy()
        want[dst] = b[src]
        assert (a == want).all()
    assert cache.errors() == 0


@pytest.mark.parametrize("kv", ["bf16", "fp8", "int8", "int4"])
def test_fork_copy_on_write_decode(kv):
    hq, hkv, d, nb, hist = 8, 2, 128, 32, 40
    m = pk.BlockManager(nb, 4, 16)
    cache = PagedKVCache(nb, hkv, d, kv, DEV, poison=True)
    g = torch.Generator(device="cpu").manual_seed(11)
    rnd = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)  # noqa: E731
    k_hist, v_hist = rnd(hist, hkv, d), rnd(hist, hkv, d)
    a = m.add_sequence()
    slots, copies = m.append_slots([a] * hist)
    assert copies == []
    pk.reshape_and_cache(cache.desc, cache.k_pool, cache.v_pool, cache.scales, k_hist.to(DEV),
                         v_hist.to(DEV), torch.from_numpy(slots).to(DEV), cache.dev_error)
    b = m.fork(a)                              # shares 3 blocks; the third holds 8 tokens
    k_new, v_new = rnd(2, hkv, d), rnd(2, hkv, d)
    slots, copies = m.append_slots([a, b])     # a writes first: a gets a private copy
    assert len(copies) == 1
    src, dst = (torch.tensor([c[i] for c in copies], dtype=torch.int32, device=DEV)
                for i in (0, 1))
    pk.paged_kv_copy_blocks(cache.desc, cache.k_pool, cache.v_pool, cache.scales, src, dst,
                            cache.dev_error)
    pk.reshape_and_cache(cache.desc, cache.k_pool, cache.v_pool, cache.scales, k_new.to(DEV),
                         v_new.to(DEV), torch.from_numpy(slots).to(DEV), cache.dev_error)
    table, lens = m.export()
    table, lens = table[[a, b]], lens[[a, b]]
    assert lens.tolist() == [hist + 1, hist + 1]
    assert table[0, 2] != table[1, 2] and table[0, 1] == table[1, 1]
    q = rnd(2, hq, d)
    out = cache.decode(q.to(DEV), torch.from_numpy(np.ascontiguousarray(table)).to(DEV),
                       torch.from_numpy(lens).to(DEV), hist + 1, 1 / math.sqrt(d))
    assert cache.errors() == 0
    # the oracle reads each sequence's own contiguous tokens: history + its new token
    k_seq = torch.cat([k_hist, k_new[:1], k_hist, k_new[1:]])
    v_seq = torch.cat([v_hist, v_new[:1], v_hist, v_new[1:]])
    offs = np.array([0, hist + 1], dtype=np.int64)
    if kv in ("fp8", "int8", "int4"):
        kc, ks = oracle.quantize_rows(k_seq.float().numpy(), kv)
        vc, vs = oracle.quantize_rows(v_seq.float().numpy(), kv)
        ref = oracle.decode_attention(storage_view(q), kc, vc, offs, lens, 1 / math.sqrt(d), hkv,
                                      kv, "bf16", k_scale=ks, v_scale=vs)
        tol = 5e-2
    else:
        ref = oracle.decode_attention(storage_view(q), storage_view(k_seq), storage_view(v_seq),
                                      offs, lens, 1 / math.sqrt(d), hkv, "bf16", "bf16")
        tol = 2e-2
    assert np.abs(out.float().cpu().numpy() - ref).max() <= tol
