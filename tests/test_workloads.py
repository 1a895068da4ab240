"""CPU: the seeded generators produce the workloads' stated shapes and structure."""
import numpy as np
import pytest
import torch

from workloads import POISON_BLOCK, WORKLOADS, make_inputs


def test_tiny_matches_its_description():
    inp = make_inputs("tiny")
    assert inp.context_lens.tolist() == [38, 101]          # 37 / 100 history + the appended token
    assert inp.num_blocks == 32
    assert inp.append_positions.tolist() == [37, 100]
    nblk = (inp.block_table != POISON_BLOCK).sum(axis=1)
    assert nblk.tolist() == [3, 7]
    used = inp.block_table[inp.block_table != POISON_BLOCK]
    assert len(set(used.tolist())) == 10 and used.max() < 32
    assert inp.q.dtype == torch.float32 and inp.k.shape == (139, 1, 64)


def test_generation_is_deterministic():
    a = make_inputs("tiny")
    b = make_inputs("tiny")
    assert torch.equal(a.k, b.k) and torch.equal(a.q, b.q)
    assert (a.block_table == b.block_table).all()


def test_llama_table_is_a_permutation_of_the_pool():
    inp = make_inputs("llama", batch=4, lens_override=[4096] * 4)
    assert inp.block_table.shape == (4, 256)
    assert len(np.unique(inp.block_table)) == 4 * 256


def test_llama_full_table_uses_every_block_once():
    spec = WORKLOADS["llama"]
    gen = torch.Generator().manual_seed(0)
    del gen
    # the full workload's block table is a permutation of all 8192 blocks
    inp = make_inputs("llama")
    assert sorted(inp.block_table.reshape(-1).tolist()) == list(range(spec.num_blocks))
    assert inp.k.shape == (32 * 4096, 8, 128) and inp.k.dtype == torch.bfloat16


def test_ragged_shares_a_prefix_and_diverges():
    inp = make_inputs("ragged", batch=70)
    L = inp.context_lens
    assert (L[:64] >= 2049).all() and (L >= 16).all() and (L <= 8192).all()
    # the 64 sharing sequences map their first 128 logical blocks to the same physical blocks
    assert (inp.block_table[:64, :128] == inp.block_table[0, :128]).all()
    # and their own blocks are private
    own = [set(inp.block_table[s, 128:(L[s] + 15) // 16].tolist()) for s in range(64)]
    assert all(not (own[i] & own[j]) for i in range(64) for j in range(i + 1, 64))
    a0, a5 = int(inp.seq_offsets[0]), int(inp.seq_offsets[5])
    assert torch.equal(inp.k[a0:a0 + 2048], inp.k[a5:a5 + 2048])
    assert not torch.equal(inp.k[a0 + 2048], inp.k[a5 + 2048])
    # the shared prefix is written once
    assert (inp.fill_seq_ids == 5).sum() == L[5] - 1 - 2048


def test_long_has_outlier_channels():
    spec = WORKLOADS["long"]
    inp = make_inputs(spec, batch=1, lens_override=[20000])
    k = inp.k.float()
    rms = k.pow(2).mean(dim=0).sqrt()               # [Hkv][D]
    for h in range(spec.num_kv_heads):
        big = (rms[h] > 10).nonzero().flatten().tolist()
        assert len(big) == spec.outlier_channels
    assert float(inp.v.float().pow(2).mean().sqrt()) < 1.1


@pytest.mark.parametrize("name", ["fp8", "int8", "int4"])
def test_quantized_lengths_in_range(name):
    inp = make_inputs(name, batch=16)
    assert (inp.context_lens >= 1024).all() and (inp.context_lens <= 16384).all()
    assert inp.k.dtype == torch.bfloat16 and inp.q.dtype == torch.bfloat16
