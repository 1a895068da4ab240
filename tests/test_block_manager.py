"""CPU: the host block manager against the allocation semantics of the pages.

``oracle.paging.ToyBlockManager`` restates the pages' paged-cache behaviour;
its pins below check it against what the pages state (block conservation, at
most one partly used block per sequence, immediate release, shared blocks)
and against a simulated pool: every sequence must read back exactly its own
tokens whatever forks and copies happened.  The C++ manager must then agree
with it exactly -- same slots, copies, tables, counts -- on random workloads.
"""
import numpy as np
import pytest

import oracle
import paged_kv_cache_401_b200 as pk
from oracle.paging import BLOCK, POISON, ToyBlockManager


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_401_b200 import build
    build.build()


# ---------------------------------------------------------------- pins of the restatement
class _Pool:
    """Simulated block contents: block -> 16 token labels."""

    def __init__(self, n):
        self.data = {b: [None] * BLOCK for b in range(n)}

    def copy(self, src, dst):
        self.data[dst] = list(self.data[src])

    def write(self, slot, label):
        self.data[slot // BLOCK][slot % BLOCK] = label

    def read(self, table, n):
        return [self.data[table[p // BLOCK]][p % BLOCK] for p in range(n)]


def _check_invariants(m: ToyBlockManager, nb: int):
    refs = [0] * nb
    for t in m.tables.values():
        for b in t:
            refs[b] += 1
    assert refs == m.ref                                     # counts = references
    assert sorted(m.free) == [b for b in range(nb) if m.ref[b] == 0]
    for s, t in m.tables.items():                            # at most one partly used block
        assert len(t) == -(-m.lens[s] // BLOCK)
        assert len(t) * BLOCK - m.lens[s] < BLOCK


def test_toy_manager_views_survive_forks_and_copies():
    rng = np.random.default_rng(0)
    nb = 96
    m, pool = ToyBlockManager(nb, 12, 40), _Pool(nb)
    truth = {}                                               # seq -> list of labels
    label = 0
    for step in range(400):
        live = list(m.tables)
        op = rng.integers(0, 10)
        if op == 0 and len(live) < 12:
            s = m.add_sequence()
            truth[s] = []
        elif op == 1 and live and len(live) < 12:
            p = int(rng.choice(live))
            c = m.fork(p)
            truth[c] = list(truth[p])
        elif op == 2 and len(live) > 1:
            s = int(rng.choice(live))
            m.free_sequence(s)
            del truth[s]
        elif live:
            s = int(rng.choice(live))
            if m.blocks_needed([s]) > len(m.free) or (m.lens[s] // BLOCK) >= 40:
                continue
            slot, cp = m.append_token(s)
            if cp:
                pool.copy(*cp)
            pool.write(slot, label)
            truth[s].append(label)
            label += 1
        _check_invariants(m, nb)
        for s, t in m.tables.items():
            assert pool.read(t, m.lens[s]) == truth[s]
    for s in list(m.tables):
        m.free_sequence(s)
    assert sorted(m.free) == list(range(nb))                 # everything released


def test_toy_manager_slots_match_closed_form():
    m = ToyBlockManager(64, 2, 16)
    s = m.add_sequence()
    slots = [m.append_token(s)[0] for _ in range(70)]
    table = np.array([m.export()[0][s]], dtype=np.int32)
    want = oracle.slot_mapping(table, np.zeros(70, np.int32), np.arange(70, dtype=np.int32))
    assert slots == want.tolist()


def test_toy_fork_then_append_copies_only_partial_shared_block():
    m = ToyBlockManager(16, 4, 8)
    a = m.add_sequence()
    for _ in range(20):                                      # 1 full block + 4 tokens
        m.append_token(a)
    b = m.fork(a)
    assert m.ref[m.tables[a][0]] == 2 and m.ref[m.tables[a][1]] == 2
    _, cp = m.append_token(b)                                # b writes into the shared partial block
    assert cp == (m.tables[a][1], m.tables[b][1])
    _, cp2 = m.append_token(a)                               # a's block is private again
    assert cp2 is None
    assert m.tables[a][0] == m.tables[b][0]                  # the full block stays shared


# ---------------------------------------------------------------- C++ manager == restatement
def _same(cpp: pk.BlockManager, toy: ToyBlockManager, nb: int):
    table, lens = cpp.export()
    t2, l2 = toy.export()
    assert (table == np.array(t2, dtype=np.int32)).all()
    assert lens.tolist() == l2
    assert cpp.num_free_blocks == len(toy.free)
    assert [cpp.refcount(b) for b in range(nb)] == toy.ref


@pytest.mark.parametrize("seed", range(6))
def test_cpp_manager_matches_restatement(seed):
    rng = np.random.default_rng(100 + seed)
    nb, ms, mb = 80, 10, 24
    cpp, toy = pk.BlockManager(nb, ms, mb), ToyBlockManager(nb, ms, mb)
    for step in range(300):
        live = sorted(toy.tables)
        op = rng.integers(0, 12)
        if op == 0 and len(live) < ms:
            assert cpp.add_sequence() == toy.add_sequence()
        elif op == 1 and live and len(live) < ms:
            p = int(rng.choice(live))
            assert cpp.fork(p) == toy.fork(p)
        elif op == 2 and live:
            s = int(rng.choice(live))
            cpp.free_sequence(s)
            toy.free_sequence(s)
        elif live:
            # a batch: several sequences, some more than once, in random order
            ids = rng.choice(live, size=int(rng.integers(1, 9))).astype(np.int32)
            too_long = any(toy.lens[s] + int((ids == s).sum()) > mb * BLOCK for s in set(ids))
            if too_long or toy.blocks_needed(ids.tolist()) > len(toy.free):
                with pytest.raises(pk.KvError) as e:
                    cpp.append_slots(ids)
                assert e.value.status == pk.KV_ERR_OUT_OF_BLOCKS
            else:
                slots, copies = cpp.append_slots(ids)
                want = [toy.append_token(int(s)) for s in ids]
                assert slots.tolist() == [w[0] for w in want]
                assert copies == [w[1] for w in want if w[1] is not None]
        _same(cpp, toy, nb)


def test_cpp_manager_errors():
    m = pk.BlockManager(2, 2, 1)
    with pytest.raises(pk.KvError):
        m.free_sequence(0)                                   # not live
    a = m.add_sequence()
    b = m.add_sequence()
    with pytest.raises(pk.KvError) as e:
        m.add_sequence()                                     # max_seqs live
    assert e.value.status == pk.KV_ERR_OUT_OF_BLOCKS
    m.append_slots([a] * 16)
    with pytest.raises(pk.KvError):
        m.append_slots([a])                                  # past max_blocks_per_seq
    m.append_slots([b])
    table, lens = m.export()
    assert lens.tolist() == [16, 1] and table[0, 0] == 0 and table[1, 0] == 1
    m.free_sequence(a)
    assert m.num_free_blocks == 1 and m.refcount(0) == 0
    assert (m.export()[0][0] == POISON).all()
