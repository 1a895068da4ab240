"""Seeded synthetic inputs for paged GQA decode -- shared by tests and bench.

This module draws inputs and lays out block tables.  It holds none of the
attention arithmetic: the CUDA path and the CPU oracle each compute slots,
cache writes, scores and outputs on their own from what is generated here.

Recipe (all draws from one ``torch.Generator`` on the CPU, seeded per
workload with 401 + the workload's index in ``WORKLOADS``):
  1. context lengths (fixed, or integers uniform in an inclusive range);
  2. q ~ N(0, 1), [B][Hq][D];
  3. outlier channels of K, where a workload has them (a seeded choice of
     channels per KV head, multiplied by 20 before rounding);
  4. K ~ N(0, 1) then V ~ N(0, 1), each as one contiguous [tokens][Hkv][D]
     array holding every sequence's tokens in logical order (sequence b at
     rows seq_offsets[b] .. + L_b), drawn sequence by sequence in chunks of
     65536 rows; a shared prefix, where a workload has one, is drawn first
     and copied into each sharing sequence;
  5. a random permutation of the physical block ids, dealt to the sequences'
     logical blocks in order (shared prefix blocks first).
Values are rounded to the stored dtype (fp32 or bf16, round to nearest even)
before either side sees them.  Context lengths count the newly appended
token: position L_b - 1 of each sequence is the token a decode step appends,
positions 0 .. L_b - 2 are the history already in the cache.
Block-table entries past a sequence's last logical block hold POISON_BLOCK,
an out-of-range id no correct reader dereferences.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_SIZE = 16
POISON_BLOCK = 2**31 - 1


@dataclass(frozen=True)
class Spec:
    name: str
    index: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    kv_dtype: str            # "f32" | "bf16" | "fp8" | "int8" | "int4" (quantised pools are fed
                             # bf16 sources)
    q_dtype: str             # "f32" | "bf16"
    lens: tuple              # ("fixed", (L0, L1, ...)) or ("uniform", lo, hi)
    scale: float
    num_blocks: int | None = None      # None: exactly the blocks the sequences need (+ slack)
    slack_blocks: int = 0
    shared_prefix_seqs: int = 0        # number of sequences sharing one prefix
    shared_prefix_tokens: int = 0
    shared_prefix_lens: tuple | None = None   # ("uniform", lo, hi) for the sharing sequences
    outlier_channels: int = 0
    outlier_factor: float = 20.0

    @property
    def seed(self) -> int:
        return 401 + self.index

    @property
    def source_dtype(self) -> str:
        return "bf16" if self.kv_dtype in ("fp8", "int8", "int4", "kivi4") else self.kv_dtype


WORKLOADS = {
    "tiny": Spec("tiny", 0, batch=2, num_q_heads=4, num_kv_heads=1, head_dim=64,
                 kv_dtype="f32", q_dtype="f32", lens=("fixed", (38, 101)), scale=1.0 / 8.0,
                 num_blocks=32),
    "llama": Spec("llama", 1, batch=32, num_q_heads=32, num_kv_heads=8, head_dim=128,
                  kv_dtype="bf16", q_dtype="bf16", lens=("fixed", (4096,) * 32),
                  scale=1.0 / math.sqrt(128.0), num_blocks=8192),
    "ragged": Spec("ragged", 2, batch=256, num_q_heads=32, num_kv_heads=8, head_dim=128,
                   kv_dtype="bf16", q_dtype="bf16", lens=("uniform", 16, 8192),
                   scale=1.0 / math.sqrt(128.0), slack_blocks=256, shared_prefix_seqs=64,
                   shared_prefix_tokens=2048, shared_prefix_lens=("uniform", 2049, 8192)),
    "long": Spec("long", 3, batch=4, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 kv_dtype="bf16", q_dtype="bf16", lens=("fixed", (131072,) * 4),
                 scale=1.0 / math.sqrt(128.0), num_blocks=32768, outlier_channels=4),
    "fp8": Spec("fp8", 4, batch=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                kv_dtype="fp8", q_dtype="bf16", lens=("uniform", 1024, 16384),
                scale=1.0 / math.sqrt(128.0)),
    "int8": Spec("int8", 5, batch=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 kv_dtype="int8", q_dtype="bf16", lens=("uniform", 1024, 16384),
                 scale=1.0 / math.sqrt(128.0)),
    "int4": Spec("int4", 6, batch=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 kv_dtype="int4", q_dtype="bf16", lens=("uniform", 1024, 16384),
                 scale=1.0 / math.sqrt(128.0)),
    "kivi": Spec("kivi", 7, batch=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 kv_dtype="kivi4", q_dtype="bf16", lens=("uniform", 1024, 16384),
                 scale=1.0 / math.sqrt(128.0)),
}


@dataclass
class Inputs:
    spec: Spec
    context_lens: np.ndarray          # int32 [B], includes the appended token
    seq_offsets: np.ndarray           # int64 [B], first row of each sequence in k/v
    q: torch.Tensor                   # [B][Hq][D], q dtype (CPU)
    k: torch.Tensor                   # [tokens][Hkv][D], source dtype (CPU)
    v: torch.Tensor
    block_table: np.ndarray           # int32 [B][max_blocks_per_seq]
    num_blocks: int
    # rows of k/v whose slot must be written before the first step (history),
    # shared prefix rows written once only; and the (seq, position) of each
    fill_rows: np.ndarray = field(default=None)
    fill_seq_ids: np.ndarray = field(default=None)
    fill_positions: np.ndarray = field(default=None)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max())

    @property
    def append_rows(self) -> np.ndarray:
        """Row in k/v of each sequence's appended token (position L_b - 1)."""
        return self.seq_offsets + self.context_lens.astype(np.int64) - 1

    @property
    def append_positions(self) -> np.ndarray:
        return (self.context_lens - 1).astype(np.int32)


def _dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _randn(gen: torch.Generator, shape, dtype: torch.dtype, chunk_rows: int = 1 << 16):
    """N(0,1) draws, rounded to `dtype`, generated in row chunks (bounded memory)."""
    out = torch.empty(shape, dtype=dtype)
    rows = shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                                 dtype=torch.float32).to(dtype)
    return out


def _draw_lens(spec_lens, n: int, gen: torch.Generator) -> np.ndarray:
    if spec_lens[0] == "fixed":
        vals = spec_lens[1]
        assert len(vals) == n
        return np.asarray(vals, dtype=np.int32)
    _, lo, hi = spec_lens
    return torch.randint(lo, hi + 1, (n,), generator=gen).numpy().astype(np.int32)


def make_inputs(name_or_spec, batch: int | None = None, lens_override=None) -> Inputs:
    """Generate one workload's inputs on the CPU.

    ``batch`` / ``lens_override`` shrink a workload for quick checks (same
    head shapes, dtypes and structure); the recipe above is unchanged.
    """
    spec = WORKLOADS[name_or_spec] if isinstance(name_or_spec, str) else name_or_spec
    gen = torch.Generator(device="cpu").manual_seed(spec.seed)
    B = spec.batch if batch is None else batch
    nshare = min(spec.shared_prefix_seqs, B)
    # 1. context lengths (the sharing sequences are the first `nshare`)
    if lens_override is not None:
        lens = np.asarray(lens_override, dtype=np.int32)
        assert lens.shape == (B,)
    else:
        if spec.lens[0] == "fixed" and B != spec.batch:
            lens = np.asarray(spec.lens[1][:B], dtype=np.int32)
        else:
            lens = _draw_lens(spec.lens, B, gen)
        if nshare:
            lens[:nshare] = _draw_lens(spec.shared_prefix_lens, nshare, gen)
    if nshare:
        assert (lens[:nshare] > spec.shared_prefix_tokens).all()
    Hq, Hkv, D = spec.num_q_heads, spec.num_kv_heads, spec.head_dim
    sdt = _dtype(spec.source_dtype)
    # 2. q
    q = _randn(gen, (B, Hq, D), _dtype(spec.q_dtype))
    # 3. outlier channels of K (a seeded choice per KV head)
    chans = None
    if spec.outlier_channels:
        chans = [torch.randperm(D, generator=gen)[:spec.outlier_channels] for _ in range(Hkv)]
    # 4. K then V: the shared prefix (drawn once), then every sequence's own rows
    P = spec.shared_prefix_tokens if nshare else 0
    seq_offsets = np.zeros(B, dtype=np.int64)
    seq_offsets[1:] = np.cumsum(lens.astype(np.int64))[:-1]
    total = int(lens.astype(np.int64).sum())
    k = torch.empty((total, Hkv, D), dtype=sdt)
    v = torch.empty((total, Hkv, D), dtype=sdt)
    for dst, outliers in ((k, chans), (v, None)):
        def draw(rows, _out=outliers):
            x = torch.randn((rows, Hkv, D), generator=gen, dtype=torch.float32)
            if _out is not None:
                for h in range(Hkv):
                    x[:, h, _out[h]] *= spec.outlier_factor
            return x.to(sdt)
        prefix = draw(P) if P else None
        for s in range(B):
            o, n = int(seq_offsets[s]), int(lens[s])
            start = 0
            if s < nshare:
                dst[o:o + P] = prefix
                start = P
            for r0 in range(start, n, 1 << 16):
                r1 = min(n, r0 + (1 << 16))
                dst[o + r0:o + r1] = draw(r1 - r0)
    # 5. block table from a permutation of physical blocks
    nblk = (lens.astype(np.int64) + BLOCK_SIZE - 1) // BLOCK_SIZE
    shared_blocks = P // BLOCK_SIZE
    needed = int(nblk.sum()) - max(nshare - 1, 0) * shared_blocks
    NB = spec.num_blocks if (spec.num_blocks is not None and batch is None
                             and lens_override is None) else needed + spec.slack_blocks
    assert NB >= needed, (NB, needed)
    perm = torch.randperm(NB, generator=gen).numpy().astype(np.int32)
    MB = int(nblk.max())
    table = np.full((B, MB), POISON_BLOCK, dtype=np.int32)
    cursor = 0
    if nshare:
        shared_ids = perm[:shared_blocks]
        cursor = shared_blocks
    for s in range(B):
        start = 0
        if s < nshare:
            table[s, :shared_blocks] = shared_ids
            start = shared_blocks
        cnt = int(nblk[s]) - start
        table[s, start:start + cnt] = perm[cursor:cursor + cnt]
        cursor += cnt
    # history rows to write before the first step (shared prefix once)
    rows, sids, poss = [], [], []
    for s in range(B):
        o, n = int(seq_offsets[s]), int(lens[s])
        first = P if (0 < s < nshare) else 0
        pos = np.arange(first, n - 1, dtype=np.int32)
        rows.append(o + pos.astype(np.int64))
        sids.append(np.full(len(pos), s, dtype=np.int32))
        poss.append(pos)
    return Inputs(spec=spec, context_lens=lens, seq_offsets=seq_offsets, q=q, k=k, v=v,
                  block_table=table, num_blocks=NB,
                  fill_rows=np.concatenate(rows) if rows else np.zeros(0, np.int64),
                  fill_seq_ids=np.concatenate(sids) if sids else np.zeros(0, np.int32),
                  fill_positions=np.concatenate(poss) if poss else np.zeros(0, np.int32))


def storage_view(t: torch.Tensor) -> np.ndarray:
    """A CPU tensor's stored bits as numpy (bf16 -> uint16 bits, fp32 as is)."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.uint8:
        return t.numpy()
    raise TypeError(t.dtype)


@dataclass
class KiviLayout:
    """Where a KIVI cache keeps each history token (positions 0 .. L-2 of every
    sequence; position L-1 is the step's new token): full blocks, 16 rows each,
    and the rows of the incomplete last block, which stay unquantised."""
    block_rows: np.ndarray     # int64 [n][16]: rows of k/v (token order) of each full block
    block_ids: np.ndarray      # int32 [n]: the physical block each one goes to
    res_seq: np.ndarray        # int32 [m]: sequence of each residual row
    res_slot: np.ndarray       # int32 [m]: its row in the sequence's residual (0..15)
    res_rows: np.ndarray       # int64 [m]: its row of k/v


def kivi_layout(inp: Inputs) -> KiviLayout:
    rows, ids, rs, rsl, rr = [], [], [], [], []
    for b in range(inp.q.shape[0]):
        hist = int(inp.context_lens[b]) - 1
        full = hist // BLOCK_SIZE
        base = int(inp.seq_offsets[b])
        for j in range(full):
            rows.append(base + j * BLOCK_SIZE + np.arange(BLOCK_SIZE))
            ids.append(int(inp.block_table[b, j]))
        n = hist - full * BLOCK_SIZE
        rs.extend([b] * n)
        rsl.extend(range(n))
        rr.extend(base + full * BLOCK_SIZE + np.arange(n))
    return KiviLayout(
        block_rows=np.array(rows, dtype=np.int64).reshape(-1, BLOCK_SIZE),
        block_ids=np.array(ids, dtype=np.int32),
        res_seq=np.array(rs, dtype=np.int32), res_slot=np.array(rsl, dtype=np.int32),
        res_rows=np.array(rr, dtype=np.int64))
