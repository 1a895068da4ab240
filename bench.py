#!/usr/bin/env python
"""Benchmark: paged GQA decode on B200 -- effective KV-read HBM GB/s and decode steps/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama]
                    [--partition P] [--impl reference]

One step = the whole decode hot path for one layer over one batch: slot
computation and cache write of every sequence's new token, split-K paged
decode attention, log-sum-exp merge.  The default workload is the
Llama-3-8B-shaped batch (32 sequences x 4096 tokens, 32 query / 8 KV heads,
head_dim 128, bf16, 16-token blocks in a randomly permuted 8192-block pool).

value    = KV bytes read per step x steps / device time, inputs resident in HBM;
e2e      = the same metric through the binding from host memory: each step
           copies one pinned buffer holding q, the new K/V rows, the block
           table and the context lengths host->device, runs the step on views
           of it, and copies the output device->host, inside the timed region;
roofline = the decode call (decode + merge kernels) against the measured HBM
           copy bandwidth: per-call time from the timed steps when a step is
           one decode call (fused append, the default), else from K decode
           calls back to back timed the same way after the steps;
timing   = --regions regions of exactly K steps, each bracketed by a barrier
           and a synchronize; value and e2e report the median region and the
           line lists every region (a 20-step region lasts ~2 ms);
config   = the workload only, the same for both arms; the split this arm chose
           (ranges, how the new tokens are appended) is under ``split``;
cpu_baseline = the double-precision CPU oracle on a bounded sample (rank 0).
``--impl reference`` times that oracle alone as the reference arm.
With N > 1 (torchrun), every rank runs an independent replica on its own GPU
(the workload needs no exchange); value is the sum over ranks / the slowest rank.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs, storage_view  # noqa: E402

# ncu summary of each workload's decode call (DRAM bytes per call, with the
# hash of the decode source it was captured on)
PROFILE_SUMMARIES = {
    "llama": "paged_decode_llama_b32x4k.md",
    "ragged": "paged_decode_ragged_b256.md",
    "long": "paged_decode_long_b4x128k.md",
    "fp8": "paged_decode_fp8_b64.md",
    "int8": "paged_decode_int8_b64.md",
    "int4": "paged_decode_int4_b64.md",
    "kivi": "paged_decode_kivi_b64.md",
}
DECODE_SRC = os.path.join(ROOT, "paged_kv_cache_401_b200", "csrc", "decode.cu")


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def dist_init(world: int, backend: str, device=None):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        kw = {"backend": backend, "timeout": datetime.timedelta(seconds=120)}
        if device is not None and backend == "nccl":
            kw["device_id"] = device
        dist.init_process_group(**kw)


def reduce_over_ranks(x: float, op: str, device=None) -> float:
    """max/sum of a scalar over ranks (identity when not distributed)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------- clocks
def gpu_id(device) -> str:
    """nvidia-smi id of a torch device (its UUID, robust to CUDA_VISIBLE_DEVICES)."""
    uuid = getattr(torch.cuda.get_device_properties(device), "uuid", None)
    if uuid is not None:
        u = str(uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    return str(device.index)


class ClockSampler:
    """nvidia-smi clocks, power and throttle reasons sampled every 20 ms; the
    summary keeps the samples taken between mark_start() and mark_end()."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def __enter__(self):
        import tempfile
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        # nvidia-smi takes a moment to start: wait (up to 5 s) for its first sample,
        # so that a short timed region is sampled too
        t_end = time.time() + 5.0
        while time.time() < t_end and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        import datetime
        if self.proc is None or self.path is None or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                t = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((t, float(parts[2]), float(parts[3]), float(parts[4]), parts[5:10]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        inside = rows
        if self.t0 is not None and self.t1 is not None:
            # a sample describes the interval before it: keep those ending in the region
            inside = [r for r in rows if self.t0 < r[0] <= self.t1 + 0.02]
            if not inside:   # region shorter than the interval: the first sample after it
                later = [r for r in rows if r[0] > self.t0]
                inside = later[:1] or rows[-1:]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for *_, r in inside for i in range(4)
                          if r[i + 1].lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in inside])),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "power_w": float(np.median([r[3] for r in inside])),
                "samples": len(inside), "interval_ms": 20}


# ---------------------------------------------------------------- workload bytes
def kv_row_bytes(spec) -> int:
    """Bytes of one stored K or V row of one KV head (plus its fp32 scale for
    an 8-bit cache)."""
    if spec.kv_dtype == "int4":    # two codes per byte + fp32 (scale, zero point)
        return spec.head_dim // 2 + 8
    if spec.kv_dtype == "kivi4":   # full blocks, per token (see kivi_bytes)
        return spec.head_dim // 2 + (spec.head_dim + 16) * 8 // 16
    elem = {"f32": 4, "bf16": 2, "fp8": 1, "int8": 1}[spec.kv_dtype]
    return spec.head_dim * elem + (4 if spec.kv_dtype in ("fp8", "int8") else 0)


def kivi_bytes(spec, lens) -> int:
    """KIVI bytes of contexts `lens`: each full block is 16 rows of 64-byte K and V
    codes plus 1152 bytes of parameters per kv head; the rest are bf16 rows."""
    lens = np.asarray(lens, dtype=np.int64)
    full, rest = lens // 16, lens % 16
    per_block = 2 * 16 * spec.head_dim // 2 + (spec.head_dim + 16) * 8
    return int((full * per_block + rest * 2 * spec.head_dim * 2).sum()) * spec.num_kv_heads


def kv_bytes_per_step(inp) -> int:
    """Algorithmic KV bytes one decode step reads: every context token's K and V
    row of every KV head (plus the fp32 per-row scales of an FP8 / INT8 cache)."""
    spec = inp.spec
    if spec.kv_dtype == "kivi4":
        return kivi_bytes(spec, inp.context_lens)
    tokens = int(inp.context_lens.astype(np.int64).sum())
    per_row = kv_row_bytes(spec)
    return tokens * spec.num_kv_heads * 2 * per_row


def unique_kv_bytes_per_step(inp) -> int:
    """KV bytes of distinct physical blocks read per step: a prefix shared by
    several sequences is one set of blocks in HBM (later readers may hit L2)."""
    spec = inp.spec
    nshare = min(spec.shared_prefix_seqs, inp.q.shape[0])
    if nshare <= 1:
        return kv_bytes_per_step(inp)
    per_row = kv_row_bytes(spec)
    dup = (nshare - 1) * spec.shared_prefix_tokens
    return kv_bytes_per_step(inp) - dup * spec.num_kv_heads * 2 * per_row


DATA = "synthetic (seeded N(0,1) q/K/V, random block permutation)"


def describe(inp, partition: int, query_tokens: int) -> dict:
    """The workload, the same for both arms (the implementation's own choices are not here)."""
    spec = inp.spec
    return {"workload": f"{spec.name}: paged GQA decode, batch {inp.q.shape[0]}, "
                        f"{spec.num_q_heads} q / {spec.num_kv_heads} kv heads, head_dim "
                        f"{spec.head_dim}, {spec.kv_dtype} KV, block 16, "
                        f"context {int(inp.context_lens.min())}..{int(inp.context_lens.max())}",
            "batch": int(inp.q.shape[0]), "max_context_len": inp.max_context_len,
            "num_q_heads": spec.num_q_heads, "num_kv_heads": spec.num_kv_heads,
            "head_dim": spec.head_dim, "block_size": 16, "num_blocks": inp.num_blocks,
            "kv_dtype": spec.kv_dtype,
            "partition_tokens": partition if partition else "0 (balanced over all SMs)",
            "l2": "inputs larger than L2 (KV read per step > 126 MB), no flush"
            if kv_bytes_per_step(inp) > 126e6 else "inputs fit in L2, not flushed",
            "parallelism": "replicas: one independent decode per GPU",
            "query_tokens": query_tokens}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def profiled_traffic(workload: str):
    """ncu DRAM bytes per decode call of a workload, if its committed summary
    was taken on the current decode kernel source (else None: no summary, or
    the kernel changed since).  Returns (bytes, summary file) or (None, None)."""
    name = PROFILE_SUMMARIES.get(workload)
    path = os.path.join(ROOT, "profiles", name) if name else None
    if path is None or not os.path.exists(path):
        return None, None
    kv = {}
    for line in open(path, encoding="utf-8"):
        if ":" in line and line.lstrip().startswith("- "):
            k, _, v = line.strip()[2:].partition(":")
            kv[k.strip()] = v.strip().strip("`")
    sha = hashlib.sha256(open(DECODE_SRC, "rb").read()).hexdigest()[:16]
    if kv.get("decode_source_sha256") != sha:
        return None, None
    try:
        return int(kv["dram_bytes_per_decode_call"]), "profiles/" + name
    except (KeyError, ValueError):
        return None, None


# ---------------------------------------------------------------- oracle (CPU) timing
def time_oracle(inp, max_seqs: int, repeats: int = 1):
    """Time the CPU oracle on the first `max_seqs` sequences; returns (GB/s, s, desc, cores)."""
    import oracle
    spec = inp.spec
    n = min(max_seqs, inp.q.shape[0])
    seqs = np.arange(n)
    q = storage_view(inp.q)[seqs]
    lens = inp.context_lens[seqs]
    args = dict(seq_offsets=inp.seq_offsets[seqs], lens=lens, scale=spec.scale,
                num_kv_heads=spec.num_kv_heads, q_dtype=spec.q_dtype)
    if spec.kv_dtype == "kivi4":
        ks, vs = [], []
        for b in seqs:
            a, L = int(inp.seq_offsets[b]), int(inp.context_lens[b])
            k64, v64 = oracle.kivi_sequence(inp.k[a:a + L].float().numpy(),
                                            inp.v[a:a + L].float().numpy())
            ks.append(k64), vs.append(v64)
        kv = dict(k=np.concatenate(ks), v=np.concatenate(vs), kv_dtype="f64")
        args["seq_offsets"] = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    elif spec.kv_dtype in ("fp8", "int8", "int4"):
        rows = slice(int(inp.seq_offsets[0]), int(inp.seq_offsets[n - 1] + lens[-1]))
        kc, ks = oracle.quantize_rows(inp.k[rows].float().numpy(), spec.kv_dtype)
        vc, vs = oracle.quantize_rows(inp.v[rows].float().numpy(), spec.kv_dtype)
        kv = dict(k=kc, v=vc, kv_dtype=spec.kv_dtype, k_scale=ks, v_scale=vs)
    else:
        kv = dict(k=storage_view(inp.k), v=storage_view(inp.v), kv_dtype=spec.kv_dtype)
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle.decode_attention(q, **kv, **args)
    dt = (time.perf_counter() - t0) / repeats
    per_row = kv_row_bytes(spec)
    nbytes = int(lens.astype(np.int64).sum()) * spec.num_kv_heads * 2 * per_row
    if spec.kv_dtype == "kivi4":
        nbytes = kivi_bytes(spec, lens)
    desc = (f"oracle (C, double, OpenMP) over {n} of {inp.q.shape[0]} sequences "
            f"({int(lens.sum())} tokens, {nbytes / 2**20:.0f} MiB of KV) x {repeats}")
    return nbytes / dt / 1e9, dt, desc, oracle.num_threads()


def run_reference(args, inp):
    rank, _, _ = dist_env()
    if rank != 0:
        return
    # calibrate: one sequence, then as many as fit ~90 s for the whole run
    _, t1, _, _ = time_oracle(inp, 1)
    budget = 90.0 / (args.steps + args.warmup)
    sample = int(max(1, min(inp.q.shape[0], budget // max(t1, 1e-6))))
    for _ in range(args.warmup):
        time_oracle(inp, sample)
    vals = []
    for _ in range(args.steps):
        v, dt, desc, cores = time_oracle(inp, sample)
        vals.append((v, dt))
    gbs = float(np.mean([v for v, _ in vals]))
    ms = float(np.mean([dt for _, dt in vals])) * 1e3
    line = {"metric": "paged GQA decode: effective KV-read HBM GB/s (% of peak), decode steps/s",
            "value": round(gbs, 3), "unit": "GB/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": DATA,
            "config": describe(inp, args.partition, 1),
            "cpu_baseline": {"value": round(gbs, 3), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(gbs, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def stage_kivi_on_device(inp, device):
    """A KIVI cache holding every sequence's history (all but its last token)
    through the library: full blocks quantised, the incomplete block's rows in
    the bf16 residual."""
    from paged_kv_cache_401_b200.cache import PagedKVCache
    from workloads import kivi_layout
    spec = inp.spec
    cache = PagedKVCache(inp.num_blocks, spec.num_kv_heads, spec.head_dim, "kivi4", device)
    res_k, res_v = cache.alloc_residual(inp.q.shape[0])
    lay = kivi_layout(inp)
    chunk = 4096
    for c0 in range(0, len(lay.block_ids), chunk):
        n = min(chunk, len(lay.block_ids) - c0)
        rows = torch.from_numpy(lay.block_rows[c0:c0 + n].reshape(-1))
        shape = (n, 16, spec.num_kv_heads, spec.head_dim)
        cache.kivi_fill(torch.from_numpy(lay.block_ids[c0:c0 + n]).to(device),
                        inp.k[rows].reshape(shape).to(device), inp.v[rows].reshape(shape).to(device))
    if len(lay.res_rows):
        rr = torch.from_numpy(lay.res_rows)
        sq, sl = torch.from_numpy(lay.res_seq).long(), torch.from_numpy(lay.res_slot).long()
        res_k[sq, :, sl] = inp.k[rr].to(device)
        res_v[sq, :, sl] = inp.v[rr].to(device)
    torch.cuda.synchronize(device)
    return cache, torch.from_numpy(inp.block_table).to(device)


def stage_on_device(inp, device, query_tokens: int = 1):
    """Fill the paged pool with every sequence's history (all but its last
    `query_tokens` tokens, which each step appends) through the library."""
    from paged_kv_cache_401_b200.cache import PagedKVCache
    spec = inp.spec
    if spec.kv_dtype == "kivi4":
        return stage_kivi_on_device(inp, device)
    cache = PagedKVCache(inp.num_blocks, spec.num_kv_heads, spec.head_dim, spec.kv_dtype,
                         device)
    bt = torch.from_numpy(inp.block_table).to(device)
    keep = inp.fill_positions < inp.context_lens[inp.fill_seq_ids] - query_tokens
    f_rows, f_sids, f_pos = (inp.fill_rows[keep], inp.fill_seq_ids[keep],
                             inp.fill_positions[keep])
    chunk = 1 << 17
    for c0 in range(0, len(f_rows), chunk):
        c1 = min(len(f_rows), c0 + chunk)
        rows = torch.from_numpy(f_rows[c0:c1])
        cache.append(bt, torch.from_numpy(f_sids[c0:c1]).to(device),
                     torch.from_numpy(f_pos[c0:c1]).to(device),
                     inp.k[rows].to(device), inp.v[rows].to(device))
    torch.cuda.synchronize(device)
    return cache, bt


def step_tokens(inp, query_tokens: int):
    """The tokens a step appends: the last `query_tokens` of every sequence
    (rows into inp.k / inp.v, sequence ids, positions), and the step's q:
    [B][Hq][D] for one token, else [B][Q][Hq][D] drawn with seed 401 + 100."""
    B = inp.q.shape[0]
    Q = query_tokens
    pos = (inp.context_lens[:, None] - Q + np.arange(Q)[None, :]).astype(np.int32)   # [B][Q]
    rows = (inp.seq_offsets[:, None] + pos).reshape(-1)
    sids = np.repeat(np.arange(B, dtype=np.int32), Q)
    if Q == 1:
        q = inp.q
    else:
        g = torch.Generator(device="cpu").manual_seed(401 + 100)
        q = torch.randn((B, Q) + tuple(inp.q.shape[1:]), generator=g).to(inp.q.dtype)
    return torch.from_numpy(rows), sids, pos.reshape(-1), q


def run_gpu(args, inp):
    import paged_kv_cache_401_b200 as pk
    rank, local, world = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl", device)
    spec = inp.spec
    B = inp.q.shape[0]
    Q = args.query_tokens
    cache, bt = stage_on_device(inp, device, Q)
    lens = torch.from_numpy(inp.context_lens).to(device)
    app, sids_np, pos_np, q_host = step_tokens(inp, Q)
    q = q_host.to(device)
    k_new, v_new = inp.k[app].to(device), inp.v[app].to(device)
    seq_ids = torch.from_numpy(sids_np).to(device)
    positions = torch.from_numpy(pos_np).to(device)
    slots = torch.empty(B * Q, dtype=torch.int64, device=device)
    out = torch.empty_like(q)
    P = args.partition
    ranges = pk.paged_decode_num_ranges(cache.desc, B, spec.num_q_heads, inp.max_context_len, P)
    ws_bytes = pk.paged_attention_workspace_bytes(cache.desc, B, spec.num_q_heads, Q,
                                                  inp.max_context_len, P)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    kivi = spec.kv_dtype == "kivi4"   # its step always appends inside the decode call
    fused = (args.append == "fused" and Q == 1) or kivi
    # separate: slot mapping, cache write, decode, merge; fused: decode (+append), merge;
    # KIVI: append (+ block flush), decode, merge
    launches_per_step = 3 if kivi else (2 if fused else 4)

    def append():
        if not fused:   # the fused call appends inside the decode
            cache.append(bt, seq_ids, positions, k_new, v_new, slots=slots)

    def attend(qq, tbl, ln):
        if Q == 1:
            cache.decode(qq, tbl, ln, inp.max_context_len, spec.scale, out=out,
                         partition_tokens=P, workspace=ws)
        else:
            cache.attend(qq, tbl, ln, inp.max_context_len, spec.scale, out=out,
                         partition_tokens=P, workspace=ws)

    def fused_call(qq, kk, vv, tbl, ln, o):
        if kivi:
            cache.kivi_decode(qq, tbl, ln, inp.max_context_len, spec.scale, kk, vv, out=o,
                              partition_tokens=P, workspace=ws)
        else:
            cache.decode_append(qq, kk, vv, tbl, ln, inp.max_context_len, spec.scale, out=o,
                                partition_tokens=P, workspace=ws)

    def decode():
        if fused:
            fused_call(q, k_new, v_new, bt, lens, out)
        else:
            attend(q, bt, lens)

    def timed_regions(body, n_regions):
        """n_regions back-to-back regions of exactly args.steps calls of body,
        each bracketed by a barrier and a device synchronize, timed with CUDA
        events on the launching stream; returns the ms of each region."""
        ms = []
        for _ in range(n_regions):
            barrier(device)
            torch.cuda.synchronize(device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                body()
            e1.record(stream)
            torch.cuda.synchronize(device)
            barrier(device)
            ms.append(e0.elapsed_time(e1))
        return ms

    def whole_step():
        append()
        decode()

    # ---- warm-up and timed region.  The clock sampler runs from before the
    # warm-up, so the timed steps follow the warm-up with no idle gap.  The
    # timed region is args.regions regions of K whole steps back to back (the
    # kernels of consecutive calls overlap their launches); the line reports
    # the median region and lists all.  When the step is one decode call
    # (fused append), the roofline takes its per-call time from these same
    # regions; otherwise K decode calls alone are timed the same way after them.
    with ClockSampler(gpu_id(device)) as clk:
        for _ in range(args.warmup):
            whole_step()
        torch.cuda.synchronize(device)
        err0 = cache.errors()
        clk.mark_start()
        step_ms = timed_regions(whole_step, args.regions)
        decode_ms_regions = step_ms if fused else timed_regions(decode, args.regions)
        clk.mark_end()
    errs = cache.errors()
    # per region: the slowest rank; then the median region
    step_ms = [reduce_over_ranks(m, "max", device) for m in step_ms]
    decode_ms_regions = [reduce_over_ranks(m, "max", device) for m in decode_ms_regions]
    elapsed_ms = float(np.median(step_ms))
    decode_ms = float(np.median(decode_ms_regions)) / args.steps

    # ---- e2e: the step's inputs live in ONE pinned host buffer (q, new K/V rows,
    # block table, context lengths, each 256-byte aligned) copied to a device
    # staging buffer every step; the calls take views of it; the output is
    # copied back every step.  As a serving loop would, the copies are double-
    # buffered on their own streams: step i+1's inputs go in and step i-1's
    # output comes out while step i computes.  Every copy is inside the timed
    # region, which ends when the last output has reached the host.
    parts = [q_host, inp.k[app], inp.v[app], torch.from_numpy(inp.block_table),
             torch.from_numpy(inp.context_lens)]
    offs, total = [], 0
    for t in parts:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_stage = torch.zeros(total, dtype=torch.uint8).pin_memory()
    for t, o in zip(parts, offs):
        nb = t.numel() * t.element_size()
        h_stage[o:o + nb].copy_(t.contiguous().view(-1).view(torch.uint8))
    d_stage = [torch.empty(total, dtype=torch.uint8, device=device) for _ in range(2)]
    views = [[d[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
              for t, o in zip(parts, offs)] for d in d_stage]
    outs = [torch.empty_like(q) for _ in range(2)]
    h_outs = [torch.empty_like(q_host).pin_memory() for _ in range(2)]
    h2d = total
    d2h = h_outs[0].numel() * h_outs[0].element_size()
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "done", "out")}

    def e2e_step(i):
        b = i % 2
        e_q, e_k, e_v, e_bt, e_lens = views[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev["done"][b])          # step i-2 no longer reads this buffer
            d_stage[b].copy_(h_stage, non_blocking=True)
            ev["in"][b].record(s_in)
        stream.wait_event(ev["in"][b])
        stream.wait_event(ev["out"][b])             # step i-2's output has been read back
        if fused:
            fused_call(e_q, e_k, e_v, e_bt, e_lens, outs[b])
        else:
            cache.append(e_bt, seq_ids, positions, e_k, e_v, slots=slots)
            if Q == 1:
                cache.decode(e_q, e_bt, e_lens, inp.max_context_len, spec.scale, out=outs[b],
                             partition_tokens=P, workspace=ws)
            else:
                cache.attend(e_q, e_bt, e_lens, inp.max_context_len, spec.scale, out=outs[b],
                             partition_tokens=P, workspace=ws)
        ev["done"][b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["done"][b])
            h_outs[b].copy_(outs[b], non_blocking=True)
            ev["out"][b].record(s_out)

    def e2e_run(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(n):
            e2e_step(i)
        stream.wait_event(ev["out"][(n - 1) % 2])
        e1.record(stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1)

    e2e_run(max(2, args.warmup))
    e2e_regions = []
    for _ in range(args.regions):
        barrier(device)
        e2e_regions.append(reduce_over_ranks(e2e_run(args.steps), "max", device))
    barrier(device)

    nbytes = kv_bytes_per_step(inp)
    max_ms = elapsed_ms
    max_e2e_ms = float(np.median(e2e_regions))
    max_decode_ms = decode_ms
    total_bytes = reduce_over_ranks(nbytes * args.steps, "sum", device)
    value = total_bytes / (max_ms * 1e-3) / 1e9
    e2e_value = total_bytes / (max_e2e_ms * 1e-3) / 1e9
    clocks = clk.summary()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        _, t1, _, _ = time_oracle(inp, 1)      # calibrate to ~10 s of CPU work
        reps = int(max(1, min(5, 10.0 // max(t1 * args.reference_seqs, 1e-6))))
        gbs, dt, desc, cores = time_oracle(inp, args.reference_seqs, reps)
        cpu = {"value": round(gbs, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": desc}
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    peak, peak_kind = measured_peak()
    achieved = nbytes / (max_decode_ms * 1e-3) / 1e9
    default_shape = (args.batch is None and args.context is None and Q == 1 and P == 0)
    traffic, traffic_src = profiled_traffic(args.workload) if default_shape else (None, None)
    line = {
        "metric": "paged GQA decode: effective KV-read HBM GB/s (% of peak), decode steps/s",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 5),
        "steps_per_s": round(args.steps / (max_ms * 1e-3), 1),
        "pct_of_peak": round(100 * value / world / peak, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": spec.kv_dtype if spec.kv_dtype != "fp8" else "fp8_e4m3",
        "data": DATA,
        "config": describe(inp, P, Q),
        "split": {"num_ranges": ranges,
                  "append": ("KIVI residual append (+ block flush) in the decode call" if kivi
                             else "fused into the decode call" if fused
                             else "separate slot-mapping and cache-write calls")},
        "timing": {"regions": args.regions,
                   "region": f"{args.steps} steps back to back, barrier + synchronize on "
                             "both sides, CUDA events on the launching stream",
                   "reported": "median region (each region: the slowest rank)",
                   "launches_per_region": launches_per_step * args.steps,
                   "ms_per_step_regions": [round(m / args.steps, 5) for m in step_ms],
                   "spread_pct": round(100 * (max(step_ms) - min(step_ms)) / elapsed_ms, 2)},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "ms_per_step": round(max_e2e_ms / args.steps, 5),
                "ms_per_step_regions": [round(m / args.steps, 5) for m in e2e_regions]},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "traffic_source": traffic_src,
                     "kernel": "paged_decode_attention (decode + merge kernels, one call)",
                     "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": nbytes,
                     "ms_per_launch": round(max_decode_ms, 5),
                     "timed_in": "the timed steps (each step is one decode call)" if fused
                                 else "decode calls alone, timed after the steps"},
        "cpu_baseline": cpu,
        "gpu_launches": launches_per_step * args.steps,
        "unique_kv": {"bytes_per_step": unique_kv_bytes_per_step(inp),
                      "value": round(unique_kv_bytes_per_step(inp) * args.steps * world
                                     / (max_ms * 1e-3) / 1e9, 2), "unit": "GB/s"},
        "clocks": clocks,
        "device_errors": {"warmup": err0, "timed": errs},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--regions", type=int, default=5,
                    help="timed regions of --steps steps each; the median region is reported")
    ap.add_argument("--workload", default="llama", choices=sorted(WORKLOADS))
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (same head shapes and dtypes)")
    ap.add_argument("--context", type=int, default=None,
                    help="override the context lengths: every sequence this many tokens")
    ap.add_argument("--partition", type=int, default=0,
                    help="max tokens per consumer range (0 = balanced over all SMs)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--reference-seqs", type=int, default=8,
                    help="sequences in the oracle's bounded sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--append", default="fused", choices=["separate", "fused"],
                    help="how a decode step stores its new tokens: separate slot-mapping and "
                         "cache-write calls, or fused into the decode call (one query token)")
    ap.add_argument("--query-tokens", type=int, default=1,
                    help="query tokens per sequence per step (1 = decode; >1 = speculative "
                         "verification of that many appended tokens)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps, reported as run
    lens = None
    if args.context is not None:
        batch = args.batch if args.batch is not None else WORKLOADS[args.workload].batch
        lens = [args.context] * batch
    inp = make_inputs(args.workload, batch=args.batch, lens_override=lens)
    if args.impl == "reference":
        run_reference(args, inp)
    else:
        run_gpu(args, inp)


if __name__ == "__main__":
    main()
