"""Pins for the CPU oracle: each checks it against something other than itself.

* printed values on the pages (tests/golden/kv_sizes.txt);
* library routines (torch scaled_dot_product_attention in float64, torch's
  float8_e4m3fn conversion);
* hand-computed INT8 and INT4 rows with exact binary scales, a brute-force
  nearest-integer search for the INT8 codes and an exact-rational re-derivation
  of the INT4 scale, zero point and codes;
* closed forms and special cases (length 1, identical keys, dominant key,
  weights summing to one, key-order invariance);
* brute force on tiny inputs (numpy, one head at a time) and an independent
  incremental restatement of the pages' paged-cache toy.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- KV size
def _kv_rows():
    rows = []
    with open(os.path.join(GOLDEN, "kv_sizes.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            nums = [int(x) for x in parts[:7]]
            rows.append((*nums, float(parts[7]), " ".join(parts[8:])))
    return rows


@pytest.mark.parametrize("row", _kv_rows(), ids=lambda r: r[-1][:40])
def test_kv_bytes_matches_printed_values(row):
    layers, kvh, hd, seq, batch, elem, printed, tol, _src = row
    got = oracle.kv_cache_bytes(layers, kvh, hd, seq, batch, elem)
    if tol == 0:
        assert got == printed
    else:
        assert abs(got - printed) <= tol * printed


def test_kv_bytes_gqa_ratio():
    # "大模型推理为何这么慢", GQA section: H query heads in G groups shrink the cache to G/H
    mha = oracle.kv_cache_bytes(32, 32, 128, 4096, 1, 2)
    gqa = oracle.kv_cache_bytes(32, 8, 128, 4096, 1, 2)
    mqa = oracle.kv_cache_bytes(32, 1, 128, 4096, 1, 2)
    assert mha == 4 * gqa == 32 * mqa


# ---------------------------------------------------------------- E4M3 codec
def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    assert (ours[~nan] == ref[~nan]).all()
    assert np.signbit(ours[0x80]) and ours[0x80] == 0.0


def test_e4m3_decode_definition_values():
    d = oracle.e4m3_decode(np.array([0x7E, 0x08, 0x01, 0x07, 0x38, 0x7F, 0xFF, 0xFE],
                                    dtype=np.uint8))
    assert d[0] == 448.0            # 1.75 * 2^8, largest finite
    assert d[1] == 2.0 ** -6        # smallest normal
    assert d[2] == 2.0 ** -9        # smallest subnormal
    assert d[3] == 7 * 2.0 ** -9    # largest subnormal
    assert d[4] == 1.0
    assert math.isnan(d[5]) and math.isnan(d[6])
    assert d[7] == -448.0


def _finite_e4m3_values():
    vals = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    return vals


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    pos = _finite_e4m3_values()
    mids = (pos[:-1] + pos[1:]) / 2
    xs = np.concatenate([
        rng.normal(size=20000) * 50,
        rng.normal(size=5000) * 1e-2,
        pos, -pos, mids, -mids,                 # exact ties: ties to even
        np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)),
        [447.9, 448.0, 455.9, -463.0, 0.0, -0.0, 1e-30],
    ]).astype(np.float32)
    xs = xs[np.abs(xs) < 464]
    ours = oracle.e4m3_encode(xs)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (ours == ref).all()


def test_e4m3_encode_saturates_and_nan():
    x = np.array([448.0, 464.0, 500.0, 1e30, np.inf, -1e9, np.nan], dtype=np.float32)
    assert oracle.e4m3_encode(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7F]


def test_e4m3_encode_bruteforce_nearest_even():
    # exact rational nearest-value search on a sample, independent of both codecs
    vals = [Fraction(float(v)) for v in _finite_e4m3_values()]
    rng = np.random.default_rng(11)
    xs = np.concatenate([rng.uniform(0, 448, 300), rng.uniform(0, 0.02, 200)]).astype(np.float32)
    got = oracle.e4m3_encode(xs)
    for x, g in zip(xs.tolist(), got.tolist()):
        fx = Fraction(x)
        dists = [abs(fx - v) for v in vals]
        best = min(dists)
        cands = [c for c, dd in enumerate(dists) if dd == best]
        want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        assert g == want, (x, g, want)


def test_quantize_rows_closed_form():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(64, 128)).astype(np.float32)
    x[5] = 0.0
    x[6, :] = 0.0
    x[6, 17] = -3.25
    codes, scales = oracle.quantize_rows(x)
    amax = np.abs(x).max(axis=1)
    expect_scale = (amax / np.float32(448.0)).astype(np.float32)
    expect_scale[amax == 0] = 0
    assert (scales == expect_scale).all()
    assert (codes[5] == 0).all()
    # the element of largest magnitude lands on (or saturates to) +-448
    for r in range(64):
        if amax[r] == 0:
            continue
        i = int(np.abs(x[r]).argmax())
        assert codes[r, i] in (0x7E, 0xFE)
    # dequantisation error bound: half a mantissa step (2^-4 relative) for normals,
    # half the subnormal spacing (2^-10 * scale) below 2^-6 * scale
    deq = oracle.e4m3_decode(codes) * scales[:, None].astype(np.float64)
    err = np.abs(deq - x.astype(np.float64))
    bound = np.maximum(np.abs(x) * 2.0 ** -4, scales[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert (err <= bound).all()


# ---------------------------------------------------------------- INT8 rows
def test_int8_quantize_hand_examples():
    # scales that are exact binary numbers, so every y = x / s is exact and the
    # codes follow by hand: ties go to the even integer, |code| <= 127
    x = np.array([[127, -0.5, 1.5, 2.5, -3.5, 0.49, 126.5, -127],
                  [254, 3, -5, 1, -254, 0.5, 253, -1],
                  [0, 0, 0, 0, 0, 0, 0, 0],
                  [-63.5, 0.25, 0.75, -0.25, 31.75, 0, 0, 0]], dtype=np.float32)
    codes, scales = oracle.quantize_rows(x, "int8")
    assert codes.dtype == np.int8
    assert scales.tolist() == [1.0, 2.0, 0.0, 0.5]
    assert codes.tolist() == [[127, 0, 2, 2, -4, 0, 126, -127],
                              [127, 2, -2, 0, -127, 0, 126, 0],
                              [0, 0, 0, 0, 0, 0, 0, 0],
                              [-127, 0, 2, 0, 64, 0, 0, 0]]


def test_int8_quantize_bruteforce_nearest_even():
    # each code is the integer of [-127, 127] nearest the exact value of the
    # fp32 quotient x / s (ties to even), searched over all 255 candidates
    rng = np.random.default_rng(21)
    x = (rng.standard_t(3, size=(24, 64)) * rng.uniform(0.01, 30, size=(24, 1))).astype(np.float32)
    codes, scales = oracle.quantize_rows(x, "int8")
    for r in range(x.shape[0]):
        s = np.float32(np.abs(x[r]).max()) / np.float32(127.0)
        assert scales[r] == s
        for i in range(x.shape[1]):
            y = Fraction(float(np.float32(x[r, i]) / s))
            best = min(abs(y - c) for c in range(-127, 128))
            cands = [c for c in range(-127, 128) if abs(y - c) == best]
            want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
            assert codes[r, i] == want, (r, i, float(y), codes[r, i], want)


def test_int8_quantize_invariants():
    rng = np.random.default_rng(5)
    x = rng.normal(size=(96, 128)).astype(np.float32)
    x[3] = 0.0
    x[7, :] = 0.0
    x[7, 100] = 1e-30                                   # tiny but nonzero row
    x[9] *= 1e6                                         # large row
    codes, scales = oracle.quantize_rows(x, "int8")
    amax = np.abs(x).max(axis=1)
    assert (codes[3] == 0).all() and scales[3] == 0
    for r in range(x.shape[0]):
        if amax[r] == 0:
            continue
        i = int(np.abs(x[r]).argmax())
        assert abs(int(codes[r, i])) == 127              # the largest element maps to +-127
    assert int(np.abs(codes.astype(np.int32)).max()) == 127
    # round to nearest: the error is at most half a step (plus the fp32 rounding of x / s)
    deq = codes.astype(np.float64) * scales[:, None].astype(np.float64)
    err = np.abs(deq - x.astype(np.float64))
    assert (err <= scales[:, None].astype(np.float64) * (0.5 + 1e-5)).all()
    # symmetric: negating the row negates the codes and keeps the scale
    c2, s2 = oracle.quantize_rows(-x, "int8")
    assert (c2 == -codes).all() and (s2 == scales).all()
    # a power-of-two factor scales the scale and leaves the codes
    c3, s3 = oracle.quantize_rows(x * np.float32(2.0 ** -7), "int8")
    assert (c3 == codes).all() and (s3 == scales * np.float32(2.0 ** -7)).all()


# ---------------------------------------------------------------- INT4 rows
def test_int4_quantize_hand_examples():
    # worked by hand from the 4-bit routine (range / 15, zero = round(-min / scale),
    # code = clamp(round(x / scale) + zero, 0, 15)), scales exact in binary:
    # row 0: hi 22.5, lo -7.5 -> scale 2, zero round(3.75) = 4;
    #        x / 2 = 0, .75, 1.5, 2.25, 11.25, -3.75 -> 0, 1, 2 (tie to even), 2, 11, -4
    # row 1: hi 15, lo 0 -> scale 1, zero 0; codes round(x): 7.5 -> 8, 8.5 -> 8,
    #        0.5 -> 0, 1.5 -> 2, 2.5 -> 2, 14.5 -> 14 (ties to even)
    # rows 2-4: constant rows are kept exactly
    x = np.array([[0, 1.5, 3, 4.5, 22.5, -7.5, 0, 0],
                  [0, 7.5, 8.5, 15, 0.5, 1.5, 2.5, 14.5],
                  [2, 2, 2, 2, 2, 2, 2, 2],
                  [-3, -3, -3, -3, -3, -3, -3, -3],
                  [0, 0, 0, 0, 0, 0, 0, 0]], dtype=np.float32)
    codes, pz = oracle.quantize_rows(x, "int4")
    assert codes.tolist() == [[4, 5, 6, 6, 15, 0, 4, 4],
                              [0, 8, 8, 15, 0, 2, 2, 14],
                              [0] * 8, [0] * 8, [0] * 8]
    assert pz.tolist() == [[2, 4], [1, 0], [2, -1], [3, 1], [0, 0]]
    assert oracle.widen(codes, "int4", pz)[2:].tolist() == [[2] * 8, [-3] * 8, [0] * 8]


def _nearest_even(y: Fraction) -> int:
    f = y.numerator // y.denominator
    r = y - f
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and f % 2 == 1):
        return f + 1
    return f


def test_int4_quantize_exact_rationals():
    # scale, zero and codes re-derived with exact rationals from the fp32
    # quotients the routine forms (round to nearest, ties to even)
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((40, 128)) * rng.uniform(0.01, 50, (40, 1))
         + rng.uniform(-5, 5, (40, 1))).astype(np.float32)
    x[3] = np.abs(x[3]) + 10                           # all positive: negative zero point
    x[4] = -np.abs(x[4]) - 10                          # all negative: zero point above 15
    codes, pz = oracle.quantize_rows(x, "int4")
    for r in range(x.shape[0]):
        hi, lo = np.float32(x[r].max()), np.float32(x[r].min())
        s = np.float32(np.float32(hi - lo) / np.float32(15))
        z = _nearest_even(Fraction(float(np.float32(-lo) / s)))
        assert pz[r, 0] == s and pz[r, 1] == z
        for i in range(x.shape[1]):
            k = _nearest_even(Fraction(float(np.float32(x[r, i]) / s)))
            assert codes[r, i] == min(15, max(0, k + z)), (r, i)


def test_int4_quantize_invariants():
    rng = np.random.default_rng(8)
    x = rng.normal(size=(64, 128)).astype(np.float32)
    x[5, :] = 0.75                                     # constant rows: exact
    x[6, :] = -1e-3
    codes, pz = oracle.quantize_rows(x, "int4")
    assert codes.max() <= 15 and codes.dtype == np.uint8
    deq = oracle.widen(codes, "int4", pz)
    s = pz[:, 0].astype(np.float64)[:, None]
    err = np.abs(deq - x.astype(np.float64))
    assert (err <= s * (1 + 1e-6)).all()               # within one step everywhere
    inner = (codes > 0) & (codes < 15)
    assert (err[inner] <= (s * np.ones_like(err))[inner] * (0.5 + 1e-5)).all()  # half a step
    assert (deq[5] == 0.75).all() and (deq[6] == np.float32(-1e-3)).all()
    # the extremes land on the ends of the code range (within one step)
    for r in range(64):
        if r in (5, 6):
            continue
        assert codes[r, np.argmax(x[r])] >= 14 and codes[r, np.argmin(x[r])] <= 1
    # a power-of-two factor scales the scale and keeps codes and zero point
    c2, p2 = oracle.quantize_rows(x * np.float32(0.25), "int4")
    assert (c2 == codes).all() and (p2[:, 1] == pz[:, 1]).all()
    assert (p2[:, 0] == pz[:, 0] * np.float32(0.25)).all()


# ---------------------------------------------------------------- KIVI blocks
def test_kivi_hand_example():
    # one block, one kv head, 4 channels: K groups are channels over the 16 tokens
    k = np.zeros((1, 16, 4), np.float32)
    k[0, :, 0] = np.arange(16)                 # hi 15, lo 0: scale 1, zero 0, codes = values
    k[0, :, 1] = 2.5                           # constant channel: exact
    k[0, :, 2] = np.arange(16) * -2.0          # hi 0, lo -30: scale 2, zero 15, codes 15 - t
    k[0, :, 3] = 0.0
    v = np.zeros((1, 16, 4), np.float32)
    v[0, 0] = [0, 1.5, 3, 22.5]                # hi 22.5, lo 0: scale 1.5, zero 0
    v[0, 1] = [-7.5, 0, 7.5, 0]                # hi 7.5, lo -7.5: scale 1, zero round(7.5) = 8
    kc, kp, vc, vp = oracle.quantize_blocks_kivi(k, v)
    assert kc[0, :, 0].tolist() == list(range(16)) and kp[0, 0].tolist() == [1, 0]
    assert (kc[0, :, 1] == 0).all() and kp[0, 1].tolist() == [2.5, -1]
    assert kc[0, :, 2].tolist() == list(range(15, -1, -1)) and kp[0, 2].tolist() == [2, 15]
    assert kp[0, 3].tolist() == [0, 0]
    assert vc[0, 0].tolist() == [0, 1, 2, 15] and vp[0, 0].tolist() == [1.5, 0]
    assert vc[0, 1].tolist() == [0, 8, 15, 8] and vp[0, 1].tolist() == [1, 8]
    kd, vd = oracle.kivi_dequantize(kc, kp, vc, vp)
    assert (kd[0, :, :3] == k[0, :, :3]).all()          # these channels are exact
    assert vd[0, 1].tolist() == [-8, 0, 7, 0]           # (c - 8) * 1


def test_kivi_groups_exact_rationals():
    # scale, zero and codes of every K channel and V row re-derived exactly
    rng = np.random.default_rng(77)
    k = (rng.standard_normal((3, 16, 64)) * rng.uniform(0.1, 20, (3, 1, 64))).astype(np.float32)
    v = (rng.standard_normal((3, 16, 64)) * rng.uniform(0.1, 20, (3, 16, 1))).astype(np.float32)
    k[1, :, 5] = np.abs(k[1, :, 5]) + 4         # a channel with a negative zero point
    kc, kp, vc, vp = oracle.quantize_blocks_kivi(k, v)

    def check(group, codes, params):
        hi, lo = np.float32(group.max()), np.float32(group.min())
        sc = np.float32(np.float32(hi - lo) / np.float32(15))
        z = _nearest_even(Fraction(float(np.float32(-lo) / sc)))
        assert params[0] == sc and params[1] == z
        for x, c in zip(group.tolist(), codes.tolist()):
            kk = _nearest_even(Fraction(float(np.float32(x) / sc)))
            assert c == min(15, max(0, kk + z))

    for b in range(3):
        for ch in range(64):
            check(k[b, :, ch], kc[b, :, ch], kp[b, ch])
        for t in range(16):
            check(v[b, t], vc[b, t], vp[b, t])


def test_kivi_sequence_keeps_the_incomplete_block_exact():
    rng = np.random.default_rng(5)
    for L in (15, 16, 32, 37):
        k = rng.normal(size=(L, 2, 32)).astype(np.float32)
        v = rng.normal(size=(L, 2, 32)).astype(np.float32)
        k64, v64 = oracle.kivi_sequence(k, v)
        full = L // 16 * 16
        assert (k64[full:] == k[full:]).all() and (v64[full:] == v[full:]).all()
        if full:
            assert (k64[:full] != k[:full]).any()          # quantised
            # per-channel error bound: at most one step of that channel's block scale
            kb = k[:full].reshape(-1, 16, 2, 32)
            step = (kb.max(axis=1) - kb.min(axis=1)) / 15
            err = np.abs(k64[:full] - k[:full]).reshape(-1, 16, 2, 32)
            assert (err <= step[:, None] * (1 + 1e-5) + 1e-7).all()


# ---------------------------------------------------------------- attention
def _rand_case(rng, b, hq, hkv, d, lens, kv_dtype="f32"):
    total = int(sum(lens))
    q = rng.normal(size=(b, hq, d)).astype(np.float32)
    k = rng.normal(size=(total, hkv, d)).astype(np.float32)
    v = rng.normal(size=(total, hkv, d)).astype(np.float32)
    offs = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    return q, k, v, offs, np.asarray(lens, dtype=np.int32)


def _bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


@pytest.mark.parametrize("hq,hkv", [(4, 1), (8, 2), (4, 4), (32, 8)])
def test_attention_matches_bruteforce_numpy(hq, hkv):
    rng = np.random.default_rng(hq * 10 + hkv)
    lens = [1, 5, 16, 17, 40]
    q, k, v, offs, lens = _rand_case(rng, 5, hq, hkv, 32, lens)
    scale = 1 / math.sqrt(32)
    ours = oracle.decode_attention(q, k, v, offs, lens, scale, hkv, "f32", "f32")
    brute = oracle.decode_attention_bruteforce(q.astype(np.float64), k.astype(np.float64),
                                               v.astype(np.float64), offs, lens, scale, hkv)
    assert np.abs(ours - brute).max() <= 1e-12


@pytest.mark.parametrize("kv_dtype", ["f32", "bf16", "fp8", "int8", "int4", "f64"])
def test_attention_matches_torch_sdpa_float64(kv_dtype):
    rng = np.random.default_rng({"f32": 1, "bf16": 2, "fp8": 3, "int8": 4, "int4": 5,
                                 "f64": 6}[kv_dtype])
    hq, hkv, d = 8, 2, 64
    lens = [3, 33, 64]
    q, k, v, offs, lens = _rand_case(rng, 3, hq, hkv, d, lens)
    scale = 0.125
    ks = vs = None
    if kv_dtype == "f32":
        kst, vst = k, v
        k64, v64 = k.astype(np.float64), v.astype(np.float64)
    elif kv_dtype == "bf16":
        kst, vst = _bf16_bits(k), _bf16_bits(v)
        k64, v64 = oracle.widen(kst, "bf16"), oracle.widen(vst, "bf16")
    elif kv_dtype == "f64":
        k64 = k.astype(np.float64) * (1 + 2.0 ** -40)       # values no float32 can hold
        v64 = v.astype(np.float64) * (1 - 2.0 ** -40)
        kst, vst = k64, v64
    elif kv_dtype == "int4":
        kst, ks = oracle.quantize_rows(k, "int4")
        vst, vs = oracle.quantize_rows(v, "int4")
        # dequantise independently of the oracle: (code - zero) * scale in float64
        k64 = (kst.astype(np.float64) - ks[..., 1:2].astype(np.float64)) * ks[..., 0:1]
        v64 = (vst.astype(np.float64) - vs[..., 1:2].astype(np.float64)) * vs[..., 0:1]
    elif kv_dtype == "int8":
        kst, ks = oracle.quantize_rows(k, "int8")
        vst, vs = oracle.quantize_rows(v, "int8")
        # dequantise independently of the oracle: code * scale in float64 (exact)
        k64 = kst.astype(np.float64) * ks.astype(np.float64)[..., None]
        v64 = vst.astype(np.float64) * vs.astype(np.float64)[..., None]
    else:
        kst, ks = oracle.quantize_rows(k)
        vst, vs = oracle.quantize_rows(v)
        k64, v64 = oracle.widen(kst, "fp8", ks), oracle.widen(vst, "fp8", vs)
    ours = oracle.decode_attention(q, kst, vst, offs, lens, scale, hkv, kv_dtype, "f32",
                                   k_scale=ks, v_scale=vs)
    for s in range(3):
        o, n = int(offs[s]), int(lens[s])
        qq = torch.from_numpy(q[s].astype(np.float64))[None, :, None, :]     # [1,Hq,1,D]
        kk = torch.from_numpy(k64[o:o + n]).permute(1, 0, 2)[None]          # [1,Hkv,n,D]
        vv = torch.from_numpy(v64[o:o + n]).permute(1, 0, 2)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale,
                                                               enable_gqa=True)
        assert np.abs(ours[s] - ref[0, :, 0, :].numpy()).max() <= 1e-12


def test_attention_bf16_q_is_widened_exactly():
    rng = np.random.default_rng(5)
    q, k, v, offs, lens = _rand_case(rng, 2, 4, 1, 64, [7, 20])
    qb = _bf16_bits(q)
    a = oracle.decode_attention(qb, k, v, offs, lens, 0.125, 1, "f32", "bf16")
    b = oracle.decode_attention(oracle.widen(qb, "bf16").astype(np.float32), k, v, offs, lens,
                                0.125, 1, "f32", "f32")
    assert (a == b).all()


def test_attention_length_one_returns_v():
    rng = np.random.default_rng(9)
    q, k, v, offs, lens = _rand_case(rng, 3, 8, 2, 64, [1, 1, 1])
    out = oracle.decode_attention(q, k, v, offs, lens, 0.3, 2, "f32", "f32")
    for s in range(3):
        for h in range(8):
            assert (out[s, h] == v[s, h // 4].astype(np.float64)).all()


def test_attention_identical_keys_give_mean_v():
    rng = np.random.default_rng(10)
    q, k, v, offs, lens = _rand_case(rng, 1, 4, 1, 64, [50])
    k[:] = k[0]
    out = oracle.decode_attention(q, k, v, offs, lens, 0.125, 1, "f32", "f32")
    mean = v[:, 0, :].astype(np.float64).mean(axis=0)
    assert np.abs(out[0] - mean).max() <= 1e-12


def test_attention_dominant_key_selects_its_value():
    rng = np.random.default_rng(12)
    q, k, v, offs, lens = _rand_case(rng, 1, 4, 1, 64, [30])
    k[17, 0, :] = 40.0 * q[0, 0, :]     # head 0 scores this key ~ 40 |q|^2 higher
    out = oracle.decode_attention(q, k, v, offs, lens, 1.0, 1, "f32", "f32")
    assert np.abs(out[0, 0] - v[17, 0]).max() <= 1e-9


def test_attention_weights_sum_to_one_and_key_order_invariance():
    rng = np.random.default_rng(13)
    q, k, v, offs, lens = _rand_case(rng, 2, 8, 2, 64, [23, 70])
    out, w = oracle.decode_attention(q, k, v, offs, lens, 0.125, 2, "f32", "f32",
                                     return_weights=True)
    for s in range(2):
        assert np.abs(w[s, :, :lens[s]].sum(axis=1) - 1).max() <= 1e-12
        assert (w[s, :, lens[s]:] == 0).all()
    perm = np.concatenate([rng.permutation(23), 23 + rng.permutation(70)])
    out2 = oracle.decode_attention(q, k[perm], v[perm], offs, lens, 0.125, 2, "f32", "f32")
    assert np.abs(out - out2).max() <= 1e-12


def test_attention_gqa_group_mapping_is_consecutive():
    # query heads 0..G-1 read KV head 0, G..2G-1 read KV head 1, ...
    rng = np.random.default_rng(14)
    q, k, v, offs, lens = _rand_case(rng, 1, 6, 3, 32, [9])
    v[:, 0, :], v[:, 1, :], v[:, 2, :] = 1.0, 2.0, 3.0
    out = oracle.decode_attention(q, k, v, offs, lens, 0.2, 3, "f32", "f32")
    assert np.allclose(out[0, :, 0], [1, 1, 2, 2, 3, 3], atol=1e-12)


@pytest.mark.parametrize("partition,tile", [(16, 16), (48, 16), (100, 16), (1024, 16), (37, 5)])
def test_split_online_softmax_equals_two_pass(partition, tile):
    rng = np.random.default_rng(partition + tile)
    q, k, v, offs, lens = _rand_case(rng, 4, 8, 2, 32, [1, 16, 250, 601])
    k[:, :, 3] *= 20.0      # outlier channel: wide score range
    q64, k64, v64 = (a.astype(np.float64) for a in (q, k, v))
    two = oracle.decode_attention(q, k, v, offs, lens, 0.18, 2, "f32", "f32")
    split = oracle.decode_attention_split(q64, k64, v64, offs, lens, 0.18, 2, partition, tile)
    assert np.abs(two - split).max() <= 1e-12


def test_oracle_rejects_empty_context():
    rng = np.random.default_rng(15)
    q, k, v, offs, lens = _rand_case(rng, 2, 4, 1, 16, [3, 4])
    lens[1] = 0
    with pytest.raises(ValueError):
        oracle.decode_attention(q, k, v, offs, lens, 1.0, 1, "f32", "f32")


# ---------------------------------------------------------------- paging
class _ToyPagedCache:
    """Incremental restatement of the "llm-inference-optimization" notes' §二
    PagedKVCache: a sequence gets a new block when it has none or its last is
    full; a token goes to the next free offset of the last block.  Physical
    ids come from a caller-supplied allocator instead of len(blocks)."""

    def __init__(self, block_size, alloc):
        self.bs, self.alloc, self.table, self.fill = block_size, alloc, {}, {}

    def append_token(self, seq):
        tab = self.table.setdefault(seq, [])
        if not tab or self.fill[tab[-1]] == self.bs:
            blk = self.alloc()
            tab.append(blk)
            self.fill[blk] = 0
        blk = tab[-1]
        off = self.fill[blk]
        self.fill[blk] += 1
        return blk * self.bs + off


def test_slot_mapping_matches_incremental_paged_toy():
    rng = np.random.default_rng(16)
    lens = [1, 15, 16, 17, 33, 160]
    pool = list(rng.permutation(200))
    toy = _ToyPagedCache(16, lambda: int(pool.pop()))
    order = [(s, p) for p in range(max(lens)) for s in range(len(lens)) if p < lens[s]]
    toy_slots = {(s, p): toy.append_token(s) for s, p in order}
    mb = max(len(t) for t in toy.table.values())
    table = np.full((len(lens), mb), 2**31 - 1, dtype=np.int32)
    for s, t in toy.table.items():
        table[s, :len(t)] = t
    sids = np.array([s for s, _ in order], dtype=np.int32)
    poss = np.array([p for _, p in order], dtype=np.int32)
    ours = oracle.slot_mapping(table, sids, poss, 16)
    assert ours.tolist() == [toy_slots[(s, p)] for s, p in order]
    # "最多浪费一个块": blocks = ceil(L / 16), fewer than 16 unused slots per sequence
    for s, n in enumerate(lens):
        assert len(toy.table[s]) == -(-n // 16)
        assert len(toy.table[s]) * 16 - n < 16


def test_scatter_then_gather_round_trip():
    rng = np.random.default_rng(17)
    nb, hkv, d = 12, 2, 8
    lens = [20, 9]
    perm = rng.permutation(nb).astype(np.int32)
    table = np.array([perm[:2], np.r_[perm[2:3], 2**31 - 1]], dtype=np.int32)
    rows = rng.normal(size=(29, hkv, d)).astype(np.float32)
    sids = np.r_[np.zeros(20, np.int32), np.ones(9, np.int32)]
    poss = np.r_[np.arange(20), np.arange(9)].astype(np.int32)
    slots = oracle.slot_mapping(table, sids, poss)
    poison = np.full((nb, hkv, 16, d), np.nan, dtype=np.float32)
    pool = oracle.scatter_to_pool(poison, rows, slots)
    for i, (s, p) in enumerate(zip(sids, poss)):
        blk = table[s, p // 16]
        assert (pool[blk, :, p % 16, :] == rows[i]).all()
    assert np.isnan(pool).sum() == (nb * 16 - 29) * hkv * d
    # negative slots are padding
    skipped = oracle.scatter_to_pool(poison, rows[:2], np.array([-1, slots[1]]))
    assert np.isnan(skipped).sum() == (nb * 16 - 1) * hkv * d


def test_scatter_scales_to_pool_flat_offsets():
    # The scale pool's layout stated by the library header: [block][kv_head][2][16]
    # float32, K's 16 row scales of a (block, kv head) and then V's.  The flat
    # index of (block b, head h, which w, slot offset o) is ((b*Hkv + h)*2 + w)*16 + o;
    # INT4 pools add a trailing (scale, zero) pair, flat index * 2 + {0, 1}.
    nb, hkv = 5, 3
    slots = np.array([0, 17, 79, -4, 38])            # slot 79: block 4, offset 15; -4 padding
    hand = [(0, 0), (1, 1), (4, 15), None, (2, 6)]   # (block, offset) written out by hand
    k_sc = np.arange(1, 16, dtype=np.float32).reshape(5, hkv)
    v_sc = -k_sc
    pool = np.full((nb, hkv, 2, 16), np.nan, np.float32)
    pool = oracle.scatter_scales_to_pool(pool, k_sc, slots, which=0)
    pool = oracle.scatter_scales_to_pool(pool, v_sc, slots, which=1)
    flat = pool.reshape(-1)
    want = np.full(nb * hkv * 2 * 16, np.nan, np.float32)
    for t, bo in enumerate(hand):
        if bo is None:
            continue
        b, o = bo
        for h in range(hkv):
            want[((b * hkv + h) * 2 + 0) * 16 + o] = k_sc[t, h]
            want[((b * hkv + h) * 2 + 1) * 16 + o] = v_sc[t, h]
    np.testing.assert_array_equal(flat, want)
    assert np.isnan(flat).sum() == (nb * 16 - 4) * hkv * 2

    # INT4: (scale, zero) per row, K then V
    kp = np.stack([k_sc, k_sc + 100], axis=-1)       # [T][Hkv][2]
    vp = np.stack([v_sc, v_sc - 100], axis=-1)
    pool4 = np.full((nb, hkv, 2, 16, 2), np.nan, np.float32)
    pool4 = oracle.scatter_scales_to_pool(pool4, kp, slots, which=0)
    pool4 = oracle.scatter_scales_to_pool(pool4, vp, slots, which=1)
    flat4 = pool4.reshape(-1)
    want4 = np.full(nb * hkv * 2 * 16 * 2, np.nan, np.float32)
    for t, bo in enumerate(hand):
        if bo is None:
            continue
        b, o = bo
        for h in range(hkv):
            for w, par in ((0, kp), (1, vp)):
                base = (((b * hkv + h) * 2 + w) * 16 + o) * 2
                want4[base] = par[t, h, 0]
                want4[base + 1] = par[t, h, 1]
    np.testing.assert_array_equal(flat4, want4)


# ---------------------------------------------------------------- multi-query (causal)
def test_multi_query_one_token_is_decode():
    rng = np.random.default_rng(21)
    q, k, v, offs, lens = _rand_case(rng, 3, 8, 2, 64, [5, 40, 1])
    mq = oracle.multi_query_attention(q[:, None], k, v, offs, lens, 0.2, 2, "f32", "f32")
    dec = oracle.decode_attention(q, k, v, offs, lens, 0.2, 2, "f32", "f32")
    assert (mq[:, 0] == dec).all()


def test_multi_query_rows_are_decodes_of_shorter_contexts():
    rng = np.random.default_rng(22)
    nq = 4
    _, k, v, offs, lens = _rand_case(rng, 3, 8, 2, 32, [4, 19, 50])
    q = rng.normal(size=(3, nq, 8, 32)).astype(np.float32)
    mq = oracle.multi_query_attention(q, k, v, offs, lens, 0.3, 2, "f32", "f32")
    for i in range(nq):
        dec = oracle.decode_attention(np.ascontiguousarray(q[:, i]), k, v, offs, lens - nq + i + 1,
                                      0.3, 2, "f32", "f32")
        assert np.abs(mq[:, i] - dec).max() <= 1e-12


def test_multi_query_matches_torch_sdpa_with_causal_offset_mask():
    rng = np.random.default_rng(23)
    nq, hq, hkv, d = 3, 4, 2, 16
    _, k, v, offs, lens = _rand_case(rng, 2, hq, hkv, d, [3, 11])
    q = rng.normal(size=(2, nq, hq, d)).astype(np.float32)
    mq = oracle.multi_query_attention(q, k, v, offs, lens, 0.25, hkv, "f32", "f32")
    for s in range(2):
        o, n = int(offs[s]), int(lens[s])
        qq = torch.from_numpy(q[s].astype(np.float64)).permute(1, 0, 2)[None]     # [1,Hq,Q,D]
        kk = torch.from_numpy(k[o:o + n].astype(np.float64)).permute(1, 0, 2)[None]
        vv = torch.from_numpy(v[o:o + n].astype(np.float64)).permute(1, 0, 2)[None]
        pos = torch.arange(n)[None, :]
        limit = (n - nq + torch.arange(nq))[:, None]
        mask = pos <= limit                                                        # [Q, n]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask,
                                                               scale=0.25, enable_gqa=True)
        assert np.abs(mq[s] - ref[0].permute(1, 0, 2).numpy()).max() <= 1e-12


def test_multi_query_rejects_short_context():
    rng = np.random.default_rng(24)
    _, k, v, offs, lens = _rand_case(rng, 2, 4, 1, 16, [2, 9])
    q = rng.normal(size=(2, 3, 4, 16)).astype(np.float32)
    with pytest.raises(ValueError):
        oracle.multi_query_attention(q, k, v, offs, lens, 1.0, 1, "f32", "f32")
