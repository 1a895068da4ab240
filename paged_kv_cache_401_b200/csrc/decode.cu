// Paged GQA decode attention: persistent split-K ("stream-K") kernel and its
// log-sum-exp merge (sm_100a).
//
// Method ("KV Cache 深度解析" §一/§三/§四; "llm-inference-optimization" notes
// §三 Flash Attention; k1-blog 2026-07-13, "PagedAttention 與 vLLM"): for each
// sequence b and kv head g, the G query heads of the group attend to the
// L_b cached tokens, read block by block through the block table, with an
// online softmax (running max m, running sum l, rescaled running output o)
// so no score leaves the chip.  Partial (m, l, o) of pieces of one sequence
// are combined by their log-sum-exp.
//
// Work decomposition.  The (sequence, kv head) pairs are laid end to end as
// one list of 16-token tiles, T tiles in all (a pair with L tokens has
// ceil(L/16)).  The list is cut into num_ranges equal contiguous ranges, one
// per consumer warp: every warp streams the same number of bytes whatever
// the mix of context lengths, so ragged batches and a handful of very long
// sequences keep every SM busy.  A warp's range may start or end inside a
// pair; such a "piece" writes its (m, l, o) to the workspace and the merge
// kernel combines the pieces of each pair.  A pair entirely inside one range
// is finished by its warp, which writes the output directly.
//
// B200 design:
//  * a CTA is one producer warp and four consumer warps; by default the grid
//    is the number of CTAs resident on the GPU (persistent), so the tile
//    stream never stalls between work items;
//  * FP8 / INT8 row scales of a tile (16 K then 16 V) are one 128-byte line;
//  * producer lane w walks consumer warp w's range and stages each (block,
//    kv head) K and V tile -- one contiguous 16-row span of the pool -- into
//    that warp's stages of a shared-memory ring (stage s feeds warp s % 4)
//    through the TMA engine (no multicast), completing on mbarriers; block
//    ids are fetched 4 tiles ahead, and no warp's refill waits behind another;
//  * the per-tile arithmetic is a policy:
//      MmaMath  (bf16, FP8, INT8, INT4 or KIVI KV, head_dim 128, bf16 q): tiles
//               land in shared memory 128-byte swizzled by 2-D TMA tensor copies
//               (4-bit codes as 16-code groups padded to 16 bytes, widened to
//               bytes by ldmatrix); the group's scores S = Q.K^T come from
//               mma.m16n8k16 (query heads as rows, fp32 accumulate), the softmax
//               runs on the accumulator fragments, and P feeds O^T = V^T.P^T
//               straight from registers; codes are widened to f16 in registers
//               (exact);
//      SimtMath (every other shape and fp32): 1-D bulk copies; q.K with
//               packed fp32x2 FMAs and a shuffle reduce-scatter, P.V with each
//               lane owning D/32 output columns, all in fp32;
//  * every wait is bounded; bad block ids and context lengths are reported
//    through the error word and never dereferenced.
#include <atomic>

#include "kernels.cuh"
#include "quant.cuh"

namespace pkv {

template <int KV_T>
struct KvElem;
template <>
struct KvElem<KV_F32> {
    static constexpr int kBytes = 4;
};
template <>
struct KvElem<KV_BF16> {
    static constexpr int kBytes = 2;
};
template <>
struct KvElem<KV_FP8_E4M3> {
    static constexpr int kBytes = 1;
};
template <>
struct KvElem<KV_INT8> {
    static constexpr int kBytes = 1;
};
template <>
struct KvElem<KV_INT4> {  // two codes per byte: row sizes are computed from bits instead
    static constexpr int kBytes = 0;
};
template <>
struct KvElem<KV_KIVI4> {
    static constexpr int kBytes = 0;
};

// Quantised pools carry per-(token, kv head) parameters: an fp32 scale (8-bit
// codes) or an fp32 (scale, zero point) pair (4-bit codes).
template <int KV_T>
inline constexpr bool kQuantized =
    KV_T == KV_FP8_E4M3 || KV_T == KV_INT8 || KV_T == KV_INT4 || KV_T == KV_KIVI4;

// Two 8-bit codes (low 16 bits) -> two floats (code values, before the row scale).
template <int KV_T>
__device__ __forceinline__ float2 codes2_to_float2(uint32_t w16) {
    if constexpr (KV_T == KV_INT8) return i8x2_to_float2(w16);
    else return e4m3x2_to_float2(w16);
}

// ---- small vector helpers --------------------------------------------------------
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Decode one 16-byte chunk into kChunkElems/2 float pairs.
template <int KV_T>
__device__ __forceinline__ void decode_chunk(const uint4 c, float2* out) {
    if constexpr (KV_T == KV_F32) {
        out[0] = make_float2(__uint_as_float(c.x), __uint_as_float(c.y));
        out[1] = make_float2(__uint_as_float(c.z), __uint_as_float(c.w));
    } else if constexpr (KV_T == KV_BF16) {
        out[0] = bf16x2_to_float2(c.x);
        out[1] = bf16x2_to_float2(c.y);
        out[2] = bf16x2_to_float2(c.z);
        out[3] = bf16x2_to_float2(c.w);
    } else {
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = codes2_to_float2<KV_T>(w[i] & 0xffffu);
            out[2 * i + 1] = codes2_to_float2<KV_T>(w[i] >> 16);
        }
    }
}

// Load and decode kDPL consecutive elements of a V row (kDPL * elem bytes).
template <int KV_T, int DPL>
__device__ __forceinline__ void load_v(const uint8_t* p, float2* out) {
    constexpr int kBytes = DPL * KvElem<KV_T>::kBytes;
    if constexpr (KV_T == KV_F32) {
        if constexpr (kBytes == 16) {
            const float4 f = *reinterpret_cast<const float4*>(p);
            out[0] = make_float2(f.x, f.y);
            out[1] = make_float2(f.z, f.w);
        } else {
            out[0] = *reinterpret_cast<const float2*>(p);
        }
    } else if constexpr (KV_T == KV_BF16) {
        if constexpr (kBytes == 8) {
            const uint2 w = *reinterpret_cast<const uint2*>(p);
            out[0] = bf16x2_to_float2(w.x);
            out[1] = bf16x2_to_float2(w.y);
        } else {
            out[0] = bf16x2_to_float2(*reinterpret_cast<const uint32_t*>(p));
        }
    } else {
        if constexpr (kBytes == 4) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
            out[0] = codes2_to_float2<KV_T>(w & 0xffffu);
            out[1] = codes2_to_float2<KV_T>(w >> 16);
        } else {
            out[0] = codes2_to_float2<KV_T>(*reinterpret_cast<const uint16_t*>(p));
        }
    }
}

// Shuffle reduce-scatter over the kLPR lanes of a row group: N partial sums per
// lane in, max(1, N/LPR) complete sums per lane out (in v[0..]).  Lane c of the
// group ends with indices c*(N/LPR)+k, or c/(LPR/N) when N < LPR.  The tree is
// fixed, so results do not depend on where blocks live in the pool.
template <int N, int MASK>
__device__ __forceinline__ void reduce_scatter(float* v, int lane) {
    if constexpr (MASK >= 1) {
        if constexpr (N >= 2) {
            const bool upper = (lane & MASK) != 0;
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                const float send = upper ? v[i] : v[i + N / 2];
                const float keep = upper ? v[i + N / 2] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, MASK);
            }
            reduce_scatter<N / 2, MASK / 2>(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], MASK);
            reduce_scatter<1, MASK / 2>(v, lane);
        }
    }
}

template <typename T>
__device__ __forceinline__ T out_cast(float x);
template <>
__device__ __forceinline__ float out_cast<float>(float x) { return x; }
template <>
__device__ __forceinline__ uint16_t out_cast<uint16_t>(float x) {
    const __nv_bfloat16 b = __float2bfloat16_rn(x);
    return *reinterpret_cast<const uint16_t*>(&b);
}

template <int Q_T>
struct QType;
template <>
struct QType<KV_F32> {
    using T = float;
};
template <>
struct QType<KV_BF16> {
    using T = uint16_t;
};

template <int Q_T>
__device__ __forceinline__ float load_q_elem(const void* q, int64_t i) {
    if constexpr (Q_T == KV_F32) {
        return static_cast<const float*>(q)[i];
    } else {
        return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(q)[i]) << 16);
    }
}



// ---- tensor-core and TMA helpers --------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// 4-bit codes staged as 16-code groups padded to 16 bytes (the TMA's 16U4_ALIGN16B
// layout), widened to one code per byte (low nibble) by the load.  Four 8-row x
// 16-code matrices: lane l gets row l / 4, codes 4 (l % 4) .. + 3 of each, as
// ldmatrix .b16 gives 8-bit rows; lanes 8m .. 8m + 7 address matrix m's rows.
__device__ __forceinline__ void ldsm_x4_u4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n16.x4.shared.b8x16.b4x16_p64 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// Two 16-row x 16-byte matrices, transposed per byte: lane (gid, tig) gets bytes of
// rows 4 tig .. + 3 in column gid (r[0]) and column gid + 8 (r[1]), then the same of
// the second matrix (r[2], r[3]); lanes 0-15 and 16-31 address the two matrices' rows.
__device__ __forceinline__ void ldsm_x2_trans_b8(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// Two 16-row x 16-code matrices of the same layout, transposed: lane (gid, tig)
// gets codes of rows 4 tig .. + 3 in column gid (r[0]) and column gid + 8 (r[1]),
// then the same of the second matrix (r[2], r[3]); lanes 0-15 and 16-31 address
// the two matrices' rows.
__device__ __forceinline__ void ldsm_x2_trans_u4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8x16.b4x16_p64 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += A(16x16, row) * B(16x8, col), fp32 accumulate; bf16 or f16 operands.
template <bool F16>
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    if constexpr (F16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

// Two fp32 -> packed pair (low half = first argument), round to nearest even.
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    uint32_t r;
    if constexpr (F16)
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    else
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four E4M3 codes -> two f16x2 (codes 0,1 -> lo; codes 2,3 -> hi), exact.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// Four signed 8-bit codes -> two f16x2, exact.  Each code c becomes the biased
// byte c + 128 in the low mantissa byte of f16 1024 (0x64xx = 1024 + c + 128),
// then 1152 is subtracted.  SEL_LO / SEL_HI pick which two bytes of w go to the
// low and high halves of lo and hi (byte_perm selectors over {w, 0x64646464}).
template <uint32_t SEL_LO, uint32_t SEL_HI>
__device__ __forceinline__ void i8x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t a = __byte_perm(u, 0x64646464u, SEL_LO);
    const uint32_t b = __byte_perm(u, 0x64646464u, SEL_HI);
    asm("add.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(0xE480E480u));  // -1152
    asm("add.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(0xE480E480u));
}

// Four 8-bit K codes (one lane's ldmatrix word) -> f16x2 {codes 0,1}, {codes 2,3}.
template <int KV_T>
__device__ __forceinline__ void widen_k4(uint32_t w, uint32_t& lo, uint32_t& hi) {
    if constexpr (KV_T == KV_INT8) i8x4_to_f16x2x2<0x4140u, 0x4342u>(w, lo, hi);
    else e4m3x4_to_f16x2x2(w, lo, hi);
}

// Four 8-bit V codes from a transposed ldmatrix word, bytes [t0 d, t0 d+1,
// t1 d, t1 d+1] -> f16x2 {t0 d, t1 d} and {t0 d+1, t1 d+1}.
template <int KV_T>
__device__ __forceinline__ void widen_v4(uint32_t w, uint32_t& lo, uint32_t& hi) {
    if constexpr (KV_T == KV_INT8) i8x4_to_f16x2x2<0x4240u, 0x4341u>(w, lo, hi);
    else e4m3x4_to_f16x2x2(__byte_perm(w, 0u, 0x3120), lo, hi);
}

__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t hsub2u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// 2^x for x <= 0 (softmax weights), flushing results below 2^-126 to zero.
__device__ __forceinline__ float fast_exp2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 2-D TMA tile load (no multicast) completing on an mbarrier; x is the
// innermost coordinate in elements (always 0 or a multiple of 16 bytes here).
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3}], [%4];" ::"r"(smem_addr(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// ---- tile list bookkeeping ----------------------------------------------------------
// A context length is valid when it holds the query tokens and fits max_context_len.
__device__ __forceinline__ bool seq_valid(int32_t L, const DecodeParams& p) {
    return L >= p.num_query_tokens && L >= 1 && L <= p.max_context_len;
}

// Tiles of a sequence with context length L: ceil(L/16) -- for KIVI pools the
// full blocks only, floor(L/16) -- or 0 when L is invalid.
__device__ __forceinline__ int32_t seq_tiles(int32_t L, const DecodeParams& p) {
    if (!seq_valid(L, p)) return 0;
    return p.kivi ? L / kBlockTokens : (L + kBlockTokens - 1) / kBlockTokens;
}

// First tile of consumer range W (ranges are equal cuts of the T-tile list):
// floor(W T / N), N = num_ranges.  With T = q N + r that is W q + floor(W r / N),
// which needs only 32-bit divisions when N <= 65535 (W r < N^2 < 2^32) -- the
// persistent grid's case; 64-bit division is a long dependent chain.
__device__ __forceinline__ int64_t range_begin(int64_t W, int64_t T, int32_t num_ranges) {
    if (W >= num_ranges) return T;
    if (T <= 0x7fffffff && num_ranges <= 65535) {
        const uint32_t n = static_cast<uint32_t>(num_ranges), t = static_cast<uint32_t>(T);
        const uint32_t w = static_cast<uint32_t>(W);
        const uint32_t q = t / n, r = t - q * n;
        return static_cast<int64_t>(w) * q + (w * r) / n;
    }
    return (W * T) / num_ranges;
}

// The range holding tile x < T: the largest W with range_begin(W) <= x, i.e.
// the largest W with W T < (x+1) N -- in 32 bits when T N fits them.
__device__ __forceinline__ int64_t range_of(int64_t x, int64_t T, int32_t num_ranges) {
    int64_t W;
    if (T <= static_cast<int64_t>(0xffffffffu / static_cast<uint32_t>(num_ranges)))
        W = (static_cast<uint32_t>(x + 1) * static_cast<uint32_t>(num_ranges) - 1u) /
            static_cast<uint32_t>(T);
    else
        W = ((x + 1) * num_ranges - 1) / T;
    return W < num_ranges - 1 ? W : num_ranges - 1;
}

__device__ __forceinline__ int64_t warp_sum_i64(int64_t x) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// Total tiles T over the batch (computed by every warp that needs it).
__device__ int64_t total_tiles(const DecodeParams& p, int lane) {
    int64_t t = 0;
    for (int b = lane; b < p.batch; b += 32)
        t += static_cast<int64_t>(p.num_kv_heads) * seq_tiles(p.context_lens[b], p);
    return warp_sum_i64(t);
}

// Position of one tile in the list: sequence b, kv head, block index jb in
// the sequence, the sequence's tile count nt and length L, and the list
// index of the pair's first tile.
struct Cursor {
    int32_t b, kvh, jb, nt, L;
    int64_t seg_start;
};

// Warp-cooperative search for the pairs holding tiles x[0..K) (each < T; a
// negative x is not looked for), all in one pass over the lengths.  When
// `prefix` is non-null the warp also writes every sequence's first tile (and T
// at [batch]) there for the merge kernel.
template <int K>
__device__ void locate_tiles(const DecodeParams& p, const int64_t (&x)[K], int lane,
                             int32_t* prefix, int64_t T, Cursor (&c)[K]) {
    bool found[K];
    int left = 0;
#pragma unroll
    for (int k = 0; k < K; ++k) {
        c[k] = Cursor{p.batch, 0, 0, 0, 0, T};
        found[k] = x[k] < 0;
        left += found[k] ? 0 : 1;
    }
    int64_t base = 0;
    for (int b0 = 0; b0 < p.batch && (left > 0 || prefix != nullptr); b0 += 32) {
        const int b = b0 + lane;
        const int32_t L = b < p.batch ? p.context_lens[b] : 0;
        const int32_t nt = b < p.batch ? seq_tiles(L, p) : 0;
        const int64_t cnt = static_cast<int64_t>(p.num_kv_heads) * nt;
        int64_t incl = cnt;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, incl, m);
            if (lane >= m) incl += y;
        }
        const int64_t excl = base + incl - cnt;
        if (prefix != nullptr && b < p.batch) prefix[b] = static_cast<int32_t>(excl);
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const uint32_t hit = __ballot_sync(
                0xffffffffu, !found[k] && cnt > 0 && x[k] >= excl && x[k] < excl + cnt);
            if (hit != 0u) {
                const int src = __ffs(hit) - 1;
                const int64_t e = __shfl_sync(0xffffffffu, excl, src);
                const int32_t n = __shfl_sync(0xffffffffu, nt, src);
                const int32_t l = __shfl_sync(0xffffffffu, L, src);
                // the tile list holds fewer than 2^31 tiles (checked by the host)
                const uint32_t off = static_cast<uint32_t>(x[k] - e);
                c[k].b = b0 + src;
                c[k].nt = n;
                c[k].L = l;
                c[k].kvh = static_cast<int32_t>(off / static_cast<uint32_t>(n));
                c[k].jb = static_cast<int32_t>(off - static_cast<uint32_t>(c[k].kvh) * n);
                c[k].seg_start = e + static_cast<int64_t>(c[k].kvh) * n;
                found[k] = true;
                --left;
            }
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (prefix != nullptr && lane == 0) prefix[p.batch] = static_cast<int32_t>(T);
}

__device__ Cursor locate_tile(const DecodeParams& p, int64_t x, int lane, int32_t* prefix,
                              int64_t T) {
    const int64_t xs[1] = {x};
    Cursor c[1];
    locate_tiles<1>(p, xs, lane, prefix, T, c);
    return c[0];
}

// Move a cursor to the next tile of the list (single thread or warp-uniform).
__device__ __forceinline__ void advance(Cursor& c, const DecodeParams& p) {
    if (++c.jb < c.nt) return;
    c.seg_start += c.nt;
    c.jb = 0;
    if (++c.kvh < p.num_kv_heads) return;
    c.kvh = 0;
    do {
        ++c.b;
        c.L = c.b < p.batch ? p.context_lens[c.b] : 0;
        c.nt = c.b < p.batch ? seq_tiles(c.L, p) : 0;
    } while (c.b < p.batch && c.nt == 0);
}


// ======================================================================================
// SimtMath: fp32 CUDA-core tile arithmetic (any KV dtype, head_dim 64 or 128).
// ======================================================================================
template <int KV_T, int Q_T, int D, int G>
struct SimtMath {
    using OutT = typename QType<Q_T>::T;
    static constexpr int kKv = KV_T;
    static constexpr int kHeadDim = D;
    static constexpr bool kCanAppend = true;                                 // one query token
    static constexpr int kElem = KvElem<KV_T>::kBytes;
    static constexpr int kRowBytes = D * kElem;
    static constexpr int kTileBytes = kBlockTokens * kRowBytes;              // K or V tile
    static constexpr int kScaleBytes = kQuantized<KV_T> ? 2 * kBlockTokens * 4 : 0;  // K|V
    static constexpr int kStageBytes = 2 * kTileBytes + kScaleBytes;
    static constexpr int kStages = (kStageBytes >= 16384) ? 4 : 8;           // multiple of 4
    static constexpr int kParamBytes = 0;  // the row scales travel inside the stage
    static constexpr int kRingAlign = 128;
    static constexpr bool kUsesTma = false;                                  // 1-D bulk copies
    static constexpr int kChunkElems = 16 / kElem;                           // per 16-byte load
    static constexpr int kRowChunks = D / kChunkElems;
    static constexpr int kLPR = kRowChunks >= 8 ? 8 : kRowChunks;           // lanes per row
    static constexpr int kNCH = kRowChunks / kLPR;                           // chunks per lane/row
    static constexpr int kRPI = 32 / kLPR;                                   // rows per load step
    static constexpr int kNR = kBlockTokens / kRPI;                          // rows per lane
    static constexpr int kQPL = kNCH * kChunkElems;                          // q elems per lane/head
    static constexpr int kNV = kNR * G;                                      // partial scores/lane
    static constexpr int kVPL = kNV >= kLPR ? kNV / kLPR : 1;                // scores/lane after RS
    static constexpr int kDPL = D / 32;                                      // output cols per lane
    static constexpr int kSMLanes = (kBlockTokens * G) < 32 ? kBlockTokens * G : 32;
    static constexpr int kSPL = kBlockTokens * G / kSMLanes;                 // softmax vals/lane
    // per consumer warp: p pairs [16][G] float2, scores [16][G], corrections [G]
    static constexpr int kWarpScratch =
        (kBlockTokens * G * 8 + kBlockTokens * G * 4 + G * 4 + 15) / 16 * 16;
    // resident blocks per SM the register budget is sized for (G = 8 needs the
    // whole register file of one block's worth of q and accumulators)
    static constexpr int kMinBlocks = G >= 8 ? 1 : 3;
    static_assert(kStageBytes % 16 == 0, "bulk copies need 16-B alignment");
    static_assert(kQPL % 2 == 0 && kDPL % 2 == 0, "pairs for fp32x2 FMA");

    // ---- producer side: one stage = K tile, V tile (+ 8-bit row scales), 1-D bulk copies
    __device__ static void issue(uint8_t* st, uint8_t* prm, int64_t tile, uint64_t* bar,
                                 const DecodeParams& p, const TmaMaps&) {
        const int64_t off = tile * kTileBytes;
        mbar_arrive_expect_tx(bar, kStageBytes);
        bulk_copy_g2s(st, p.k_pool + off, kTileBytes, bar);
        bulk_copy_g2s(st + kTileBytes, p.v_pool + off, kTileBytes, bar);
        if constexpr (kQuantized<KV_T>)
            bulk_copy_g2s(prm, p.scales + tile * 2 * kBlockTokens, kScaleBytes, bar);
    }

    // Byte offset of byte `byte` of row `row` in a staged K or V tile (rows are contiguous).
    __device__ static __forceinline__ int32_t tile_byte(int32_t row, int32_t byte) {
        return row * D * kElem + byte;
    }

    // ---- consumer side
    int32_t lane, c, r0, sm_lane, sm_g;
    float2* p_buf;  // [16][G]
    float* s_buf;   // [16][G]
    float* c_buf;   // [G]
    float2 q2[G][kQPL / 2];
    float m_run, l_run;
    float2 o2[G][kDPL / 2];

    __device__ void init(int32_t lane_, uint8_t* scratch) {
        lane = lane_;
        c = lane % kLPR;    // chunk column of this lane in a K row
        r0 = lane / kLPR;   // first K row of this lane
        sm_lane = lane % kSMLanes;
        sm_g = sm_lane % G; // query head this lane's softmax values belong to
        p_buf = reinterpret_cast<float2*>(scratch);
        s_buf = reinterpret_cast<float*>(p_buf + kBlockTokens * G);
        c_buf = s_buf + kBlockTokens * G;
    }

    __device__ void load_q(const DecodeParams& p, int32_t b, int32_t kvh) {
        const int64_t qbase = (static_cast<int64_t>(b) * p.num_q_heads + kvh * G) * D;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k = 0; k < kNCH; ++k)
#pragma unroll
                for (int e = 0; e < kChunkElems; e += 2) {
                    const int64_t col = (c + k * kLPR) * kChunkElems + e;
                    q2[g][(k * kChunkElems + e) / 2] =
                        make_float2(load_q_elem<Q_T>(p.q, qbase + g * D + col) * p.scale_log2,
                                    load_q_elem<Q_T>(p.q, qbase + g * D + col + 1) * p.scale_log2);
                }
    }

    __device__ void reset() {
        m_run = -INFINITY;  // running max of this lane's head (base-2 units)
        l_run = 0.0f;       // this lane's share of the running sum
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int i = 0; i < kDPL / 2; ++i) o2[g][i] = make_float2(0.0f, 0.0f);
    }

    __device__ void tile(const uint8_t* kt, uint8_t* prm, int32_t jb, int32_t L,
                         const DecodeParams&) {
        const int32_t nvalid = min(kBlockTokens, L - jb * kBlockTokens);
        const uint8_t* vt = kt + kTileBytes;
        const float* ksc = reinterpret_cast<const float*>(prm);
        const float* vsc = ksc + kBlockTokens;

        // scores: partial dot products over this lane's columns, then reduce-scatter
        float acc[kNV];
#pragma unroll
        for (int i = 0; i < kNR; ++i) {
            const int row = r0 + kRPI * i;
            float2 ap[G];
#pragma unroll
            for (int g = 0; g < G; ++g) ap[g] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int kk = 0; kk < kNCH; ++kk) {
                const uint4 chunk =
                    *reinterpret_cast<const uint4*>(kt + row * (D * kElem) + (c + kk * kLPR) * 16);
                float2 kv[kChunkElems / 2];
                decode_chunk<KV_T>(chunk, kv);
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int e = 0; e < kChunkElems / 2; ++e)
                        ap[g] = ffma2(q2[g][kk * kChunkElems / 2 + e], kv[e], ap[g]);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) acc[i * G + g] = ap[g].x + ap[g].y;
        }
        reduce_scatter<kNV, kLPR / 2>(acc, lane);
#pragma unroll
        for (int v = 0; v < kVPL; ++v) {
            const int idx = (kNV >= kLPR) ? c * kVPL + v : c / (kLPR / kNV);
            const int t = r0 + kRPI * (idx / G);
            float sc = acc[v];
            if constexpr (kQuantized<KV_T>) sc *= ksc[t];
            s_buf[t * G + (idx % G)] = sc;
        }
        __syncwarp();

        // online softmax: lane handles head sm_g, tokens sm_lane/G + i*(kSMLanes/G)
        float sv[kSPL];
        float tmax = -INFINITY;
#pragma unroll
        for (int i = 0; i < kSPL; ++i) {
            const int t = sm_lane / G + i * (kSMLanes / G);
            sv[i] = (t < nvalid) ? s_buf[t * G + sm_g] : -INFINITY;
            tmax = fmaxf(tmax, sv[i]);
        }
#pragma unroll
        for (int m = G; m < kSMLanes; m <<= 1)
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, m));
        const float m_new = fmaxf(m_run, tmax);
        const float corr = exp2f(m_run - m_new);
        l_run *= corr;
#pragma unroll
        for (int i = 0; i < kSPL; ++i) {
            const int t = sm_lane / G + i * (kSMLanes / G);
            const float pr = exp2f(sv[i] - m_new);
            l_run += pr;
            float pv = pr;
            if constexpr (kQuantized<KV_T>) pv *= vsc[t];
            if (lane < kSMLanes) p_buf[t * G + sm_g] = make_float2(pv, pv);
        }
        m_run = m_new;
        if (lane < G) c_buf[lane] = corr;
        __syncwarp();

        // P.V: this lane's kDPL output columns for every head of the group
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float cg = c_buf[g];
#pragma unroll
            for (int i = 0; i < kDPL / 2; ++i) o2[g][i] = __fmul2_rn(o2[g][i], make_float2(cg, cg));
        }
        const uint8_t* vrow = vt + lane * kDPL * kElem;
        if (nvalid == kBlockTokens) {
#pragma unroll
            for (int t = 0; t < kBlockTokens; ++t) {
                float2 vv[kDPL / 2];
                load_v<KV_T, kDPL>(vrow + t * D * kElem, vv);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float2 pp = p_buf[t * G + g];
#pragma unroll
                    for (int i = 0; i < kDPL / 2; ++i) o2[g][i] = ffma2(pp, vv[i], o2[g][i]);
                }
            }
        } else {
            for (int t = 0; t < nvalid; ++t) {
                float2 vv[kDPL / 2];
                load_v<KV_T, kDPL>(vrow + t * D * kElem, vv);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float2 pp = p_buf[t * G + g];
#pragma unroll
                    for (int i = 0; i < kDPL / 2; ++i) o2[g][i] = ffma2(pp, vv[i], o2[g][i]);
                }
            }
        }
    }

    // End of a piece: the whole pair's output, or a partial (m, l, o) for the merge.
    __device__ void finish(const DecodeParams& p, int32_t b, int32_t kvh, bool whole,
                           int64_t pid) {
        float l = l_run;  // sum of l over the lanes that share this lane's head
#pragma unroll
        for (int m = G; m < kSMLanes; m <<= 1) l += __shfl_xor_sync(0xffffffffu, l, m);
        const int64_t bh0 = static_cast<int64_t>(b) * p.num_q_heads + kvh * G;
        if (whole) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float lg = __shfl_sync(0xffffffffu, l, g);
                OutT* o = static_cast<OutT*>(p.out) + (bh0 + g) * D + lane * kDPL;
#pragma unroll
                for (int i = 0; i < kDPL / 2; ++i) {
                    o[2 * i] = out_cast<OutT>(lg > 0.0f ? o2[g][i].x / lg : 0.0f);
                    o[2 * i + 1] = out_cast<OutT>(lg > 0.0f ? o2[g][i].y / lg : 0.0f);
                }
            }
        } else {
            if (lane < G) p.ws_ml[pid * G + lane] = make_float2(m_run, l);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int i = 0; i < kDPL / 2; ++i)
                    *reinterpret_cast<float2*>(&p.ws_o[(pid * G + g) * D + lane * kDPL + 2 * i]) =
                        o2[g][i];
        }
    }
};

// ======================================================================================
// MmaMath: tensor-core tile arithmetic for bf16, FP8, INT8, INT4 or KIVI KV, head_dim
// 128, bf16 q.
//
// A tile is 16 tokens x 128 dims.  K and V land in shared memory as [16 rows]
// x [128-byte] boxes written by TMA with the 128-byte swizzle (16-byte chunk
// c of row r stored at chunk c ^ (r & 7)), so every ldmatrix row set hits 32
// distinct banks.  The rows of the MMAs are the query rows of a (sequence, kv
// head) pair: row r = i * G + g is query token i (of Q) and head g (of G) of
// the group, R = G * Q <= 16 rows.  Per tile and warp (gid = lane / 4, tig =
// lane % 4):
//   S   = Q.K^T      m16n8k16, 2 token tiles x 8 dim steps; fp32 accumulators;
//                    lane holds rows gid and gid + 8 ("row sets" 0 and 1).
//   softmax on the accumulator fragments: a row holds tokens 2tig,2tig+1 and
//                    8+2tig,9+2tig; max/sum across the 4 lanes of the row.
//                    Query token i sits at position L - Q + i and sees
//                    positions <= L - Q + i (causal).
//   O^T += V^T.P^T   m16n8k16, rows = 16 head dims, columns = 8 query rows per
//                    row set; the P fragment of the score accumulators is
//                    exactly the B operand, so P never leaves registers.
// bf16 KV: bf16 MMAs, P rounded to bf16.  FP8 / INT8 KV: codes widened to f16 in
// registers (exact), f16 MMAs with q rounded to f16 and P (times the V row
// scale) rounded to f16; the K row scale multiplies the scores.  Element
// orders inside a k-step are permuted consistently between the two operands
// (a dot product does not depend on the order of its terms), which is what
// lets 8-bit rows be read with 16-bit ldmatrix.  4-bit KV (INT4, KIVI): the
// TMA stages each 16 codes padded to 16 bytes, and ldmatrix widens them to one
// code per byte, which the FP8 conversion turns into c * 2^-9 exactly; the row
// (INT4) or channel (KIVI keys) parameters enter as in the comments below.
// FP8 and 4-bit V tiles are read by a per-byte transposed ldmatrix, whose token
// order the score columns follow (tok()).  QM: kSingle = one query token
// (the decode: no causal bookkeeping), kNarrow = up to 8 query rows, kWide = up
// to 16 (two row sets).
// ======================================================================================
enum QueryMode { kSingle = 1, kNarrow = 2, kWide = 3 };

template <int KV_T, int G, int QM>
struct MmaMath {
    static constexpr bool WIDE = QM == kWide;
    static constexpr bool SINGLE = QM == kSingle;
    static_assert(KV_T == KV_BF16 || kQuantized<KV_T>, "bf16, FP8, INT8 or INT4 KV");
    static_assert(G <= 8, "a row set holds 8 query rows");
    using OutT = uint16_t;                                        // bf16 output
    static constexpr bool kF16 = kQuantized<KV_T>;              // codes widened to f16
    static constexpr bool kKivi = KV_T == KV_KIVI4;             // 4-bit, per-channel K params
    static constexpr bool kI4 = KV_T == KV_INT4 || kKivi;       // 4-bit codes, 64-byte rows
    // 4-bit tiles land in shared memory as 16-code groups padded to 16 bytes (128-byte
    // rows, 128-byte swizzle) and are widened to bytes by ldmatrix
    static constexpr bool kU4 = kI4;
    // V tiles read by the transposed byte load (4-bit and FP8 codes): the lanes then
    // own tokens in the order tok() gives, and the K rows are addressed to match
    static constexpr bool kByteV = kU4 || KV_T == KV_FP8_E4M3;
    static_assert(!kKivi || QM == kSingle, "KIVI pools: one query token");
    // parameter block: INT4 (scale, zero) per K row then per V row; KIVI per K
    // channel (128) then per V row (16), as float2
    static constexpr int kVParams = kKivi ? 128 : kBlockTokens;
    static constexpr int D = 128;
    static constexpr int kKv = KV_T;
    static constexpr int kHeadDim = D;
    static constexpr bool kCanAppend = SINGLE && !kKivi;          // fused append: decode only
    static constexpr int kSets = WIDE ? 2 : 1;                    // row sets used
    static constexpr int kRowBytes = kI4 ? D / 2 : D * KvElem<KV_T>::kBytes;  // 256 / 128 / 64
    static constexpr int kBoxRow = 128;                           // shared-memory bytes of a box row
    static constexpr int kBoxCols = kU4 ? 128 : 128 / KvElem<KV_T>::kBytes;  // box row, elements
    static constexpr int kBoxes = kU4 ? 1 : kRowBytes / kBoxRow;
    static constexpr int kBoxBytes = kBlockTokens * kBoxRow;
    static constexpr int kTileBytes = kBoxes * kBoxBytes;         // a K or V tile in shared memory
    static constexpr int kTileTx = kBlockTokens * kRowBytes;      // ... and the bytes it copies
    // K then V row parameters: fp32 scales (8-bit) or fp32 (scale, zero) pairs (4-bit)
    static constexpr int kScaleBytes =
        kKivi ? (128 + kBlockTokens) * 8 : (kI4 ? 2 * kBlockTokens * 8 : (kF16 ? 2 * kBlockTokens * 4 : 0));
    // A stage holds the K and V tiles (1024-byte aligned, as the swizzle needs) and,
    // after them, the tile's parameter line.  KIVI parameter lines sit in a ring of their
    // own instead (measured 3 % faster; for the other tiles the same move measured no
    // better): the line's 1152 bytes plus the f16 key parameters (128 x {scale,
    // zero 2^-9}) that the tile converts once, past the bytes the copy writes.
    static constexpr int kParamBytes = kKivi ? (kScaleBytes + 128 * 4 + 127) / 128 * 128 : 0;
    static constexpr int kStageBytes =
        kKivi ? 2 * kTileBytes : (2 * kTileBytes + kScaleBytes + 1023) / 1024 * 1024;
    static constexpr int kKiviF16Params = kScaleBytes;
    static constexpr int kStages = kF16 ? 12 : 8;                  // multiple of 4
    static_assert(kKiviF16Params % 16 == 0, "16-byte stores");
    static constexpr int kRingAlign = 1024;                       // 128-byte swizzle atom
    static constexpr bool kUsesTma = true;                        // tensor-map tile copies
    static constexpr int kWarpScratch = 0;
    static constexpr int kMinBlocks = WIDE ? 2 : 3;

    // ---- producer side: TMA boxes of K and V (+ the scale line of 8-bit codes by bulk copy)
    __device__ static void issue(uint8_t* st, uint8_t* prm, int64_t tile, uint64_t* bar,
                                 const DecodeParams& p, const TmaMaps& maps) {
        const int32_t row = static_cast<int32_t>(tile * kBlockTokens);
        mbar_arrive_expect_tx(bar, 2 * kTileTx + kScaleBytes);
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) {
            tma_load_2d(st + bx * kBoxBytes, &maps.k, bx * kBoxCols, row, bar);
            tma_load_2d(st + kTileBytes + bx * kBoxBytes, &maps.v, bx * kBoxCols, row, bar);
        }
        if constexpr (kF16)
            bulk_copy_g2s(prm, p.scales + tile * (kScaleBytes / 4), kScaleBytes, bar);
    }

    // Byte offset of byte `byte` of row `row` (as the pool stores it) in a staged
    // (swizzled) K or V tile; padded INT4 rows hold 8 bytes of codes per 16 bytes.
    __device__ static __forceinline__ int32_t tile_byte(int32_t row, int32_t byte) {
        if constexpr (kU4) return static_cast<int32_t>(swz(row, byte >> 3)) + (byte & 7);
        return static_cast<int32_t>(swz(row, byte >> 4)) + (byte & 15);
    }

    // Byte offset of 16-byte chunk `chunk` of row `row` in a swizzled K or V tile:
    // the 128-byte swizzle (chunk ^ row % 8 within 128-byte rows).
    __device__ static __forceinline__ uint32_t swz(int32_t row, int32_t chunk) {
        return (chunk >> 3) * kBoxBytes + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
    }

    // head-dim of row r (0..15) of output m-tile mi: 8-bit tiles interleave even/odd
    // dims (the byte order of a transposed 16-bit unit); bf16 and widened 4-bit tiles
    // keep them in order
    __device__ static __forceinline__ int32_t dim_of(int32_t mi, int32_t r) {
        if constexpr (kF16 && !kByteV) return 16 * mi + (r < 8 ? 2 * r : 2 * (r - 8) + 1);
        return 16 * mi + r;
    }

    // Byte-transposed V tiles: the transposed byte load hands lane tig the V rows of tokens
    // 4 tig .. 4 tig + 3, where the MMA's k pairs are 2 tig, 2 tig + 1 and 2 tig + 8,
    // 2 tig + 9.  Score column n is therefore token tok(n) (the K rows are addressed in
    // that order), so P's fragment matches the V fragment without moving data.
    __device__ static __forceinline__ int32_t tok(int32_t n) {
        if constexpr (kByteV) return 4 * ((n & 7) >> 1) + (n & 1) + 2 * (n >> 3);
        return n;
    }

    // ---- consumer side
    int32_t lane, gid, tig, nq, rows;
    int32_t qtok[kSets];        // query token of row gid + 8k (>= nq: padding row)
    uint32_t qa[kSets][8][2];   // A fragments of q per 16-dim k-step, row gid + 8k: {k lo, k hi}
    float o[kSets][8][4];       // O^T: [set][m-tile][c]; c0,c1 = (dim gid, rows 8k+2tig, +1)
    float m_run[kSets], l_run[kSets];  // running max (base 2), lane part of the sum, row gid+8k
    float qsum[kSets];          // 4-bit: sum of row gid+8k's q (as rounded to f16)
    float b_run[kSets];         // 4-bit: lane part of sum_t p_t * scale_t * zero_t, row gid+8k

    __device__ void init(int32_t lane_, uint8_t*) {
        lane = lane_;
        gid = lane >> 2;
        tig = lane & 3;
    }

    __device__ void load_q(const DecodeParams& p, int32_t b, int32_t kvh) {
        nq = SINGLE ? 1 : p.num_query_tokens;
        rows = G * nq;
#pragma unroll
        for (int k = 0; k < kSets; ++k) {
            const int32_t r = gid + 8 * k;
            qtok[k] = r < rows ? r / G : nq;
            const uint16_t* q = static_cast<const uint16_t*>(p.q) +
                                ((static_cast<int64_t>(b) * nq + (r / G)) * p.num_q_heads +
                                 kvh * G + r % G) * D;
            float qs = 0.0f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                if (r >= rows) {
                    qa[k][ks][0] = qa[k][ks][1] = 0u;
                } else if constexpr (!kF16) {
                    // k index 2tig+{0,1} -> dim 16ks+2tig+{0,1}; 8+2tig+{0,1} -> 16ks+8+2tig+{0,1}
                    qa[k][ks][0] = *reinterpret_cast<const uint32_t*>(q + 16 * ks + 2 * tig);
                    qa[k][ks][1] = *reinterpret_cast<const uint32_t*>(q + 16 * ks + 8 + 2 * tig);
                } else {
                    // 8-bit rows are read 4 codes per lane: k 2tig+{0,1} -> dim 16ks+4tig+{0,1},
                    // k 8+2tig+{0,1} -> dim 16ks+4tig+{2,3}
                    const uint2 w = *reinterpret_cast<const uint2*>(q + 16 * ks + 4 * tig);
                    qa[k][ks][0] = pack2<true>(__uint_as_float(w.x << 16),
                                               __uint_as_float(w.x & 0xffff0000u));
                    qa[k][ks][1] = pack2<true>(__uint_as_float(w.y << 16),
                                               __uint_as_float(w.y & 0xffff0000u));
                    if constexpr (kU4 && !kKivi) {  // widened INT4 codes: the row's q sum too
                        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&qa[k][ks][0]));
                        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&qa[k][ks][1]));
                        qs += (f0.x + f0.y) + (f1.x + f1.y);
                    }
                }
            }
            if constexpr (kI4 && !kKivi) {
                qs += __shfl_xor_sync(0xffffffffu, qs, 1);
                qs += __shfl_xor_sync(0xffffffffu, qs, 2);
                qsum[k] = qs;
            }
        }
    }

    __device__ void reset() {
#pragma unroll
        for (int k = 0; k < kSets; ++k) {
            m_run[k] = -INFINITY;
            l_run[k] = 0.0f;
            b_run[k] = 0.0f;
#pragma unroll
            for (int mi = 0; mi < 8; ++mi)
#pragma unroll
                for (int j = 0; j < 4; ++j) o[k][mi][j] = 0.0f;
        }
    }

    // A tile whose 16 tokens every query row sees (for one query token: every tile but
    // a pair's last) needs no position masks, and runs an instantiation without them.
    __device__ void tile(const uint8_t* kt, uint8_t* prm, int32_t jb, int32_t L,
                         const DecodeParams& p) {
        if ((jb + 1) * kBlockTokens <= L - nq + 1)
            tile_body<true>(kt, prm, jb, L, p);
        else
            tile_body<false>(kt, prm, jb, L, p);
    }

    template <bool FULL>
    __device__ __forceinline__ void tile_body(const uint8_t* kt, uint8_t* prm, int32_t jb, int32_t L,
                                              const DecodeParams& p) {
        const uint32_t k_s = smem_addr(kt);
        const uint32_t v_s = k_s + kTileBytes;
        // the parameter line (in-stage lines are addressed from the stage itself)
        if constexpr (kParamBytes == 0) prm = const_cast<uint8_t*>(kt) + 2 * kTileBytes;
        const float* ksc = reinterpret_cast<const float*>(prm);
        const float* vsc = ksc + kBlockTokens;
        const int32_t pos0 = jb * kBlockTokens;            // position of the tile's token 0
        const int32_t nvalid = min(kBlockTokens, L - pos0);
        const int32_t mtx = lane >> 3, r = lane & 7;       // ldmatrix: matrix and row this lane addresses

        // ---- S = Q.K^T: s[nt] = rows gid (c0, c1) and gid + 8 (c2, c3)
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        // KIVI: the 128 key channels' (scale, zero) as f16 {scale, zero 2^-9}, converted once
        // per tile into the parameter line's tail, past the bytes the copies write (so no
        // async-proxy write can meet these stores); lane l converts channels 4l .. 4l + 3
        [[maybe_unused]] const uint4* kp16 = reinterpret_cast<const uint4*>(prm + kKiviF16Params);
        if constexpr (kKivi) {
            constexpr uint32_t kTwoM9 = 0x18001800u;  // f16 2^-9, both halves
            const float4* pc = reinterpret_cast<const float4*>(ksc) + 2 * lane;
            const float4 p01 = pc[0], p23 = pc[1];  // (scale, zero) of 2 channels each
            uint4 h;
            h.x = pack2<true>(p01.x, p01.z);
            h.y = pack2<true>(p23.x, p23.z);
            h.z = hmul2u(pack2<true>(p01.y, p01.w), kTwoM9);
            h.w = hmul2u(pack2<true>(p23.y, p23.w), kTwoM9);
            reinterpret_cast<uint4*>(prm + kKiviF16Params)[lane] = h;
            __syncwarp();
        }
        auto a_hi = [&](int ks, int h) -> uint32_t {
            if constexpr (WIDE) return qa[1][ks][h];
            return 0u;
        };
        if constexpr (!kF16) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t b[4];  // {nt0 dims lo, nt0 dims hi, nt1 dims lo, nt1 dims hi}
                ldsm_x4(b, k_s + swz(8 * (mtx >> 1) + r, 2 * ks + (mtx & 1)));
                mma_16816<false>(s[0], qa[0][ks][0], a_hi(ks, 0), qa[0][ks][1], a_hi(ks, 1), b[0], b[1]);
                mma_16816<false>(s[1], qa[0][ks][0], a_hi(ks, 0), qa[0][ks][1], a_hi(ks, 1), b[2], b[3]);
            }
        } else {
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
                uint32_t w[4];  // {(ks 2kq, nt0), (2kq+1, nt0), (2kq, nt1), (2kq+1, nt1)}
                if constexpr (kU4)  // score column n is token tok(n): rows addressed in that order
                    ldsm_x4_u4(w, k_s + swz(tok(8 * (mtx >> 1) + r), 2 * kq + (mtx & 1)));
                else
                    ldsm_x4(w, k_s + swz(tok(8 * (mtx >> 1) + r), 2 * kq + (mtx & 1)));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int ks = 2 * kq + h;
                    uint32_t b0, b1, b2, b3;
                    widen_k4<KV_T>(w[h], b0, b1);
                    widen_k4<KV_T>(w[2 + h], b2, b3);
                    uint32_t qa0 = qa[0][ks][0], qa1 = qa[0][ks][1];
                    if constexpr (kKivi) {
                        // key channel d: (c - zero_d) * scale_d.  q takes the scales (q' = q *
                        // scale, f16), the codes the zero points: c 2^-9 - zero 2^-9 =
                        // (c - zero) 2^-9, exact in f16 while |c - zero| <= 2048 (the score
                        // takes the 2^-9 back).  This lane's dims of k-step ks: 16ks + 4tig +
                        // {0, 1} and {2, 3}, converted by lane 4ks + tig
                        const uint4 h = kp16[4 * ks + tig];
                        qa0 = hmul2u(qa0, h.x);
                        qa1 = hmul2u(qa1, h.y);
                        b0 = hsub2u(b0, h.z);
                        b1 = hsub2u(b1, h.w);
                        b2 = hsub2u(b2, h.z);
                        b3 = hsub2u(b3, h.w);
                    }
                    mma_16816<true>(s[0], qa0, a_hi(ks, 0), qa1, a_hi(ks, 1), b0, b1);
                    mma_16816<true>(s[1], qa0, a_hi(ks, 0), qa1, a_hi(ks, 1), b2, b3);
                }
            }
        }

        // ---- online softmax per row set: row gid + 8k holds tokens 8nt + 2tig + j
        float pr[kSets][2][2];
        float corr[kSets], m_old[kSets], m_ref[kSets], psum[kSets];
        bool grow = false;
#pragma unroll
        for (int k = 0; k < kSets; ++k) {
            // last position this row sees (one query token: the context's last, for every row)
            const int32_t last = SINGLE ? L - 1 : L - nq + qtok[k];
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int t = tok(8 * nt + 2 * tig + j);  // token of this score
                    float v;
                    if constexpr (kKivi) {
                        // parameters are in q' and the codes; the codes carry 2^-9
                        v = s[nt][2 * k + j] * (512.0f * p.scale_log2);
                    } else if constexpr (kI4) {
                        // (c - zero) * scale, summed over d with q: 512 acc - zero * sum_d q_d
                        const float2 pz = reinterpret_cast<const float2*>(ksc)[t];
                        v = (512.0f * s[nt][2 * k + j] - pz.y * qsum[k]) * pz.x * p.scale_log2;
                    } else {
                        v = s[nt][2 * k + j] * p.scale_log2;
                        if constexpr (kF16) v *= ksc[t];
                    }
                    pr[k][nt][j] = (FULL || pos0 + t <= last) ? v : -INFINITY;
                    mx = fmaxf(mx, pr[k][nt][j]);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run[k], mx);
            // with several query tokens a row may have seen nothing yet (max -inf):
            // exponentiate against 0 then; one query token always sees a token
            const float m_use = (!SINGLE && m_new == -INFINITY) ? 0.0f : m_new;
            grow = grow || m_new != m_run[k];
            m_old[k] = m_run[k];
            m_ref[k] = m_use;
            psum[k] = 0.0f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    pr[k][nt][j] = fast_exp2(pr[k][nt][j] - m_use);
                    psum[k] += pr[k][nt][j];
                }
            m_run[k] = m_new;
        }

        // Corrections 2^(m_old - m_new).  While no row of the warp has a new max they
        // are all exactly 1 and the exponentials, shuffles and rescale are skipped
        // (the result is the same to the bit).  Otherwise rescale the O^T columns:
        // column 8k + 2tig + j is row gid' = 2tig + j of set k.
        if (__any_sync(0xffffffffu, grow)) {
            float cf[kSets][2];
#pragma unroll
            for (int k = 0; k < kSets; ++k) {
                corr[k] = fast_exp2(m_old[k] - m_ref[k]);
                l_run[k] = l_run[k] * corr[k] + psum[k];
                cf[k][0] = __shfl_sync(0xffffffffu, corr[k], 8 * tig);
                cf[k][1] = __shfl_sync(0xffffffffu, corr[k], 8 * tig + 4);
            }
#pragma unroll
            for (int k = 0; k < kSets; ++k)
#pragma unroll
                for (int mi = 0; mi < 8; ++mi) {
                    o[k][mi][0] *= cf[k][0];
                    o[k][mi][1] *= cf[k][1];
                    o[k][mi][2] *= cf[k][0];
                    o[k][mi][3] *= cf[k][1];
                }
        } else {
#pragma unroll
            for (int k = 0; k < kSets; ++k) {
                corr[k] = 1.0f;
                l_run[k] += psum[k];
            }
        }

        // ---- P^T fragments (B operand: k = token, n = row gid of set k).  Tokens
        // past the context end have p = 0; their V rows and scales may hold
        // anything (NaN included), so they are removed by select, never multiplied.
        uint32_t pb[kSets][2];
#pragma unroll
        for (int k = 0; k < kSets; ++k) {
            if constexpr (kI4) {
                // O = sum_t p_t scale_t (c_t - zero_t) = sum_t P'_t c_t - sum_t P'_t zero_t,
                // P' = p * scale as the MMA sees it (f16); the second sum is kept per
                // row (b_run)
                const float2* vpz = reinterpret_cast<const float2*>(ksc) + kVParams;
                float2 pz[2][2];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int t = tok(8 * nt + 2 * tig + j);
                        pz[nt][j] = vpz[t];
                        const float pv = pr[k][nt][j] * pz[nt][j].x;
                        pr[k][nt][j] = (FULL || t < nvalid) ? pv : 0.0f;
                    }
                pb[k][0] = pack2<true>(pr[k][0][0], pr[k][0][1]);
                pb[k][1] = pack2<true>(pr[k][1][0], pr[k][1][1]);
                // (parameters past the context end may hold anything: select, never multiply)
                float bsum = 0.0f;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&pb[k][nt]));
                    const int t = tok(8 * nt + 2 * tig);  // tok(n + 1) = tok(n) + 1 for even n
                    bsum += (FULL || t < nvalid) ? f.x * pz[nt][0].y : 0.0f;
                    bsum += (FULL || t + 1 < nvalid) ? f.y * pz[nt][1].y : 0.0f;
                }
                b_run[k] = b_run[k] * corr[k] + bsum;
                continue;
            } else if constexpr (kF16) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int t = tok(8 * nt + 2 * tig + j);
                        pr[k][nt][j] = (FULL || t < nvalid) ? pr[k][nt][j] * vsc[t] : 0.0f;
                    }
            }
            pb[k][0] = pack2<kF16>(pr[k][0][0], pr[k][0][1]);
            pb[k][1] = pack2<kF16>(pr[k][1][0], pr[k][1][1]);
        }
        // V^T fragment halves of tokens 2tig, 2tig+1 (mask_a) and 8+2tig, 9+2tig (mask_b)
        const bool partial = !FULL && nvalid < kBlockTokens;
        const uint32_t mask_a = (2 * tig < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 1 < nvalid ? 0xffff0000u : 0u);
        const uint32_t mask_b = (2 * tig + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 9 < nvalid ? 0xffff0000u : 0u);

        // ---- O^T += V^T.P^T over 8 m-tiles of 16 head dims
        if constexpr (kByteV) {
            // FP8 codes past the context end may be NaN: masked by token when the tile is
            // partial.  4-bit codes all widen to finite values and those tokens have
            // P' = 0, so they need no mask
            const bool vmask = !kU4 && partial;
            const uint32_t m_lo = (4 * tig < nvalid ? 0x0000ffffu : 0u) |
                                  (4 * tig + 1 < nvalid ? 0xffff0000u : 0u);
            const uint32_t m_hi = (4 * tig + 2 < nvalid ? 0x0000ffffu : 0u) |
                                  (4 * tig + 3 < nvalid ? 0xffff0000u : 0u);
#pragma unroll
            for (int mp = 0; mp < 4; ++mp) {
                // chunks 2mp, 2mp + 1 (16 dims each), all 16 tokens, transposed per byte
                // (4-bit codes widened to bytes first): w = {(dim gid), (dim gid + 8)} of
                // chunk 2mp, then of chunk 2mp + 1, each the codes of tokens 4tig ..
                // 4tig + 3 = score columns 2tig, 2tig + 1, 2tig + 8, 2tig + 9
                uint32_t w[4];
                if constexpr (kU4)
                    ldsm_x2_trans_u4(w, v_s + swz(lane & 15, 2 * mp + (lane >> 4)));
                else
                    ldsm_x2_trans_b8(w, v_s + swz(lane & 15, 2 * mp + (lane >> 4)));
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    uint32_t lo0, hi0, lo1, hi1;  // (dim, token pair), E4M3 -> f16 exact
                    e4m3x4_to_f16x2x2(w[2 * m], lo0, hi0);
                    e4m3x4_to_f16x2x2(w[2 * m + 1], lo1, hi1);
                    if (vmask) {
                        lo0 &= m_lo;
                        lo1 &= m_lo;
                        hi0 &= m_hi;
                        hi1 &= m_hi;
                    }
#pragma unroll
                    for (int k = 0; k < kSets; ++k)
                        mma_16816<true>(o[k][2 * mp + m], lo0, lo1, hi0, hi1, pb[k][0], pb[k][1]);
                }
            }
        } else if constexpr (!kF16) {
#pragma unroll
            for (int mi = 0; mi < 8; ++mi) {
                uint32_t a[4];  // {tok 0-7 dims lo, tok 0-7 dims hi, tok 8-15 lo, tok 8-15 hi}
                ldsm_x4_trans(a, v_s + swz(8 * (mtx >> 1) + r, 2 * mi + (mtx & 1)));
                if (partial) {
                    a[0] &= mask_a;
                    a[1] &= mask_a;
                    a[2] &= mask_b;
                    a[3] &= mask_b;
                }
#pragma unroll
                for (int k = 0; k < kSets; ++k)
                    mma_16816<false>(o[k][mi], a[0], a[1], a[2], a[3], pb[k][0], pb[k][1]);
            }
        } else {
#pragma unroll
            for (int mq = 0; mq < 4; ++mq) {
                uint32_t w[4];  // {(tok 0-7, mt 2mq), (tok 8-15, 2mq), (tok 0-7, 2mq+1), (tok 8-15, 2mq+1)}
                ldsm_x4_trans(w, v_s + swz(8 * (mtx & 1) + r, 2 * mq + (mtx >> 1)));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // bytes of w: [t0 d2g, t0 d2g+1, t1 d2g, t1 d2g+1] -> [t0 d2g, t1 d2g,
                    // t0 d2g+1, t1 d2g+1]; row gid <- even dim, row gid + 8 <- odd dim
                    uint32_t lo0, hi0, lo1, hi1;
                    widen_v4<KV_T>(w[2 * h], lo0, hi0);
                    widen_v4<KV_T>(w[2 * h + 1], lo1, hi1);
                    if (partial) {
                        lo0 &= mask_a;
                        hi0 &= mask_a;
                        lo1 &= mask_b;
                        hi1 &= mask_b;
                    }
#pragma unroll
                    for (int k = 0; k < kSets; ++k)
                        mma_16816<true>(o[k][2 * mq + h], lo0, hi0, lo1, hi1, pb[k][0], pb[k][1]);
                }
            }
        }
    }

    __device__ void finish(const DecodeParams& p, int32_t b, int32_t kvh, bool whole,
                           int64_t pid) {
#pragma unroll
        for (int k = 0; k < kSets; ++k) {
            float l = l_run[k];  // row gid + 8k's sum over its 4 lanes
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            const float lr[2] = {__shfl_sync(0xffffffffu, l, 8 * tig),        // row 8k + 2tig
                                 __shfl_sync(0xffffffffu, l, 8 * tig + 4)};   // row 8k + 2tig + 1
            // 4-bit: O = 512 (the MMA sums of P' c 2^-9) - sum_t P'_t zero_t
            if constexpr (kI4) {
                float bq = b_run[k];
                bq += __shfl_xor_sync(0xffffffffu, bq, 1);
                bq += __shfl_xor_sync(0xffffffffu, bq, 2);
                const float br[2] = {__shfl_sync(0xffffffffu, bq, 8 * tig),
                                     __shfl_sync(0xffffffffu, bq, 8 * tig + 4)};
#pragma unroll
                for (int mi = 0; mi < 8; ++mi)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        o[k][mi][j] = 512.0f * o[k][mi][j] - br[j];
                        o[k][mi][2 + j] = 512.0f * o[k][mi][2 + j] - br[j];
                    }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int32_t row = 8 * k + 2 * tig + j;
                if (row >= rows) continue;
                const int32_t i = row / G, g = row % G;
                const float lh = lr[j];
                if (whole) {
                    uint16_t* out = static_cast<uint16_t*>(p.out) +
                                    ((static_cast<int64_t>(b) * nq + i) * p.num_q_heads + kvh * G + g) * D;
#pragma unroll
                    for (int mi = 0; mi < 8; ++mi) {
                        out[dim_of(mi, gid)] = out_cast<uint16_t>(lh > 0.0f ? o[k][mi][j] / lh : 0.0f);
                        out[dim_of(mi, gid + 8)] =
                            out_cast<uint16_t>(lh > 0.0f ? o[k][mi][2 + j] / lh : 0.0f);
                    }
                } else {
                    float* ws = p.ws_o + (pid * rows + row) * D;
#pragma unroll
                    for (int mi = 0; mi < 8; ++mi) {
                        ws[dim_of(mi, gid)] = o[k][mi][j];
                        ws[dim_of(mi, gid + 8)] = o[k][mi][2 + j];
                    }
                }
            }
            if (!whole && tig == 0 && gid + 8 * k < rows)
                p.ws_ml[pid * rows + gid + 8 * k] = make_float2(m_run[k], l);
        }
    }
};

// ======================================================================================
// Decode kernel: grid ceil(num_ranges / 4) CTAs of 160 threads.
// ======================================================================================
constexpr int kConsumerWarps = 4;
// Poll limits of the ring's waits (0: the hardware's own).  The producer warp spends
// most of a compute-bound call waiting for released stages; letting its polls sleep
// up to 20 us (a completed phase still wakes it) leaves the issue slots to the
// consumer warps.  Consumer polls keep the hardware's limit: a 20 us one measured
// no better.
constexpr uint32_t kConsumerSuspendNs = 0;
constexpr uint32_t kProducerSuspendNs = 20000u;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

template <class M>
struct Smem {
    static constexpr int kRingBytes = M::kStages * M::kStageBytes;
    static constexpr int kParamRingBytes = M::kStages * M::kParamBytes;
    static constexpr int kScratch = kConsumerWarps * M::kWarpScratch;
    static constexpr int kFlags = (2 * M::kStages * 4 + 16 + 15) / 16 * 16;  // ok, issued, abort
    static constexpr int kBars = 2 * M::kStages * 8;
    // dynamic shared memory is only guaranteed 16-byte aligned: pad for the ring's alignment
    static constexpr int kBytes =
        M::kRingAlign + kRingBytes + kParamRingBytes + kScratch + kFlags + kBars;
    static_assert(M::kParamBytes % 16 == 0, "bulk copies need 16-B alignment");
    static_assert(M::kMinBlocks * (kBytes + 1024) <= 228 * 1024, "resident CTAs per SM");
    static_assert(M::kStages % kConsumerWarps == 0, "stage s feeds consumer warp s % 4");
    static_assert(M::kStageBytes % M::kRingAlign == 0, "stages keep the ring's alignment");
    static_assert((kRingBytes + kParamRingBytes + kScratch + kFlags) % 8 == 0,
                  "mbarriers need 8-B alignment");
    static_assert(kBytes <= 227 * 1024, "shared memory per block");
};

// Fused append: the warp that attends to the last tile of pair (b, kvh) -- the
// tile holding position L - 1 -- writes that position's new K and V rows to the
// pool (for 8-bit pools: quantised exactly as reshape_and_cache does, codes and
// scales) and patches the staged copy of the tile, whose TMA read of that slot
// may have seen the old contents.  The block id was validated by the producer.
// Never inlined: it runs once per pair, and keeping it out of line keeps the
// tile loop's register allocation as it is without the append.
// What the fused append needs, passed by value so the out-of-line call does
// not force a local copy of the kernel's parameters.
struct AppendRow {
    const void* k_new;
    const void* v_new;
    uint8_t* k_dst;
    uint8_t* v_dst;
    float* scales_dst;
    const int32_t* table_row;  // block_table row of the sequence
    int64_t src_row;           // row of k_new / v_new: b * Hkv + kvh
    int32_t num_kv_heads, kvh, L, src_dtype;
};

// Bring the bytes of the new rows this lane will read in append_row into L1,
// so the warp that owns the pair's last tile does not wait on them there.
template <class M>
__device__ __forceinline__ void prefetch_append(const DecodeParams& p, int32_t b, int32_t kvh,
                                                int32_t lane) {
    constexpr int D = M::kHeadDim;
    const int64_t srow = static_cast<int64_t>(b) * p.num_kv_heads + kvh;
    const uint8_t* k = static_cast<const uint8_t*>(p.k_new);
    const uint8_t* v = static_cast<const uint8_t*>(p.v_new);
    int64_t off;
    if constexpr (kQuantized<M::kKv>) {
        const int32_t src_bytes = p.append_src_dtype == KV_F32 ? 4 : 2;
        off = (srow * D + lane * (D / 32)) * src_bytes;
    } else {
        constexpr int kRowBytes = D * KvElem<M::kKv>::kBytes;
        off = srow * kRowBytes + (lane * 16) % kRowBytes;
    }
    asm volatile("prefetch.global.L1 [%0];" ::"l"(k + off));
    asm volatile("prefetch.global.L1 [%0];" ::"l"(v + off));
}

template <class M>
__device__ __noinline__ void append_row(uint8_t* st, uint8_t* prm, const AppendRow a,
                                       int32_t lane) {
    constexpr int D = M::kHeadDim;
    constexpr int kRowBytes = M::kRowBytes;
    constexpr int kTileBytes = M::kTileBytes;
    const int32_t pos = a.L - 1, r = pos % kBlockTokens;
    const int64_t blk = a.table_row[pos / kBlockTokens];
    const int64_t rowi = (blk * a.num_kv_heads + a.kvh) * kBlockTokens + r;  // pool row
    if constexpr (M::kKv == KV_INT4) {
        // 2 bytes of packed codes per lane; (scale, zero) per row, K rows then V rows
        const int32_t src_bytes = a.src_dtype == KV_F32 ? 4 : 2;
        float2* pz_stage = reinterpret_cast<float2*>(prm);
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const uint8_t* src = static_cast<const uint8_t*>(which ? a.v_new : a.k_new);
            float x[D / 32];
            load_row_part<D>(src + a.src_row * D * src_bytes, a.src_dtype, lane, x);
            float sc, zr;
            const uint16_t codes = static_cast<uint16_t>(quantize_row_int4_warp<D>(x, &sc, &zr));
            *reinterpret_cast<uint16_t*>((which ? a.v_dst : a.k_dst) + rowi * kRowBytes + lane * 2) =
                codes;
            *reinterpret_cast<uint16_t*>(st + which * kTileBytes + M::tile_byte(r, lane * 2)) = codes;
            if (lane == 0) {
                reinterpret_cast<float2*>(a.scales_dst)
                    [((blk * a.num_kv_heads + a.kvh) * 2 + which) * kBlockTokens + r] =
                    make_float2(sc, zr);
                pz_stage[which * kBlockTokens + r] = make_float2(sc, zr);
            }
        }
    } else if constexpr (kQuantized<M::kKv>) {
        constexpr int kPer = D / 32;
        const int32_t src_bytes = a.src_dtype == KV_F32 ? 4 : 2;
        float* sc_stage = reinterpret_cast<float*>(prm);  // K then V row scales
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const uint8_t* src = static_cast<const uint8_t*>(which ? a.v_new : a.k_new);
            float x[kPer];
            load_row_part<D>(src + a.src_row * D * src_bytes, a.src_dtype, lane, x);
            float sc;
            const uint32_t codes = quantize_row_warp<M::kKv, D>(x, &sc);
            store_codes<D>((which ? a.v_dst : a.k_dst) + rowi * kRowBytes + lane * kPer, codes);
            store_codes<D>(st + which * kTileBytes + M::tile_byte(r, lane * kPer), codes);
            if (lane == 0) {
                a.scales_dst[((blk * a.num_kv_heads + a.kvh) * 2 + which) * kBlockTokens + r] = sc;
                sc_stage[which * kBlockTokens + r] = sc;
            }
        }
    } else {
        // same dtype as the pool: the row's bytes, 16 at a time
        constexpr int kChunks = kRowBytes / 16;
        for (int i = lane; i < 2 * kChunks; i += 32) {
            const int which = i / kChunks, c = i % kChunks;
            const uint8_t* src = static_cast<const uint8_t*>(which ? a.v_new : a.k_new);
            const uint4 v = *reinterpret_cast<const uint4*>(src + a.src_row * kRowBytes + c * 16);
            *reinterpret_cast<uint4*>((which ? a.v_dst : a.k_dst) + rowi * kRowBytes + c * 16) = v;
            *reinterpret_cast<uint4*>(st + which * kTileBytes + M::tile_byte(r, c * 16)) = v;
        }
    }
    // the stage is refilled by the async proxy (TMA) later: order these writes first
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
}

template <class M, int Q_T>
__device__ __forceinline__ void decode_body(const DecodeParams& p, const TmaMaps& maps) {
    using S = Smem<M>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + M::kRingAlign - 1) &
        ~static_cast<uintptr_t>(M::kRingAlign - 1));
    uint8_t* params = ring + S::kRingBytes;  // parameter lines (tile types that have a ring)
    uint8_t* scratch = params + S::kParamRingBytes;
    int32_t* stage_ok = reinterpret_cast<int32_t*>(scratch + S::kScratch);
    int32_t* issued_round = stage_ok + M::kStages;
    volatile int32_t* abort_flag = issued_round + M::kStages;
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stage_ok) + S::kFlags);
    uint64_t* empty = full + M::kStages;
    // stage s's parameter line: in the parameter ring, or after the stage's two tiles
    auto param_line = [&](int s) -> uint8_t* {
        if constexpr (M::kParamBytes > 0) return params + s * M::kParamBytes;
        else return ring + s * M::kStageBytes + 2 * M::kTileBytes;
    };

    const int32_t warp = threadIdx.x >> 5;
    const int32_t lane = threadIdx.x & 31;
    // No early launch_dependents here: this grid is persistent, and a dependent
    // (the merge) launched at its start parks CTAs on the SMs for its whole
    // duration; releasing it at exit measured 7 % faster per call.
    // The tensor maps are parameters, not data of the preceding grid: their
    // descriptors are fetched while it finishes.
    if constexpr (M::kUsesTma)
        if (threadIdx.x == kConsumerWarps * 32) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.v)) : "memory");
        }
    pdl_wait();
    const int64_t T = total_tiles(p, lane);
    const int64_t W0 = static_cast<int64_t>(blockIdx.x) * kConsumerWarps;

    if (warp == kConsumerWarps) {
        // ================= producer warp =================
        // the four ranges' first tiles, found in one pass over the lengths (the first
        // CTA also publishes every sequence's first tile for the merge)
        Cursor cur[kConsumerWarps];
        int32_t cnt[kConsumerWarps];
        int64_t first[kConsumerWarps];
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const int64_t lo = range_begin(W0 + w, T, p.num_ranges);
            cnt[w] = static_cast<int32_t>(range_begin(W0 + w + 1, T, p.num_ranges) - lo);
            first[w] = cnt[w] > 0 ? lo : -1;
        }
        locate_tiles<kConsumerWarps>(p, first, lane, blockIdx.x == 0 ? p.ws_seq_start : nullptr,
                                     T, cur);

        // Lane w feeds consumer warp w: its j-th tile goes through stage
        // w + 4 * (j % kPerWarp), so no warp's stage ever waits behind another
        // warp's; block ids are loaded kLook tiles ahead, the first ones before
        // the barrier setup.
        constexpr int kPerWarp = M::kStages / kConsumerWarps;
        constexpr int kLook = 4;
        Cursor c = cur[0];
        int32_t count = cnt[0];
#pragma unroll
        for (int w = 1; w < kConsumerWarps; ++w)
            if (lane == w) {
                c = cur[w];
                count = cnt[w];
            }
        if (lane >= kConsumerWarps) count = 0;
        int32_t q_id[kLook];
        int32_t q_head[kLook];
        auto fetch = [&](int j, int i) {
            if (j < count) {
                q_id[i] = p.block_table[static_cast<int64_t>(c.b) * p.max_blocks + c.jb];
                q_head[i] = c.kvh;
                advance(c, p);
            }
        };
#pragma unroll
        for (int i = 0; i < kLook; ++i) fetch(i, i);
        if (lane == 0) {
            for (int s = 0; s < M::kStages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
                issued_round[s] = -1;
            }
            *abort_flag = 0;
            mbar_init_fence();
        }
        __syncthreads();
        if (lane >= kConsumerWarps) return;
        for (int j0 = 0; j0 < count; j0 += kLook) {
#pragma unroll
            for (int i = 0; i < kLook; ++i) {
                const int j = j0 + i;
                if (j < count && !*abort_flag) {
                    const int s = lane + kConsumerWarps * (j % kPerWarp);
                    const int round = j / kPerWarp;
                    if (round > 0 && !mbar_wait_bounded<kProducerSuspendNs>(&empty[s], (round - 1) & 1)) {
                        report(p.dev_error, KV_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    } else {
                        const int32_t id = q_id[i];
                        const bool ok = id >= 0 && id < p.num_blocks;
                        stage_ok[s] = ok;
                        issued_round[s] = round;
                        if (ok) {
                            M::issue(ring + s * M::kStageBytes, param_line(s),
                                     static_cast<int64_t>(id) * p.num_kv_heads + q_head[i], &full[s],
                                     p, maps);
                        } else {
                            report(p.dev_error, KV_DEVERR_BAD_BLOCK_ID);
                            mbar_arrive(&full[s]);  // nothing to copy: the consumer skips it
                        }
                    }
                }
                fetch(j + kLook, i);
            }
        }
        if (*abort_flag) {
            // drain: wait (bounded) until no copy issued by this lane is in flight
            for (int s = lane; s < M::kStages; s += kConsumerWarps)
                if (issued_round[s] >= 0) mbar_wait_bounded(&full[s], issued_round[s] & 1);
        }
        return;
    }

    // ================= consumer warps =================
    const int64_t W = W0 + warp;
    const int64_t lo = range_begin(W, T, p.num_ranges);
    const int32_t n = static_cast<int32_t>(range_begin(W + 1, T, p.num_ranges) - lo);
    Cursor cur{};
    if (n > 0) cur = locate_tile(p, lo, lane, nullptr, T);
    __syncthreads();
    if (n <= 0) return;

    // When the range goes on past the current pair, bring the next pair's q rows
    // into L1 now, so switching pairs does not wait on them (one query token).
    auto prefetch_next_q = [&]() {
        if (p.num_query_tokens != 1 || lo + n <= cur.seg_start + cur.nt) return;
        const int32_t G = p.num_q_heads / p.num_kv_heads;
        const bool same_b = cur.kvh + 1 < p.num_kv_heads;
        const int32_t b = same_b ? cur.b : cur.b + 1, kvh = same_b ? cur.kvh + 1 : 0;
        constexpr int kQBytes = Q_T == KV_F32 ? 4 : 2;
        const int32_t bytes = G * M::kHeadDim * kQBytes;
        if (b < p.batch && lane * 128 < bytes)
            asm volatile("prefetch.global.L1 [%0];" ::"l"(
                static_cast<const uint8_t*>(p.q) +
                (static_cast<int64_t>(b) * p.num_q_heads + kvh * G) * M::kHeadDim * kQBytes +
                lane * 128));
    };

    M math;
    math.init(lane, scratch + warp * M::kWarpScratch);
    math.load_q(p, cur.b, cur.kvh);
    math.reset();
    prefetch_next_q();
    if constexpr (M::kCanAppend)
        if (p.k_new != nullptr) prefetch_append<M>(p, cur.b, cur.kvh, lane);
    int64_t piece_start = lo;

    constexpr int kPerWarp = M::kStages / kConsumerWarps;
    for (int j = 0; j < n; ++j) {
        const int s = warp + kConsumerWarps * (j % kPerWarp);
        const bool arrived =
            __all_sync(0xffffffffu, mbar_wait_bounded<kConsumerSuspendNs>(&full[s], (j / kPerWarp) & 1));
        if (!arrived) {  // output invalid (reported); the producer stops at its next tile
            if (lane == 0) report(p.dev_error, KV_DEVERR_TIMEOUT);
            *abort_flag = 1;
            return;
        }
        if (stage_ok[s]) {
            if constexpr (M::kCanAppend) {
                if (p.k_new != nullptr && cur.jb + 1 == cur.nt) {
                    const AppendRow a{p.k_new, p.v_new, p.k_dst, p.v_dst, p.scales_dst,
                                      p.block_table + static_cast<int64_t>(cur.b) * p.max_blocks,
                                      static_cast<int64_t>(cur.b) * p.num_kv_heads + cur.kvh,
                                      p.num_kv_heads, cur.kvh, cur.L, p.append_src_dtype};
                    append_row<M>(ring + s * M::kStageBytes, param_line(s), a, lane);
                }
            }
            math.tile(ring + s * M::kStageBytes, param_line(s), cur.jb, cur.L, p);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        // ---- end of a piece: at the end of a (sequence, kv head) pair or of the range
        const bool seg_end = cur.jb + 1 == cur.nt;
        if (seg_end || j == n - 1) {
            // KIVI pairs always end in the merge, which adds the bf16 residual tokens
            const bool whole = seg_end && piece_start == cur.seg_start && !p.kivi;
            const int64_t pid = static_cast<int64_t>(cur.b) * p.num_kv_heads + cur.kvh + W;
            math.finish(p, cur.b, cur.kvh, whole, pid);
            if (j + 1 < n) {
                advance(cur, p);  // next pair (the range goes on)
                piece_start = lo + j + 1;
                math.load_q(p, cur.b, cur.kvh);
                math.reset();
                prefetch_next_q();
                if constexpr (M::kCanAppend)
                    if (p.k_new != nullptr) prefetch_append<M>(p, cur.b, cur.kvh, lane);
            }
        } else {
            ++cur.jb;
        }
    }
}

// Registers per thread for kMinBlocks resident CTAs of kThreads.
constexpr int decode_max_regs(int min_blocks) {
    return min_blocks >= 3 ? 128 : (min_blocks == 2 ? 168 : 255);
}

// The decode grid.  The tensor-core tiles take the block size (__launch_bounds__
// without a CTA count) and a register cap (__maxnreg__); the code needs both to be
// spill-free.  Giving the resident CTA count to __launch_bounds__ instead yields
// the same register counts with 4 to 32 bytes of spills per thread, about one local
// load per tile (removing them measured time-neutral).  nvcc rejects the pair when
// the register count is a literal; with the count depending on the tile type it
// accepts it, and a compiler that did not would fail the build, not change the code.
// The CUDA-core tiles spill less with the CTA count given.
template <class M, int Q_T>
__global__ void __launch_bounds__(kThreads) __maxnreg__(decode_max_regs(M::kMinBlocks))
    paged_decode_kernel(const DecodeParams p, const __grid_constant__ TmaMaps maps) {
    decode_body<M, Q_T>(p, maps);
}

template <class M, int Q_T>
__global__ void __launch_bounds__(kThreads, M::kMinBlocks)
    paged_decode_kernel_simt(const DecodeParams p, const __grid_constant__ TmaMaps maps) {
    decode_body<M, Q_T>(p, maps);
}

// The entry point of a tile type (only that one is instantiated): tensor-core tiles
// the register-capped one, CUDA-core tiles the other.
template <class M, int Q_T>
constexpr auto decode_entry() {
    if constexpr (M::kUsesTma)
        return &paged_decode_kernel<M, Q_T>;
    else
        return &paged_decode_kernel_simt<M, Q_T>;
}

// ======================================================================================
// Merge kernel: pairs split over several consumer ranges are combined:
//   M = max_p m_p;  w_p = 2^(m_p - M);  out = sum_p w_p o_p / sum_p w_p l_p.
// A CTA is four warps.  With few pieces per pair each warp merges one output row
// (sequence, query token, head); when the split gives pairs many pieces (a few
// very long sequences) the four warps of a CTA share one row, fold a quarter of
// its pieces each and combine the four partial (max, sum, output) in warp order.
// Pairs of invalid length get zeros.
// ======================================================================================
constexpr int kMergeWarps = 4;

template <int Q_T, int D, bool KIVI, int WPR>
__global__ void __launch_bounds__(kMergeWarps * 32) paged_decode_merge_kernel(const DecodeParams p) {
    using OutT = typename QType<Q_T>::T;
    constexpr int kDPL = D / 32;
    constexpr int kBatch = 8;  // pieces whose partial outputs are loaded together
    __shared__ float sm_o[kMergeWarps][D];
    __shared__ float sm_ml[kMergeWarps][2];
    pdl_wait();
    pdl_trigger();
    const int32_t lane = threadIdx.x & 31;
    const int32_t warp = threadIdx.x >> 5;
    constexpr int32_t wpr = WPR;                // warps per output row: 1 or 4
    const int32_t part = warp % wpr;            // this warp's share of the row's pieces
    // the output row (sequence b, query token i, head h): out is [B][Q][Hq][D]
    const int64_t bh = static_cast<int64_t>(blockIdx.x) * (kMergeWarps / wpr) + warp / wpr;
    const int32_t nq = p.num_query_tokens;
    const int64_t rows_total = static_cast<int64_t>(p.batch) * nq * p.num_q_heads;
    if (bh >= rows_total) return;
    int32_t b, h, qi;
    if (rows_total <= 0x7fffffff) {  // 32-bit divisions (64-bit ones are long chains)
        const uint32_t x = static_cast<uint32_t>(bh), hq = static_cast<uint32_t>(p.num_q_heads);
        const uint32_t bq = x / hq;  // b * nq + qi
        h = static_cast<int32_t>(x - bq * hq);
        b = static_cast<int32_t>(bq / static_cast<uint32_t>(nq));
        qi = static_cast<int32_t>(bq) - b * nq;
    } else {
        b = static_cast<int32_t>(bh / (static_cast<int64_t>(nq) * p.num_q_heads));
        h = static_cast<int32_t>(bh % p.num_q_heads);
        qi = static_cast<int32_t>((bh / p.num_q_heads) % nq);
    }
    const int32_t G = p.num_q_heads / p.num_kv_heads;
    const int32_t kvh = h / G;
    const int32_t R = G * nq;          // query rows of a (sequence, kv head) pair
    const int32_t g = qi * G + h % G;  // this warp's row within the pair
    // KIVI: bring all 16 residual K and V rows of the pair into L1 now, in the same
    // round trip as the lengths, so the residual tokens at the end wait on no memory
    // (rows past L mod 16 are fetched and not used); lane l fetches 128-byte line
    // l % 2 of row l / 2 (D = 128: two lines per row)
    if constexpr (KIVI) {
        const int64_t row = (static_cast<int64_t>(b) * p.num_kv_heads + kvh) * kBlockTokens +
                            lane / 2;
        const int64_t e = row * D + (lane % 2) * 64;
        if (lane / 2 < kBlockTokens && (lane % 2) * 64 < D) {
            asm volatile("prefetch.global.L1 [%0];" ::"l"(p.res_k + e));
            asm volatile("prefetch.global.L1 [%0];" ::"l"(p.res_v + e));
        }
    }
    // three independent loads in one round trip
    const int32_t L = p.context_lens[b];
    const int64_t T = p.ws_seq_start[p.batch];
    const int64_t seq0 = p.ws_seq_start[b];
    const int32_t nt = seq_tiles(L, p);
    OutT* out = static_cast<OutT*>(p.out) + bh * D + lane * kDPL;
    if (!seq_valid(L, p)) {
        if (part == 0) {
#pragma unroll
            for (int j = 0; j < kDPL; ++j) out[j] = out_cast<OutT>(0.0f);
            if (lane == 0 && g == 0 && kvh == 0) report(p.dev_error, KV_DEVERR_BAD_CONTEXT_LEN);
        }
        return;
    }
    const int64_t a = seq0 + static_cast<int64_t>(kvh) * nt;
    const int64_t w_first = nt > 0 ? range_of(a, T, p.num_ranges) : 0;
    const int64_t w_last = nt > 0 ? range_of(a + nt - 1, T, p.num_ranges) : -1;
    // a pair within one range was written by the decode kernel (KIVI: never)
    if (!KIVI && w_first == w_last) return;
    const int64_t s = static_cast<int64_t>(b) * p.num_kv_heads + kvh;
    const int32_t npieces = static_cast<int32_t>(w_last - w_first + 1);
    // pieces are (pair s, range W) for the non-empty ranges W in [w_first, w_last],
    // with piece id s + W (see the decode kernel); ranges are never empty when T >= N
    const bool all_ranges_full = T >= p.num_ranges;
    auto piece_id = [&](int32_t i) -> int64_t {
        const int64_t W = w_first + i;
        if (all_ranges_full) return s + W;
        return range_begin(W, T, p.num_ranges) < range_begin(W + 1, T, p.num_ranges) ? s + W : -1;
    };
    // this warp's pieces [pb, pe)
    const int32_t pb = static_cast<int32_t>((static_cast<int64_t>(npieces) * part) / wpr);
    const int32_t pe = static_cast<int32_t>((static_cast<int64_t>(npieces) * (part + 1)) / wpr);
    float o[kDPL];
#pragma unroll
    for (int j = 0; j < kDPL; ++j) o[j] = 0.0f;
    float l = 0.0f;
    float M = -INFINITY;
    for (int i0 = pb; i0 < pe; i0 += 32) {
        // lane i: piece i0+i's (m, l); every lane: this round's first kBatch partial
        // outputs -- both sets of loads are in flight together
        const int64_t pl = (i0 + lane < pe) ? piece_id(i0 + lane) : -1;
        const float2 ml = pl >= 0 ? p.ws_ml[pl * R + g] : make_float2(-INFINITY, 0.0f);
        const int cnt = min(32, pe - i0);
        float v[kBatch][kDPL];
        int64_t pids[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            pids[u] = __shfl_sync(0xffffffffu, pl, u);
            const bool use = u < cnt && pids[u] >= 0;
            const float* src = p.ws_o + ((use ? pids[u] : 0) * R + g) * D + lane * kDPL;
#pragma unroll
            for (int j = 0; j < kDPL; ++j) v[u][j] = use ? src[j] : 0.0f;
        }
        // running max over the pieces seen so far; rescale what is accumulated
        float mr = ml.x;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, m));
        const float M_new = fmaxf(M, mr);
        if (M_new == -INFINITY) continue;  // nothing but empty pieces so far
        const float c = exp2f(M - M_new);
        l *= c;
#pragma unroll
        for (int j = 0; j < kDPL; ++j) o[j] *= c;
        M = M_new;
        const float wl = pl >= 0 ? exp2f(ml.x - M) : 0.0f;
        l += wl * ml.y;  // lane-partial, reduced at the end
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const float w = __shfl_sync(0xffffffffu, wl, u);
#pragma unroll
            for (int j = 0; j < kDPL; ++j) o[j] = fmaf(w, v[u][j], o[j]);
        }
        for (int u0 = kBatch; u0 < cnt; u0 += kBatch) {
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = (u0 + u) & 31;
                pids[u] = __shfl_sync(0xffffffffu, pl, i);
                const bool use = u0 + u < cnt && pids[u] >= 0;
                const float* src = p.ws_o + ((use ? pids[u] : 0) * R + g) * D + lane * kDPL;
#pragma unroll
                for (int j = 0; j < kDPL; ++j) v[u][j] = use ? src[j] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const float w = __shfl_sync(0xffffffffu, wl, (u0 + u) & 31);
#pragma unroll
                for (int j = 0; j < kDPL; ++j) o[j] = fmaf(w, v[u][j], o[j]);
            }
        }
    }
    if constexpr (WPR > 1) {
        // the row's warps' (M, l, o), combined by its first warp in warp order
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) l += __shfl_xor_sync(0xffffffffu, l, m);
#pragma unroll
        for (int j = 0; j < kDPL; ++j) sm_o[warp][lane * kDPL + j] = o[j];
        if (lane == 0) {
            sm_ml[warp][0] = M;
            sm_ml[warp][1] = l;
        }
        __syncthreads();
        if (part != 0) return;
        float Mt = -INFINITY;
        for (int w = warp; w < warp + wpr; ++w) Mt = fmaxf(Mt, sm_ml[w][0]);
        float lt = 0.0f;
#pragma unroll
        for (int j = 0; j < kDPL; ++j) o[j] = 0.0f;
        for (int w = warp; w < warp + wpr; ++w) {
            const float mw = sm_ml[w][0];
            const float c = mw == -INFINITY ? 0.0f : exp2f(mw - Mt);
            lt += c * sm_ml[w][1];
#pragma unroll
            for (int j = 0; j < kDPL; ++j) o[j] = fmaf(c, sm_o[w][lane * kDPL + j], o[j]);
        }
        M = Mt;
        l = lane == 0 ? lt : 0.0f;  // lane-partial again: counted once in the sum below
    }
    if constexpr (KIVI) {
        // KIVI: the newest L mod 16 tokens, kept in bf16 at res_k / res_v
        // [batch][Hkv][16][D] (fetched into L1 at the start), join the softmax (same
        // base-2 scores): all their scores first, then one rescale, then the value rows.
        const int32_t nres = L % kBlockTokens;
        if (nres > 0) {
            float qf[kDPL];
#pragma unroll
            for (int j = 0; j < kDPL; ++j) qf[j] = load_q_elem<Q_T>(p.q, bh * D + lane * kDPL + j);
            const int64_t rbase =
                ((static_cast<int64_t>(b) * p.num_kv_heads + kvh) * kBlockTokens) * D + lane * kDPL;
            float sc[kBlockTokens];
#pragma unroll
            for (int r = 0; r < kBlockTokens; ++r) {
                float dot = 0.0f;
                if (r < nres) {
                    const uint16_t* kr = p.res_k + rbase + r * D;
#pragma unroll
                    for (int j = 0; j < kDPL; ++j)
                        dot = fmaf(qf[j], __uint_as_float(static_cast<uint32_t>(kr[j]) << 16), dot);
                }
                sc[r] = dot;
            }
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
                for (int r = 0; r < kBlockTokens; ++r)
                    sc[r] += __shfl_xor_sync(0xffffffffu, sc[r], m);
            float M_new = M;
#pragma unroll
            for (int r = 0; r < kBlockTokens; ++r)
                if (r < nres) M_new = fmaxf(M_new, sc[r] * p.scale_log2);
            const float c = exp2f(M - M_new);  // 0 while nothing came before (M = -inf)
            l *= c;
#pragma unroll
            for (int j = 0; j < kDPL; ++j) o[j] *= c;
#pragma unroll
            for (int r = 0; r < kBlockTokens; ++r) {
                if (r < nres) {
                    const float w = exp2f(sc[r] * p.scale_log2 - M_new);
                    l += lane == 0 ? w : 0.0f;  // l is lane-partial: count the token once
                    const uint16_t* vr = p.res_v + rbase + r * D;
#pragma unroll
                    for (int j = 0; j < kDPL; ++j)
                        o[j] = fmaf(w, __uint_as_float(static_cast<uint32_t>(vr[j]) << 16), o[j]);
                }
            }
            M = M_new;
        }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) l += __shfl_xor_sync(0xffffffffu, l, m);
#pragma unroll
    for (int j = 0; j < kDPL; ++j) out[j] = out_cast<OutT>(l > 0.0f ? o[j] / l : 0.0f);
}

// ---- launch ------------------------------------------------------------------------------
constexpr int kMaxDevices = 64;

template <class M, int Q_T, int D>
static cudaError_t launch_one(const DecodeParams& p, const TmaMaps& maps, cudaStream_t stream) {
    using S = Smem<M>;
    constexpr auto kernel = decode_entry<M, Q_T>();
    // Whether this device's context has the kernel's dynamic shared-memory limit raised.
    // A context destroyed and created again (cudaDeviceReset) loses it while the flag
    // stays set; the launch then fails before anything runs, and is retried once after
    // raising the limit again.
    static std::atomic<bool> attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto set_attr = [&]() -> cudaError_t {
        const cudaError_t a = cudaFuncSetAttribute(
            kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
        if (a == cudaSuccess && dev < kMaxDevices)
            attr_set[dev].store(true, std::memory_order_relaxed);
        return a;
    };
    if (dev >= kMaxDevices || !attr_set[dev].load(std::memory_order_relaxed)) {
        e = set_attr();
        if (e != cudaSuccess) return e;
    }
    const unsigned grid =
        static_cast<unsigned>((p.num_ranges + kConsumerWarps - 1) / kConsumerWarps);
    e = launch_pdl(kernel, dim3(grid), dim3(kThreads), S::kBytes, stream, p, maps);
    if (e == cudaErrorInvalidValue) {
        cudaGetLastError();
        e = set_attr();
        if (e == cudaSuccess)
            e = launch_pdl(kernel, dim3(grid), dim3(kThreads), S::kBytes, stream, p, maps);
    }
    if (e != cudaSuccess) return e;
    const int64_t rows = static_cast<int64_t>(p.batch) * p.num_query_tokens * p.num_q_heads;
    const int64_t rows_per_cta = kMergeWarps / p.merge_warps_per_row;
    const dim3 merge_grid(static_cast<unsigned>((rows + rows_per_cta - 1) / rows_per_cta));
    const dim3 merge_block(kMergeWarps * 32);
    // the KIVI merge also attends to the bf16 residual, the split one shares rows
    // between warps: their own instantiations, so the common one keeps its smaller
    // register footprint (and occupancy)
    const bool split = p.merge_warps_per_row > 1;
    if (p.kivi)
        return split ? launch_pdl(paged_decode_merge_kernel<Q_T, D, true, kMergeWarps>,
                                  merge_grid, merge_block, 0, stream, p)
                     : launch_pdl(paged_decode_merge_kernel<Q_T, D, true, 1>, merge_grid,
                                  merge_block, 0, stream, p);
    return split ? launch_pdl(paged_decode_merge_kernel<Q_T, D, false, kMergeWarps>, merge_grid,
                              merge_block, 0, stream, p)
                 : launch_pdl(paged_decode_merge_kernel<Q_T, D, false, 1>, merge_grid,
                              merge_block, 0, stream, p);
}

template <int KV_T, int Q_T, int D>
static cudaError_t dispatch_g(const DecodeParams& p, const TmaMaps& maps, int32_t group,
                              cudaStream_t s) {
    switch (group) {
        case 1: return launch_one<SimtMath<KV_T, Q_T, D, 1>, Q_T, D>(p, maps, s);
        case 2: return launch_one<SimtMath<KV_T, Q_T, D, 2>, Q_T, D>(p, maps, s);
        case 4: return launch_one<SimtMath<KV_T, Q_T, D, 4>, Q_T, D>(p, maps, s);
        default: return launch_one<SimtMath<KV_T, Q_T, D, 8>, Q_T, D>(p, maps, s);
    }
}

template <int KV_T, int QM>
static cudaError_t dispatch_mma_g(const DecodeParams& p, const TmaMaps& maps, int32_t group,
                                  cudaStream_t s) {
    switch (group) {
        case 1: return launch_one<MmaMath<KV_T, 1, QM>, KV_BF16, 128>(p, maps, s);
        case 2: return launch_one<MmaMath<KV_T, 2, QM>, KV_BF16, 128>(p, maps, s);
        case 4: return launch_one<MmaMath<KV_T, 4, QM>, KV_BF16, 128>(p, maps, s);
        default: return launch_one<MmaMath<KV_T, 8, QM>, KV_BF16, 128>(p, maps, s);
    }
}

template <int KV_T>
static cudaError_t dispatch_mma(const DecodeParams& p, const TmaMaps& maps, int32_t group,
                                cudaStream_t s) {
    if (p.num_query_tokens == 1) return dispatch_mma_g<KV_T, kSingle>(p, maps, group, s);
    if constexpr (KV_T == KV_KIVI4) {
        return cudaErrorInvalidValue;  // one query token only
    } else {
        return group * p.num_query_tokens > 8 ? dispatch_mma_g<KV_T, kWide>(p, maps, group, s)
                                              : dispatch_mma_g<KV_T, kNarrow>(p, maps, group, s);
    }
}

template <int KV_T, int Q_T>
static cudaError_t dispatch_d(const DecodeParams& p, const TmaMaps& maps, int32_t head_dim,
                              int32_t group, cudaStream_t s) {
    return head_dim == 128 ? dispatch_g<KV_T, Q_T, 128>(p, maps, group, s)
                           : dispatch_g<KV_T, Q_T, 64>(p, maps, group, s);
}

template <int KV_T>
static cudaError_t dispatch_q(const DecodeParams& p, const TmaMaps& maps, int32_t q_dtype,
                              int32_t head_dim, int32_t group, cudaStream_t s) {
    return q_dtype == KV_F32 ? dispatch_d<KV_T, KV_F32>(p, maps, head_dim, group, s)
                             : dispatch_d<KV_T, KV_BF16>(p, maps, head_dim, group, s);
}

bool decode_uses_tensor_cores(int32_t kv_dtype, int32_t q_dtype, int32_t head_dim) {
    return (kv_dtype == KV_BF16 || kv_dtype == KV_FP8_E4M3 || kv_dtype == KV_INT8 ||
            kv_dtype == KV_INT4 || kv_dtype == KV_KIVI4) &&
           q_dtype == KV_BF16 &&
           head_dim == 128;
}

cudaError_t launch_paged_decode(const DecodeParams& p, const TmaMaps& maps, int32_t kv_dtype,
                                int32_t q_dtype, int32_t head_dim, int32_t group,
                                cudaStream_t stream) {
    if (decode_uses_tensor_cores(kv_dtype, q_dtype, head_dim)) {
        switch (kv_dtype) {
            case KV_BF16: return dispatch_mma<KV_BF16>(p, maps, group, stream);
            case KV_INT8: return dispatch_mma<KV_INT8>(p, maps, group, stream);
            case KV_INT4: return dispatch_mma<KV_INT4>(p, maps, group, stream);
            case KV_KIVI4: return dispatch_mma<KV_KIVI4>(p, maps, group, stream);
            default: return dispatch_mma<KV_FP8_E4M3>(p, maps, group, stream);
        }
    }
    // (4-bit pools have only the tensor-core tile; the host rejects other shapes)
    if (kv_dtype == KV_INT4 || kv_dtype == KV_KIVI4) return cudaErrorInvalidValue;
    switch (kv_dtype) {
        case KV_F32: return dispatch_q<KV_F32>(p, maps, q_dtype, head_dim, group, stream);
        case KV_BF16: return dispatch_q<KV_BF16>(p, maps, q_dtype, head_dim, group, stream);
        case KV_INT8: return dispatch_q<KV_INT8>(p, maps, q_dtype, head_dim, group, stream);
        default: return dispatch_q<KV_FP8_E4M3>(p, maps, q_dtype, head_dim, group, stream);
    }
}

int32_t decode_ctas_per_sm(int32_t, int32_t, int32_t group, int32_t query_tokens) {
    return group * query_tokens > 8 ? 2 : 3;
}

}  // namespace pkv
