// Split-K paged GQA decode attention and its log-sum-exp merge (sm_100a).
//
// Method ("KV Cache 深度解析" §一/§三/§四; "llm-inference-optimization" notes
// §三 Flash Attention; k1-blog 2026-07-13, "PagedAttention 與 vLLM"):
// one thread block per (sequence partition, kv head, sequence).  Its tokens are
// read once from HBM, block by block through the block table, and shared by
// the G query heads of the GQA group.  A running max m, running sum l and
// rescaled running output o per query head implement the online softmax, so
// no score ever leaves the chip.  Partitions of one sequence are combined by
// their log-sum-exp in a second, small kernel.
//
// B200 design:
//  * one producer warp stages each (block, kv head) K and V tile (a contiguous
//    16*D-element span in the pool) into shared memory with 1-D bulk async
//    copies (the TMA engine, no multicast) completing on mbarriers, through a
//    ring of kStages stages;
//  * four consumer warps take the ring's tiles round-robin, each keeping its
//    own (m, l, o), and are combined through shared memory at the end;
//  * q·K: every lane multiplies 16-byte chunks of 8 lanes-per-row against q
//    held in registers with packed fp32x2 FMAs, then a shuffle reduce-scatter
//    leaves each score on one lane; P·V: every lane owns D/32 output columns;
//  * scores are in base-2 units (q pre-scaled by scale*log2 e) and exp2 is used.
// Every wait is bounded; bad block ids and context lengths are reported through
// the error word and never dereferenced.
#include "kernels.cuh"

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

template <int KV_T, int D, int G>
struct Cfg {
    static constexpr int kElem = KvElem<KV_T>::kBytes;
    static constexpr int kTileBytes = kBlockTokens * D * kElem;              // K or V tile
    static constexpr int kScaleBytes = (KV_T == KV_FP8_E4M3) ? kBlockTokens * 4 : 0;
    static constexpr int kStageBytes = 2 * kTileBytes + 2 * kScaleBytes;
    static constexpr int kConsumerWarps = 4;
    static constexpr int kThreads = (kConsumerWarps + 1) * 32;
    static constexpr int kStages = (kStageBytes >= 16384) ? 4 : 8;           // multiple of 4
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
    // shared memory
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kEpiBytes = kConsumerWarps * G * (D * 4 + 8);
    static constexpr int kBodyBytes = kRingBytes > kEpiBytes ? kRingBytes : kEpiBytes;
    // per consumer warp: p pairs [16][G] float2, scores [16][G], corrections [G];
    // rounded to 16 bytes so every warp's region (and its float2 array) is aligned
    static constexpr int kWarpScratch = (kBlockTokens * G * 8 + kBlockTokens * G * 4 + G * 4 + 15) / 16 * 16;
    static constexpr int kMaxIds = 512;                                      // partition <= 8192
    static constexpr int kSmemBytes =
        kBodyBytes + kConsumerWarps * kWarpScratch + kMaxIds * 4 + 2 * kStages * 8 + 16;
    // resident blocks per SM the register budget is sized for (G = 8 needs the
    // whole register file of one block's worth of q and accumulators)
    static constexpr int kMinBlocks = G >= 8 ? 1 : 3;
    static_assert(kStages % kConsumerWarps == 0, "stage ring must split evenly across warps");
    static_assert(kStageBytes % 16 == 0 && kBodyBytes % 16 == 0, "bulk copies need 16-B alignment");
    static_assert((kBodyBytes + kConsumerWarps * kWarpScratch + kMaxIds * 4) % 8 == 0,
                  "mbarriers need 8-B alignment");
    static_assert(kQPL % 2 == 0 && kDPL % 2 == 0, "pairs for fp32x2 FMA");
};

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
            out[2 * i] = e4m3x2_to_float2(w[i] & 0xffffu);
            out[2 * i + 1] = e4m3x2_to_float2(w[i] >> 16);
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
            out[0] = e4m3x2_to_float2(w & 0xffffu);
            out[1] = e4m3x2_to_float2(w >> 16);
        } else {
            out[0] = e4m3x2_to_float2(*reinterpret_cast<const uint16_t*>(p));
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
__device__ __forceinline__ float load_q(const void* q, int64_t i) {
    if constexpr (Q_T == KV_F32) {
        return static_cast<const float*>(q)[i];
    } else {
        return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(q)[i]) << 16);
    }
}

// ======================================================================================
// Split kernel: grid (max_parts, Hkv, B), kThreads threads.
// ======================================================================================
template <int KV_T, int Q_T, int D, int G>
__global__ void __launch_bounds__(Cfg<KV_T, D, G>::kThreads, Cfg<KV_T, D, G>::kMinBlocks)
    paged_decode_split_kernel(const DecodeParams p) {
    using C = Cfg<KV_T, D, G>;
    using OutT = typename QType<Q_T>::T;
    extern __shared__ __align__(128) uint8_t smem[];

    const int32_t part = blockIdx.x;
    const int32_t kvh = blockIdx.y;
    const int32_t b = blockIdx.z;
    const int32_t warp = threadIdx.x >> 5;
    const int32_t lane = threadIdx.x & 31;
    const int32_t L = p.context_lens[b];
    const int32_t hq0 = kvh * G;  // first query head of the group

    if (L < 1 || L > p.max_context_len) {
        // invalid length: the first partition writes zeros and reports
        if (part == 0) {
            OutT* out = static_cast<OutT*>(p.out);
            for (int i = threadIdx.x; i < G * D; i += C::kThreads)
                out[(static_cast<int64_t>(b) * p.num_q_heads + hq0) * D + i] = out_cast<OutT>(0.0f);
            if (threadIdx.x == 0) report(p.dev_error, KV_DEVERR_BAD_CONTEXT_LEN);
        }
        return;
    }
    const int32_t P = p.partition_tokens;
    const int32_t nparts = (L + P - 1) / P;
    if (part >= nparts) return;
    const int32_t tok0 = part * P;
    const int32_t tok1 = min(tok0 + P, L);
    const int32_t blk0 = tok0 / kBlockTokens;
    const int32_t nblk = (tok1 - tok0 + kBlockTokens - 1) / kBlockTokens;

    uint8_t* ring = smem;
    uint8_t* scratch = smem + C::kBodyBytes;
    int32_t* ids = reinterpret_cast<int32_t*>(scratch + C::kConsumerWarps * C::kWarpScratch);
    uint64_t* full = reinterpret_cast<uint64_t*>(ids + C::kMaxIds);
    uint64_t* empty = full + C::kStages;
    volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(empty + C::kStages);

    // ---- prologue: block ids (producer warp), q (consumer warps), barriers -------
    float2 q2[G][C::kQPL / 2];
    const int32_t c = lane % C::kLPR;   // chunk column of this lane
    const int32_t r0 = lane / C::kLPR;  // first row of this lane
    if (warp == C::kConsumerWarps) {
        const int32_t* bt = p.block_table + static_cast<int64_t>(b) * p.max_blocks + blk0;
        for (int k = lane; k < nblk; k += 32) {
            int32_t id = bt[k];
            if (id < 0 || id >= p.num_blocks) {
                report(p.dev_error, KV_DEVERR_BAD_BLOCK_ID);
                id = -1;
            }
            ids[k] = id;
        }
        if (lane == 0) {
            for (int s = 0; s < C::kStages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            *abort_flag = 0;
            mbar_init_fence();
        }
    } else {
        const int64_t qbase = (static_cast<int64_t>(b) * p.num_q_heads + hq0) * D;
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int k = 0; k < C::kNCH; ++k) {
#pragma unroll
                for (int e = 0; e < C::kChunkElems; e += 2) {
                    const int64_t col = (c + k * C::kLPR) * C::kChunkElems + e;
                    q2[g][(k * C::kChunkElems + e) / 2] =
                        make_float2(load_q<Q_T>(p.q, qbase + g * D + col) * p.scale_log2,
                                    load_q<Q_T>(p.q, qbase + g * D + col + 1) * p.scale_log2);
                }
            }
        }
    }
    __syncthreads();

    // ---- producer: stream the partition's tiles through the ring -----------------
    if (warp == C::kConsumerWarps) {
        if (lane == 0) {
            const int64_t tile_elems = static_cast<int64_t>(kBlockTokens) * D;
            int issued = 0;
            for (int k = 0; k < nblk; ++k) {
                const int s = k % C::kStages;
                const int round = k / C::kStages;
                if (round > 0 && !mbar_wait_bounded(&empty[s], (round - 1) & 1)) {
                    report(p.dev_error, KV_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                if (*abort_flag) break;
                const int32_t id = ids[k];
                uint8_t* st = ring + s * C::kStageBytes;
                if (id >= 0) {
                    const int64_t tile = static_cast<int64_t>(id) * p.num_kv_heads + kvh;
                    mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                    bulk_copy_g2s(st, p.k_pool + tile * tile_elems * C::kElem, C::kTileBytes,
                                  &full[s]);
                    bulk_copy_g2s(st + C::kTileBytes, p.v_pool + tile * tile_elems * C::kElem,
                                  C::kTileBytes, &full[s]);
                    if constexpr (KV_T == KV_FP8_E4M3) {
                        bulk_copy_g2s(st + 2 * C::kTileBytes, p.k_scales + tile * kBlockTokens,
                                      C::kScaleBytes, &full[s]);
                        bulk_copy_g2s(st + 2 * C::kTileBytes + C::kScaleBytes,
                                      p.v_scales + tile * kBlockTokens, C::kScaleBytes,
                                      &full[s]);
                    }
                } else {
                    mbar_arrive(&full[s]);  // skipped block: nothing to wait for
                }
                issued = k + 1;
            }
            if (*abort_flag) {
                // drain: wait (bounded) until no copy issued by this block is in flight
                for (int k = (issued > C::kStages ? issued - C::kStages : 0); k < issued; ++k)
                    mbar_wait_bounded(&full[k % C::kStages], (k / C::kStages) & 1);
            }
        }
        return;
    }

    // ---- consumers ------------------------------------------------------------------
    float2* p_buf = reinterpret_cast<float2*>(scratch + warp * C::kWarpScratch);  // [16][G]
    float* s_buf = reinterpret_cast<float*>(p_buf + kBlockTokens * G);            // [16][G]
    float* c_buf = s_buf + kBlockTokens * G;                                       // [G]

    const int32_t sm_lane = lane % C::kSMLanes;
    const int32_t sm_g = sm_lane % G;
    float m_run = -INFINITY;  // running max of this lane's head (base-2 units)
    float l_run = 0.0f;       // this lane's share of the running sum
    float2 o2[G][C::kDPL / 2];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < C::kDPL / 2; ++i) o2[g][i] = make_float2(0.0f, 0.0f);

    for (int k = warp; k < nblk; k += C::kConsumerWarps) {
        const int s = k % C::kStages;
        const bool arrived = __all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (k / C::kStages) & 1));
        if (!arrived) {
            if (lane == 0) report(p.dev_error, KV_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
        if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
        if (ids[k] >= 0) {
            const uint8_t* kt = ring + s * C::kStageBytes;
            const uint8_t* vt = kt + C::kTileBytes;
            const float* ksc = reinterpret_cast<const float*>(kt + 2 * C::kTileBytes);
            const float* vsc = ksc + kBlockTokens;
            const int32_t nvalid = min(kBlockTokens, tok1 - (tok0 + k * kBlockTokens));

            // scores: partial dot products over this lane's columns, then reduce-scatter
            float acc[C::kNV];
#pragma unroll
            for (int i = 0; i < C::kNR; ++i) {
                const int row = r0 + C::kRPI * i;
                float2 ap[G];
#pragma unroll
                for (int g = 0; g < G; ++g) ap[g] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int kk = 0; kk < C::kNCH; ++kk) {
                    const uint4 chunk = *reinterpret_cast<const uint4*>(
                        kt + row * (D * C::kElem) + (c + kk * C::kLPR) * 16);
                    float2 kv[C::kChunkElems / 2];
                    decode_chunk<KV_T>(chunk, kv);
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int e = 0; e < C::kChunkElems / 2; ++e)
                            ap[g] = ffma2(q2[g][kk * C::kChunkElems / 2 + e], kv[e], ap[g]);
                }
#pragma unroll
                for (int g = 0; g < G; ++g) acc[i * G + g] = ap[g].x + ap[g].y;
            }
            reduce_scatter<C::kNV, C::kLPR / 2>(acc, lane);
#pragma unroll
            for (int v = 0; v < C::kVPL; ++v) {
                const int idx = (C::kNV >= C::kLPR) ? c * C::kVPL + v : c / (C::kLPR / C::kNV);
                const int t = r0 + C::kRPI * (idx / G);
                float sc = acc[v];
                if constexpr (KV_T == KV_FP8_E4M3) sc *= ksc[t];
                s_buf[t * G + (idx % G)] = sc;
            }
            __syncwarp();

            // online softmax: lane handles head sm_g, tokens sm_lane/G + j*(kSMLanes/G)
            float sv[C::kSPL];
            float tmax = -INFINITY;
#pragma unroll
            for (int j = 0; j < C::kSPL; ++j) {
                const int t = sm_lane / G + j * (C::kSMLanes / G);
                sv[j] = (t < nvalid) ? s_buf[t * G + sm_g] : -INFINITY;
                tmax = fmaxf(tmax, sv[j]);
            }
#pragma unroll
            for (int m = G; m < C::kSMLanes; m <<= 1)
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, m));
            const float m_new = fmaxf(m_run, tmax);
            const float corr = exp2f(m_run - m_new);
            l_run *= corr;
#pragma unroll
            for (int j = 0; j < C::kSPL; ++j) {
                const int t = sm_lane / G + j * (C::kSMLanes / G);
                const float pr = exp2f(sv[j] - m_new);
                l_run += pr;
                float pv = pr;
                if constexpr (KV_T == KV_FP8_E4M3) pv *= vsc[t];
                if (lane < C::kSMLanes) p_buf[t * G + sm_g] = make_float2(pv, pv);
            }
            m_run = m_new;
            if (lane < G) c_buf[lane] = corr;
            __syncwarp();

            // P·V: this lane's kDPL output columns for every head of the group
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float cg = c_buf[g];
#pragma unroll
                for (int i = 0; i < C::kDPL / 2; ++i) o2[g][i] = __fmul2_rn(o2[g][i], make_float2(cg, cg));
            }
            const uint8_t* vrow = vt + lane * C::kDPL * C::kElem;
            if (nvalid == kBlockTokens) {
#pragma unroll
                for (int t = 0; t < kBlockTokens; ++t) {
                    float2 vv[C::kDPL / 2];
                    load_v<KV_T, C::kDPL>(vrow + t * D * C::kElem, vv);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float2 pp = p_buf[t * G + g];
#pragma unroll
                        for (int i = 0; i < C::kDPL / 2; ++i) o2[g][i] = ffma2(pp, vv[i], o2[g][i]);
                    }
                }
            } else {
                for (int t = 0; t < nvalid; ++t) {
                    float2 vv[C::kDPL / 2];
                    load_v<KV_T, C::kDPL>(vrow + t * D * C::kElem, vv);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float2 pp = p_buf[t * G + g];
#pragma unroll
                        for (int i = 0; i < C::kDPL / 2; ++i) o2[g][i] = ffma2(pp, vv[i], o2[g][i]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- combine the consumer warps of this block ---------------------------------------
    // full sum of l over the lanes sharing this lane's head
#pragma unroll
    for (int m = G; m < C::kSMLanes; m <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, m);
    asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumerWarps * 32) : "memory");
    if (*abort_flag) return;  // output invalid, reported as KV_DEVERR_TIMEOUT
    float* wo = reinterpret_cast<float*>(ring);                                  // [W][G][D]
    float2* wml = reinterpret_cast<float2*>(ring + C::kConsumerWarps * G * D * 4);  // [W][G]
    if (lane < G) wml[warp * G + lane] = make_float2(m_run, l_run);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int i = 0; i < C::kDPL / 2; ++i)
            *reinterpret_cast<float2*>(&wo[(warp * G + g) * D + lane * C::kDPL + 2 * i]) = o2[g][i];
    asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumerWarps * 32) : "memory");

    const int32_t tid = threadIdx.x;  // 0 .. 127
    for (int idx = tid; idx < G * D; idx += C::kConsumerWarps * 32) {
        const int g = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < C::kConsumerWarps; ++w) M = fmaxf(M, wml[w * G + g].x);
        float o = 0.0f, l = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < C::kConsumerWarps; ++w) {
                const float2 ml = wml[w * G + g];
                const float f = exp2f(ml.x - M);
                o += f * wo[(w * G + g) * D + d];
                l += f * ml.y;
            }
        }
        const int64_t bh = static_cast<int64_t>(b) * p.num_q_heads + hq0 + g;
        if (nparts == 1) {
            static_cast<OutT*>(p.out)[bh * D + d] = out_cast<OutT>(l > 0.0f ? o / l : 0.0f);
        } else {
            p.ws_o[(bh * p.max_parts + part) * D + d] = o;
            if (d == 0) p.ws_ml[bh * p.max_parts + part] = make_float2(M, l);
        }
    }
}

// ======================================================================================
// Merge kernel: one warp per (sequence, query head) with more than one partition.
//   M = max_p m_p;  w_p = 2^(m_p - M);  out = sum_p w_p o_p / sum_p w_p l_p
// ======================================================================================
template <int Q_T, int D>
__global__ void __launch_bounds__(128) paged_decode_merge_kernel(const DecodeParams p) {
    using OutT = typename QType<Q_T>::T;
    constexpr int kDPL = D / 32;
    const int32_t lane = threadIdx.x & 31;
    const int64_t bh = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (bh >= static_cast<int64_t>(p.batch) * p.num_q_heads) return;
    const int32_t b = static_cast<int32_t>(bh / p.num_q_heads);
    const int32_t L = p.context_lens[b];
    if (L < 1 || L > p.max_context_len) return;
    const int32_t n = (L + p.partition_tokens - 1) / p.partition_tokens;
    if (n <= 1) return;
    const float2* ml = p.ws_ml + bh * p.max_parts;
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) M = fmaxf(M, ml[i].x);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    float o[kDPL];
#pragma unroll
    for (int i = 0; i < kDPL; ++i) o[i] = 0.0f;
    float l = 0.0f;
    if (M != -INFINITY) {
        const float* ob = p.ws_o + bh * p.max_parts * D + lane * kDPL;
        for (int i = 0; i < n; ++i) {
            const float2 mli = ml[i];
            const float w = exp2f(mli.x - M);
            l += w * mli.y;
#pragma unroll
            for (int j = 0; j < kDPL; ++j) o[j] += w * ob[static_cast<int64_t>(i) * D + j];
        }
    }
    OutT* out = static_cast<OutT*>(p.out) + bh * D + lane * kDPL;
#pragma unroll
    for (int j = 0; j < kDPL; ++j) out[j] = out_cast<OutT>(l > 0.0f ? o[j] / l : 0.0f);
}

// ---- dispatch ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;

template <int KV_T, int Q_T, int D, int G>
static cudaError_t launch_one(const DecodeParams& p, cudaStream_t stream) {
    using C = Cfg<KV_T, D, G>;
    static bool attr_set[kMaxDevices] = {};  // benign race: every caller sets the same value
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !attr_set[dev]) {
        e = cudaFuncSetAttribute(paged_decode_split_kernel<KV_T, Q_T, D, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) attr_set[dev] = true;
    }
    const dim3 grid(p.max_parts, p.num_kv_heads, p.batch);
    paged_decode_split_kernel<KV_T, Q_T, D, G><<<grid, C::kThreads, C::kSmemBytes, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.max_parts <= 1) return e;
    const int64_t warps = static_cast<int64_t>(p.batch) * p.num_q_heads;
    paged_decode_merge_kernel<Q_T, D><<<static_cast<unsigned>((warps + 3) / 4), 128, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int KV_T, int Q_T, int D>
static cudaError_t dispatch_g(const DecodeParams& p, int32_t group, cudaStream_t s) {
    switch (group) {
        case 1: return launch_one<KV_T, Q_T, D, 1>(p, s);
        case 2: return launch_one<KV_T, Q_T, D, 2>(p, s);
        case 4: return launch_one<KV_T, Q_T, D, 4>(p, s);
        default: return launch_one<KV_T, Q_T, D, 8>(p, s);
    }
}

template <int KV_T, int Q_T>
static cudaError_t dispatch_d(const DecodeParams& p, int32_t head_dim, int32_t group,
                              cudaStream_t s) {
    return head_dim == 128 ? dispatch_g<KV_T, Q_T, 128>(p, group, s)
                           : dispatch_g<KV_T, Q_T, 64>(p, group, s);
}

template <int KV_T>
static cudaError_t dispatch_q(const DecodeParams& p, int32_t q_dtype, int32_t head_dim,
                              int32_t group, cudaStream_t s) {
    return q_dtype == KV_F32 ? dispatch_d<KV_T, KV_F32>(p, head_dim, group, s)
                             : dispatch_d<KV_T, KV_BF16>(p, head_dim, group, s);
}

cudaError_t launch_paged_decode(const DecodeParams& p, int32_t kv_dtype, int32_t q_dtype,
                                int32_t head_dim, int32_t group, cudaStream_t stream) {
    switch (kv_dtype) {
        case KV_F32: return dispatch_q<KV_F32>(p, q_dtype, head_dim, group, stream);
        case KV_BF16: return dispatch_q<KV_BF16>(p, q_dtype, head_dim, group, stream);
        default: return dispatch_q<KV_FP8_E4M3>(p, q_dtype, head_dim, group, stream);
    }
}

}  // namespace pkv
