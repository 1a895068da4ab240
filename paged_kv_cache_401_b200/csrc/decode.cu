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
//    is exactly the number of CTAs resident on the GPU (persistent), so the
//    tile stream never stalls between work items;
//  * the producer's lane 0 walks the four consumer warps' ranges and stages
//    each (block, kv head) K and V tile -- one contiguous 16*D span of the
//    pool -- into a shared-memory ring with 1-D bulk async copies (the TMA
//    engine, no multicast) completing on mbarriers; block ids are fetched 8
//    tiles ahead so table-lookup latency never gaps the stream;
//  * stage s of the ring always feeds consumer warp s % 4; a consumer warp
//    computes q.K with packed fp32x2 FMAs on 16-byte chunks (8 lanes per
//    row) and a shuffle reduce-scatter, the online softmax with exp2 on
//    scores pre-scaled by scale*log2(e), and P.V with each lane owning D/32
//    output columns, all in fp32;
//  * every wait is bounded; bad block ids and context lengths are reported
//    through the error word and never dereferenced.
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
    // shared memory: the ring, per-consumer-warp scratch, per-stage flags, barriers
    static constexpr int kRingBytes = kStages * kStageBytes;
    // per consumer warp: p pairs [16][G] float2, scores [16][G], corrections [G];
    // rounded to 16 bytes so every warp's region (and its float2 array) is aligned
    static constexpr int kWarpScratch =
        (kBlockTokens * G * 8 + kBlockTokens * G * 4 + G * 4 + 15) / 16 * 16;
    static constexpr int kFlagsBytes = (2 * kStages * 4 + 16 + 15) / 16 * 16;  // ok, issued, abort
    static constexpr int kSmemBytes =
        kRingBytes + kConsumerWarps * kWarpScratch + kFlagsBytes + 2 * kStages * 8;
    // resident blocks per SM the register budget is sized for (G = 8 needs the
    // whole register file of one block's worth of q and accumulators)
    static constexpr int kMinBlocks = G >= 8 ? 1 : 3;
    static_assert(kStages % kConsumerWarps == 0, "stage s feeds consumer warp s % 4");
    static_assert(kStageBytes % 16 == 0 && kRingBytes % 16 == 0, "bulk copies need 16-B alignment");
    static_assert((kRingBytes + kConsumerWarps * kWarpScratch + kFlagsBytes) % 8 == 0,
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


// ---- tile list bookkeeping ----------------------------------------------------------
// Tiles of a sequence with context length L: ceil(L/16), or 0 when L is invalid.
__device__ __forceinline__ int32_t seq_tiles(int32_t L, int32_t max_context_len) {
    return (L >= 1 && L <= max_context_len) ? (L + kBlockTokens - 1) / kBlockTokens : 0;
}

// First tile of consumer range W (ranges are equal cuts of the T-tile list).
__device__ __forceinline__ int64_t range_begin(int64_t W, int64_t T, int32_t num_ranges) {
    return W >= num_ranges ? T : (W * T) / num_ranges;
}

// The range holding tile x < T: the largest W with range_begin(W) <= x, i.e.
// the largest W with W*T < (x+1)*num_ranges.
__device__ __forceinline__ int64_t range_of(int64_t x, int64_t T, int32_t num_ranges) {
    const int64_t W = ((x + 1) * num_ranges - 1) / T;
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
        t += static_cast<int64_t>(p.num_kv_heads) * seq_tiles(p.context_lens[b], p.max_context_len);
    return warp_sum_i64(t);
}

// Position of one tile in the list: sequence b, kv head, block index jb in
// the sequence, the sequence's tile count nt and length L, and the list
// index of the pair's first tile.
struct Cursor {
    int32_t b, kvh, jb, nt, L;
    int64_t seg_start;
};

// Warp-cooperative search for the pair holding tile x (< T).  When `prefix`
// is non-null the warp also writes every sequence's first tile (and T at
// [batch]) there for the merge kernel.
__device__ Cursor locate_tile(const DecodeParams& p, int64_t x, int lane, int32_t* prefix,
                              int64_t T) {
    Cursor c{p.batch, 0, 0, 0, 0, T};
    bool found = false;
    int64_t base = 0;
    for (int b0 = 0; b0 < p.batch; b0 += 32) {
        const int b = b0 + lane;
        const int32_t L = b < p.batch ? p.context_lens[b] : 0;
        const int32_t nt = b < p.batch ? seq_tiles(L, p.max_context_len) : 0;
        const int64_t cnt = static_cast<int64_t>(p.num_kv_heads) * nt;
        int64_t incl = cnt;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, incl, m);
            if (lane >= m) incl += y;
        }
        const int64_t excl = base + incl - cnt;
        if (prefix != nullptr && b < p.batch) prefix[b] = static_cast<int32_t>(excl);
        const uint32_t hit = __ballot_sync(0xffffffffu, !found && cnt > 0 && x >= excl && x < excl + cnt);
        if (hit != 0u && !found) {
            const int src = __ffs(hit) - 1;
            const int64_t e = __shfl_sync(0xffffffffu, excl, src);
            const int32_t n = __shfl_sync(0xffffffffu, nt, src);
            const int32_t l = __shfl_sync(0xffffffffu, L, src);
            const int64_t off = x - e;
            c.b = b0 + src;
            c.nt = n;
            c.L = l;
            c.kvh = static_cast<int32_t>(off / n);
            c.jb = static_cast<int32_t>(off % n);
            c.seg_start = e + static_cast<int64_t>(c.kvh) * n;
            found = true;
            if (prefix == nullptr) break;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (prefix != nullptr && lane == 0) prefix[p.batch] = static_cast<int32_t>(T);
    return c;
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
        c.nt = c.b < p.batch ? seq_tiles(c.L, p.max_context_len) : 0;
    } while (c.b < p.batch && c.nt == 0);
}

// ======================================================================================
// Decode kernel: grid ceil(num_ranges / 4) CTAs of kThreads threads.
// ======================================================================================
template <int KV_T, int Q_T, int D, int G>
__global__ void __launch_bounds__(Cfg<KV_T, D, G>::kThreads, Cfg<KV_T, D, G>::kMinBlocks)
    paged_decode_kernel(const DecodeParams p) {
    using C = Cfg<KV_T, D, G>;
    using OutT = typename QType<Q_T>::T;
    extern __shared__ __align__(128) uint8_t smem[];

    const int32_t warp = threadIdx.x >> 5;
    const int32_t lane = threadIdx.x & 31;
    uint8_t* ring = smem;
    uint8_t* scratch = smem + C::kRingBytes;
    int32_t* stage_ok = reinterpret_cast<int32_t*>(scratch + C::kConsumerWarps * C::kWarpScratch);
    int32_t* issued_round = stage_ok + C::kStages;
    volatile int32_t* abort_flag = issued_round + C::kStages;
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stage_ok) + C::kFlagsBytes);
    uint64_t* empty = full + C::kStages;

    pdl_wait();
    pdl_trigger();
    const int64_t T = total_tiles(p, lane);
    const int64_t W0 = static_cast<int64_t>(blockIdx.x) * C::kConsumerWarps;

    if (warp == C::kConsumerWarps) {
        // ================= producer warp =================
        Cursor cur[C::kConsumerWarps];
        int32_t cnt[C::kConsumerWarps];
        int32_t kmax = 0;
#pragma unroll
        for (int w = 0; w < C::kConsumerWarps; ++w) {
            const int64_t lo = range_begin(W0 + w, T, p.num_ranges);
            const int64_t hi = range_begin(W0 + w + 1, T, p.num_ranges);
            cnt[w] = static_cast<int32_t>(hi - lo);
            // the first CTA also publishes every sequence's first tile for the merge
            int32_t* prefix = (blockIdx.x == 0 && w == 0) ? p.ws_seq_start : nullptr;
            if (cnt[w] > 0 || prefix != nullptr) cur[w] = locate_tile(p, lo, lane, prefix, T);
            kmax = max(kmax, C::kConsumerWarps * cnt[w]);
        }
        if (lane == 0) {
            for (int s = 0; s < C::kStages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
                issued_round[s] = -1;
            }
            *abort_flag = 0;
            mbar_init_fence();
        }
        __syncthreads();
        if (lane != 0) return;

        // slot k feeds consumer warp k % 4 with its (k / 4)-th tile, through
        // stage k % kStages; block ids are loaded kLook slots ahead
        constexpr int kLook = 8;
        int32_t q_id[kLook];
        int32_t q_head[kLook];
        bool q_valid[kLook];
        auto fetch = [&](int k, int i) {
            const int w = i % C::kConsumerWarps;  // == k % 4: i == k % kLook
            q_valid[i] = k < kmax && (k / C::kConsumerWarps) < cnt[w];
            if (q_valid[i]) {
                const Cursor& c = cur[w];
                q_id[i] = p.block_table[static_cast<int64_t>(c.b) * p.max_blocks + c.jb];
                q_head[i] = c.kvh;
                advance(cur[w], p);
            }
        };
#pragma unroll
        for (int i = 0; i < kLook; ++i) fetch(i, i);
        const int64_t tile_elems = static_cast<int64_t>(kBlockTokens) * D;
        for (int k0 = 0; k0 < kmax; k0 += kLook) {
#pragma unroll
            for (int i = 0; i < kLook; ++i) {
                const int k = k0 + i;
                if (q_valid[i] && !*abort_flag) {
                    const int s = k % C::kStages;
                    const int round = k / C::kStages;
                    if (round > 0 && !mbar_wait_bounded(&empty[s], (round - 1) & 1)) {
                        report(p.dev_error, KV_DEVERR_TIMEOUT);
                        *abort_flag = 1;
                    } else {
                        const int32_t id = q_id[i];
                        const bool ok = id >= 0 && id < p.num_blocks;
                        stage_ok[s] = ok;
                        issued_round[s] = round;
                        if (ok) {
                            const int64_t tile = static_cast<int64_t>(id) * p.num_kv_heads + q_head[i];
                            uint8_t* st = ring + s * C::kStageBytes;
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
                            report(p.dev_error, KV_DEVERR_BAD_BLOCK_ID);
                            mbar_arrive(&full[s]);  // nothing to copy: the consumer skips it
                        }
                    }
                }
                fetch(k + kLook, i);
            }
        }
        if (*abort_flag) {
            // drain: wait (bounded) until no copy issued by this block is in flight
            for (int s = 0; s < C::kStages; ++s)
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

    float2* p_buf = reinterpret_cast<float2*>(scratch + warp * C::kWarpScratch);  // [16][G]
    float* s_buf = reinterpret_cast<float*>(p_buf + kBlockTokens * G);            // [16][G]
    float* c_buf = s_buf + kBlockTokens * G;                                       // [G]
    const int32_t c = lane % C::kLPR;   // chunk column of this lane in a K row
    const int32_t r0 = lane / C::kLPR;  // first K row of this lane
    const int32_t sm_lane = lane % C::kSMLanes;
    const int32_t sm_g = sm_lane % G;   // query head this lane's softmax values belong to

    float2 q2[G][C::kQPL / 2];
    auto load_q_group = [&]() {
        const int64_t qbase = (static_cast<int64_t>(cur.b) * p.num_q_heads + cur.kvh * G) * D;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k = 0; k < C::kNCH; ++k)
#pragma unroll
                for (int e = 0; e < C::kChunkElems; e += 2) {
                    const int64_t col = (c + k * C::kLPR) * C::kChunkElems + e;
                    q2[g][(k * C::kChunkElems + e) / 2] =
                        make_float2(load_q<Q_T>(p.q, qbase + g * D + col) * p.scale_log2,
                                    load_q<Q_T>(p.q, qbase + g * D + col + 1) * p.scale_log2);
                }
    };
    float m_run, l_run;
    float2 o2[G][C::kDPL / 2];
    auto reset = [&]() {
        m_run = -INFINITY;  // running max of this lane's head (base-2 units)
        l_run = 0.0f;       // this lane's share of the running sum
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int i = 0; i < C::kDPL / 2; ++i) o2[g][i] = make_float2(0.0f, 0.0f);
    };
    load_q_group();
    reset();
    int64_t piece_start = lo;

    for (int j = 0; j < n; ++j) {
        const int k = j * C::kConsumerWarps + warp;
        const int s = k % C::kStages;
        const bool arrived =
            __all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (k / C::kStages) & 1));
        if (!arrived) {
            if (lane == 0) report(p.dev_error, KV_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
        if (__any_sync(0xffffffffu, *abort_flag != 0)) return;  // output invalid (reported)
        if (stage_ok[s]) {
            const uint8_t* kt = ring + s * C::kStageBytes;
            const uint8_t* vt = kt + C::kTileBytes;
            const float* ksc = reinterpret_cast<const float*>(kt + 2 * C::kTileBytes);
            const float* vsc = ksc + kBlockTokens;
            const int32_t nvalid = min(kBlockTokens, cur.L - cur.jb * kBlockTokens);

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

            // online softmax: lane handles head sm_g, tokens sm_lane/G + i*(kSMLanes/G)
            float sv[C::kSPL];
            float tmax = -INFINITY;
#pragma unroll
            for (int i = 0; i < C::kSPL; ++i) {
                const int t = sm_lane / G + i * (C::kSMLanes / G);
                sv[i] = (t < nvalid) ? s_buf[t * G + sm_g] : -INFINITY;
                tmax = fmaxf(tmax, sv[i]);
            }
#pragma unroll
            for (int m = G; m < C::kSMLanes; m <<= 1)
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, m));
            const float m_new = fmaxf(m_run, tmax);
            const float corr = exp2f(m_run - m_new);
            l_run *= corr;
#pragma unroll
            for (int i = 0; i < C::kSPL; ++i) {
                const int t = sm_lane / G + i * (C::kSMLanes / G);
                const float pr = exp2f(sv[i] - m_new);
                l_run += pr;
                float pv = pr;
                if constexpr (KV_T == KV_FP8_E4M3) pv *= vsc[t];
                if (lane < C::kSMLanes) p_buf[t * G + sm_g] = make_float2(pv, pv);
            }
            m_run = m_new;
            if (lane < G) c_buf[lane] = corr;
            __syncwarp();

            // P.V: this lane's kDPL output columns for every head of the group
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

        // ---- end of a piece: at the end of a (sequence, kv head) pair or of the range
        const bool seg_end = cur.jb + 1 == cur.nt;
        if (seg_end || j == n - 1) {
            float l = l_run;  // sum of l over the lanes that share this lane's head
#pragma unroll
            for (int m = G; m < C::kSMLanes; m <<= 1) l += __shfl_xor_sync(0xffffffffu, l, m);
            const int64_t bh0 = static_cast<int64_t>(cur.b) * p.num_q_heads + cur.kvh * G;
            if (seg_end && piece_start == cur.seg_start) {
                // the whole pair was this warp's: write the output
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float lg = __shfl_sync(0xffffffffu, l, g);
                    OutT* o = static_cast<OutT*>(p.out) + (bh0 + g) * D + lane * C::kDPL;
#pragma unroll
                    for (int i = 0; i < C::kDPL / 2; ++i) {
                        o[2 * i] = out_cast<OutT>(lg > 0.0f ? o2[g][i].x / lg : 0.0f);
                        o[2 * i + 1] = out_cast<OutT>(lg > 0.0f ? o2[g][i].y / lg : 0.0f);
                    }
                }
            } else {
                // a piece of the pair: partial (m, l, o) for the merge kernel
                const int64_t pid = static_cast<int64_t>(cur.b) * p.num_kv_heads + cur.kvh + W;
                if (lane < G) p.ws_ml[pid * G + lane] = make_float2(m_run, l);
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int i = 0; i < C::kDPL / 2; ++i)
                        *reinterpret_cast<float2*>(&p.ws_o[(pid * G + g) * D + lane * C::kDPL + 2 * i]) =
                            o2[g][i];
            }
            if (j + 1 < n) {
                advance(cur, p);  // next pair (the range goes on)
                piece_start = lo + j + 1;
                load_q_group();
                reset();
            }
        } else {
            ++cur.jb;
        }
    }
}

// ======================================================================================
// Merge kernel: one warp per (sequence, query head).  Pairs split over several
// consumer ranges are combined:  M = max_p m_p;  w_p = 2^(m_p - M);
// out = sum_p w_p o_p / sum_p w_p l_p.  Pairs of invalid length get zeros.
// ======================================================================================
template <int Q_T, int D>
__global__ void __launch_bounds__(128) paged_decode_merge_kernel(const DecodeParams p) {
    using OutT = typename QType<Q_T>::T;
    constexpr int kDPL = D / 32;
    constexpr int kBatch = 8;  // pieces whose loads are in flight together
    pdl_wait();
    pdl_trigger();
    const int32_t lane = threadIdx.x & 31;
    const int64_t bh = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (bh >= static_cast<int64_t>(p.batch) * p.num_q_heads) return;
    const int32_t b = static_cast<int32_t>(bh / p.num_q_heads);
    const int32_t h = static_cast<int32_t>(bh % p.num_q_heads);
    const int32_t G = p.num_q_heads / p.num_kv_heads;
    const int32_t kvh = h / G, g = h % G;
    const int32_t nt = seq_tiles(p.context_lens[b], p.max_context_len);
    OutT* out = static_cast<OutT*>(p.out) + bh * D + lane * kDPL;
    if (nt == 0) {
#pragma unroll
        for (int j = 0; j < kDPL; ++j) out[j] = out_cast<OutT>(0.0f);
        if (lane == 0 && g == 0 && kvh == 0) report(p.dev_error, KV_DEVERR_BAD_CONTEXT_LEN);
        return;
    }
    const int64_t T = p.ws_seq_start[p.batch];
    const int64_t a = static_cast<int64_t>(p.ws_seq_start[b]) + static_cast<int64_t>(kvh) * nt;
    const int64_t w_first = range_of(a, T, p.num_ranges);
    const int64_t w_last = range_of(a + nt - 1, T, p.num_ranges);
    if (w_first == w_last) return;  // the pair was one range's: written by the decode kernel
    const int64_t s = static_cast<int64_t>(b) * p.num_kv_heads + kvh;
    const int32_t npieces = static_cast<int32_t>(w_last - w_first + 1);
    // pieces are (pair s, range W) for the non-empty ranges W in [w_first, w_last];
    // piece id s + W (see the decode kernel)
    auto piece_id = [&](int32_t i) -> int64_t {
        const int64_t W = w_first + i;
        return range_begin(W, T, p.num_ranges) < range_begin(W + 1, T, p.num_ranges) ? s + W : -1;
    };
    float M = -INFINITY;
    for (int i = lane; i < npieces; i += 32) {
        const int64_t pid = piece_id(i);
        if (pid >= 0) M = fmaxf(M, p.ws_ml[pid * G + g].x);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    float o[kDPL];
#pragma unroll
    for (int j = 0; j < kDPL; ++j) o[j] = 0.0f;
    float l = 0.0f;
    if (M != -INFINITY) {
        for (int i0 = 0; i0 < npieces; i0 += 32) {
            // lane i holds piece i0+i's id and weight; the warp then folds the pieces
            // in kBatch at a time with all their loads issued before the first FMA
            const int64_t pl = (i0 + lane < npieces) ? piece_id(i0 + lane) : -1;
            float wl = 0.0f;
            if (pl >= 0) {
                const float2 ml = p.ws_ml[pl * G + g];
                wl = exp2f(ml.x - M);
                l += wl * ml.y;
            }
            const int cnt = min(32, npieces - i0);
            for (int i1 = 0; i1 < cnt; i1 += kBatch) {
                float v[kBatch][kDPL];
                float w[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int i = (i1 + u) & 31;
                    w[u] = __shfl_sync(0xffffffffu, wl, i);
                    const int64_t pid = __shfl_sync(0xffffffffu, pl, i);
                    const bool use = i1 + u < cnt && pid >= 0;
                    const float* src = p.ws_o + ((use ? pid : 0) * G + g) * D + lane * kDPL;
#pragma unroll
                    for (int j = 0; j < kDPL; ++j) v[u][j] = use ? src[j] : 0.0f;
                    if (!use) w[u] = 0.0f;
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u)
#pragma unroll
                    for (int j = 0; j < kDPL; ++j) o[j] = fmaf(w[u], v[u][j], o[j]);
            }
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) l += __shfl_xor_sync(0xffffffffu, l, m);
    }
#pragma unroll
    for (int j = 0; j < kDPL; ++j) out[j] = out_cast<OutT>(l > 0.0f ? o[j] / l : 0.0f);
}

// ---- launch ------------------------------------------------------------------------------
constexpr int kMaxDevices = 64;

template <int KV_T, int D, int G>
int32_t resident_ctas_per_sm() {
    return Cfg<KV_T, D, G>::kMinBlocks;
}

template <int KV_T, int Q_T, int D, int G>
static cudaError_t launch_one(const DecodeParams& p, cudaStream_t stream) {
    using C = Cfg<KV_T, D, G>;
    static bool attr_set[kMaxDevices] = {};  // benign race: every caller sets the same value
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices || !attr_set[dev]) {
        e = cudaFuncSetAttribute(paged_decode_kernel<KV_T, Q_T, D, G>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev < kMaxDevices) attr_set[dev] = true;
    }
    const unsigned grid = static_cast<unsigned>((p.num_ranges + C::kConsumerWarps - 1) /
                                                C::kConsumerWarps);
    e = launch_pdl(paged_decode_kernel<KV_T, Q_T, D, G>, dim3(grid), dim3(C::kThreads),
                   C::kSmemBytes, stream, p);
    if (e != cudaSuccess) return e;
    const int64_t warps = static_cast<int64_t>(p.batch) * p.num_q_heads;
    return launch_pdl(paged_decode_merge_kernel<Q_T, D>, dim3(static_cast<unsigned>((warps + 3) / 4)),
                      dim3(128), 0, stream, p);
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

int32_t decode_ctas_per_sm(int32_t kv_dtype, int32_t head_dim, int32_t group) {
    (void)kv_dtype;
    (void)head_dim;
    return group >= 8 ? 1 : 3;
}

}  // namespace pkv
