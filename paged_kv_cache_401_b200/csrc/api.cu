// C ABI of libpagedkv.so (declared in include/paged_kv.h): host-side argument
// checks, geometry, the split of the tile list into consumer ranges, the
// workspace layout and kernel launches.
#include <cudaTypedefs.h>

#include <cmath>

#include "kernels.cuh"

namespace {

using pkv::kBlockTokens;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Bits of one stored K/V element; 0 for an unknown dtype.
int32_t kv_bits(int32_t dtype) {
    switch (dtype) {
        case KV_F32: return 32;
        case KV_BF16: return 16;
        case KV_FP8_E4M3: return 8;
        case KV_INT8: return 8;
        case KV_INT4: return 4;
        case KV_KIVI4: return 4;
        default: return 0;
    }
}

// The descriptor's elem_bytes: 0 for 4-bit codes (two per byte).
int32_t elem_bytes(int32_t dtype) { return kv_bits(dtype) / 8; }

// Bytes of one stored row (one token, one kv head) of a pool.
int64_t row_bytes(const kv_pool_desc* d) {
    return static_cast<int64_t>(d->head_dim) * kv_bits(d->dtype) / 8;
}

// Pools of codes with per-(token, kv head) parameters: one fp32 scale (FP8,
// INT8) or an fp32 (scale, zero point) pair (INT4).
bool quantized(int32_t dtype) {
    return dtype == KV_FP8_E4M3 || dtype == KV_INT8 || dtype == KV_INT4 || dtype == KV_KIVI4;
}

// Bytes of the scale / parameter pool per (block, kv head): fp32 scales of 16
// K and 16 V rows (8-bit), (scale, zero) pairs of the 32 rows (INT4), or of 128
// key channels and 16 value rows (KIVI).
int64_t params_per_tile(int32_t dtype) {
    switch (dtype) {
        case KV_FP8_E4M3:
        case KV_INT8: return 2 * kBlockTokens * 4;
        case KV_INT4: return 2 * kBlockTokens * 8;
        case KV_KIVI4: return (128 + kBlockTokens) * 8;
        default: return 0;
    }
}

// SM count of the current device; 148 (B200) when no device can be queried.
int32_t current_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();  // clear the sticky "no device" error of the query
        return 148;
    }
    return n;
}

bool valid_pool(const kv_pool_desc* d) {
    return d != nullptr && d->num_blocks > 0 && d->block_size == kBlockTokens &&
           d->num_kv_heads > 0 && (d->head_dim == 64 || d->head_dim == 128) &&
           kv_bits(d->dtype) != 0 && elem_bytes(d->dtype) == d->elem_bytes &&
           ((d->dtype != KV_INT4 && d->dtype != KV_KIVI4) || d->head_dim == 128);
}

int32_t ceil_div(int64_t a, int64_t b) { return static_cast<int32_t>((a + b - 1) / b); }


// The driver's tensor-map encoder, looked up once through the runtime (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
        }
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// A pool as a 2-D tensor [num_blocks*Hkv*16 rows][head_dim]: 16-row x 128-byte
// boxes with the 128-byte swizzle; 4-bit pools (64-byte rows of packed codes,
// as bytes) use 16-row x 64-byte boxes with the 64-byte swizzle.  Returns a
// kv_status.
kv_status encode_pool_map(CUtensorMap* map, const void* base, const kv_pool_desc* pool) {
    const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (encode == nullptr) return KV_ERR_CUDA;
    const cuuint64_t rows = static_cast<cuuint64_t>(pool->num_blocks) * pool->num_kv_heads *
                            kBlockTokens;
    // 4-bit rows (INT4, KIVI) are copied as 4-bit elements, each 16 of them padded to
    // 16 bytes in shared memory (the kernel widens them to bytes as it loads them);
    // every row lands as 128 bytes with the 128-byte swizzle
    const bool four_bit = kv_bits(pool->dtype) == 4;
    const int64_t rb = row_bytes(pool);
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(pool->head_dim), rows};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(rb)};
    const cuuint32_t box[2] = {four_bit ? 128u : static_cast<cuuint32_t>(128 / pool->elem_bytes),
                               static_cast<cuuint32_t>(kBlockTokens)};
    const cuuint32_t elem_strides[2] = {1, 1};
    const CUtensorMapDataType type =
        pool->dtype == KV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                               : (four_bit ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B
                                           : CU_TENSOR_MAP_DATA_TYPE_UINT8);
    const CUresult r = encode(map, type, 2, const_cast<void*>(base), dims, strides, box,
                              elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? KV_OK : KV_ERR_INVALID_ARGUMENT;
}

}  // namespace

extern "C" {

kv_status kv_pool_create(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                         int32_t head_dim, kv_dtype dtype, kv_pool_desc* out) {
    if (out == nullptr || num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return KV_ERR_INVALID_ARGUMENT;
    if (block_size != kBlockTokens || (head_dim != 64 && head_dim != 128) || num_kv_heads > 256 ||
        kv_bits(dtype) == 0 || (kv_bits(dtype) == 4 && head_dim != 128))
        return KV_ERR_UNSUPPORTED;
    kv_pool_desc d{};
    d.num_blocks = num_blocks;
    d.block_size = block_size;
    d.num_kv_heads = num_kv_heads;
    d.head_dim = head_dim;
    d.dtype = dtype;
    d.elem_bytes = elem_bytes(dtype);
    d.stride_slot = head_dim;
    d.stride_head = static_cast<int64_t>(block_size) * head_dim;
    d.stride_block = d.stride_head * num_kv_heads;
    d.kv_bytes = static_cast<uint64_t>(d.stride_block) * num_blocks * kv_bits(dtype) / 8u;
    d.scale_bytes = static_cast<uint64_t>(num_blocks) * num_kv_heads *
                    static_cast<uint64_t>(params_per_tile(dtype));
    *out = d;
    return KV_OK;
}

kv_status compute_slot_mapping(const int32_t* block_table, int32_t batch,
                               int32_t max_blocks_per_seq, int32_t block_size,
                               const int32_t* seq_ids, const int32_t* positions,
                               int32_t num_tokens, int64_t* slot_mapping, int32_t* dev_error,
                               kv_stream_t stream) {
    if (num_tokens < 0 || batch < 0 || max_blocks_per_seq < 0) return KV_ERR_INVALID_ARGUMENT;
    if (block_size != kBlockTokens) return KV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return KV_OK;
    if (block_table == nullptr || seq_ids == nullptr || positions == nullptr ||
        slot_mapping == nullptr)
        return KV_ERR_INVALID_ARGUMENT;
    cudaError_t e = pkv::launch_slot_mapping(block_table, batch, max_blocks_per_seq, seq_ids,
                                             positions, num_tokens, slot_mapping, dev_error,
                                             reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

kv_status reshape_and_cache(const kv_pool_desc* pool, void* k_pool, void* v_pool,
                            float* scales, const void* k_new,
                            const void* v_new, kv_dtype src_dtype, const int64_t* slot_mapping,
                            int32_t num_tokens, int32_t* dev_error, kv_stream_t stream) {
    if (!valid_pool(pool) || num_tokens < 0) return KV_ERR_INVALID_ARGUMENT;
    if (num_tokens == 0) return KV_OK;
    if (k_pool == nullptr || v_pool == nullptr || k_new == nullptr || v_new == nullptr ||
        slot_mapping == nullptr)
        return KV_ERR_INVALID_ARGUMENT;
    if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(k_new) || !aligned16(v_new))
        return KV_ERR_INVALID_ARGUMENT;
    const int64_t num_slots = static_cast<int64_t>(pool->num_blocks) * kBlockTokens;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (pool->dtype == KV_KIVI4) return KV_ERR_UNSUPPORTED;  // kivi_quantize_blocks / the append
    if (quantized(pool->dtype)) {
        if (src_dtype != KV_F32 && src_dtype != KV_BF16) return KV_ERR_UNSUPPORTED;
        if (scales == nullptr) return KV_ERR_INVALID_ARGUMENT;
        e = pkv::launch_cache_quant(pool->dtype, src_dtype, pool->head_dim, k_pool, v_pool, scales,
                                  k_new, v_new, slot_mapping, num_tokens, pool->num_kv_heads,
                                  num_slots, dev_error, s);
    } else {
        if (src_dtype != pool->dtype) return KV_ERR_UNSUPPORTED;
        if (scales != nullptr) return KV_ERR_INVALID_ARGUMENT;
        e = pkv::launch_cache_copy(k_pool, v_pool, k_new, v_new, slot_mapping, num_tokens,
                                   pool->num_kv_heads, static_cast<int32_t>(row_bytes(pool)),
                                   num_slots, current_sm_count(), dev_error, s);
    }
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

kv_status paged_kv_copy_blocks(const kv_pool_desc* pool, void* k_pool, void* v_pool,
                               float* scales, const int32_t* copy_src, const int32_t* copy_dst,
                               int32_t num_copies, int32_t* dev_error, kv_stream_t stream) {
    if (!valid_pool(pool) || num_copies < 0) return KV_ERR_INVALID_ARGUMENT;
    if (num_copies == 0) return KV_OK;
    if (k_pool == nullptr || v_pool == nullptr || copy_src == nullptr || copy_dst == nullptr)
        return KV_ERR_INVALID_ARGUMENT;
    if (!aligned16(k_pool) || !aligned16(v_pool)) return KV_ERR_INVALID_ARGUMENT;
    const bool fp8 = quantized(pool->dtype);  // FP8, INT8 or INT4: a parameter pool
    if (fp8 != (scales != nullptr) || (fp8 && !aligned16(scales))) return KV_ERR_INVALID_ARGUMENT;
    const int64_t block_bytes = row_bytes(pool) * kBlockTokens * pool->num_kv_heads;
    const int64_t scale_bytes = static_cast<int64_t>(pool->num_kv_heads) * params_per_tile(pool->dtype);
    cudaError_t e = pkv::launch_copy_blocks(k_pool, v_pool, scales, copy_src, copy_dst,
                                            num_copies, block_bytes, scale_bytes,
                                            pool->num_blocks, dev_error,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

}  // extern "C"

namespace {

// Consumer ranges of the tile list (see paged_decode_num_ranges).
int32_t num_ranges_for(const kv_pool_desc* pool, int32_t batch, int32_t num_q_heads,
                       int32_t query_tokens, int32_t max_context_len, int32_t partition_tokens) {
    if (!valid_pool(pool) || batch <= 0 || num_q_heads <= 0 || max_context_len <= 0 ||
        query_tokens < 1 || num_q_heads % pool->num_kv_heads != 0 || partition_tokens < 0 ||
        partition_tokens % kBlockTokens != 0)
        return 0;
    const int32_t group = num_q_heads / pool->num_kv_heads;
    if (partition_tokens == 0) {
        // persistent: one range per consumer warp of every CTA the GPU holds at once
        return current_sm_count() *
               pkv::decode_ctas_per_sm(pool->dtype, pool->head_dim, group, query_tokens) * 4;
    }
    // ranges of at most partition_tokens tokens over the largest possible tile list
    const int64_t max_tiles = static_cast<int64_t>(batch) * pool->num_kv_heads *
                              ceil_div(max_context_len, kBlockTokens);
    const int64_t per = partition_tokens / kBlockTokens;
    const int64_t n = (max_tiles + per - 1) / per;
    return static_cast<int32_t>(n < 1 ? 1 : (n > (1 << 28) ? (1 << 28) : n));
}

// Workspace layout: [B + 1] int32 sequence starts | [pieces][R] float2 (m, l) |
// [pieces][R][D] float partial outputs; pieces = B * Hkv + num_ranges, R = G * Q
// query rows per (sequence, kv head) pair.
struct WsLayout {
    size_t ml_off, o_off, total;
};
WsLayout ws_layout(const kv_pool_desc* pool, int32_t batch, int32_t num_q_heads,
                   int32_t query_tokens, int32_t num_ranges) {
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t rows = static_cast<size_t>(num_q_heads / pool->num_kv_heads) * query_tokens;
    const size_t pieces = static_cast<size_t>(batch) * pool->num_kv_heads + num_ranges;
    WsLayout w{};
    w.ml_off = up(sizeof(int32_t) * (static_cast<size_t>(batch) + 1));
    w.o_off = w.ml_off + up(pieces * rows * sizeof(float2));
    w.total = w.o_off + pieces * rows * pool->head_dim * sizeof(float);
    return w;
}

size_t workspace_bytes_for(const kv_pool_desc* pool, int32_t batch, int32_t num_q_heads,
                           int32_t query_tokens, int32_t max_context_len,
                           int32_t partition_tokens) {
    const int32_t ranges = num_ranges_for(pool, batch, num_q_heads, query_tokens,
                                          max_context_len, partition_tokens);
    if (ranges <= 0) return 0;
    return ws_layout(pool, batch, num_q_heads, query_tokens, ranges).total;
}

// The bf16 residual (newest L mod 16 tokens) of a KIVI call, and its new rows.
struct KiviArgs {
    void* k_pool;
    void* v_pool;
    float* params;
    uint16_t* res_k;
    uint16_t* res_v;
    const void* k_new;  // nullable: no append
    const void* v_new;
};

// The new token rows of a fused append+decode call.
struct AppendArgs {
    void* k_pool;
    void* v_pool;
    float* scales;
    const void* k_new;
    const void* v_new;
    kv_dtype src_dtype;
};

kv_status attention_impl(const kv_pool_desc* pool, void* out, const void* q, kv_dtype q_dtype,
                         int32_t query_tokens, const void* k_pool, const void* v_pool,
                         const float* scales, const int32_t* block_table,
                         int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch,
                         int32_t num_q_heads, int32_t max_context_len, float scale,
                         int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                         int32_t* dev_error, kv_stream_t stream,
                         const AppendArgs* app = nullptr, const KiviArgs* kivi = nullptr) {
    if (!valid_pool(pool) || batch < 0 || num_q_heads <= 0 || max_blocks_per_seq < 0 ||
        query_tokens < 1 || (app != nullptr && query_tokens != 1))
        return KV_ERR_INVALID_ARGUMENT;
    // KIVI pools go through kivi_decode_attention (one query token), and only they
    if ((pool->dtype == KV_KIVI4) != (kivi != nullptr)) return KV_ERR_UNSUPPORTED;
    if (kivi != nullptr && query_tokens != 1) return KV_ERR_UNSUPPORTED;
    if (app != nullptr) {
        // no conversion for 16/32-bit pools (as reshape_and_cache); 8-bit pools quantise
        const bool src_ok = quantized(pool->dtype)
                                ? (app->src_dtype == KV_F32 || app->src_dtype == KV_BF16)
                                : app->src_dtype == pool->dtype;
        if (!src_ok) return KV_ERR_UNSUPPORTED;
    }
    if (q_dtype != KV_F32 && q_dtype != KV_BF16) return KV_ERR_UNSUPPORTED;
    if (num_q_heads % pool->num_kv_heads != 0) return KV_ERR_INVALID_ARGUMENT;
    const int32_t group = num_q_heads / pool->num_kv_heads;
    if (group != 1 && group != 2 && group != 4 && group != 8) return KV_ERR_UNSUPPORTED;
    // several query tokens: tensor-core shapes, at most 16 query rows per kv head
    if (query_tokens > 1 && (!pkv::decode_uses_tensor_cores(pool->dtype, q_dtype, pool->head_dim) ||
                             group * query_tokens > 16))
        return KV_ERR_UNSUPPORTED;
    // 4-bit codes have only the tensor-core tile (bf16 q, head_dim 128)
    if (kv_bits(pool->dtype) == 4 &&
        !pkv::decode_uses_tensor_cores(pool->dtype, q_dtype, pool->head_dim))
        return KV_ERR_UNSUPPORTED;
    if (batch == 0) return KV_OK;
    if (max_context_len < query_tokens ||
        static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * kBlockTokens)
        return KV_ERR_INVALID_ARGUMENT;
    if (partition_tokens < 0 || partition_tokens % kBlockTokens != 0)
        return KV_ERR_INVALID_ARGUMENT;
    // the tile list (and its int32 per-sequence starts) must stay below 2^31 tiles
    if (static_cast<int64_t>(batch) * pool->num_kv_heads *
            ceil_div(max_context_len, kBlockTokens) >= (int64_t{1} << 31))
        return KV_ERR_UNSUPPORTED;
    if (!std::isfinite(scale)) return KV_ERR_INVALID_ARGUMENT;
    if (out == nullptr || q == nullptr || k_pool == nullptr || v_pool == nullptr ||
        block_table == nullptr || context_lens == nullptr)
        return KV_ERR_INVALID_ARGUMENT;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool))
        return KV_ERR_INVALID_ARGUMENT;
    // the 4-bit element copies of INT4 and KIVI pools need 32-byte aligned pools
    if (kv_bits(pool->dtype) == 4 && ((reinterpret_cast<uintptr_t>(k_pool) & 31) != 0 ||
                                      (reinterpret_cast<uintptr_t>(v_pool) & 31) != 0))
        return KV_ERR_INVALID_ARGUMENT;
    const bool fp8 = quantized(pool->dtype);  // FP8, INT8 or INT4: a parameter pool
    if (fp8 != (scales != nullptr)) return KV_ERR_INVALID_ARGUMENT;
    if (fp8 && !aligned16(scales)) return KV_ERR_INVALID_ARGUMENT;
    if (app != nullptr && (app->k_new == nullptr || app->v_new == nullptr ||
                           !aligned16(app->k_new) || !aligned16(app->v_new)))
        return KV_ERR_INVALID_ARGUMENT;
    if (kivi != nullptr &&
        (kivi->res_k == nullptr || kivi->res_v == nullptr || !aligned16(kivi->res_k) ||
         !aligned16(kivi->res_v) || ((kivi->k_new == nullptr) != (kivi->v_new == nullptr)) ||
         (kivi->k_new != nullptr && (!aligned16(kivi->k_new) || !aligned16(kivi->v_new)))))
        return KV_ERR_INVALID_ARGUMENT;

    const int32_t ranges = num_ranges_for(pool, batch, num_q_heads, query_tokens,
                                          max_context_len, partition_tokens);
    if (ranges <= 0) return KV_ERR_INVALID_ARGUMENT;
    const WsLayout wl = ws_layout(pool, batch, num_q_heads, query_tokens, ranges);
    if (workspace == nullptr || workspace_bytes < wl.total || !aligned16(workspace))
        return KV_ERR_INVALID_ARGUMENT;

    pkv::DecodeParams p{};
    p.out = out;
    p.q = q;
    p.k_pool = static_cast<const uint8_t*>(k_pool);
    p.v_pool = static_cast<const uint8_t*>(v_pool);
    p.scales = scales;
    p.block_table = block_table;
    p.context_lens = context_lens;
    p.dev_error = dev_error;
    p.batch = batch;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = pool->num_kv_heads;
    p.num_blocks = pool->num_blocks;
    p.max_blocks = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    p.num_query_tokens = query_tokens;
    p.num_ranges = ranges;
    // pieces per pair, at most about ranges / pairs + 1 (all contexts of the longest
    // length): many of them -> four merge warps per output row
    const int64_t pairs = static_cast<int64_t>(batch) * pool->num_kv_heads;
    p.merge_warps_per_row = ranges / pairs + 1 > 16 ? 4 : 1;
    p.scale_log2 = scale * 1.4426950408889634f;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.ws_seq_start = reinterpret_cast<int32_t*>(ws);
    p.ws_ml = reinterpret_cast<float2*>(ws + wl.ml_off);
    p.ws_o = reinterpret_cast<float*>(ws + wl.o_off);
    if (app != nullptr) {
        p.k_new = app->k_new;
        p.v_new = app->v_new;
        p.k_dst = static_cast<uint8_t*>(app->k_pool);
        p.v_dst = static_cast<uint8_t*>(app->v_pool);
        p.scales_dst = app->scales;
        p.append_src_dtype = app->src_dtype;
    }
    if (kivi != nullptr) {
        p.kivi = 1;
        p.res_k = kivi->res_k;
        p.res_v = kivi->res_v;
    }
    pkv::TmaMaps maps{};
    if (pkv::decode_uses_tensor_cores(pool->dtype, q_dtype, pool->head_dim)) {
        // TMA row coordinates are 32-bit
        if (static_cast<int64_t>(pool->num_blocks) * pool->num_kv_heads * kBlockTokens >=
            (int64_t{1} << 31))
            return KV_ERR_UNSUPPORTED;
        kv_status st = encode_pool_map(&maps.k, k_pool, pool);
        if (st == KV_OK) st = encode_pool_map(&maps.v, v_pool, pool);
        if (st != KV_OK) return st;
    }
    cudaError_t e = cudaSuccess;
    if (kivi != nullptr && kivi->k_new != nullptr)  // residual row, and the block it completes
        e = pkv::launch_kivi_append(kivi->k_pool, kivi->v_pool, kivi->params, kivi->res_k,
                                    kivi->res_v, kivi->k_new, kivi->v_new, block_table,
                                    max_blocks_per_seq, context_lens, batch, pool->num_kv_heads,
                                    max_context_len, pool->num_blocks, dev_error,
                                    reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaSuccess)
        e = pkv::launch_paged_decode(p, maps, pool->dtype, q_dtype, pool->head_dim, group,
                                     reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

}  // namespace

extern "C" {

int32_t paged_decode_num_ranges(const kv_pool_desc* pool, int32_t batch, int32_t num_q_heads,
                                int32_t max_context_len, int32_t partition_tokens) {
    return num_ranges_for(pool, batch, num_q_heads, 1, max_context_len, partition_tokens);
}

size_t paged_decode_workspace_bytes(const kv_pool_desc* pool, int32_t batch,
                                    int32_t num_q_heads, int32_t max_context_len,
                                    int32_t partition_tokens) {
    return workspace_bytes_for(pool, batch, num_q_heads, 1, max_context_len, partition_tokens);
}

size_t paged_attention_workspace_bytes(const kv_pool_desc* pool, int32_t batch,
                                       int32_t num_q_heads, int32_t num_query_tokens,
                                       int32_t max_context_len, int32_t partition_tokens) {
    return workspace_bytes_for(pool, batch, num_q_heads, num_query_tokens, max_context_len,
                               partition_tokens);
}

kv_status paged_decode_attention(const kv_pool_desc* pool, void* out, const void* q,
                                 kv_dtype q_dtype, const void* k_pool, const void* v_pool,
                                 const float* scales, const int32_t* block_table,
                                 int32_t max_blocks_per_seq, const int32_t* context_lens,
                                 int32_t batch, int32_t num_q_heads, int32_t max_context_len,
                                 float scale, int32_t partition_tokens, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_error,
                                 kv_stream_t stream) {
    return attention_impl(pool, out, q, q_dtype, 1, k_pool, v_pool, scales, block_table,
                          max_blocks_per_seq, context_lens, batch, num_q_heads, max_context_len,
                          scale, partition_tokens, workspace, workspace_bytes, dev_error, stream);
}

kv_status paged_decode_attention_append(const kv_pool_desc* pool, void* out, const void* q,
                                        kv_dtype q_dtype, void* k_pool, void* v_pool,
                                        float* scales, const void* k_new, const void* v_new,
                                        kv_dtype src_dtype, const int32_t* block_table,
                                        int32_t max_blocks_per_seq, const int32_t* context_lens,
                                        int32_t batch, int32_t num_q_heads,
                                        int32_t max_context_len, float scale,
                                        int32_t partition_tokens, void* workspace,
                                        size_t workspace_bytes, int32_t* dev_error,
                                        kv_stream_t stream) {
    const AppendArgs app{k_pool, v_pool, scales, k_new, v_new, src_dtype};
    return attention_impl(pool, out, q, q_dtype, 1, k_pool, v_pool, scales, block_table,
                          max_blocks_per_seq, context_lens, batch, num_q_heads, max_context_len,
                          scale, partition_tokens, workspace, workspace_bytes, dev_error, stream,
                          &app);
}

kv_status kivi_decode_attention(const kv_pool_desc* pool, void* out, const void* q,
                                kv_dtype q_dtype, void* k_pool, void* v_pool, float* params,
                                void* res_k, void* res_v, const void* k_new, const void* v_new,
                                const int32_t* block_table, int32_t max_blocks_per_seq,
                                const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                                int32_t max_context_len, float scale, int32_t partition_tokens,
                                void* workspace, size_t workspace_bytes, int32_t* dev_error,
                                kv_stream_t stream) {
    const KiviArgs kv{k_pool, v_pool, params, static_cast<uint16_t*>(res_k),
                      static_cast<uint16_t*>(res_v), k_new, v_new};
    return attention_impl(pool, out, q, q_dtype, 1, k_pool, v_pool, params, block_table,
                          max_blocks_per_seq, context_lens, batch, num_q_heads, max_context_len,
                          scale, partition_tokens, workspace, workspace_bytes, dev_error, stream,
                          nullptr, &kv);
}

kv_status kivi_quantize_blocks(const kv_pool_desc* pool, void* k_pool, void* v_pool, float* params,
                               const void* k_rows, const void* v_rows, kv_dtype src_dtype,
                               const int32_t* block_ids, int32_t num_blocks, int32_t* dev_error,
                               kv_stream_t stream) {
    if (!valid_pool(pool) || pool->dtype != KV_KIVI4 || num_blocks < 0)
        return pool != nullptr && valid_pool(pool) && pool->dtype != KV_KIVI4
                   ? KV_ERR_UNSUPPORTED
                   : KV_ERR_INVALID_ARGUMENT;
    if (src_dtype != KV_F32 && src_dtype != KV_BF16) return KV_ERR_UNSUPPORTED;
    if (num_blocks == 0) return KV_OK;
    if (k_pool == nullptr || v_pool == nullptr || params == nullptr || k_rows == nullptr ||
        v_rows == nullptr || block_ids == nullptr)
        return KV_ERR_INVALID_ARGUMENT;
    if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(params) || !aligned16(k_rows) ||
        !aligned16(v_rows))
        return KV_ERR_INVALID_ARGUMENT;
    const cudaError_t e = pkv::launch_kivi_quantize_blocks(
        src_dtype, k_pool, v_pool, params, k_rows, v_rows, block_ids, num_blocks,
        pool->num_kv_heads, pool->num_blocks, dev_error, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

kv_status paged_attention_multi_query(const kv_pool_desc* pool, void* out, const void* q,
                                      kv_dtype q_dtype, int32_t num_query_tokens,
                                      const void* k_pool, const void* v_pool,
                                      const float* scales, const int32_t* block_table,
                                      int32_t max_blocks_per_seq, const int32_t* context_lens,
                                      int32_t batch, int32_t num_q_heads,
                                      int32_t max_context_len, float scale,
                                      int32_t partition_tokens, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_error,
                                      kv_stream_t stream) {
    return attention_impl(pool, out, q, q_dtype, num_query_tokens, k_pool, v_pool, scales,
                          block_table, max_blocks_per_seq, context_lens, batch, num_q_heads,
                          max_context_len, scale, partition_tokens, workspace, workspace_bytes,
                          dev_error, stream);
}

const char* kv_status_string(kv_status status) {
    switch (status) {
        case KV_OK: return "KV_OK";
        case KV_ERR_INVALID_ARGUMENT: return "KV_ERR_INVALID_ARGUMENT";
        case KV_ERR_UNSUPPORTED: return "KV_ERR_UNSUPPORTED";
        case KV_ERR_CUDA: return "KV_ERR_CUDA";
        case KV_ERR_OUT_OF_BLOCKS: return "KV_ERR_OUT_OF_BLOCKS";
        default: return "KV_STATUS_UNKNOWN";
    }
}

}  // extern "C"
