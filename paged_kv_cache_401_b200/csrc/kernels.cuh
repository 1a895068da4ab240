// Launchers of the paged-KV kernels, called by the C ABI layer (api.cu).
#pragma once

#include "common.cuh"

namespace pkv {

cudaError_t launch_slot_mapping(const int32_t* block_table, int32_t batch, int32_t max_blocks,
                                const int32_t* seq_ids, const int32_t* positions,
                                int32_t num_tokens, int64_t* slots, int32_t* dev_error,
                                cudaStream_t stream);

cudaError_t launch_cache_copy(void* k_pool, void* v_pool, const void* k_new, const void* v_new,
                              const int64_t* slots, int32_t num_tokens, int32_t num_kv_heads,
                              int32_t row_bytes, int64_t num_slots, int32_t num_sms,
                              int32_t* dev_error, cudaStream_t stream);

cudaError_t launch_cache_fp8(int32_t src_dtype, int32_t head_dim, void* k_pool, void* v_pool,
                             float* k_scales, float* v_scales, const void* k_new,
                             const void* v_new, const int64_t* slots, int32_t num_tokens,
                             int32_t num_kv_heads, int64_t num_slots, int32_t* dev_error,
                             cudaStream_t stream);

// Everything the split-K decode and its merge need for one launch.
struct DecodeParams {
    void* out;                    // [B][Hq][D] in q dtype
    const void* q;                // [B][Hq][D]
    const uint8_t* k_pool;        // [NB][Hkv][16][D]
    const uint8_t* v_pool;
    const float* k_scales;        // [NB][Hkv][16] (FP8 only)
    const float* v_scales;
    const int32_t* block_table;   // [B][max_blocks]
    const int32_t* context_lens;  // [B]
    float2* ws_ml;                // [B][Hq][max_parts] (running max in log2 units, sum)
    float* ws_o;                  // [B][Hq][max_parts][D]
    int32_t* dev_error;
    int32_t batch, num_q_heads, num_kv_heads, num_blocks, max_blocks;
    int32_t max_context_len, partition_tokens, max_parts;
    float scale_log2;             // scale * log2(e): scores are kept in base-2 units
};

// kv_dtype, q_dtype, head_dim and group size select the kernel instantiation.
cudaError_t launch_paged_decode(const DecodeParams& p, int32_t kv_dtype, int32_t q_dtype,
                                int32_t head_dim, int32_t group, cudaStream_t stream);

}  // namespace pkv
