// Launchers of the paged-KV kernels, called by the C ABI layer (api.cu).
#pragma once

#include <cuda.h>

#include <utility>

#include "common.cuh"

namespace pkv {

// Launch with programmatic stream serialisation (see pdl_wait / pdl_trigger).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_slot_mapping(const int32_t* block_table, int32_t batch, int32_t max_blocks,
                                const int32_t* seq_ids, const int32_t* positions,
                                int32_t num_tokens, int64_t* slots, int32_t* dev_error,
                                cudaStream_t stream);

cudaError_t launch_cache_copy(void* k_pool, void* v_pool, const void* k_new, const void* v_new,
                              const int64_t* slots, int32_t num_tokens, int32_t num_kv_heads,
                              int32_t row_bytes, int64_t num_slots, int32_t num_sms,
                              int32_t* dev_error, cudaStream_t stream);

cudaError_t launch_cache_quant(int32_t kv_dtype, int32_t src_dtype, int32_t head_dim,
                               void* k_pool, void* v_pool, float* scales, const void* k_new,
                               const void* v_new, const int64_t* slots, int32_t num_tokens,
                               int32_t num_kv_heads, int64_t num_slots, int32_t* dev_error,
                               cudaStream_t stream);

cudaError_t launch_copy_blocks(void* k_pool, void* v_pool, float* scales, const int32_t* src,
                               const int32_t* dst, int32_t num_copies, int64_t block_bytes,
                               int64_t scale_bytes, int32_t num_blocks, int32_t* dev_error,
                               cudaStream_t stream);

// Everything the decode kernel and its merge need for one launch.
struct DecodeParams {
    void* out;                    // [B][Hq][D] in q dtype
    const void* q;                // [B][Hq][D]
    const uint8_t* k_pool;        // [NB][Hkv][16][D]
    const uint8_t* v_pool;
    const float* scales;          // [NB][Hkv][2][16]: K then V row scales (FP8 / INT8)
    const int32_t* block_table;   // [B][max_blocks]
    const int32_t* context_lens;  // [B]
    int32_t* ws_seq_start;        // [B + 1]: first tile of each sequence, total tiles at [B]
    float2* ws_ml;                // [pieces][G*Q]: (running max in base-2 units, running sum)
    float* ws_o;                  // [pieces][G*Q][D]: unnormalised partial outputs
    int32_t* dev_error;
    int32_t batch, num_q_heads, num_kv_heads, num_blocks, max_blocks;
    int32_t max_context_len;
    int32_t num_query_tokens;     // Q: query tokens per sequence (1 for decode)
    int32_t num_ranges;           // consumer-warp ranges the tile list is cut into
    int32_t merge_warps_per_row;  // 1: four output rows per merge CTA; 4: one row per CTA,
                                  // its pieces split over the four warps
    float scale_log2;             // scale * log2(e): scores are kept in base-2 units
    // Fused append (one query token): every sequence's new K/V row [B][Hkv][D] in
    // append_src_dtype is written to the slot of position L - 1 (codes and scale
    // for 8-bit pools) by the warp that attends to it.  k_new == nullptr: no append.
    const void* k_new;
    const void* v_new;
    uint8_t* k_dst;               // the pools again, writable
    uint8_t* v_dst;
    float* scales_dst;
    int32_t append_src_dtype;
    // KIVI pools: only full blocks are tiles; every pair ends in the merge, which
    // also attends to the sequence's newest L mod 16 tokens, kept in bf16 at
    // res_k / res_v [batch][Hkv][16][D]
    int32_t kivi;
    const uint16_t* res_k;
    const uint16_t* res_v;
};

cudaError_t launch_kivi_quantize_blocks(int32_t src_dtype, void* k_pool, void* v_pool,
                                        float* params, const void* k_rows, const void* v_rows,
                                        const int32_t* block_ids, int32_t num_blocks,
                                        int32_t num_kv_heads, int32_t pool_blocks,
                                        int32_t* dev_error, cudaStream_t stream);

cudaError_t launch_kivi_append(void* k_pool, void* v_pool, float* params, uint16_t* res_k,
                               uint16_t* res_v, const void* k_new, const void* v_new,
                               const int32_t* block_table, int32_t max_blocks,
                               const int32_t* context_lens, int32_t batch, int32_t num_kv_heads,
                               int32_t max_context_len, int32_t pool_blocks, int32_t* dev_error,
                               cudaStream_t stream);

// TMA descriptors of the K and V pools as 2-D tensors [num_blocks*Hkv*16 rows][head_dim],
// boxes of 16 rows x 128 bytes with the 128-byte swizzle (tensor-core path only).
struct TmaMaps {
    CUtensorMap k;
    CUtensorMap v;
};

// Resident decode CTAs per SM the kernels are built for (their register budget).
int32_t decode_ctas_per_sm(int32_t kv_dtype, int32_t head_dim, int32_t group,
                           int32_t query_tokens);

// Whether this shape runs the tensor-core tile arithmetic (and needs TmaMaps).
bool decode_uses_tensor_cores(int32_t kv_dtype, int32_t q_dtype, int32_t head_dim);

// kv_dtype, q_dtype, head_dim and group size select the kernel instantiation.
cudaError_t launch_paged_decode(const DecodeParams& p, const TmaMaps& maps, int32_t kv_dtype,
                                int32_t q_dtype, int32_t head_dim, int32_t group,
                                cudaStream_t stream);

}  // namespace pkv
