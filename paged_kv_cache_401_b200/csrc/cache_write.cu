// Slot computation and cache write ("KV Cache 深度解析" §一/§三/§四;
// "llm-inference-optimization" notes §二 PagedKVCache.append_token).
//
// Pool layout [num_blocks][num_kv_heads][16][head_dim]: the new token's row of
// kv head h goes to block slot/16, row slot%16.  HBM-bound scatter: every
// thread moves one 16-byte vector (bf16/fp32) or one warp quantises one row
// (FP8, INT8, INT4), so loads and stores are full 32-byte sectors.
#include <algorithm>

#include "kernels.cuh"
#include "quant.cuh"

namespace pkv {

__global__ void slot_mapping_kernel(const int32_t* __restrict__ block_table, int32_t batch,
                                    int32_t max_blocks, const int32_t* __restrict__ seq_ids,
                                    const int32_t* __restrict__ positions, int32_t num_tokens,
                                    int64_t* __restrict__ slots, int32_t* dev_error) {
    pdl_wait();
    pdl_trigger();
    const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= num_tokens) return;
    const int32_t s = seq_ids[i];
    const int32_t p = positions[i];
    if (s < 0 || s >= batch || p < 0 || p >= max_blocks * kBlockTokens) {
        slots[i] = -1;
        report(dev_error, KV_DEVERR_BAD_POSITION);
        return;
    }
    const int64_t blk = block_table[static_cast<int64_t>(s) * max_blocks + p / kBlockTokens];
    slots[i] = blk * kBlockTokens + p % kBlockTokens;
}

// Exact copy: one 16-byte vector per thread, K and V.
__global__ void cache_copy_kernel(uint8_t* __restrict__ k_pool, uint8_t* __restrict__ v_pool,
                                  const uint8_t* __restrict__ k_new,
                                  const uint8_t* __restrict__ v_new,
                                  const int64_t* __restrict__ slots, int32_t num_tokens,
                                  int32_t num_kv_heads, int32_t row_bytes, int64_t num_slots,
                                  int32_t* dev_error) {
    pdl_wait();
    pdl_trigger();
    const int32_t vecs_per_row = row_bytes / 16;
    const int64_t per_token = static_cast<int64_t>(num_kv_heads) * vecs_per_row;
    const int64_t total = per_token * num_tokens;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / per_token;
        const int64_t rem = i - t * per_token;
        const int32_t h = static_cast<int32_t>(rem / vecs_per_row);
        const int32_t v = static_cast<int32_t>(rem - static_cast<int64_t>(h) * vecs_per_row);
        const int64_t slot = slots[t];
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (h == 0 && v == 0) report(dev_error, KV_DEVERR_BAD_SLOT);
            continue;
        }
        const int64_t blk = slot / kBlockTokens, off = slot % kBlockTokens;
        const int64_t src = (t * num_kv_heads + h) * row_bytes + v * 16;
        const int64_t dst = ((blk * num_kv_heads + h) * kBlockTokens + off) * row_bytes + v * 16;
        const uint4 kv = *reinterpret_cast<const uint4*>(k_new + src);
        const uint4 vv = *reinterpret_cast<const uint4*>(v_new + src);
        *reinterpret_cast<uint4*>(k_pool + dst) = kv;
        *reinterpret_cast<uint4*>(v_pool + dst) = vv;
    }
}

// Quantising write: one warp per (token, kv head, K|V) row of D elements; the
// codes and parameters come from quant.cuh (FP8: absmax/448, E4M3; INT8:
// absmax/127, round to nearest even, clamp to 127; INT4: asymmetric scale and
// zero point, two codes per byte).
template <int KV_T, int SRC_T, int D>
__global__ void cache_quant_kernel(uint8_t* __restrict__ k_pool, uint8_t* __restrict__ v_pool,
                                   float* __restrict__ scales,
                                   const void* __restrict__ k_new, const void* __restrict__ v_new,
                                   const int64_t* __restrict__ slots, int32_t num_tokens,
                                   int32_t num_kv_heads, int64_t num_slots, int32_t* dev_error) {
    constexpr int kPer = D / 32;  // elements per lane (4 or 2)
    constexpr int kSrcBytes = SRC_T == KV_F32 ? 4 : 2;
    pdl_wait();
    pdl_trigger();
    const int32_t lane = threadIdx.x & 31;
    const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t rows = 2ll * num_tokens * num_kv_heads;
    if (row >= rows) return;
    const int32_t which = static_cast<int32_t>(row & 1);  // 0 = K, 1 = V
    const int64_t th = row >> 1;                          // token * heads + head
    const int64_t t = th / num_kv_heads;
    const int32_t h = static_cast<int32_t>(th - t * num_kv_heads);
    const int64_t slot = slots[t];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (lane == 0 && h == 0 && which == 0) report(dev_error, KV_DEVERR_BAD_SLOT);
        return;
    }
    float x[kPer];
    const uint8_t* src = static_cast<const uint8_t*>(which ? v_new : k_new);
    load_row_part<D>(src + th * D * kSrcBytes, SRC_T, lane, x);
    const int64_t blk = slot / kBlockTokens, off = slot % kBlockTokens;
    const int64_t rowi = (blk * num_kv_heads + h) * kBlockTokens + off;
    const int64_t pidx = ((blk * num_kv_heads + h) * 2 + which) * kBlockTokens + off;
    if constexpr (KV_T == KV_INT4) {
        // 64-byte rows, 2 bytes per lane; parameter pool [block][head][K|V][16][scale, zero]
        float s, z;
        const uint32_t codes = quantize_row_int4_warp<D>(x, &s, &z);
        *reinterpret_cast<uint16_t*>((which ? v_pool : k_pool) + rowi * (D / 2) + lane * 2) =
            static_cast<uint16_t>(codes);
        if (lane == 0) reinterpret_cast<float2*>(scales)[pidx] = make_float2(s, z);
    } else {
        float s;
        const uint32_t codes = quantize_row_warp<KV_T, D>(x, &s);
        store_codes<D>((which ? v_pool : k_pool) + rowi * D + lane * kPer, codes);
        // scale pool [block][head][K|V][16]: one 128-byte line per (block, head)
        if (lane == 0) scales[pidx] = s;
    }
}

// Whole-block copies (copy-on-write of shared blocks): CTA (pair, part) moves
// 16-byte vectors of the K block, the V block and its scale / parameter line.
__global__ void copy_blocks_kernel(uint8_t* __restrict__ k_pool, uint8_t* __restrict__ v_pool,
                                   uint8_t* __restrict__ scales, const int32_t* __restrict__ src,
                                   const int32_t* __restrict__ dst, int64_t block_bytes,
                                   int64_t scale_bytes, int32_t num_blocks, int32_t* dev_error) {
    pdl_wait();
    pdl_trigger();
    const int32_t pair = blockIdx.y;
    const int32_t s = src[pair], d = dst[pair];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
        if (blockIdx.x == 0 && threadIdx.x == 0) report(dev_error, KV_DEVERR_BAD_BLOCK_ID);
        return;
    }
    const int64_t vecs = block_bytes / 16;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < vecs;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t so = s * block_bytes + i * 16, dof = d * block_bytes + i * 16;
        *reinterpret_cast<uint4*>(k_pool + dof) = *reinterpret_cast<const uint4*>(k_pool + so);
        *reinterpret_cast<uint4*>(v_pool + dof) = *reinterpret_cast<const uint4*>(v_pool + so);
    }
    if (scales != nullptr) {
        for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
             i < scale_bytes / 16; i += static_cast<int64_t>(gridDim.x) * blockDim.x)
            *reinterpret_cast<uint4*>(scales + d * scale_bytes + i * 16) =
                *reinterpret_cast<const uint4*>(scales + s * scale_bytes + i * 16);
    }
}

// ---- launchers ------------------------------------------------------------------
cudaError_t launch_copy_blocks(void* k_pool, void* v_pool, float* scales, const int32_t* src,
                               const int32_t* dst, int32_t num_copies, int64_t block_bytes,
                               int64_t scale_bytes, int32_t num_blocks, int32_t* dev_error,
                               cudaStream_t stream) {
    const int threads = 256;
    const int64_t vecs = block_bytes / 16;
    const unsigned parts = static_cast<unsigned>(std::min<int64_t>(8, (vecs + threads - 1) / threads));
    return launch_pdl(copy_blocks_kernel, dim3(parts, static_cast<unsigned>(num_copies)),
                      dim3(threads), 0, stream, static_cast<uint8_t*>(k_pool),
                      static_cast<uint8_t*>(v_pool), reinterpret_cast<uint8_t*>(scales), src, dst,
                      block_bytes, scale_bytes, num_blocks, dev_error);
}

cudaError_t launch_slot_mapping(const int32_t* block_table, int32_t batch, int32_t max_blocks,
                                const int32_t* seq_ids, const int32_t* positions,
                                int32_t num_tokens, int64_t* slots, int32_t* dev_error,
                                cudaStream_t stream) {
    const int threads = 256;
    const int blocks = (num_tokens + threads - 1) / threads;
    return launch_pdl(slot_mapping_kernel, dim3(blocks), dim3(threads), 0, stream, block_table,
                      batch, max_blocks, seq_ids, positions, num_tokens, slots, dev_error);
}

cudaError_t launch_cache_copy(void* k_pool, void* v_pool, const void* k_new, const void* v_new,
                              const int64_t* slots, int32_t num_tokens, int32_t num_kv_heads,
                              int32_t row_bytes, int64_t num_slots, int32_t num_sms,
                              int32_t* dev_error, cudaStream_t stream) {
    const int threads = 256;
    const int64_t vecs = static_cast<int64_t>(num_tokens) * num_kv_heads * (row_bytes / 16);
    int64_t blocks = (vecs + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    return launch_pdl(cache_copy_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0,
                      stream, static_cast<uint8_t*>(k_pool), static_cast<uint8_t*>(v_pool),
                      static_cast<const uint8_t*>(k_new), static_cast<const uint8_t*>(v_new),
                      slots, num_tokens, num_kv_heads, row_bytes, num_slots, dev_error);
}

cudaError_t launch_cache_quant(int32_t kv_dtype, int32_t src_dtype, int32_t head_dim,
                               void* k_pool, void* v_pool, float* scales, const void* k_new,
                               const void* v_new, const int64_t* slots, int32_t num_tokens,
                               int32_t num_kv_heads, int64_t num_slots, int32_t* dev_error,
                               cudaStream_t stream) {
    const int threads = 256;
    const int64_t rows = 2ll * num_tokens * num_kv_heads;
    const int64_t blocks = (rows * 32 + threads - 1) / threads;
    auto* kp = static_cast<uint8_t*>(k_pool);
    auto* vp = static_cast<uint8_t*>(v_pool);
    auto go = [&](auto kernel) {
        return launch_pdl(kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream,
                          kp, vp, scales, k_new, v_new, slots, num_tokens, num_kv_heads,
                          num_slots, dev_error);
    };
    const bool f32 = src_dtype == KV_F32, d128 = head_dim == 128;
    if (kv_dtype == KV_INT4)  // head_dim 128 only
        return f32 ? go(cache_quant_kernel<KV_INT4, KV_F32, 128>)
                   : go(cache_quant_kernel<KV_INT4, KV_BF16, 128>);
    if (kv_dtype == KV_INT8) {
        if (f32) return d128 ? go(cache_quant_kernel<KV_INT8, KV_F32, 128>)
                             : go(cache_quant_kernel<KV_INT8, KV_F32, 64>);
        return d128 ? go(cache_quant_kernel<KV_INT8, KV_BF16, 128>)
                    : go(cache_quant_kernel<KV_INT8, KV_BF16, 64>);
    }
    if (f32) return d128 ? go(cache_quant_kernel<KV_FP8_E4M3, KV_F32, 128>)
                         : go(cache_quant_kernel<KV_FP8_E4M3, KV_F32, 64>);
    return d128 ? go(cache_quant_kernel<KV_FP8_E4M3, KV_BF16, 128>)
                : go(cache_quant_kernel<KV_FP8_E4M3, KV_BF16, 64>);
}

}  // namespace pkv
