// KIVI cache writes ("大模型推理为何这么慢", KV Cache量化: keys quantised per
// channel, values per token, the newest tokens kept at full precision; the
// 4-bit routine is the one printed in the "llm-inference-optimization" notes
// §四, applied to those groups).
//
// A KIVI pool holds full 16-token blocks only: K and V codes as 64-byte rows
// of two 4-bit codes per byte (dim 2i low nibble), and per (block, kv head)
// 1152 bytes of fp32 parameters: 128 (scale, zero) pairs, one per key channel
// over the block's 16 tokens, then 16 pairs, one per value row.  A sequence's
// incomplete last block lives in a bf16 residual [batch][Hkv][16][D] owned by
// the caller; when it fills, it is quantised into its block.
#include "kernels.cuh"
#include "quant.cuh"

namespace pkv {

namespace {

constexpr int kD = 128;                      // head_dim of KIVI pools
constexpr int kRowBytes = kD / 2;            // 64 bytes of codes per row
constexpr int kParamFloats = (kD + kBlockTokens) * 2;  // 288 floats = 1152 bytes

__device__ __forceinline__ float bf16_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// One warp quantises one (block, kv head): xk[t][e] / xv[t][e] are element
// 4*lane + e of token row t.  Key channel 4*lane + e is one group of 16; each
// value row is one group of 128 (a warp reduction).
__device__ void quantize_block_warp(const float (&xk)[kBlockTokens][4],
                                    const float (&xv)[kBlockTokens][4], int32_t lane,
                                    uint8_t* k_rows, uint8_t* v_rows, float2* params) {
    uint32_t kc[kBlockTokens] = {};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float x[kBlockTokens];
#pragma unroll
        for (int t = 0; t < kBlockTokens; ++t) x[t] = xk[t][e];
        uint32_t c[kBlockTokens];
        float s, z;
        quantize_group16_int4(x, c, &s, &z);
#pragma unroll
        for (int t = 0; t < kBlockTokens; ++t) kc[t] |= c[t] << (4 * e);
        params[4 * lane + e] = make_float2(s, z);
    }
#pragma unroll
    for (int t = 0; t < kBlockTokens; ++t) {
        *reinterpret_cast<uint16_t*>(k_rows + t * kRowBytes + 2 * lane) = static_cast<uint16_t>(kc[t]);
        float s, z;
        const uint32_t vc = quantize_row_int4_warp<kD>(xv[t], &s, &z);
        *reinterpret_cast<uint16_t*>(v_rows + t * kRowBytes + 2 * lane) = static_cast<uint16_t>(vc);
        if (lane == 0) params[kD + t] = make_float2(s, z);
    }
}

// Full blocks from source rows [n][16][Hkv][D]: warp (i, h) writes block block_ids[i].
template <int SRC_T>
__global__ void kivi_quantize_blocks_kernel(uint8_t* __restrict__ k_pool, uint8_t* __restrict__ v_pool,
                                            float* __restrict__ params,
                                            const void* __restrict__ k_src,
                                            const void* __restrict__ v_src,
                                            const int32_t* __restrict__ block_ids, int32_t n,
                                            int32_t num_kv_heads, int32_t pool_blocks,
                                            int32_t* dev_error) {
    pdl_wait();
    pdl_trigger();
    const int32_t lane = threadIdx.x & 31;
    const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (w >= static_cast<int64_t>(n) * num_kv_heads) return;
    const int64_t i = w / num_kv_heads;
    const int32_t h = static_cast<int32_t>(w - i * num_kv_heads);
    const int32_t blk = block_ids[i];
    if (blk < 0 || blk >= pool_blocks) {
        if (lane == 0 && h == 0) report(dev_error, KV_DEVERR_BAD_BLOCK_ID);
        return;
    }
    constexpr int kSrcBytes = SRC_T == KV_F32 ? 4 : 2;
    float xk[kBlockTokens][4], xv[kBlockTokens][4];
#pragma unroll
    for (int t = 0; t < kBlockTokens; ++t) {
        const int64_t row = ((i * kBlockTokens + t) * num_kv_heads + h) * kD * kSrcBytes;
        load_row_part<kD>(static_cast<const uint8_t*>(k_src) + row, SRC_T, lane, xk[t]);
        load_row_part<kD>(static_cast<const uint8_t*>(v_src) + row, SRC_T, lane, xv[t]);
    }
    const int64_t tile = static_cast<int64_t>(blk) * num_kv_heads + h;
    quantize_block_warp(xk, xv, lane, k_pool + tile * kBlockTokens * kRowBytes,
                        v_pool + tile * kBlockTokens * kRowBytes,
                        reinterpret_cast<float2*>(params + tile * kParamFloats));
}

// Decode-time append: warp (b, h) stores the new bf16 rows at residual row
// (L - 1) % 16; when that completes the block, the 16 residual rows are
// quantised into block block_table[b][(L - 1) / 16].
__global__ void kivi_append_kernel(uint8_t* __restrict__ k_pool, uint8_t* __restrict__ v_pool,
                                   float* __restrict__ params, uint16_t* __restrict__ res_k,
                                   uint16_t* __restrict__ res_v,
                                   const uint16_t* __restrict__ k_new,
                                   const uint16_t* __restrict__ v_new,
                                   const int32_t* __restrict__ block_table, int32_t max_blocks,
                                   const int32_t* __restrict__ context_lens, int32_t batch,
                                   int32_t num_kv_heads, int32_t max_context_len,
                                   int32_t pool_blocks, int32_t* dev_error) {
    pdl_wait();
    pdl_trigger();
    const int32_t lane = threadIdx.x & 31;
    const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (w >= static_cast<int64_t>(batch) * num_kv_heads) return;
    const int32_t b = static_cast<int32_t>(w / num_kv_heads);
    const int32_t h = static_cast<int32_t>(w - static_cast<int64_t>(b) * num_kv_heads);
    const int32_t L = context_lens[b];
    if (L < 1 || L > max_context_len) return;  // reported by the decode
    const int32_t pos = L - 1, r = pos % kBlockTokens;
    const int64_t rbase = w * kBlockTokens * kD;  // residual rows of (b, h)
    const uint2 kn = *reinterpret_cast<const uint2*>(k_new + w * kD + 4 * lane);
    const uint2 vn = *reinterpret_cast<const uint2*>(v_new + w * kD + 4 * lane);
    *reinterpret_cast<uint2*>(res_k + rbase + r * kD + 4 * lane) = kn;
    *reinterpret_cast<uint2*>(res_v + rbase + r * kD + 4 * lane) = vn;
    if (r != kBlockTokens - 1) return;
    const int32_t blk = block_table[static_cast<int64_t>(b) * max_blocks + pos / kBlockTokens];
    if (blk < 0 || blk >= pool_blocks) {
        if (lane == 0) report(dev_error, KV_DEVERR_BAD_BLOCK_ID);
        return;
    }
    // the block is complete: rows 0..14 from the residual (this lane's own
    // columns), row 15 from the registers
    float xk[kBlockTokens][4], xv[kBlockTokens][4];
#pragma unroll
    for (int t = 0; t < kBlockTokens; ++t) {
        uint2 a = kn, c = vn;
        if (t < kBlockTokens - 1) {
            a = *reinterpret_cast<const uint2*>(res_k + rbase + t * kD + 4 * lane);
            c = *reinterpret_cast<const uint2*>(res_v + rbase + t * kD + 4 * lane);
        }
        xk[t][0] = bf16_to_float(a.x & 0xffff);
        xk[t][1] = bf16_to_float(a.x >> 16);
        xk[t][2] = bf16_to_float(a.y & 0xffff);
        xk[t][3] = bf16_to_float(a.y >> 16);
        xv[t][0] = bf16_to_float(c.x & 0xffff);
        xv[t][1] = bf16_to_float(c.x >> 16);
        xv[t][2] = bf16_to_float(c.y & 0xffff);
        xv[t][3] = bf16_to_float(c.y >> 16);
    }
    const int64_t tile = static_cast<int64_t>(blk) * num_kv_heads + h;
    quantize_block_warp(xk, xv, lane, k_pool + tile * kBlockTokens * kRowBytes,
                        v_pool + tile * kBlockTokens * kRowBytes,
                        reinterpret_cast<float2*>(params + tile * kParamFloats));
}

}  // namespace

cudaError_t launch_kivi_quantize_blocks(int32_t src_dtype, void* k_pool, void* v_pool,
                                        float* params, const void* k_rows, const void* v_rows,
                                        const int32_t* block_ids, int32_t num_blocks,
                                        int32_t num_kv_heads, int32_t pool_blocks,
                                        int32_t* dev_error, cudaStream_t stream) {
    const int threads = 128;
    const int64_t warps = static_cast<int64_t>(num_blocks) * num_kv_heads;
    const dim3 grid(static_cast<unsigned>((warps * 32 + threads - 1) / threads));
    auto* kp = static_cast<uint8_t*>(k_pool);
    auto* vp = static_cast<uint8_t*>(v_pool);
    if (src_dtype == KV_F32)
        return launch_pdl(kivi_quantize_blocks_kernel<KV_F32>, grid, dim3(threads), 0, stream, kp,
                          vp, params, k_rows, v_rows, block_ids, num_blocks, num_kv_heads,
                          pool_blocks, dev_error);
    return launch_pdl(kivi_quantize_blocks_kernel<KV_BF16>, grid, dim3(threads), 0, stream, kp, vp,
                      params, k_rows, v_rows, block_ids, num_blocks, num_kv_heads, pool_blocks,
                      dev_error);
}

cudaError_t launch_kivi_append(void* k_pool, void* v_pool, float* params, uint16_t* res_k,
                               uint16_t* res_v, const void* k_new, const void* v_new,
                               const int32_t* block_table, int32_t max_blocks,
                               const int32_t* context_lens, int32_t batch, int32_t num_kv_heads,
                               int32_t max_context_len, int32_t pool_blocks, int32_t* dev_error,
                               cudaStream_t stream) {
    const int threads = 128;
    const int64_t warps = static_cast<int64_t>(batch) * num_kv_heads;
    const dim3 grid(static_cast<unsigned>((warps * 32 + threads - 1) / threads));
    return launch_pdl(kivi_append_kernel, grid, dim3(threads), 0, stream,
                      static_cast<uint8_t*>(k_pool), static_cast<uint8_t*>(v_pool), params, res_k,
                      res_v, static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new),
                      block_table, max_blocks, context_lens, batch, num_kv_heads, max_context_len,
                      pool_blocks, dev_error);
}

}  // namespace pkv
