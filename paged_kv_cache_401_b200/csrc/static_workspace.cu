// paged_decode_attention_static_workspace: the split-K decode for callers that
// cannot allocate device memory.
//
// Some callers have no way to obtain device memory for the split-K workspace:
// an engine that reserved all of HBM for its KV pool up front (a cudaMalloc would
// fail, or fragment the pool), a plugin inside another runtime that owns the
// allocator and hands plugins no allocation hook, or a latency-bound loop that
// cannot take cudaMalloc's implicit device synchronisation.  For them the
// partial (max, sum, output) of every sequence partition lives in a fixed array
// in this library's device image instead of a caller buffer.
//
// The array is file-scope device memory: every GPU that loads the library holds
// KV_STATIC_WORKSPACE_BYTES of it until the process exits, and every call on a
// device shares it.  Host code cannot use the array's name as a device address
// (on the host it names a stand-in object), so each call looks up the device
// address with cudaGetSymbolAddress on the current device.  Nothing is cached
// across calls: a context that is destroyed and created again (cudaDeviceReset)
// loads the module again, possibly at another address, and the next call finds
// the new one.
#include "kernels.cuh"

namespace {

__device__ __align__(256) static uint8_t g_static_workspace[KV_STATIC_WORKSPACE_BYTES];

}  // namespace

extern "C" {

KV_API kv_status paged_decode_attention_static_workspace(
    const kv_pool_desc* pool, void* out, const void* q, kv_dtype q_dtype, const void* k_pool,
    const void* v_pool, const float* scales, const int32_t* block_table,
    int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t max_context_len, float scale, int32_t partition_tokens, int32_t* dev_error,
    kv_stream_t stream) {
    // size check first, on the host: a request needing more than the array holds is refused
    const size_t need = paged_decode_workspace_bytes(pool, batch, num_q_heads, max_context_len,
                                                     partition_tokens);
    if (need > KV_STATIC_WORKSPACE_BYTES) return KV_ERR_INVALID_ARGUMENT;
    void* ws = nullptr;
    if (need > 0) {
        // the array's address in the current device's context (a host-side lookup
        // once the module is loaded)
        if (cudaGetSymbolAddress(&ws, g_static_workspace) != cudaSuccess || ws == nullptr) {
            cudaGetLastError();
            return KV_ERR_CUDA;
        }
    }
    // Every partial the merge reads is written earlier in the same call, so
    // nothing in the array needs clearing between calls.
    return paged_decode_attention(pool, out, q, q_dtype, k_pool, v_pool, scales,
                                  block_table, max_blocks_per_seq, context_lens, batch,
                                  num_q_heads, max_context_len, scale, partition_tokens, ws,
                                  need > 0 ? KV_STATIC_WORKSPACE_BYTES : 0, dev_error, stream);
}

}  // extern "C"
