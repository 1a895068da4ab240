/*
 * paged_kv.h -- C ABI of libpagedkv.so: single-token GQA decode attention
 * over a PagedAttention KV cache, for NVIDIA B200 (sm_100a).
 *
 * The method (the four web pages on KV caching it follows):
 *  - "KV Cache 深度解析：显存黑洞、PagedAttention 与三路省内存方案" (d7kj.com):
 *    §一 decode attends the new token's q to every cached K/V with
 *    softmax(q·Kᵀ/√d)·V; §三 the cache is cut into fixed 16-token blocks and
 *    a block table maps each sequence's logical blocks to physical blocks
 *    scattered in a pool ("逻辑连续、物理离散"), several sequences may share a
 *    physical block; §四 GQA (query heads share KV heads) and fp8 E4M3 KV
 *    with per-token scales.
 *  - "llm-inference-optimization" notes (qingdujian.com): §二 the paged
 *    cache's append (new block when the last one is full, write at the next
 *    offset); §三 the tiled online-softmax update (running max, running sum,
 *    rescaled running output).
 *  - k1-blog daily note 2026-07-13, "PagedAttention 與 vLLM": the attention
 *    kernel must be rewritten to read non-contiguous memory.
 *
 * Conventions for every entry point:
 *  - Every device buffer is owned by the caller.  The library allocates no
 *    device memory, keeps no state between calls and never synchronises:
 *    work is enqueued on the caller's stream (NULL = legacy default stream).
 *  - Device pointers must be 16-byte aligned (the K and V pools of INT4 and KIVI
 *    caches 32-byte aligned); contiguous row-major layouts.
 *  - Argument errors found on the host return KV_ERR_INVALID_ARGUMENT or
 *    KV_ERR_UNSUPPORTED before anything is enqueued; a failed launch returns
 *    KV_ERR_CUDA.  Nothing throws, nothing aborts the process.
 *  - Data errors found on the device (a slot or block id out of range, a bad
 *    context length, a bounded wait that ran out) never trap: the kernel skips
 *    the offending work and ORs a KV_DEVERR_* bit into *dev_error when
 *    dev_error is non-NULL (an int32 in device memory the caller zeroes).
 */
#ifndef PAGED_KV_H
#define PAGED_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KV_API __attribute__((visibility("default")))
#else
#define KV_API
#endif

/* The CUDA stream type (identical to cudaStream_t / CUstream). */
struct CUstream_st;
typedef struct CUstream_st* kv_stream_t;

typedef enum {
    KV_OK = 0,
    KV_ERR_INVALID_ARGUMENT = 1,
    KV_ERR_UNSUPPORTED = 2,
    KV_ERR_CUDA = 3,
    KV_ERR_OUT_OF_BLOCKS = 4   /* block manager: no free block / sequence slot left */
} kv_status;

typedef enum {
    KV_F32 = 0,        /* IEEE binary32 */
    KV_BF16 = 1,       /* bfloat16 */
    KV_FP8_E4M3 = 2,   /* OCP FP8 E4M3 codes (KV pools only) with fp32 row scales */
    KV_INT8 = 3,       /* signed 8-bit codes (KV pools only) with fp32 row scales */
    KV_INT4 = 4,       /* unsigned 4-bit codes, two per byte (KV pools only, head_dim 128),
                          with an fp32 (scale, zero point) pair per row */
    KV_KIVI4 = 5       /* KIVI: 4-bit codes as KV_INT4, keys with a (scale, zero point) per
                          channel of each full block, values per row; see kivi_* below */
} kv_dtype;

/* Bits ORed into *dev_error by the kernels. */
#define KV_DEVERR_BAD_SLOT        0x1  /* slot >= num_blocks * block_size: write skipped */
#define KV_DEVERR_BAD_CONTEXT_LEN 0x2  /* context_lens[b] < 1 or > max_context_len: out[b] = 0 */
#define KV_DEVERR_BAD_BLOCK_ID    0x4  /* block id outside [0, num_blocks): block skipped */
#define KV_DEVERR_TIMEOUT         0x8  /* a bounded wait on staged data ran out: output invalid */
#define KV_DEVERR_BAD_POSITION    0x10 /* slot mapping: position outside the block table */

/*
 * Geometry of one layer's K pool and V pool (plain data, owns nothing).
 *
 * Layout of each pool, row-major: [num_blocks][num_kv_heads][block_size][head_dim]
 * so the 16 tokens of one (physical block, kv head) pair are one contiguous
 * span of block_size*head_dim elements.  A quantised cache (FP8 or INT8) also
 * has ONE fp32 scale pool laid out [num_blocks][num_kv_heads][2][block_size]:
 * for each (block, kv head) the 16 K row scales then the 16 V row scales, 128
 * contiguous bytes.  An INT4 pool stores a row's 128 codes in 64 bytes (dim
 * 2i in the low nibble of byte i, dim 2i+1 in the high nibble) and has one
 * fp32 parameter pool [num_blocks][num_kv_heads][2][block_size][2]: per row
 * (scale, zero point), K rows then V rows, 256 bytes per (block, kv head).
 * A KIVI pool (KV_KIVI4) has the INT4 code layout and a parameter pool
 * [num_blocks][num_kv_heads][128 + 16][2] fp32: (scale, zero point) of each of
 * the 128 key channels over the block's 16 tokens, then of each of the 16
 * value rows, 1152 bytes per (block, kv head).
 */
typedef struct {
    int32_t num_blocks;
    int32_t block_size;      /* tokens per block; 16 */
    int32_t num_kv_heads;
    int32_t head_dim;        /* 64 or 128 */
    int32_t dtype;           /* kv_dtype */
    int32_t elem_bytes;      /* 4, 2 or 1; 0 for 4-bit codes (two per byte) */
    uint64_t kv_bytes;       /* bytes of ONE pool (K or V) */
    uint64_t scale_bytes;    /* bytes of the scale / parameter pool (FP8, INT8, INT4, KIVI) */
    int64_t stride_block;    /* elements between consecutive physical blocks */
    int64_t stride_head;     /* elements between consecutive kv heads of a block */
    int64_t stride_slot;     /* elements between consecutive tokens of a block */
} kv_pool_desc;

/*
 * Fill *out with the geometry of a pool (host only, no device work).
 * Errors: KV_ERR_INVALID_ARGUMENT for out == NULL or non-positive sizes;
 * KV_ERR_UNSUPPORTED for block_size != 16, head_dim not in {64, 128},
 * num_kv_heads > 256, an unknown dtype, or KV_INT4 / KV_KIVI4 with head_dim != 128.
 */
KV_API kv_status kv_pool_create(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                         int32_t head_dim, kv_dtype dtype, kv_pool_desc* out);

/*
 * Slot of each token to append ("KV Cache 深度解析" §三; "llm-inference-
 * optimization" notes §二): token i is position positions[i] of sequence
 * seq_ids[i]; its slot is
 *     block_table[seq][pos / block_size] * block_size + pos % block_size.
 *   block_table  : device int32 [batch][max_blocks_per_seq]
 *   seq_ids      : device int32 [num_tokens], each in [0, batch)
 *   positions    : device int32 [num_tokens]
 *   slot_mapping : device int64 [num_tokens] (written)
 * A position outside [0, max_blocks_per_seq*block_size) or a seq id outside
 * [0, batch) gives slot -1 (padding, skipped by reshape_and_cache) and
 * KV_DEVERR_BAD_POSITION.  num_tokens == 0 enqueues nothing.
 */
KV_API kv_status compute_slot_mapping(const int32_t* block_table, int32_t batch,
                               int32_t max_blocks_per_seq, int32_t block_size,
                               const int32_t* seq_ids, const int32_t* positions,
                               int32_t num_tokens, int64_t* slot_mapping,
                               int32_t* dev_error, kv_stream_t stream);

/*
 * Cache write ("KV Cache 深度解析" §一: decode computes only the new token's
 * K/V and appends it to the cache).  For token t and kv head h with
 * s = slot_mapping[t] >= 0:
 *     pool[s / 16][h][s % 16][:] = row(t, h)
 *   k_new, v_new : device [num_tokens][num_kv_heads][head_dim] in src_dtype
 *   slot_mapping : device int64 [num_tokens]; s < 0 is padding (skipped);
 *                  s >= num_blocks*16 is skipped with KV_DEVERR_BAD_SLOT
 * F32 / BF16 pools: src_dtype must equal the pool dtype; the copy is exact.
 * FP8 pools ("KV Cache 深度解析" §四): src_dtype F32 or BF16; for each row
 *     a = max |x| (fp32),  scale = a / 448 (IEEE fp32 division),
 *     code = E4M3(x / scale) (IEEE division, round to nearest even,
 *            saturating to ±448),  and scale = 0, codes 0x00 when a == 0;
 * INT8 pools ("k1-blog" KV 量化 and "大模型推理为何这么慢" KV Cache量化: 8-bit KV
 * halves the cache like FP8): src_dtype F32 or BF16; for each row
 *     a = max |x|,  scale = a / 127 (IEEE fp32 division),
 *     code = clamp(round_to_nearest_even(x / scale), -127, 127),
 *     and scale = 0, codes 0 when a == 0.
 * INT4 pools ("llm-inference-optimization" notes §四: the printed 4-bit
 * routine, asymmetric with a zero point, applied to each row; "大模型推理为何
 * 这么慢", KV Cache量化: a 4-bit cache is 4x smaller than fp16): src_dtype F32
 * or BF16; for each row, in IEEE fp32
 *     hi = max x, lo = min x,  scale = (hi - lo) / 15,
 *     zero = round_to_nearest_even(-lo / scale),
 *     code = clamp(round_to_nearest_even(x / scale) + zero, 0, 15),
 *     value = (code - zero) * scale;
 *     a constant row (hi == lo), where the routine would divide by zero, is
 *     stored exactly: scale = |lo|, zero = -1 (lo > 0), +1 (lo < 0) or 0 (with
 *     scale 0, lo == 0), every code 0.
 *   scales : device fp32 scale pool [num_blocks][num_kv_heads][2][16] (K row
 *   scales, then V row scales), or for INT4 the parameter pool above; NULL for
 *   F32/BF16 pools.  Rows must be finite.
 * Two tokens given the same slot race (last writer unspecified).
 */
KV_API kv_status reshape_and_cache(const kv_pool_desc* pool, void* k_pool, void* v_pool,
                            float* scales,
                            const void* k_new, const void* v_new, kv_dtype src_dtype,
                            const int64_t* slot_mapping, int32_t num_tokens,
                            int32_t* dev_error, kv_stream_t stream);

/*
 * Number of consumer ranges the decode cuts its work into (host only).
 * The decode lays the (sequence, kv head) pairs end to end as one list of
 * 16-token tiles and cuts it into this many equal contiguous ranges, one per
 * consumer warp.  partition_tokens == 0: as many ranges as the current
 * device runs consumer warps at once (148 SMs assumed when no device can be
 * queried), so every SM streams the same number of bytes; partition_tokens >
 * 0 (a multiple of 16): ranges of at most that many tokens over the longest
 * possible list (batch * kv heads * ceil(max_context_len / 16) tiles).
 * Returns 0 for invalid arguments.
 */
KV_API int32_t paged_decode_num_ranges(const kv_pool_desc* pool, int32_t batch,
                                       int32_t num_q_heads, int32_t max_context_len,
                                       int32_t partition_tokens);

/*
 * Bytes of device workspace paged_decode_attention needs for these sizes
 * (host only; partition_tokens as above; 0 for invalid arguments):
 * (batch + 1) int32 sequence starts, then, for each of
 * batch * num_kv_heads + num_ranges pieces, the partial (max, sum) and
 * head_dim-wide partial output of every query head of the group.  Its
 * contents need no initialisation.
 */
KV_API size_t paged_decode_workspace_bytes(const kv_pool_desc* pool, int32_t batch,
                                           int32_t num_q_heads, int32_t max_context_len,
                                           int32_t partition_tokens);

/*
 * Single-token GQA decode attention over the paged cache ("KV Cache 深度解析"
 * §一, §三, §四; "llm-inference-optimization" notes §三).  For sequence b,
 * query head h, kv head g = h / (num_q_heads / num_kv_heads) and the
 * L = context_lens[b] tokens of logical positions 0..L-1 (token p stored in
 * physical block block_table[b][p / 16], slot p % 16):
 *     s_p = scale * q[b,h,:] . K_p[g,:]
 *     out[b,h,:] = sum_p softmax(s)_p * V_p[g,:]
 * computed exactly up to fp32 rounding with an online softmax.  The
 * (sequence, kv head) pairs are split over paged_decode_num_ranges(...)
 * consumer ranges; a pair split over several ranges has its pieces' (max,
 * sum, output) merged by log-sum-exp in a second kernel.
 *   out          : device [batch][num_q_heads][head_dim] in q_dtype
 *   q            : device [batch][num_q_heads][head_dim], q_dtype F32 or BF16
 *   k_pool/v_pool: device pools (layout above)
 *   scales       : device fp32 scale / parameter pool (layout above), non-NULL iff the
 *                  pool is FP8, INT8 or INT4
 *   block_table  : device int32 [batch][max_blocks_per_seq]; entries past
 *                  ceil(L/16) are never read
 *   context_lens : device int32 [batch], each in [1, max_context_len]
 *   max_context_len : upper bound of context_lens, <= max_blocks_per_seq*16
 *   partition_tokens : 0 (balanced over the GPU) or a multiple of 16, see
 *                  paged_decode_num_ranges
 *   workspace    : device buffer of >= paged_decode_workspace_bytes(...) bytes
 * Host checks: num_q_heads % num_kv_heads == 0 with a group size of 1, 2, 4
 * or 8 (else KV_ERR_UNSUPPORTED); partition_tokens a multiple of 16;
 * max_context_len <= max_blocks_per_seq * 16; batch * num_kv_heads *
 * ceil(max_context_len / 16) < 2^31 (else KV_ERR_UNSUPPORTED); an INT4
 * pool needs bf16 q (else KV_ERR_UNSUPPORTED); pointer alignment;
 * workspace size.  Device errors: KV_DEVERR_BAD_CONTEXT_LEN (that sequence's output is
 * zero), KV_DEVERR_BAD_BLOCK_ID (that block's tokens are skipped),
 * KV_DEVERR_TIMEOUT.
 */
KV_API kv_status paged_decode_attention(const kv_pool_desc* pool, void* out, const void* q,
                                 kv_dtype q_dtype, const void* k_pool, const void* v_pool,
                                 const float* scales,
                                 const int32_t* block_table, int32_t max_blocks_per_seq,
                                 const int32_t* context_lens, int32_t batch,
                                 int32_t num_q_heads, int32_t max_context_len, float scale,
                                 int32_t partition_tokens, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_error,
                                 kv_stream_t stream);

/*
 * Fused append + decode: one call for a decode step's cache write and attention.
 * "KV Cache 深度解析" §一/§六 (decode stores the new token's K/V, then scores the
 * query against every cached key including it) and §三 (the slot of position p
 * is block_table[b][p / 16] * 16 + p % 16).  For every sequence b with
 * L = context_lens[b], the new rows k_new[b], v_new[b] go to the slot of
 * position L - 1 -- stored exactly as reshape_and_cache would store them
 * (for FP8 / INT8 pools: the same codes and scales, bit for bit) -- and
 * paged_decode_attention is computed over positions 0 .. L - 1, new token
 * included.  The result (pools and output) is identical to
 * compute_slot_mapping + reshape_and_cache + paged_decode_attention.
 *   k_new, v_new : device [batch][num_kv_heads][head_dim] in src_dtype, 16-byte
 *                  aligned.  src_dtype: the pool dtype for F32 / BF16 pools (no
 *                  conversion), F32 or BF16 for FP8 / INT8 pools, else
 *                  KV_ERR_UNSUPPORTED.
 *   k_pool, v_pool, scales : written (the slot of position L - 1) and read.
 * Everything else as paged_decode_attention; it uses the same workspace size.
 * The slot of position L - 1 must not be read by another sequence of the same
 * call (a shared, partly filled last block is copied on write first).  When
 * the block id of position L - 1 is invalid nothing is written for that pair
 * (KV_DEVERR_BAD_BLOCK_ID); an invalid context length writes nothing for that
 * sequence (KV_DEVERR_BAD_CONTEXT_LEN, zeros).  This entry point has no
 * counterpart on the pages; it fuses two of their steps into one launch.
 */
KV_API kv_status paged_decode_attention_append(const kv_pool_desc* pool, void* out,
                                               const void* q, kv_dtype q_dtype, void* k_pool,
                                               void* v_pool, float* scales, const void* k_new,
                                               const void* v_new, kv_dtype src_dtype,
                                               const int32_t* block_table,
                                               int32_t max_blocks_per_seq,
                                               const int32_t* context_lens, int32_t batch,
                                               int32_t num_q_heads, int32_t max_context_len,
                                               float scale, int32_t partition_tokens,
                                               void* workspace, size_t workspace_bytes,
                                               int32_t* dev_error, kv_stream_t stream);

/*
 * KIVI cache ("大模型推理为何这么慢", KV Cache量化: keys quantised per channel,
 * values per token, the newest tokens kept at full precision).  The 4-bit
 * routine is the INT4 one above (reshape_and_cache), run on a key channel's
 * 16 values within a full block and on each value row.  A KIVI pool holds
 * FULL blocks only; the newest L mod 16 tokens of sequence b (L its context
 * length) live unquantised in caller-owned bf16 residual buffers
 * res_k / res_v [batch][num_kv_heads][16][head_dim], row t holding position
 * 16 * floor(L / 16) + t.
 *
 * kivi_quantize_blocks: quantise num_blocks full blocks (prefill):
 *   k_rows, v_rows : device [num_blocks][16][num_kv_heads][head_dim], 16
 *                    consecutive tokens per block, in src_dtype (F32 or BF16)
 *   block_ids      : device int32 [num_blocks], the block each one goes to
 * An out-of-range block id skips that block (KV_DEVERR_BAD_BLOCK_ID).
 * KV_ERR_UNSUPPORTED for a pool that is not KV_KIVI4 or another src_dtype.
 */
KV_API kv_status kivi_quantize_blocks(const kv_pool_desc* pool, void* k_pool, void* v_pool,
                                      float* params, const void* k_rows, const void* v_rows,
                                      kv_dtype src_dtype, const int32_t* block_ids,
                                      int32_t num_blocks, int32_t* dev_error, kv_stream_t stream);

/*
 * kivi_decode_attention: one decode step over a KIVI pool.  When k_new/v_new
 * (device bf16 [batch][num_kv_heads][head_dim]) are given, each sequence's new
 * rows are first stored at residual row (L - 1) % 16, and when that completes
 * the block, the 16 residual rows are quantised into block
 * block_table[b][(L - 1) / 16]; NULL for both appends nothing.  Then
 * paged_decode_attention's result over positions 0 .. L - 1: full blocks from
 * the pool, the last L mod 16 positions from the residual.  Arguments and
 * workspace as paged_decode_attention; bf16 q and head_dim 128 only, else
 * KV_ERR_UNSUPPORTED (so is a KIVI pool passed to the other entry points).
 */
KV_API kv_status kivi_decode_attention(const kv_pool_desc* pool, void* out, const void* q,
                                       kv_dtype q_dtype, void* k_pool, void* v_pool,
                                       float* params, void* res_k, void* res_v,
                                       const void* k_new, const void* v_new,
                                       const int32_t* block_table, int32_t max_blocks_per_seq,
                                       const int32_t* context_lens, int32_t batch,
                                       int32_t num_q_heads, int32_t max_context_len, float scale,
                                       int32_t partition_tokens, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_error,
                                       kv_stream_t stream);

/*
 * Multi-query paged attention: Q = num_query_tokens new tokens per sequence
 * attend to the cache at once -- the verification of Q speculative tokens, or a
 * chunk of a chunked prefill ("KV Cache 深度解析" §五 chunked prefill; "大模型推理为何
 * 这么慢", speculative decoding).  The Q tokens are the LAST Q tokens of each
 * sequence's context and must already be in the cache: query token i of
 * sequence b sits at position L - Q + i (L = context_lens[b]) and attends to
 * positions 0 .. L - Q + i (causal), with the softmax of paged_decode_attention.
 *   q, out : device [batch][Q][num_q_heads][head_dim] (q_dtype; out in q_dtype)
 * Everything else as paged_decode_attention (Q = 1 is exactly that call).
 * Supported shapes: bf16, FP8, INT8 or INT4 KV, head_dim 128, bf16 q, and
 * (num_q_heads / num_kv_heads) * Q <= 16, else KV_ERR_UNSUPPORTED.  A context
 * length below Q is invalid (zeros, KV_DEVERR_BAD_CONTEXT_LEN).
 */
KV_API size_t paged_attention_workspace_bytes(const kv_pool_desc* pool, int32_t batch,
                                              int32_t num_q_heads, int32_t num_query_tokens,
                                              int32_t max_context_len, int32_t partition_tokens);

KV_API kv_status paged_attention_multi_query(const kv_pool_desc* pool, void* out, const void* q,
                                             kv_dtype q_dtype, int32_t num_query_tokens,
                                             const void* k_pool, const void* v_pool,
                                             const float* scales, const int32_t* block_table,
                                             int32_t max_blocks_per_seq,
                                             const int32_t* context_lens, int32_t batch,
                                             int32_t num_q_heads, int32_t max_context_len,
                                             float scale, int32_t partition_tokens,
                                             void* workspace, size_t workspace_bytes,
                                             int32_t* dev_error, kv_stream_t stream);

/*
 * Bytes of device memory the library holds on every GPU that loads it, for
 * paged_decode_attention_static_workspace (16 MiB: enough for the default
 * split of e.g. 256 sequences x 8 kv heads x 4 query heads per group at
 * head_dim 128 on a 148-SM GPU, about 8 MB).
 */
#define KV_STATIC_WORKSPACE_BYTES (16u * 1024u * 1024u)

/*
 * paged_decode_attention for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point: it exists for callers
 * that have no way to obtain a workspace buffer -- an engine that reserved
 * all device memory for its KV pool at start-up, a plugin inside another
 * runtime that owns the allocator and gives plugins no allocation hook, a
 * latency-bound loop that cannot take cudaMalloc's implicit synchronisation.
 *
 * Same arguments, layouts and results as paged_decode_attention, without
 * workspace / workspace_bytes: the split-K partials go to a fixed array of
 * KV_STATIC_WORKSPACE_BYTES in the library's own device memory, which every
 * GPU that loads the library holds until the process exits.  The caller
 * still passes q, the pools, the tables and out.  Nothing is allocated: no
 * cudaMalloc, cudaFree or allocating library routine is called.
 *  - Sizes whose workspace (paged_decode_workspace_bytes for the same
 *    arguments) exceeds KV_STATIC_WORKSPACE_BYTES return
 *    KV_ERR_INVALID_ARGUMENT before anything is enqueued; a larger
 *    partition_tokens needs less workspace.
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress); nothing is cached, so a context that was reset
 *    and created again is handled.  The first call on a device may load the
 *    library's device code into the context (lazy loading): make that first
 *    call before any stream capture.  A failed look-up returns KV_ERR_CUDA.
 *  - All calls on a device share the one array, which keeps the last call's
 *    contents: calls that may overlap on the GPU (on different streams, or
 *    from different host threads without ordering) race and must be
 *    serialised by the caller.  Each call writes every partial it reads, so
 *    nothing has to be cleared between calls.
 */
KV_API kv_status paged_decode_attention_static_workspace(
    const kv_pool_desc* pool, void* out, const void* q, kv_dtype q_dtype, const void* k_pool,
    const void* v_pool, const float* scales, const int32_t* block_table,
    int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
    int32_t max_context_len, float scale, int32_t partition_tokens, int32_t* dev_error,
    kv_stream_t stream);

/*
 * Copy whole physical blocks: for i < num_copies, block copy_dst[i] of the K
 * pool, the V pool and (quantised pools) the scale / parameter pool becomes a copy of block
 * copy_src[i], every kv head ("KV Cache 深度解析" §三: blocks shared by
 * several sequences; a sequence that writes into a shared, partly filled
 * block first gets its own copy -- see kv_block_manager_append_slots).
 *   copy_src, copy_dst : device int32 [num_copies]; a pair with an id outside
 *   [0, num_blocks) is skipped with KV_DEVERR_BAD_BLOCK_ID.  Destinations
 *   must be distinct and not also sources in the same call.
 */
KV_API kv_status paged_kv_copy_blocks(const kv_pool_desc* pool, void* k_pool, void* v_pool,
                                      float* scales, const int32_t* copy_src,
                                      const int32_t* copy_dst, int32_t num_copies,
                                      int32_t* dev_error, kv_stream_t stream);

/*
 * Host block manager (host memory only; no device work).  Follows "KV Cache
 * 深度解析" §三 (16-token blocks allocated on demand, at most one partly used
 * block per sequence, physical blocks shared between sequences), "大模型推理为何
 * 这么慢" (PagedAttention section: a finished request's blocks are freed at
 * once) and the "llm-inference-optimization" notes §二 (a sequence takes a new
 * block when it has none or its last one is full).  Sharing is by reference
 * count; appending into a shared block that still has free slots first moves
 * the sequence to a private copy (copy-on-write).  Policies: free blocks are a
 * LIFO stack that initially yields 0, 1, 2, ...; a new sequence gets the
 * lowest unused id.  Not thread-safe: one manager per caller thread.
 */
typedef struct kv_block_manager kv_block_manager;

/* num_blocks physical blocks, up to max_seqs live sequences of up to
 * max_blocks_per_seq blocks.  KV_ERR_INVALID_ARGUMENT for non-positive sizes. */
KV_API kv_status kv_block_manager_create(int32_t num_blocks, int32_t max_seqs,
                                         int32_t max_blocks_per_seq, kv_block_manager** out);
KV_API void kv_block_manager_destroy(kv_block_manager* manager);
KV_API int32_t kv_block_manager_num_free_blocks(const kv_block_manager* manager);
/* Reference count of a physical block (0 = free), -1 for an invalid id. */
KV_API int32_t kv_block_manager_refcount(const kv_block_manager* manager, int32_t block);

/* A new empty sequence (KV_ERR_OUT_OF_BLOCKS when max_seqs are live). */
KV_API kv_status kv_block_manager_add_sequence(kv_block_manager* manager, int32_t* seq_id);

/* A new sequence sharing every block of `parent` (same length). */
KV_API kv_status kv_block_manager_fork(kv_block_manager* manager, int32_t parent,
                                       int32_t* child);

/* Release a sequence: its blocks' counts drop, blocks reaching 0 are freed. */
KV_API kv_status kv_block_manager_free_sequence(kv_block_manager* manager, int32_t seq_id);

/*
 * Reserve the slots of num_tokens new tokens, token i appended to sequence
 * seq_ids[i] (several tokens of one sequence are taken in order):
 *   slots[i]  : host int64, the token's slot (block * 16 + offset)
 *   copy_src / copy_dst : host int32 of capacity >= num_tokens; on return the
 *   first *num_copies pairs are the copy-on-write block copies to perform
 *   (paged_kv_copy_blocks) BEFORE writing the new tokens.
 * A batch that needs more free blocks than exist, or grows a sequence past
 * max_blocks_per_seq, returns KV_ERR_OUT_OF_BLOCKS and changes nothing.
 */
KV_API kv_status kv_block_manager_append_slots(kv_block_manager* manager,
                                               const int32_t* seq_ids, int32_t num_tokens,
                                               int64_t* slots, int32_t* copy_src,
                                               int32_t* copy_dst, int32_t* num_copies);

/*
 * Block table and context lengths of every sequence id in [0, max_seqs):
 *   block_table  : host int32 [max_seqs][max_blocks_per_seq]; entries past a
 *                  sequence's last block hold 0x7fffffff
 *   context_lens : host int32 [max_seqs] (0 for ids not in use)
 */
KV_API kv_status kv_block_manager_export(const kv_block_manager* manager, int32_t* block_table,
                                         int32_t* context_lens);

/* Static, human-readable name of a status code. */
KV_API const char* kv_status_string(kv_status status);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_H */
