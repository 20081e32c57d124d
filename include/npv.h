/*
 * npv.h: C ABI of libnpv, attention over a block-paged bf16 KV cache on
 * NVIDIA B200 (sm_100a).
 *
 * The library implements the two jobs of the attention layer of a
 * nano-vLLM-style engine ("3.1 Project overview and the four-layer
 * architecture", section 3, Layer 4: write the new K/V into the cache, then run
 * attention; "Nano-vLLM Architecture and Performance", Key Features 4):
 *
 *   npv_store_kvcache            scatter new K/V rows into cache slots
 *   npv_paged_decode_attention   one query row per sequence over its blocks
 *   npv_paged_prefill_attention  varlen causal rows (chunked prefill, mixed
 *                                with decode rows) over the same cache
 *
 * Conventions shared by every call
 *   - Every tensor and metadata pointer is a DEVICE pointer on the current CUDA
 *     device; shape and size arguments are host integers.  The caller owns all
 *     buffers; the library allocates no device memory per call.
 *   - bf16 tensors are passed as `void *` holding IEEE bfloat16 values.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream): inputs
 *     must stay alive, and outputs must not be read, until the stream has
 *     passed the call.
 *   - Host-side validation failures return synchronously and launch nothing.
 *     Data-dependent faults found on the device (a block id, slot or context
 *     length out of range) never trap: the offending entry is skipped, a
 *     library-wide device error word records it, and
 *     npv_check_device_errors() reports and clears it.
 *   - No C++ exception crosses this interface.
 *
 * Cache layout (both caches): [num_blocks, block_size, num_kv_heads, head_dim]
 * bf16, contiguous.  A cache slot s addresses block s / block_size, row
 * s % block_size ("Nano-vLLM Architecture and Performance", Key Features 2:
 * fixed-size blocks, 256 tokens by default).  Sequence b's j-th token lives in
 * block block_tables[b * max_blocks_per_seq + j / block_size], row
 * j % block_size.  Block-table entries past ceil(context_lens[b] / block_size)
 * are never read.  Several sequences may list the same physical block (prefix
 * caching, "nano-vllm" README, Features: Prefix Caching); attention only reads
 * such blocks, and a store must never target them.
 *
 * Grouped-query attention ("nano-vllm" README, X-Ray Mode): query head h reads
 * KV head h / (num_q_heads / num_kv_heads).  The default softmax scale is
 * 1 / sqrt(head_dim) (same section, step 2).
 *
 * Supported: head_dim in {64, 128}; num_q_heads / num_kv_heads in {1, 2, 4, 8};
 * block_size a positive multiple of 16; every bf16 pointer 16-byte aligned;
 * for npv_paged_prefill_attention, num_blocks * block_size < 2^31 (its tensor
 * maps address cache rows with signed 32-bit coordinates).
 */
#ifndef NPV_H
#define NPV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define NPV_API __attribute__((visibility("default")))
#else
#define NPV_API
#endif

/* ABI-identical to cudaStream_t / CUstream. */
typedef struct CUstream_st *npv_stream_t;

typedef enum {
    NPV_OK = 0,
    NPV_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misaligned pointer or stride */
    NPV_ERR_UNSUPPORTED = 2,   /* valid but outside the supported set above */
    NPV_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small */
    NPV_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    NPV_ERR_DEVICE_BOUNDS = 5  /* device found an out-of-range id (npv_check_device_errors) */
} npv_status;

/* Device error word bits (npv_check_device_errors). */
#define NPV_DEVERR_SLOT 0x1u        /* slot_mapping entry >= num_blocks * block_size */
#define NPV_DEVERR_BLOCK_ID 0x2u    /* a live block-table entry outside [0, num_blocks) */
#define NPV_DEVERR_CONTEXT_LEN 0x4u /* context length < 0, > max_blocks_per_seq * block_size,
                                       or smaller than the sequence's query rows */
#define NPV_DEVERR_QUERY_LENS 0x8u  /* cu_seqlens_q not nondecreasing from 0 to total_q, or an
                                       n_b above a max_seqlen_q that sent the call to the
                                       decode kernel alone */
#define NPV_DEVERR_TIMEOUT 0x10u    /* an internal pipeline wait gave up after ~2 s (library bug) */

/* Static description of a status code. Never NULL. */
NPV_API const char *npv_status_string(npv_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
NPV_API int npv_version(void);

/*
 * Store new keys and values into the paged cache
 * ("Nano-vLLM Architecture and Performance", Key Features 4: store_kvcache
 * writes KV entries into the paged cache blocks; "3.1 Project overview ...",
 * section 4 step 4: the new K/V are stored before attention runs).
 *
 *   key, value    [num_tokens, num_kv_heads, head_dim] bf16; token t's rows start
 *                 key_token_stride (value_token_stride) ELEMENTS apart, heads
 *                 contiguous.  A stride of 0 means num_kv_heads * head_dim.
 *                 Strides * 2 bytes must be multiples of 16.
 *   k_cache, v_cache  [num_blocks, block_size, num_kv_heads, head_dim] bf16.
 *   slot_mapping  [num_tokens] int32 on the device.  Token t goes to slot
 *                 slot_mapping[t]; a negative slot is a padding row and writes
 *                 nothing.  Slots >= num_blocks * block_size set
 *                 NPV_DEVERR_SLOT and are skipped.  Two tokens with the same
 *                 slot in one call leave that slot undefined.
 * Result: a bit-exact copy; no other cache byte changes.  num_tokens == 0 is a
 * no-op.
 */
NPV_API npv_status npv_store_kvcache(const void *key, const void *value, int64_t key_token_stride,
                             int64_t value_token_stride, void *k_cache, void *v_cache,
                             const int32_t *slot_mapping, int32_t num_tokens, int32_t num_blocks,
                             int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                             npv_stream_t stream);

/*
 * Rotary position embedding of the new tokens' q and k, then the store of the
 * rotated k and of v into their cache slots, in one launch ("Nano-vLLM
 * Architecture and Performance", project structure: RoPE in
 * layers/rotary_embedding.py, applied to q and k before the attention layer
 * stores k and v; the store as for npv_store_kvcache).  The pages name RoPE
 * without its formula; this is the rotary embedding of Su et al. ("RoFormer",
 * section 3.4) in the rotate-half pairing that Qwen3 uses: for a row x of
 * head_dim D at position p and i < D/2, the pair (x[i], x[i + D/2]) is turned
 * by the angle p * theta_i, theta_i = rope_base^(-2i/D):
 *     x[i]       <- x[i] cos - x[i + D/2] sin
 *     x[i + D/2] <- x[i + D/2] cos + x[i] sin
 * The angle, cos and sin are taken in double precision, the rotation in fp32,
 * and each result is rounded to bf16 (nearest, ties to even) once.
 *
 *   q             [num_tokens, num_q_heads, head_dim] bf16, rows q_token_stride
 *                 ELEMENTS apart (0: num_q_heads * head_dim); rotated IN PLACE.
 *                 May be null when num_q_heads == 0 (k and v only).
 *   key, value    [num_tokens, num_kv_heads, head_dim] bf16, strides as for
 *                 npv_store_kvcache; read only (the rotated k goes to the cache).
 *   positions     [num_tokens] int32 (device): token t's position (any int32;
 *                 for a decode row, L_b - 1; for row i of an n_b-row chunk,
 *                 L_b - n_b + i).
 *   k_cache, v_cache, slot_mapping, num_blocks, block_size: as for
 *                 npv_store_kvcache (a negative slot stores nothing, but the
 *                 token's q rows are still rotated; a slot past the cache sets
 *                 NPV_DEVERR_SLOT and stores nothing).
 *   head_dim      a multiple of 16, at most 256 (else NPV_ERR_UNSUPPORTED).
 *   rope_base     base of the frequencies (> 0 and finite; Qwen3 uses 1e6).
 * All pointers 16-byte aligned, all strides * 2 bytes multiples of 16.
 * num_tokens == 0 is a no-op.
 */
NPV_API npv_status npv_rope_store_kvcache(void *q, int64_t q_token_stride, int32_t num_q_heads, const void *key,
                                          const void *value, int64_t key_token_stride, int64_t value_token_stride,
                                          const int32_t *positions, void *k_cache, void *v_cache,
                                          const int32_t *slot_mapping, int32_t num_tokens, int32_t num_blocks,
                                          int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                                          double rope_base, npv_stream_t stream);

/*
 * Bytes of device workspace npv_paged_decode_attention needs on the current
 * device for this head configuration.  The size does not depend on context
 * lengths.  Returns 0 for arguments the call would reject.
 */
NPV_API size_t npv_paged_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim);

/*
 * Grouped-query decode attention over the paged cache: for each sequence b and
 * query head h, softmax(scale * q[b,h] . K_b^T) V_b over the context_lens[b]
 * tokens of sequence b (the tokens stored by this step included).
 *
 *   out           [num_seqs, num_q_heads, head_dim] bf16, contiguous (written).
 *   q             [num_seqs, num_q_heads, head_dim] bf16; sequence b's row starts
 *                 q_seq_stride ELEMENTS after sequence b-1's (0 = num_q_heads *
 *                 head_dim), heads contiguous.
 *   block_tables  [num_seqs, max_blocks_per_seq] int32 (device).
 *   context_lens  [num_seqs] int32 (device).  0 writes a zero row.  Values < 0 or
 *                 > max_blocks_per_seq * block_size set NPV_DEVERR_CONTEXT_LEN
 *                 and write a zero row.
 *   scale         softmax scale; <= 0 selects 1 / sqrt(head_dim).
 *   workspace     device scratch of at least npv_paged_decode_workspace_size()
 *                 bytes, 256-byte aligned.  Its contents need no initialisation
 *                 and are meaningless after the call.  Two calls in flight at
 *                 once must not share a workspace.
 * Work is split over the device's SMs by KV tokens (split-KV): a sequence whose
 * tokens land on several CTAs is combined by a merge kernel from its partial
 * (max, sum, unnormalised output) triples.  Q K^T and P V run on warp-level
 * tensor-core MMAs with fp32 accumulation (the probabilities P are rounded to
 * bf16 for the P V product and the row sums add the rounded values); the
 * output is rounded once to bf16 (round to nearest even).
 */
NPV_API npv_status npv_paged_decode_attention(void *out, const void *q, int64_t q_seq_stride, const void *k_cache,
                                      const void *v_cache, const int32_t *block_tables,
                                      int32_t max_blocks_per_seq, const int32_t *context_lens,
                                      int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
                                      void *workspace, size_t workspace_bytes, npv_stream_t stream);

/*
 * One decode step's two jobs in one launch set: store each sequence's new key
 * and value rows, then decode attention over the caches that include them
 * ("3.1 Project overview and the four-layer architecture", section 3, Layer 4:
 * the attention layer writes the new K/V, then attends).  The result equals
 * npv_store_kvcache(key, value, ..., slot_mapping, num_tokens = num_seqs)
 * followed by npv_paged_decode_attention, bit for bit.
 *
 *   key, value    [num_seqs, num_kv_heads, head_dim] bf16: token b is sequence
 *                 b's new token, at position context_lens[b] - 1.  Strides as
 *                 for npv_store_kvcache.
 *   slot_mapping  [num_seqs] int32 (device): token b's slot, which must be the
 *                 slot that sequence b's block table gives position
 *                 context_lens[b] - 1 (the CTA that reads that position stores
 *                 the token first).  A negative slot stores nothing.
 *   other arguments and the workspace as for npv_paged_decode_attention.
 */
NPV_API npv_status npv_store_kvcache_and_decode_attention(
    void *out, const void *q, int64_t q_seq_stride, const void *key, const void *value, int64_t key_token_stride,
    int64_t value_token_stride, const int32_t *slot_mapping, void *k_cache, void *v_cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
    void *workspace, size_t workspace_bytes, npv_stream_t stream);

/*
 * Bytes of device workspace npv_paged_prefill_attention needs on the current
 * device.  Returns 0 for arguments the call would reject.
 */
NPV_API size_t npv_paged_prefill_workspace_size(int32_t num_seqs, int32_t total_q, int32_t num_q_heads,
                                        int32_t num_kv_heads, int32_t head_dim);

/*
 * Varlen causal attention for packed query rows over the paged cache: chunked
 * prefill with prior cached context, prefix-shared blocks, and decode rows in
 * the same batch ("nano-vllm" README, Features: Chunked Prefill and Prefix
 * Caching; "Nano-vLLM Architecture and Performance", Key Features 1).
 *
 *   out           [total_q, num_q_heads, head_dim] bf16, contiguous (written).
 *   q             [total_q, num_q_heads, head_dim] bf16, contiguous.  Rows of
 *                 sequence b are cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1.
 *   cu_seqlens_q  [num_seqs + 1] int32 (device), nondecreasing from 0 to total_q.
 *                 A first entry other than 0, a last entry other than total_q, or
 *                 a decreasing entry sets NPV_DEVERR_QUERY_LENS; the rows of a
 *                 sequence whose range is reversed or leaves [0, total_q) are
 *                 not written.
 *                 n_b = cu_seqlens_q[b+1] - cu_seqlens_q[b] may be 0 (no rows) or
 *                 1 (a decode row).
 *   context_lens  [num_seqs] int32 (device): L_b, all cached tokens of sequence b
 *                 including its n_b new rows, which must already be stored.
 *                 Row i of sequence b sits at position L_b - n_b + i and sees
 *                 keys 0 .. L_b - n_b + i.  L_b < n_b sets NPV_DEVERR_CONTEXT_LEN.
 *   max_seqlen_q  host upper bound on every n_b, as in flash-attn's varlen calls;
 *                 checked to be >= 0.  When max_seqlen_q * g <= 8 the short
 *                 sequences run on a lighter variant of the decode kernel (see
 *                 below).  When max_seqlen_q <= m every sequence fits the decode
 *                 kernel, and the call launches that kernel alone (no tcgen05
 *                 kernel, no plan); a sequence with n_b > m then sets
 *                 NPV_DEVERR_QUERY_LENS and its rows are written as zeros.  With
 *                 max_seqlen_q > m a bound that is broken costs nothing: the row
 *                 counts are read on the device and route each sequence.
 *   other arguments as for npv_paged_decode_attention.
 * Sequences with n_b > m (g = num_q_heads / num_kv_heads; m = 8 / g when
 * max_seqlen_q * g <= 8, else 16 / g) run on the tcgen05 tensor cores (QK^T and
 * PV with fp32 accumulators in tensor memory); sequences with 1 <= n_b <= m
 * (decode rows, speculative-decode verification) run on the split-KV decode
 * kernel within the same call, whose warp-level MMA tiles hold the g * n_b rows
 * of one KV head.  Both round P to bf16 for the PV product.
 */
NPV_API npv_status npv_paged_prefill_attention(void *out, const void *q, const int32_t *cu_seqlens_q,
                                       int32_t max_seqlen_q, int32_t total_q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       int32_t max_blocks_per_seq, const int32_t *context_lens,
                                       int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
                                       void *workspace, size_t workspace_bytes, npv_stream_t stream);

/* Size of the scratch array compiled into the library for
 * npv_paged_decode_attention_noalloc (16 MiB on every device that loads it). */
#define NPV_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * Decode attention for callers that cannot allocate device memory.  The pages
 * have no counterpart to this entry point; it is a convenience of this library.
 *
 * Some callers cannot call cudaMalloc or hand the library a workspace: a plugin
 * or custom-op host whose framework owns all device memory and passes only its
 * input and output buffers, or code on a path where an allocation is not
 * allowed because cudaMalloc may synchronise the device.  This call computes
 * exactly what npv_paged_decode_attention computes (same arguments, minus the
 * workspace) and allocates nothing: its scratch is a fixed array of
 * NPV_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library holds until the process exits.
 *   - The first call on each device looks up that array's device address (a
 *     one-time set-up that may load the library's GPU code).  Make the first
 *     call on a device before any stream capture begins.
 *   - A head configuration whose scratch would not fit returns
 *     NPV_ERR_WORKSPACE (on a 148-SM B200 every supported configuration fits).
 *   - All calls share the one array, which keeps whatever the last call left in
 *     it; nothing in it needs to start at zero.  Calls that overlap on the GPU
 *     (on different streams, or from several host threads at once) race on it
 *     and produce wrong results; calls ordered on one stream are safe.
 */
NPV_API npv_status npv_paged_decode_attention_noalloc(void *out, const void *q, int64_t q_seq_stride,
                                                      const void *k_cache, const void *v_cache,
                                                      const int32_t *block_tables, int32_t max_blocks_per_seq,
                                                      const int32_t *context_lens, int32_t num_seqs,
                                                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                                      int32_t num_blocks, int32_t block_size, float scale,
                                                      npv_stream_t stream);

/*
 * Test hook for failure detection; the pages have no counterpart.  With
 * enable != 0, later decode-kernel launches on the current device (the decode
 * calls, and the short sequences of a prefill call) run with one pipeline stage
 * per CTA left unfilled on purpose, and their consumer warps wait for a stage at
 * most about a millisecond instead of 2 s.  The wait therefore gives up: the
 * kernel records NPV_DEVERR_TIMEOUT, waits (bounded, 2 s) for the copies it did
 * issue, and returns; the outputs of such calls are meaningless, nothing
 * faults, and the CUDA context stays usable.  npv_check_device_errors() then
 * reports the timeout.  enable == 0 restores normal operation.  The setting is
 * copied to the device synchronously; change it only while no call is in
 * flight.  Returns NPV_ERR_CUDA if the copy fails.
 */
NPV_API npv_status npv_debug_inject_decode_timeout(int enable);

/*
 * Synchronise `stream`, then read and clear the device error word of the
 * current device.  Returns NPV_OK if no error was recorded since the last
 * check, NPV_ERR_DEVICE_BOUNDS otherwise (with the NPV_DEVERR_* bits in
 * *bits_out when bits_out is not NULL), or NPV_ERR_CUDA if the synchronisation
 * failed.
 */
NPV_API npv_status npv_check_device_errors(npv_stream_t stream, uint32_t *bits_out);

#ifdef __cplusplus
}
#endif

#endif /* NPV_H */
