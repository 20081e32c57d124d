// npv_paged_decode_attention_noalloc: decode attention for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) and cannot
// hand the library a workspace: for example a plugin or custom-op host whose
// framework owns every byte of device memory and passes the library only its
// input and output buffers, or code running on a path where an allocation is
// not allowed because cudaMalloc can synchronise the device and stall every
// other stream.  For them this entry point runs the same split-KV and merge
// kernels as npv_paged_decode_attention, with the scratch those kernels need
// taken from a fixed array compiled into the library instead of a
// caller-provided workspace.
//
// This file is compiled as part of npv_lib.cu's translation unit (it is
// included at the end of that file), so the kernels and the library's device
// error word are the same ones the other entry points use.

#include <mutex>

namespace {

// Scratch for the split-KV partials and the per-CTA schedule of one call.  Every
// GPU that loads the library holds these bytes until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NPV_NOALLOC_SCRATCH_BYTES];

// Host code must not use g_noalloc_scratch as a pointer: on the host it names a
// stand-in, not device memory.  Its device address is looked up once per device
// with that device current, and passed to the kernels.
void *g_noalloc_ptr[kMaxDevices] = {};
cudaError_t g_noalloc_err[kMaxDevices] = {};
std::once_flag g_noalloc_once[kMaxDevices];

npv_status noalloc_scratch(void **ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NPV_ERR_CUDA;
    std::call_once(g_noalloc_once[dev], [dev] {
        void *p = nullptr;
        g_noalloc_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        g_noalloc_ptr[dev] = p;
    });
    if (g_noalloc_err[dev] != cudaSuccess || g_noalloc_ptr[dev] == nullptr) return NPV_ERR_CUDA;
    *ptr = g_noalloc_ptr[dev];
    return NPV_OK;
}

}  // namespace

extern "C" NPV_API npv_status npv_paged_decode_attention_noalloc(
    void *out, const void *q, int64_t q_seq_stride, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks, int32_t block_size,
    float scale, npv_stream_t stream) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
        return NPV_ERR_INVALID_ARG;
    if (num_q_heads <= 0 || num_q_heads % num_kv_heads != 0) return NPV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return NPV_ERR_INVALID_ARG;
    if (block_size % 16 != 0) return NPV_ERR_UNSUPPORTED;
    DecodeConfig cfg;
    npv_status st = decode_config(num_q_heads, num_kv_heads, head_dim, &cfg);
    if (st != NPV_OK) return st;
    // the scratch this configuration needs must fit the fixed array
    if (cfg.ws_total > (size_t)NPV_NOALLOC_SCRATCH_BYTES) return NPV_ERR_WORKSPACE;
    if (num_seqs == 0) return NPV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return NPV_ERR_INVALID_ARG;
    const int64_t qrow = (int64_t)num_q_heads * head_dim;
    if (q_seq_stride == 0) q_seq_stride = qrow;
    if (q_seq_stride < qrow || (q_seq_stride * 2) % 16 != 0) return NPV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return NPV_ERR_INVALID_ARG;
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != NPV_OK) return st;
    // Nothing in the scratch has to start at zero: every slot the merge kernel
    // reads is written earlier in the same call by the split kernel.
    return run_decode(out, q, q_seq_stride, nullptr, num_seqs, k_cache, v_cache, block_tables, max_blocks_per_seq,
                      context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, scale,
                      scratch, cfg, (cudaStream_t)stream);
}
