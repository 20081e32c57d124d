// libnpv: the C ABI declared in include/npv.h.
//
// One translation unit: the kernels are included here so that the library-wide
// device error word is a single symbol without relocatable device code.
// Host functions validate every argument before launching, translate CUDA
// errors into npv_status codes and never throw.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "npv.h"
#include "npv_device.cuh"
#include "store_kvcache.cuh"
#include "rope_store.cuh"
#include "decode_attention.cuh"
#include "prefill_attention.cuh"

#define NPV_VERSION_MAJOR 0
#define NPV_VERSION_MINOR 1
#define NPV_VERSION_PATCH 0

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sm_count = 0;
    int max_smem_optin = 0;
};

DeviceInfo g_devices[kMaxDevices];
std::once_flag g_device_once[kMaxDevices];

// Properties of the current device (queried once per device).
const DeviceInfo *current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::call_once(g_device_once[dev], [dev] {
        DeviceInfo info;
        cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&info.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        g_devices[dev] = info;
    });
    return g_devices[dev].sm_count > 0 ? &g_devices[dev] : nullptr;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

npv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NPV_OK : NPV_ERR_CUDA; }

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel on the stream drains; every kernel of this library
// calls griddepcontrol.wait before touching memory, so ordering is preserved.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---- decode configuration ------------------------------------------------------

struct DecodeConfig {
    int group = 0;           // g = Hq / Hkv
    int heads_per_cta = 0;   // HC
    int head_groups = 0;     // Hkv / HC
    int max_rows = 0;        // most query rows of a sequence the kernel serves
    int rows_per_head = 0;   // partial-slot rows per KV head: g * max_rows
    bool sole_path = false;  // mixed batch with no prefill kernel launched
    bool wide_merge = false; // merge CTAs of 1,024 threads (units of many query rows)
    int stages = 0;
    int grid = 0;
    size_t smem = 0;
    size_t ws_ml = 0, ws_o = 0, ws_total = 0;
};

bool supported_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

// Largest divisor of Hkv within the kernel's consumer-warp budget (one warp per KV head).
int pick_heads_per_cta(int num_kv_heads) {
    for (int hc = npv::decode::kMaxConsumerWarps; hc >= 1; --hc)
        if (num_kv_heads % hc == 0) return hc;
    return 1;
}

// multi_row: the decode kernel also serves sequences of up to 16 / g query rows
// (the rows of a prefill call that fit its two 8-column MMA tiles per KV head);
// the workspace is sized for that.
npv_status decode_config(int num_q_heads, int num_kv_heads, int head_dim, DecodeConfig *cfg,
                         bool multi_row = false) {
    if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return NPV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return NPV_ERR_UNSUPPORTED;
    const int g = num_q_heads / num_kv_heads;
    if (!supported_group(g)) return NPV_ERR_UNSUPPORTED;
    const DeviceInfo *dev = current_device();
    if (!dev) return NPV_ERR_CUDA;
    cfg->group = g;
    cfg->heads_per_cta = pick_heads_per_cta(num_kv_heads);
    cfg->head_groups = num_kv_heads / cfg->heads_per_cta;
    cfg->max_rows = multi_row ? npv::decode::kTileRows / g : 1;
    cfg->rows_per_head = g * cfg->max_rows;
    const int hc = cfg->heads_per_cta;
    const size_t stage_bytes = 2ull * npv::decode::kChunk * hc * head_dim * 2;
    int stages = (int)(npv::decode::kStageBudgetBytes / stage_bytes);
    if (stages > npv::decode::kMaxStages) stages = npv::decode::kMaxStages;
    if (stages < 2) stages = 2;
    cfg->stages = stages;
    cfg->smem = npv::decode::kHeaderBytes + stages * stage_bytes;
    if ((int)cfg->smem > dev->max_smem_optin) return NPV_ERR_UNSUPPORTED;
    cfg->grid = dev->sm_count;
    const size_t rows = (size_t)hc * cfg->rows_per_head;
    cfg->ws_ml = align_up((size_t)cfg->grid * 2 * rows * sizeof(float2), 256);
    cfg->ws_o = align_up((size_t)cfg->grid * 2 * rows * head_dim * sizeof(float), 256);
    cfg->ws_total = cfg->ws_ml + cfg->ws_o;
    return NPV_OK;
}

template <int D, int G, int NR>
cudaError_t launch_decode_split(const npv::decode::Params &p, const DecodeConfig &cfg, cudaStream_t stream) {
    auto kernel = npv::decode::decode_split_kernel<D, G, NR>;
    static int configured_smem[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && configured_smem[dev] < (int)cfg.smem) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cfg.smem);
        if (e != cudaSuccess) return e;
        configured_smem[dev] = (int)cfg.smem;
    }
    return launch_pdl(kernel, dim3(cfg.grid), dim3((cfg.heads_per_cta + 1) * 32), cfg.smem, stream, p);
}

cudaError_t dispatch_decode_split(int D, const npv::decode::Params &p, const DecodeConfig &cfg,
                                  cudaStream_t stream) {
    const int nr = cfg.rows_per_head > 8 ? 2 : 1;
#define NPV_DECODE_CASE(DD, GG)                                                         \
    if (D == DD && cfg.group == GG)                                                     \
        return nr == 1 ? launch_decode_split<DD, GG, 1>(p, cfg, stream)                 \
                       : launch_decode_split<DD, GG, 2>(p, cfg, stream);
    NPV_DECODE_CASE(128, 1)
    NPV_DECODE_CASE(128, 2)
    NPV_DECODE_CASE(128, 4)
    NPV_DECODE_CASE(128, 8)
    NPV_DECODE_CASE(64, 1)
    NPV_DECODE_CASE(64, 2)
    NPV_DECODE_CASE(64, 4)
    NPV_DECODE_CASE(64, 8)
#undef NPV_DECODE_CASE
    return cudaErrorInvalidValue;
}

// New K/V rows stored by a fused store + decode call (one token per sequence).
struct FusedStore {
    const void *key;
    const void *value;
    int64_t key_stride;
    int64_t value_stride;
    const int32_t *slot_mapping;
};

// Shared by the decode calls and the decode rows of the prefill call.
npv_status run_decode(void *out, const void *q, int64_t q_row_stride, const int32_t *cu_seqlens_q, int32_t total_q,
                      const void *k_cache, const void *v_cache, const int32_t *block_tables,
                      int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                      int32_t block_size, float scale, void *workspace, const DecodeConfig &cfg,
                      cudaStream_t stream, const FusedStore *store = nullptr) {
    npv::decode::Params p = {};
    p.out = static_cast<uint16_t *>(out);
    p.q = static_cast<const uint16_t *>(q);
    p.q_row_stride = q_row_stride;
    p.k_cache = static_cast<const uint16_t *>(k_cache);
    p.v_cache = static_cast<const uint16_t *>(v_cache);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.cu_seqlens_q = cu_seqlens_q;
    p.total_q = total_q;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.block_size = block_size;
    p.heads_per_cta = cfg.heads_per_cta;
    p.num_head_groups = cfg.head_groups;
    p.max_rows = cfg.max_rows;
    p.rows_per_head = cfg.rows_per_head;
    p.sole_path = cfg.sole_path ? 1 : 0;
    p.num_stages = cfg.stages;
    const float s = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)head_dim));
    p.scale_log2 = s * 1.4426950408889634f;
    char *ws = static_cast<char *>(workspace);
    p.part_ml = reinterpret_cast<float2 *>(ws);
    p.part_o = reinterpret_cast<float *>(ws + cfg.ws_ml);
    if (store) {
        p.key = static_cast<const uint16_t *>(store->key);
        p.value = static_cast<const uint16_t *>(store->value);
        p.key_stride = store->key_stride;
        p.value_stride = store->value_stride;
        p.slot_mapping = store->slot_mapping;
    }
    cudaError_t e = dispatch_decode_split(head_dim, p, cfg, stream);
    if (e != cudaSuccess) return NPV_ERR_CUDA;
    if (cfg.wide_merge)
        e = launch_pdl(npv::decode::decode_merge_kernel<1024>, dim3(cfg.grid), dim3(1024), 0, stream, p,
                       (int)head_dim);
    else
        e = launch_pdl(npv::decode::decode_merge_kernel<512>, dim3(cfg.grid), dim3(512), 0, stream, p, (int)head_dim);
    return cuda_status(e);
}

// ---- prefill configuration ----------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, found through the runtime (no libcuda link).
EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 3-D bf16 tensor [d2][d1][d0] (d0 contiguous), 128-byte swizzled boxes of b0 x b1 x b2.
bool encode_map_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                   uint32_t b1, uint32_t b2) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct PrefillConfig {
    DecodeConfig decode;  // for the rows of single-row sequences
    int32_t max_pairs = 0;
    int grid = 0;
    size_t smem = 0;
    size_t ws_pairs = 0;
    size_t ws_total = 0;
};

npv_status prefill_config(int32_t num_seqs, int32_t total_q, int num_q_heads, int num_kv_heads, int head_dim,
                          PrefillConfig *cfg) {
    if (num_seqs < 0 || total_q < 0) return NPV_ERR_INVALID_ARG;
    npv_status st = decode_config(num_q_heads, num_kv_heads, head_dim, &cfg->decode, true);
    if (st != NPV_OK) return st;
    const DeviceInfo *dev = current_device();
    if (!dev) return NPV_ERR_CUDA;
    const int ppt = npv::prefill::kTileM / cfg->decode.group;
    const int64_t pairs = (int64_t)total_q / ppt + 1 + num_seqs;
    if (pairs > 0x7FFFFFFF) return NPV_ERR_UNSUPPORTED;
    cfg->max_pairs = (int32_t)pairs;
    cfg->grid = dev->sm_count;
    cfg->smem = (head_dim == 128 ? npv::prefill::Smem<128>::total : npv::prefill::Smem<64>::total) + 1024;
    if ((int)cfg->smem > dev->max_smem_optin) return NPV_ERR_UNSUPPORTED;
    cfg->ws_pairs = align_up((size_t)pairs * sizeof(int2), 256);
    cfg->ws_total = cfg->decode.ws_total + 256 + cfg->ws_pairs;
    return NPV_OK;
}

template <int D, int G>
cudaError_t launch_prefill(const npv::prefill::Params &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                           const CUtensorMap &vmap, const PrefillConfig &cfg, cudaStream_t stream) {
    cudaError_t e = launch_pdl(npv::prefill::prefill_plan_kernel<G>, dim3(1), dim3(1024), 0, stream, p, D);
    if (e != cudaSuccess) return e;
    auto kernel = npv::prefill::prefill_attention_kernel<D, G>;
    static int configured_smem[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && configured_smem[dev] < (int)cfg.smem) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cfg.smem);
        if (e != cudaSuccess) return e;
        configured_smem[dev] = (int)cfg.smem;
    }
    return launch_pdl(kernel, dim3(cfg.grid), dim3(npv::prefill::kThreads), cfg.smem, stream, p, qmap, kmap, vmap);
}

cudaError_t dispatch_prefill(int D, int G, const npv::prefill::Params &p, const CUtensorMap &qmap,
                             const CUtensorMap &kmap, const CUtensorMap &vmap, const PrefillConfig &cfg,
                             cudaStream_t stream) {
#define NPV_PREFILL_CASE(DD, GG) \
    if (D == DD && G == GG) return launch_prefill<DD, GG>(p, qmap, kmap, vmap, cfg, stream);
    NPV_PREFILL_CASE(128, 1)
    NPV_PREFILL_CASE(128, 2)
    NPV_PREFILL_CASE(128, 4)
    NPV_PREFILL_CASE(128, 8)
    NPV_PREFILL_CASE(64, 1)
    NPV_PREFILL_CASE(64, 2)
    NPV_PREFILL_CASE(64, 4)
    NPV_PREFILL_CASE(64, 8)
#undef NPV_PREFILL_CASE
    return cudaErrorInvalidValue;
}

bool cache_shape_ok(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads, int32_t head_dim) {
    return num_blocks > 0 && block_size > 0 && num_kv_heads > 0 && head_dim > 0;
}

}  // namespace

extern "C" {

const char *npv_status_string(npv_status status) {
    switch (status) {
        case NPV_OK: return "ok";
        case NPV_ERR_INVALID_ARG: return "invalid argument (null pointer, bad shape, misaligned pointer or stride)";
        case NPV_ERR_UNSUPPORTED: return "unsupported configuration";
        case NPV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case NPV_ERR_CUDA: return "CUDA runtime error";
        case NPV_ERR_DEVICE_BOUNDS: return "device reported an out-of-range slot, block id or length";
    }
    return "unknown status";
}

int npv_version(void) { return NPV_VERSION_MAJOR * 10000 + NPV_VERSION_MINOR * 100 + NPV_VERSION_PATCH; }

npv_status npv_store_kvcache(const void *key, const void *value, int64_t key_token_stride,
                             int64_t value_token_stride, void *k_cache, void *v_cache,
                             const int32_t *slot_mapping, int32_t num_tokens, int32_t num_blocks,
                             int32_t block_size, int32_t num_kv_heads, int32_t head_dim, npv_stream_t stream) {
    if (num_tokens < 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
        return NPV_ERR_INVALID_ARG;
    if (num_tokens == 0) return NPV_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return NPV_ERR_INVALID_ARG;
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (key_token_stride == 0) key_token_stride = row;
    if (value_token_stride == 0) value_token_stride = row;
    if (key_token_stride < row || value_token_stride < row) return NPV_ERR_INVALID_ARG;
    if ((row * 2) % 16 != 0 || (key_token_stride * 2) % 16 != 0 || (value_token_stride * 2) % 16 != 0)
        return NPV_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
        return NPV_ERR_INVALID_ARG;
    const DeviceInfo *dev = current_device();
    if (!dev) return NPV_ERR_CUDA;
    npv::store::Params p = {};
    p.key = static_cast<const uint16_t *>(key);
    p.value = static_cast<const uint16_t *>(value);
    p.key_stride = key_token_stride;
    p.value_stride = value_token_stride;
    p.k_cache = static_cast<uint16_t *>(k_cache);
    p.v_cache = static_cast<uint16_t *>(v_cache);
    p.slot_mapping = slot_mapping;
    p.num_tokens = num_tokens;
    p.row_vecs = (int32_t)(row / 8);
    p.num_slots = (int64_t)num_blocks * block_size;
    const int64_t vecs = (int64_t)num_tokens * p.row_vecs;
    const int64_t per_block = (int64_t)npv::store::kThreads * npv::store::kVecsPerThread;
    int64_t blocks = (vecs + per_block - 1) / per_block;
    const int64_t cap = (int64_t)dev->sm_count * 8;
    if (blocks > cap) blocks = cap;
    cudaError_t e = launch_pdl(npv::store::store_kvcache_kernel, dim3((unsigned)blocks),
                               dim3(npv::store::kThreads), 0, (cudaStream_t)stream, p);
    return cuda_status(e);
}

npv_status npv_rope_store_kvcache(void *q, int64_t q_token_stride, int32_t num_q_heads, const void *key,
                                  const void *value, int64_t key_token_stride, int64_t value_token_stride,
                                  const int32_t *positions, void *k_cache, void *v_cache,
                                  const int32_t *slot_mapping, int32_t num_tokens, int32_t num_blocks,
                                  int32_t block_size, int32_t num_kv_heads, int32_t head_dim, double rope_base,
                                  npv_stream_t stream) {
    if (num_tokens < 0 || num_q_heads < 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
        return NPV_ERR_INVALID_ARG;
    if (!(rope_base > 0.0) || !std::isfinite(rope_base)) return NPV_ERR_INVALID_ARG;
    if (head_dim % 16 != 0 || head_dim > npv::rope::kMaxHeadDim) return NPV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return NPV_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping || !positions) return NPV_ERR_INVALID_ARG;
    if (num_q_heads > 0 && !q) return NPV_ERR_INVALID_ARG;
    const int64_t kvrow = (int64_t)num_kv_heads * head_dim;
    const int64_t qrow = (int64_t)num_q_heads * head_dim;
    if (key_token_stride == 0) key_token_stride = kvrow;
    if (value_token_stride == 0) value_token_stride = kvrow;
    if (q_token_stride == 0) q_token_stride = qrow;
    if (key_token_stride < kvrow || value_token_stride < kvrow || q_token_stride < qrow) return NPV_ERR_INVALID_ARG;
    if ((key_token_stride * 2) % 16 != 0 || (value_token_stride * 2) % 16 != 0 || (q_token_stride * 2) % 16 != 0)
        return NPV_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (num_q_heads > 0 && !aligned16(q)))
        return NPV_ERR_INVALID_ARG;
    npv::rope::Params p = {};
    p.q = num_q_heads > 0 ? static_cast<uint16_t *>(q) : nullptr;
    p.q_stride = q_token_stride;
    p.key = static_cast<const uint16_t *>(key);
    p.value = static_cast<const uint16_t *>(value);
    p.key_stride = key_token_stride;
    p.value_stride = value_token_stride;
    p.positions = positions;
    p.slot_mapping = slot_mapping;
    p.k_cache = static_cast<uint16_t *>(k_cache);
    p.v_cache = static_cast<uint16_t *>(v_cache);
    p.num_tokens = num_tokens;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.num_slots = (int64_t)num_blocks * block_size;
    p.base = rope_base;
    const unsigned blocks = (unsigned)((num_tokens + npv::rope::kTokens - 1) / npv::rope::kTokens);
    return cuda_status(launch_pdl(npv::rope::rope_store_kernel, dim3(blocks), dim3(npv::rope::kThreads), 0,
                                  (cudaStream_t)stream, p));
}

size_t npv_paged_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim) {
    if (num_seqs < 0) return 0;
    DecodeConfig cfg;
    if (decode_config(num_q_heads, num_kv_heads, head_dim, &cfg) != NPV_OK) return 0;
    return cfg.ws_total;
}

npv_status npv_paged_decode_attention(void *out, const void *q, int64_t q_seq_stride, const void *k_cache,
                                      const void *v_cache, const int32_t *block_tables,
                                      int32_t max_blocks_per_seq, const int32_t *context_lens,
                                      int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
                                      void *workspace, size_t workspace_bytes, npv_stream_t stream) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
        return NPV_ERR_INVALID_ARG;
    if (num_q_heads <= 0 || num_q_heads % num_kv_heads != 0) return NPV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return NPV_ERR_INVALID_ARG;
    if (block_size % 16 != 0) return NPV_ERR_UNSUPPORTED;
    DecodeConfig cfg;
    npv_status st = decode_config(num_q_heads, num_kv_heads, head_dim, &cfg);
    if (st != NPV_OK) return st;
    if (num_seqs == 0) return NPV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return NPV_ERR_INVALID_ARG;
    const int64_t qrow = (int64_t)num_q_heads * head_dim;
    if (q_seq_stride == 0) q_seq_stride = qrow;
    if (q_seq_stride < qrow || (q_seq_stride * 2) % 16 != 0) return NPV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return NPV_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < cfg.ws_total)
        return NPV_ERR_WORKSPACE;
    return run_decode(out, q, q_seq_stride, nullptr, num_seqs, k_cache, v_cache, block_tables, max_blocks_per_seq,
                      context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, scale,
                      workspace, cfg, (cudaStream_t)stream);
}

npv_status npv_store_kvcache_and_decode_attention(
    void *out, const void *q, int64_t q_seq_stride, const void *key, const void *value, int64_t key_token_stride,
    int64_t value_token_stride, const int32_t *slot_mapping, void *k_cache, void *v_cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
    void *workspace, size_t workspace_bytes, npv_stream_t stream) {
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
        return NPV_ERR_INVALID_ARG;
    if (num_q_heads <= 0 || num_q_heads % num_kv_heads != 0) return NPV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return NPV_ERR_INVALID_ARG;
    if (block_size % 16 != 0) return NPV_ERR_UNSUPPORTED;
    DecodeConfig cfg;
    npv_status st = decode_config(num_q_heads, num_kv_heads, head_dim, &cfg);
    if (st != NPV_OK) return st;
    if (num_seqs == 0) return NPV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !key || !value || !slot_mapping)
        return NPV_ERR_INVALID_ARG;
    const int64_t qrow = (int64_t)num_q_heads * head_dim;
    const int64_t kvrow = (int64_t)num_kv_heads * head_dim;
    if (q_seq_stride == 0) q_seq_stride = qrow;
    if (key_token_stride == 0) key_token_stride = kvrow;
    if (value_token_stride == 0) value_token_stride = kvrow;
    if (q_seq_stride < qrow || (q_seq_stride * 2) % 16 != 0) return NPV_ERR_INVALID_ARG;
    if (key_token_stride < kvrow || value_token_stride < kvrow || (key_token_stride * 2) % 16 != 0 ||
        (value_token_stride * 2) % 16 != 0)
        return NPV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(key) ||
        !aligned16(value))
        return NPV_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < cfg.ws_total)
        return NPV_ERR_WORKSPACE;
    const FusedStore fs = {key, value, key_token_stride, value_token_stride, slot_mapping};
    return run_decode(out, q, q_seq_stride, nullptr, num_seqs, k_cache, v_cache, block_tables, max_blocks_per_seq,
                      context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, scale,
                      workspace, cfg, (cudaStream_t)stream, &fs);
}

size_t npv_paged_prefill_workspace_size(int32_t num_seqs, int32_t total_q, int32_t num_q_heads,
                                        int32_t num_kv_heads, int32_t head_dim) {
    PrefillConfig cfg;
    if (prefill_config(num_seqs, total_q, num_q_heads, num_kv_heads, head_dim, &cfg) != NPV_OK) return 0;
    return cfg.ws_total;
}

npv_status npv_paged_prefill_attention(void *out, const void *q, const int32_t *cu_seqlens_q,
                                       int32_t max_seqlen_q, int32_t total_q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       int32_t max_blocks_per_seq, const int32_t *context_lens,
                                       int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
                                       void *workspace, size_t workspace_bytes, npv_stream_t stream) {
    if (num_seqs < 0 || total_q < 0 || max_seqlen_q < 0 || max_blocks_per_seq <= 0 ||
        !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
        return NPV_ERR_INVALID_ARG;
    if (num_q_heads <= 0 || num_q_heads % num_kv_heads != 0) return NPV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return NPV_ERR_INVALID_ARG;
    if (block_size % 16 != 0) return NPV_ERR_UNSUPPORTED;
    // TMA coordinates are signed 32-bit: every cache slot row must be addressable
    if ((int64_t)num_blocks * block_size > 0x7FFFFFFFll) return NPV_ERR_UNSUPPORTED;
    PrefillConfig cfg;
    npv_status st = prefill_config(num_seqs, total_q, num_q_heads, num_kv_heads, head_dim, &cfg);
    if (st != NPV_OK) return st;
    if (num_seqs == 0 || total_q == 0) return NPV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !cu_seqlens_q)
        return NPV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return NPV_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < cfg.ws_total)
        return NPV_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    const int D = head_dim, G = cfg.decode.group;

    // The decode kernel takes the sequences whose g * n_b rows fit its MMA
    // columns: one 8-column tile when max_seqlen_q says that suffices (fewer
    // registers), else two.  The row counts themselves are read on the device.
    if ((int64_t)max_seqlen_q * G <= 8) {
        cfg.decode.max_rows = 8 / G;
        cfg.decode.rows_per_head = 8;
    }
    // When the hint bounds every sequence by the decode kernel's rows, no
    // sequence is left for the tensor-memory kernel: its plan and launch are
    // skipped, and the decode kernel reports a sequence that breaks the bound.
    cfg.decode.sole_path = max_seqlen_q <= cfg.decode.max_rows;
    // a call of multi-row sequences only (speculative-decode verification) has
    // merges of g * n_b >= 8 rows per KV head: the wide merge CTA
    cfg.decode.wide_merge = cfg.decode.sole_path && (int64_t)max_seqlen_q * G >= 8;
    if (!cfg.decode.sole_path) {
        // tensor maps, 128-byte swizzle: the caches [NB * BS, Hkv, D] in boxes of
        // {64 elements, 1 head, box_tokens slots}; q [total_q, Hq, D] in boxes of
        // {64 elements, G heads, 128 / G positions} (one 128-row tile of a KV head)
        CUtensorMap qmap, kmap, vmap;
        const int box_tokens = (block_size % 128 == 0) ? 128 : 16;
        if (!encode_map_3d(&qmap, q, D, num_q_heads, (uint64_t)total_q, 64, G, npv::prefill::kTileM / G) ||
            !encode_map_3d(&kmap, k_cache, D, num_kv_heads, (uint64_t)num_blocks * block_size, 64, 1, box_tokens) ||
            !encode_map_3d(&vmap, v_cache, D, num_kv_heads, (uint64_t)num_blocks * block_size, 64, 1, box_tokens))
            return NPV_ERR_CUDA;

        npv::prefill::Params p = {};
        p.out = static_cast<uint16_t *>(out);
        p.cu_seqlens_q = cu_seqlens_q;
        p.context_lens = context_lens;
        p.block_tables = block_tables;
        p.total_q = total_q;
        p.num_seqs = num_seqs;
        p.num_q_heads = num_q_heads;
        p.num_kv_heads = num_kv_heads;
        p.num_blocks = num_blocks;
        p.block_size = block_size;
        p.max_blocks_per_seq = max_blocks_per_seq;
        p.box_tokens = box_tokens;
        p.q = static_cast<const uint16_t *>(q);
        const float sc = scale > 0.f ? scale : (float)(1.0 / std::sqrt((double)head_dim));
        p.scale_log2 = sc * 1.4426950408889634f;
        char *ws = static_cast<char *>(workspace);
        p.plan_count = reinterpret_cast<int32_t *>(ws + cfg.decode.ws_total);
        p.plan_pairs = reinterpret_cast<int2 *>(ws + cfg.decode.ws_total + 256);
        p.max_pairs = cfg.max_pairs;
        p.decode_rows_max = cfg.decode.max_rows;
        cudaError_t e = dispatch_prefill(D, G, p, qmap, kmap, vmap, cfg, s);
        if (e != cudaSuccess) return NPV_ERR_CUDA;
    }
    // sequences of 1 .. 16 / g query rows: the split-KV decode kernel
    return run_decode(out, q, (int64_t)num_q_heads * head_dim, cu_seqlens_q, total_q, k_cache, v_cache,
                      block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads, num_kv_heads,
                      head_dim, num_blocks, block_size, scale, workspace, cfg.decode, s);
}

npv_status npv_debug_inject_decode_timeout(int enable) {
    const unsigned int v = enable ? 1u : 0u;
    return cuda_status(cudaMemcpyToSymbol(npv::decode::g_debug_timeout, &v, sizeof(v)));
}

npv_status npv_check_device_errors(npv_stream_t stream, uint32_t *bits_out) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return NPV_ERR_CUDA;
    unsigned int bits = 0;
    if (cudaMemcpyFromSymbol(&bits, npv::g_error_word, sizeof(bits)) != cudaSuccess) return NPV_ERR_CUDA;
    if (bits != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(npv::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return NPV_ERR_CUDA;
    }
    if (bits_out) *bits_out = bits;
    return bits ? NPV_ERR_DEVICE_BOUNDS : NPV_OK;
}

}  // extern "C"

// The allocation-free decode entry point shares this translation unit.
#include "npv_noalloc.cu"
