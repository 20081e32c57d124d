// store_kvcache: scatter each new token's K and V rows into its cache slot.
//
// "Nano-vLLM Architecture and Performance", Key Features 4: a store kernel
// writes KV cache entries into the paged cache blocks; "3.1 Project overview and
// the four-layer architecture", section 4 step 4: the store happens before the
// attention of the same layer.  Slot s is block s / block_size, row
// s % block_size of a [num_blocks, block_size, num_kv_heads, head_dim] cache.
//
// A token's [num_kv_heads, head_dim] row is contiguous both in the source and in
// the cache, so the scatter is a set of row copies.  Each thread moves 16-byte
// vectors (8 bf16), consecutive threads take consecutive vectors of a row, so
// every warp reads and writes whole 512-byte runs.  The work is pure bandwidth:
// 2 * num_tokens * row_bytes read and the same written.
#pragma once

#include "npv_device.cuh"

namespace npv {
namespace store {

struct Params {
    const uint16_t *key;
    const uint16_t *value;
    int64_t key_stride;    // elements between consecutive tokens
    int64_t value_stride;  // elements between consecutive tokens
    uint16_t *k_cache;
    uint16_t *v_cache;
    const int32_t *slot_mapping;
    int32_t num_tokens;
    int32_t row_vecs;      // 16-byte vectors per token row: num_kv_heads * head_dim / 8
    int64_t num_slots;     // num_blocks * block_size
};

constexpr int kThreads = 256;
constexpr int kVecsPerThread = 4;

// Grid-stride over (token, vector) pairs; the K and V copies of one vector are
// issued together so each thread has 2 * kVecsPerThread loads in flight.
__global__ void __launch_bounds__(kThreads) store_kvcache_kernel(const Params p) {
    // Launched with programmatic stream serialisation: wait until the previous
    // grid on the stream (which may still be reading the cache, or writing
    // key / value / slot_mapping) has completed and its writes are visible.
    grid_dependency_wait();
    const int64_t total = (int64_t)p.num_tokens * p.row_vecs;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t base = (int64_t)blockIdx.x * kThreads * kVecsPerThread + threadIdx.x; base < total;
         base += stride * kVecsPerThread) {
        uint4 kv[kVecsPerThread], vv[kVecsPerThread];
        int64_t dst[kVecsPerThread];
#pragma unroll
        for (int r = 0; r < kVecsPerThread; ++r) {
            const int64_t idx = base + (int64_t)r * kThreads;
            dst[r] = -1;
            if (idx < total) {
                const int32_t t = (int32_t)(idx / p.row_vecs);
                const int32_t v = (int32_t)(idx - (int64_t)t * p.row_vecs);
                const int32_t s = __ldg(p.slot_mapping + t);
                if (s >= 0) {
                    if ((int64_t)s < p.num_slots) {
                        kv[r] = ld_nc_v4(p.key + t * p.key_stride + (int64_t)v * 8);
                        vv[r] = ld_nc_v4(p.value + t * p.value_stride + (int64_t)v * 8);
                        dst[r] = ((int64_t)s * p.row_vecs + v) * 8;
                    } else if (v == 0) {
                        report_error(NPV_DEVERR_SLOT);
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kVecsPerThread; ++r) {
            if (dst[r] >= 0) {
                st_global_v4(p.k_cache + dst[r], kv[r]);
                st_global_v4(p.v_cache + dst[r], vv[r]);
            }
        }
    }
}

}  // namespace store
}  // namespace npv
