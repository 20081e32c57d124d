// rope_store: rotary position embedding of the new tokens' q and k, then the
// store of the rotated k and of v into their cache slots, in one launch.
//
// "Nano-vLLM Architecture and Performance", project structure: the Qwen3 layer
// applies RoPE (layers/rotary_embedding.py) to q and k right before the
// attention layer, whose first job is the store of k and v into the paged
// cache (Key Features 4; "3.1 Project overview and the four-layer
// architecture", section 4 step 4).  Fusing the two moves each new k row
// through HBM once instead of three times (read, rotated write, store read).
//
// Rotary embedding (Su et al., "RoFormer", section 3.4), rotate-half pairing:
// for a row x of D values at position p and i < D/2, the pair
// (x[i], x[i + D/2]) turns by p * theta_i, theta_i = base^(-2i/D).  The angle
// and its cosine and sine are taken in double precision (positions reach 1e5
// and more, where a single-precision angle would already be off by ~1e-2
// radians); the rotation itself runs in fp32 and rounds to bf16 once.
//
// Work layout: a CTA takes kTokens consecutive tokens.  Its first phase fills
// a shared table of (cos, sin) for those tokens' D/2 frequencies; in the
// second, every thread takes "units": 8 consecutive elements of a row's first
// half and the 8 partner elements of its second half (two 16-byte loads and
// stores).  A token has Hq + 2 Hkv rows (q rows rotated in place, k rows
// rotated into the cache, v rows copied into the cache) of D/16 units each;
// consecutive threads take consecutive units, so each half-row moves as one
// contiguous run.  The kernel is bound by HBM bandwidth (plus its launch):
// per token it reads and writes the q row and reads k and v and writes them to
// the cache.
#pragma once

#include "npv_device.cuh"

namespace npv {
namespace rope {

struct Params {
    uint16_t *q;            // [T, Hq, D] rows q_stride apart (rotated in place); null when Hq == 0
    int64_t q_stride;
    const uint16_t *key;    // [T, Hkv, D]
    const uint16_t *value;  // [T, Hkv, D]
    int64_t key_stride;
    int64_t value_stride;
    const int32_t *positions;     // [T]
    const int32_t *slot_mapping;  // [T]
    uint16_t *k_cache;
    uint16_t *v_cache;
    int32_t num_tokens;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int64_t num_slots;  // num_blocks * block_size
    double base;
};

constexpr int kThreads = 256;
constexpr int kTokens = 4;
constexpr int kMaxHeadDim = 256;

__global__ void __launch_bounds__(kThreads) rope_store_kernel(const Params p) {
    __shared__ float2 cs[kTokens][kMaxHeadDim / 2];
    // Launched with programmatic stream serialisation: the previous grid may
    // still be reading the cache or writing q / key / value.
    grid_dependency_wait();
    const int D = p.head_dim, half = D / 2;
    const int32_t t0 = blockIdx.x * kTokens;
    const int nt = min(kTokens, p.num_tokens - t0);

    for (int j = threadIdx.x; j < nt * half; j += kThreads) {
        const int tl = j / half, i = j - tl * half;
        const double theta = pow(p.base, -2.0 * (double)i / (double)D);
        const double angle = (double)__ldg(p.positions + t0 + tl) * theta;
        double s, c;
        sincos(angle, &s, &c);
        cs[tl][i] = make_float2((float)c, (float)s);
    }
    __syncthreads();

    const int upr = D / 16;  // units per row
    const int rows = p.num_q_heads + 2 * p.num_kv_heads;
    const int units = nt * rows * upr;
    for (int u = threadIdx.x; u < units; u += kThreads) {
        const int tl = u / (rows * upr);
        const int rem = u - tl * rows * upr;
        const int r = rem / upr, j = rem - r * upr;
        const int32_t t = t0 + tl;
        const int e0 = j * 8;  // first element of the unit in the first half

        const uint16_t *src;
        uint16_t *dst;
        bool rotate = true;
        if (r < p.num_q_heads) {
            src = p.q + (int64_t)t * p.q_stride + (int64_t)r * D;
            dst = p.q + (int64_t)t * p.q_stride + (int64_t)r * D;
        } else {
            const int32_t s = __ldg(p.slot_mapping + t);
            if (s < 0) continue;  // padding row: nothing stored
            if ((int64_t)s >= p.num_slots) {
                if (r == p.num_q_heads && j == 0) report_error(NPV_DEVERR_SLOT);
                continue;
            }
            const int kr = r - p.num_q_heads;
            if (kr < p.num_kv_heads) {
                src = p.key + (int64_t)t * p.key_stride + (int64_t)kr * D;
                dst = p.k_cache + ((int64_t)s * p.num_kv_heads + kr) * D;
            } else {
                const int vr = kr - p.num_kv_heads;
                src = p.value + (int64_t)t * p.value_stride + (int64_t)vr * D;
                dst = p.v_cache + ((int64_t)s * p.num_kv_heads + vr) * D;
                rotate = false;
            }
        }
        // q is rewritten in place, so it is read through the coherent path
        const uint4 a = (r < p.num_q_heads) ? *reinterpret_cast<const uint4 *>(src + e0) : ld_nc_v4(src + e0);
        const uint4 b = (r < p.num_q_heads) ? *reinterpret_cast<const uint4 *>(src + half + e0)
                                            : ld_nc_v4(src + half + e0);
        if (!rotate) {
            st_global_v4(dst + e0, a);
            st_global_v4(dst + half + e0, b);
            continue;
        }
        float x1[8], x2[8], y1[8], y2[8];
        unpack8(a, x1);
        unpack8(b, x2);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 w = cs[tl][e0 + k];  // (cos, sin)
            y1[k] = __fmaf_rn(x1[k], w.x, -(x2[k] * w.y));
            y2[k] = __fmaf_rn(x2[k], w.x, x1[k] * w.y);
        }
        st_global_v4(dst + e0, pack8(y1));
        st_global_v4(dst + half + e0, pack8(y2));
    }
}

}  // namespace rope
}  // namespace npv
