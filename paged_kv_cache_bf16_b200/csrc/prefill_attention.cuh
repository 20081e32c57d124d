// Chunked-prefill varlen causal attention over the paged cache on the tcgen05
// tensor cores.
//
// What it computes ("nano-vllm" README, Features: Chunked Prefill and Prefix
// Caching, Tutorial Mode chapter 3 on the causal mask; "Nano-vLLM Architecture
// and Performance", Key Features 1): for sequence b with n_b >= 2 new rows that
// are already stored at positions L_b - n_b .. L_b - 1, row i attends to keys
// 0 .. L_b - n_b + i of the sequence's paged K/V, query head h reading KV head
// h / g, scale 1/sqrt(D) by default.  Rows of sequences with n_b == 1 go to
// the split-KV decode kernel in the same call.
//
// How (B200 design):
//   * Work item = (sequence, KV head, tile of 128 MMA rows).  The 128 rows pack
//     128/g positions x the g query heads of one GQA group, so every K/V tile
//     loaded from HBM feeds all g heads (row r = position * g + head).
//   * A one-CTA plan kernel lists the (sequence, row-tile) pairs, counting-sorted
//     by their number of 128-key KV tiles, longest first.  The persistent main
//     kernel (one CTA per SM) takes items from that list in snake order.
//   * Warp roles: warp 4 issues TMA loads (Q once per item, K and V tiles of 128
//     keys through a 2-stage ring; block ids come from the block table a
//     32-entry window at a time, one TMA box per block piece); warp 5 owns tensor
//     memory and issues tcgen05.mma from one thread; warps 0-3 run the softmax,
//     one TMEM lane (= one query row) per thread.
//   * Tensor memory holds S twice (so S for tile j+1 is computed while the
//     softmax reads tile j) and the O accumulator.  S = Q K^T reads Q and K as
//     K-major 128-byte-swizzled operands; O += P V reads P (bf16, written by the
//     softmax threads in the same swizzle) as K-major and V as MN-major.
//   * The softmax keeps a per-row running max in the log2 domain and rescales
//     the O accumulator only when the max grows by more than 2^8 (otherwise the
//     stale max is kept; the final division by the row sum corrects it exactly
//     in real arithmetic).  V rows past the context of the last tile are zeroed
//     before the P.V product so unwritten cache slots never meet it.
#pragma once

#include "npv_device.cuh"
#include "npv_tcgen05.cuh"

namespace npv {
namespace prefill {

constexpr int kTileM = 128;   // query rows per item (MMA M)
constexpr int kTileN = 128;   // keys per KV tile (MMA N of S, K of P.V)
constexpr int kStages = 2;    // K/V ring depth
constexpr int kThreads = 192; // 4 softmax warps, producer, MMA
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kTmemCols = 512;
constexpr int kBuckets = 4096;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Params {
    uint16_t *out;
    const int32_t *cu_seqlens_q;
    const int32_t *context_lens;
    const int32_t *block_tables;
    int32_t total_q;
    int32_t num_seqs;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t num_blocks;
    int32_t block_size;
    int32_t max_blocks_per_seq;
    int32_t box_tokens;  // tokens per K/V TMA box: 128 when block_size % 128 == 0, else 16
    float scale_log2;
    int32_t *plan_count;  // [1]: number of (sequence, row-tile) pairs
    int2 *plan_pairs;     // [max_pairs]: (sequence, row tile), longest first
    int32_t max_pairs;
};

// Shared-memory layout (bytes from a 1024-aligned base).
template <int D>
struct Smem {
    static constexpr int kHeader = 1024;
    static constexpr int kQ = kTileM * D * 2;
    static constexpr int kKV = kTileN * D * 2;
    static constexpr int kP = kTileM * kTileN * 2;
    static constexpr int q = kHeader;
    static constexpr int k = q + kQ;
    static constexpr int v = k + kStages * kKV;
    static constexpr int p = v + kStages * kKV;
    static constexpr int total = p + kP;
};

// Per-item quantities every warp role derives the same way.
struct Item {
    int32_t b, qt, h;
    int32_t row0;    // first packed query row of the sequence
    int32_t n;       // query rows of the sequence
    int32_t L;       // context length (new rows included)
    int32_t p0;      // first position of this row tile (relative to the new rows)
    int32_t npos;    // positions in this tile
    int32_t kv_end;  // keys the tile needs: [0, kv_end)
    int32_t ntiles;  // 128-key tiles
};

template <int G>
__device__ __forceinline__ Item load_item(const Params &p, long long idx) {
    Item it;
    const int2 pr = p.plan_pairs[idx / p.num_kv_heads];
    it.b = pr.x;
    it.qt = pr.y;
    it.h = (int32_t)(idx % p.num_kv_heads);
    it.row0 = __ldg(p.cu_seqlens_q + it.b);
    it.n = __ldg(p.cu_seqlens_q + it.b + 1) - it.row0;
    it.L = __ldg(p.context_lens + it.b);
    constexpr int ppt = kTileM / G;
    it.p0 = it.qt * ppt;
    it.npos = min(ppt, it.n - it.p0);
    it.kv_end = min(it.L, it.L - it.n + it.p0 + it.npos);
    it.ntiles = (it.kv_end + kTileN - 1) / kTileN;
    return it;
}

// Item index of round r for this CTA (snake order over the sorted list).
__device__ __forceinline__ long long item_index(long long r) {
    const long long G = gridDim.x;
    return r * G + ((r & 1) ? (G - 1 - blockIdx.x) : blockIdx.x);
}

// A sequence runs on the tensor-core path when it has >= 2 valid query rows.
__device__ __forceinline__ bool prefill_seq(const Params &p, int32_t b, int32_t *n_out, bool *bad) {
    const int32_t cb = __ldg(p.cu_seqlens_q + b), ce = __ldg(p.cu_seqlens_q + b + 1);
    *bad = false;
    if (cb < 0 || ce < cb || ce > p.total_q) {
        *n_out = 0;
        *bad = true;
        return false;
    }
    const int32_t n = ce - cb;
    *n_out = n;
    if (n < 2) return false;
    const int32_t L = __ldg(p.context_lens + b);
    if (L < n || (long long)L > (long long)p.max_blocks_per_seq * p.block_size) {
        *bad = true;
        return false;
    }
    return true;
}

// ---------------------------------------------------------------------------
// plan: list the (sequence, row tile) pairs, longest KV range first
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(1024) prefill_plan_kernel(const Params p, int head_dim) {
    __shared__ int hist[kBuckets];
    __shared__ long long scratch[40];
    grid_dependency_wait();
    constexpr int ppt = kTileM / G;
    const int tid = threadIdx.x;
    for (int i = tid; i < kBuckets; i += blockDim.x) hist[i] = 0;
    const int per = (p.num_seqs + blockDim.x - 1) / blockDim.x;
    const int lo = min(p.num_seqs, tid * per), hi = min(p.num_seqs, lo + per);
    long long mine = 0;
    for (int b = lo; b < hi; ++b) {
        int32_t n;
        bool bad;
        if (prefill_seq(p, b, &n, &bad)) mine += (n + ppt - 1) / ppt;
        if (bad) {
            const int32_t cb = __ldg(p.cu_seqlens_q + b), ce = __ldg(p.cu_seqlens_q + b + 1);
            if (cb < 0 || ce < cb || ce > p.total_q) {
                report_error(NPV_DEVERR_QUERY_LENS);
            } else {
                report_error(NPV_DEVERR_CONTEXT_LEN);
                // rows of an invalid multi-row sequence are written as zeros
                uint4 *o = reinterpret_cast<uint4 *>(p.out + (int64_t)cb * p.num_q_heads * head_dim);
                const int64_t nvec = (int64_t)(ce - cb) * p.num_q_heads * head_dim / 8;
                for (int64_t i = 0; i < nvec; ++i) o[i] = make_uint4(0, 0, 0, 0);
            }
        }
    }
    long long total;
    long long base = decode::block_exclusive_scan(mine, scratch, &total);
    (void)base;
    __syncthreads();
    // histogram of KV-tile counts (reversed so that the longest come first)
    for (int b = lo; b < hi; ++b) {
        int32_t n;
        bool bad;
        if (!prefill_seq(p, b, &n, &bad)) continue;
        const int32_t L = __ldg(p.context_lens + b);
        for (int qt = 0; qt * ppt < n; ++qt) {
            const int npos = min(ppt, n - qt * ppt);
            const int kv_end = min(L, L - n + qt * ppt + npos);
            const int nt = min(kBuckets - 1, (kv_end + kTileN - 1) / kTileN);
            atomicAdd(&hist[kBuckets - 1 - nt], 1);
        }
    }
    __syncthreads();
    // exclusive scan of the histogram: 4 buckets per thread
    {
        constexpr int kPer = kBuckets / 1024;
        long long s = 0;
        int v[kPer];
        for (int i = 0; i < kPer; ++i) {
            const int idx = tid * kPer + i;
            v[i] = idx < kBuckets && tid < 1024 ? hist[idx] : 0;
            s += v[i];
        }
        long long tot2;
        long long ex = decode::block_exclusive_scan(s, scratch, &tot2);
        __syncthreads();
        for (int i = 0; i < kPer; ++i) {
            const int idx = tid * kPer + i;
            if (idx < kBuckets) hist[idx] = (int)ex;
            ex += v[i];
        }
    }
    __syncthreads();
    for (int b = lo; b < hi; ++b) {
        int32_t n;
        bool bad;
        if (!prefill_seq(p, b, &n, &bad)) continue;
        const int32_t L = __ldg(p.context_lens + b);
        for (int qt = 0; qt * ppt < n; ++qt) {
            const int npos = min(ppt, n - qt * ppt);
            const int kv_end = min(L, L - n + qt * ppt + npos);
            const int nt = min(kBuckets - 1, (kv_end + kTileN - 1) / kTileN);
            const int pos = atomicAdd(&hist[kBuckets - 1 - nt], 1);
            if (pos < p.max_pairs) p.plan_pairs[pos] = make_int2(b, qt);
        }
    }
    if (tid == 0) p.plan_count[0] = (int32_t)min(total, (long long)p.max_pairs);
}

// ---------------------------------------------------------------------------
// main kernel
// ---------------------------------------------------------------------------

#define NPV_WAIT(bar, parity)                     \
    do {                                          \
        if (!mbar_wait((bar), (parity))) {        \
            *abort_flag = 1;                      \
            goto finish;                          \
        }                                         \
        if (*(volatile int *)abort_flag) goto finish; \
    } while (0)

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_attention_kernel(const Params p, const __grid_constant__ CUtensorMap qmap,
                             const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
    using L = Smem<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 128-byte-swizzled tiles need 1024-byte-aligned shared addresses
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint64_t *q_full = bars + 0;
    uint64_t *q_empty = bars + 1;
    uint64_t *k_full = bars + 2;     // [2]
    uint64_t *v_full = bars + 4;     // [2]
    uint64_t *kv_empty = bars + 6;   // [2]
    uint64_t *s_full = bars + 8;     // [2]
    uint64_t *s_free = bars + 10;    // [2]
    uint64_t *p_full = bars + 12;
    uint64_t *p_empty = bars + 13;
    uint64_t *o_full = bars + 14;
    uint64_t *o_free = bars + 15;
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(bars + 16);
    int *abort_flag = reinterpret_cast<int *>(bars + 17);
    uint8_t *sQ = smem + L::q;
    uint8_t *sK = smem + L::k;
    uint8_t *sV = smem + L::v;
    uint8_t *sP = smem + L::p;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kDBlocks = D / 64;        // 64-element (128-byte) column blocks
    constexpr int kBlockBytes = kTileN * 128;  // one column block of a 128-row tile

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], 4);
        }
        mbar_init(p_full, 4);
        mbar_init(p_empty, 1);
        mbar_init(o_full, 1);
        mbar_init(o_free, 4);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kProducerWarp && lane == 0) {
        tc::prefetch_tensormap(&qmap);
        tc::prefetch_tensormap(&kmap);
        tc::prefetch_tensormap(&vmap);
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(tmem_base_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_base_slot;
    grid_dependency_wait();

    const long long n_items = (long long)p.plan_count[0] * p.num_kv_heads;
    const long long rounds = (n_items + gridDim.x - 1) / gridDim.x;

    if (warp == kProducerWarp) {
        // ============================ TMA producer ============================
        uint32_t q_iter = 0, kv_iter = 0;
        const int BS = p.block_size;
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) continue;
            const Item it = load_item<G>(p, idx);
            const int32_t *bt_row = p.block_tables + (size_t)it.b * p.max_blocks_per_seq;
            int win = -1, win_val = -1;
            NPV_WAIT(q_empty, (q_iter & 1) ^ 1);
            if (lane == 0) {
                mbar_arrive_expect_tx(q_full, (uint32_t)L::kQ);
                for (int db = 0; db < kDBlocks; ++db)
                    tc::tma_load_3d(sQ + db * (kTileM * 128), &qmap, db * 64, it.h * G, it.row0 + it.p0, q_full);
            }
            ++q_iter;
            for (int t = 0; t < it.ntiles; ++t, ++kv_iter) {
                const int s = kv_iter & 1;
                NPV_WAIT(&kv_empty[s], ((kv_iter >> 1) & 1) ^ 1);
                const int kv0 = t * kTileN;
                const int nbox = kTileN / p.box_tokens;
                int blk_of_box[8];
                int nload = 0;
                for (int i = 0; i < nbox; ++i) {
                    const int ks = kv0 + i * p.box_tokens;
                    blk_of_box[i] = -1;
                    if (ks >= it.kv_end) continue;  // warp-uniform
                    const int li = ks / BS;
                    if ((li >> 5) != win) {
                        win = li >> 5;
                        const int e = (win << 5) + lane;
                        win_val = e < p.max_blocks_per_seq ? __ldg(bt_row + e) : -1;
                    }
                    const int blk = __shfl_sync(0xffffffffu, win_val, li & 31);
                    if (blk >= 0 && blk < p.num_blocks) {
                        blk_of_box[i] = blk;
                        ++nload;
                    } else if (lane == 0) {
                        report_error(NPV_DEVERR_BLOCK_ID);
                    }
                }
                if (lane == 0) {
                    const uint32_t bytes = (uint32_t)(nload * p.box_tokens * 128 * kDBlocks);
                    uint8_t *dk = sK + s * L::kKV;
                    uint8_t *dv = sV + s * L::kKV;
                    if (bytes) {
                        mbar_arrive_expect_tx(&k_full[s], bytes);
                        mbar_arrive_expect_tx(&v_full[s], bytes);
                    } else {
                        mbar_arrive(&k_full[s]);
                        mbar_arrive(&v_full[s]);
                    }
                    for (int i = 0; i < nbox; ++i) {
                        if (blk_of_box[i] < 0) continue;
                        const int ks = kv0 + i * p.box_tokens;
                        const int slot_row = blk_of_box[i] * BS + ks % BS;
                        for (int db = 0; db < kDBlocks; ++db) {
                            const int off = db * kBlockBytes + i * p.box_tokens * 128;
                            tc::tma_load_3d(dk + off, &kmap, db * 64, it.h, slot_row, &k_full[s]);
                            tc::tma_load_3d(dv + off, &vmap, db * 64, it.h, slot_row, &v_full[s]);
                        }
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================ MMA issuer ============================
        constexpr uint32_t idesc_s = tc::idesc_bf16_f32(kTileM, kTileN, 0, 0);
        constexpr uint32_t idesc_o = tc::idesc_bf16_f32(kTileM, D, 0, 1);
        const uint32_t q_addr = smem_addr(sQ), k_addr = smem_addr(sK), v_addr = smem_addr(sV),
                       p_addr = smem_addr(sP);
        uint32_t q_iter = 0, kv_iter = 0, item_iter = 0;
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) continue;
            const Item it = load_item<G>(p, idx);
            NPV_WAIT(q_full, q_iter & 1);
            ++q_iter;
            tc::fence_after_sync();
            for (int t = 0; t <= it.ntiles; ++t) {
                if (t < it.ntiles) {
                    // ---- S[t % 2] = Q K_t^T
                    const uint32_t T = kv_iter + t;
                    const int s = T & 1;
                    NPV_WAIT(&k_full[s], (T >> 1) & 1);
                    NPV_WAIT(&s_free[s], ((T >> 1) & 1) ^ 1);
                    tc::fence_after_sync();
                    if (lane == 0) {
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t off = (k >> 2) * kBlockBytes + (k & 3) * 32;
                            tc::mma_bf16_ss(tmem + s * kTileN, tc::smem_desc_sw128(q_addr + off, 16, 1024),
                                            tc::smem_desc_sw128(k_addr + s * L::kKV + off, 16, 1024), idesc_s,
                                            k > 0);
                        }
                        tc::mma_commit(&s_full[s]);
                        if (t == it.ntiles - 1) tc::mma_commit(q_empty);
                    }
                    __syncwarp();
                }
                if (t > 0) {
                    // ---- O (+)= P_{t-1} V_{t-1}
                    const int tp = t - 1;
                    const uint32_t T = kv_iter + tp;
                    const int s = T & 1;
                    NPV_WAIT(p_full, T & 1);
                    NPV_WAIT(&v_full[s], (T >> 1) & 1);
                    if (tp == 0) NPV_WAIT(o_free, (item_iter & 1) ^ 1);
                    const int valid = min(kTileN, it.kv_end - tp * kTileN);
                    const int ksteps = (valid + 15) / 16;
                    if (valid < ksteps * 16) {
                        // zero the V rows of the last K step that lie past the context
                        uint8_t *vs = sV + s * L::kKV;
                        const int nrows = ksteps * 16 - valid;
                        for (int e = lane; e < nrows * 8 * kDBlocks; e += 32) {
                            const int db = e / (nrows * 8);
                            const int rr = valid + (e % (nrows * 8)) / 8;
                            const int ch = e % 8;
                            *reinterpret_cast<uint4 *>(vs + db * kBlockBytes + rr * 128 + ch * 16) =
                                make_uint4(0, 0, 0, 0);
                        }
                        tc::fence_proxy_async_smem();
                        __syncwarp();
                    }
                    tc::fence_after_sync();
                    if (lane == 0) {
                        for (int k = 0; k < ksteps; ++k) {
                            const uint32_t poff = (k >> 2) * (kTileM * 128) + (k & 3) * 32;
                            const uint32_t voff = k * 16 * 128;
                            tc::mma_bf16_ss(tmem + 2 * kTileN, tc::smem_desc_sw128(p_addr + poff, 16, 1024),
                                            tc::smem_desc_sw128(v_addr + s * L::kKV + voff, kBlockBytes, 1024),
                                            idesc_o, tp > 0 || k > 0);
                        }
                        tc::mma_commit(&kv_empty[s]);
                        tc::mma_commit(p_empty);
                        if (tp == it.ntiles - 1) tc::mma_commit(o_full);
                    }
                    __syncwarp();
                }
            }
            kv_iter += it.ntiles;
            ++item_iter;
        }
    } else {
        // ============================ softmax (warps 0-3) ============================
        const int row = warp * 32 + lane;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        uint32_t kv_iter = 0, item_iter = 0;
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) continue;
            const Item it = load_item<G>(p, idx);
            const int pos = row / G, jh = row % G;
            const bool valid_row = pos < it.npos;
            const int lim = valid_row ? (it.L - it.n + it.p0 + pos) : (it.L - 1);
            const int lim_min = it.L - it.n + it.p0;  // smallest limit among the tile's rows
            float m = -INFINITY, l = 0.f;
            for (int t = 0; t < it.ntiles; ++t) {
                const uint32_t T = kv_iter + t;
                const int sb = T & 1;
                NPV_WAIT(&s_full[sb], (T >> 1) & 1);
                tc::fence_after_sync();
                float sv[kTileN];
                {
                    uint32_t raw[32];
#pragma unroll
                    for (int c = 0; c < kTileN / 32; ++c) {
                        tc::tmem_ld32(tmem + lane_off + sb * kTileN + c * 32, raw);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(raw[e]);
                    }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[sb]);
                const int kv0 = t * kTileN;
                if (kv0 + kTileN - 1 > lim_min) {
#pragma unroll
                    for (int c = 0; c < kTileN; ++c)
                        if (kv0 + c > lim) sv[c] = -INFINITY;
                }
                float mx = sv[0];
#pragma unroll
                for (int c = 1; c < kTileN; ++c) mx = fmaxf(mx, sv[c]);
                const float m_tile = mx * p.scale_log2;
                if (t == 0) {
                    m = m_tile;
                } else {
                    const float m_new = fmaxf(m, m_tile);
                    const bool need = m_new > m + kRescaleThreshold;
                    if (__any_sync(0xffffffffu, need)) {
                        // the previous P.V must have landed before O is rescaled
                        NPV_WAIT(p_empty, (T - 1) & 1);
                        tc::fence_after_sync();
                        const float alpha = need ? fast_exp2(m - m_new) : 1.0f;
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t raw[32];
                            const uint32_t ta = tmem + lane_off + 2 * kTileN + c * 32;
                            tc::tmem_ld32(ta, raw);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
                            tc::tmem_st32(ta, raw);
                        }
                        tc::tmem_wait_st();
                        if (need) {
                            l *= alpha;
                            m = m_new;
                        }
                    }
                }
                // probabilities, packed to bf16 pairs
                uint32_t pk[kTileN / 2];
                float lsum = 0.f;
#pragma unroll
                for (int c = 0; c < kTileN; c += 2) {
                    const float p0v = fast_exp2(fmaf(sv[c], p.scale_log2, -m));
                    const float p1v = fast_exp2(fmaf(sv[c + 1], p.scale_log2, -m));
                    lsum += p0v + p1v;
                    pk[c / 2] = pack_bf16x2(p0v, p1v);
                }
                l += lsum;
                if (T > 0) NPV_WAIT(p_empty, (T - 1) & 1);  // P buffer free again
                // row `row` of P, K-major with the 128-byte swizzle: 16-byte chunk c of
                // a 128-byte row lands at chunk c ^ (row % 8)
                {
                    uint8_t *prow = sP + row * 128;
#pragma unroll
                    for (int c = 0; c < kTileN / 8; ++c) {
                        const int kb = c >> 3, ch = c & 7;
                        uint4 v4 = make_uint4(pk[c * 4 + 0], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
                        *reinterpret_cast<uint4 *>(prow + kb * (kTileM * 128) + ((ch ^ (row & 7)) * 16)) = v4;
                    }
                }
                tc::fence_proxy_async_smem();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full);
            }
            // ---- epilogue: O / l -> bf16
            NPV_WAIT(o_full, item_iter & 1);
            tc::fence_after_sync();
            {
                const float inv = 1.0f / l;
                uint16_t *orow = p.out + ((int64_t)(it.row0 + it.p0 + pos) * p.num_q_heads + it.h * G + jh) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t raw[32];
                    tc::tmem_ld32(tmem + lane_off + 2 * kTileN + c * 32, raw);
                    tc::tmem_wait_ld();
                    if (valid_row) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(raw[v * 8 + e]) * inv;
                            st_global_v4(orow + c * 32 + v * 8, pack8(f));
                        }
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
            kv_iter += it.ntiles;
            ++item_iter;
        }
    }
finish:
    tc::fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

#undef NPV_WAIT

}  // namespace prefill
}  // namespace npv
