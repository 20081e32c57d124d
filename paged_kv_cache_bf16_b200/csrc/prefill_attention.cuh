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
//   * A one-CTA plan kernel lists the (sequence, row-tile) pairs: sequences
//     counting-sorted by KV length, longest first, each sequence's tiles
//     contiguous (so the items that read the same K/V run at the same time and
//     share it through L2).  The persistent main kernel (one CTA per SM) takes
//     items (pair, KV head) from that list in snake order.
//   * Operands: an M128 x N128 x K16 tcgen05.mma with both operands in shared
//     memory reads 8 KB per 64 cycles, the whole shared-memory bandwidth of the
//     tensor path, so anything else in shared memory slows the MMAs.  Q and P
//     therefore live in tensor memory (the A operand of both products): Q is
//     written there once per item by the softmax threads straight from global
//     memory, P by the softmax threads after the exponentials.  Shared memory
//     carries only K and V: TMA writes them, the MMAs read them.
//   * Warp roles: warp 8 issues the TMA loads of the K tiles (128 keys) through
//     a 3-stage ring, warp 10 those of the V tiles through a 3-stage ring; block
//     ids come from the block table a 32-entry window at a time, one TMA box per
//     block piece.  A K stage is released as soon as S = Q K^T completes.  Warp 9
//     owns tensor memory and issues tcgen05.mma from one thread.  Two softmax
//     warpgroups (warps 0-3 and 4-7) each take 64 of the 128 key columns of every
//     S tile, one TMEM lane (= one query row) per thread, and exchange per-row
//     partial maxima and sums through shared memory guarded by mbarriers.
//   * Tensor memory (512 columns): S double-buffered (2 x 128 fp32), O (D fp32),
//     Q (D/2 columns of bf16 pairs), P (64 columns of bf16 pairs).  K is read as
//     a K-major 128-byte-swizzled operand, V as MN-major.
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
constexpr int kKStages = 3;   // K ring depth (a K stage is free once S = Q K^T is done)
constexpr int kVStages = 3;   // V ring depth (a V stage is free once O += P V is done)
constexpr int kThreads = 352; // 8 softmax warps, K producer, MMA, V producer
constexpr int kSoftmaxWarps = 8;
constexpr int kKProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;
constexpr int kHalf = kTileN / 2;  // key columns of an S tile per softmax warpgroup
constexpr int kTmemCols = 512;
constexpr int kTmemO = 2 * kTileN;  // O: [256, 256 + D)
constexpr int kTmemQ = 384;         // Q: [384, 384 + D/2), bf16 pairs
constexpr int kTmemP = 448;         // P: [448, 512), bf16 pairs
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
    const uint16_t *q;   // [total_q, Hq, D]
    float scale_log2;
    int32_t *plan_count;  // [1]: number of (sequence, row-tile) pairs
    int2 *plan_pairs;     // [max_pairs]: (sequence, row tile), longest first
    int32_t max_pairs;
};

// Shared-memory layout (bytes from a 1024-aligned base): barriers and the
// softmax warpgroups' exchange slots, then the K and V rings.
template <int D>
struct Smem {
    static constexpr int kHeader = 4096;
    static constexpr int kXmax = 512;    // float [2 parity][2 warpgroups][128 rows]
    static constexpr int kXsum = 2560;   // float [2 warpgroups][128 rows]
    static constexpr int kKV = kTileN * D * 2;
    static constexpr int k = kHeader;
    static constexpr int v = k + kKStages * kKV;
    static constexpr int total = v + kVStages * kKV;
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
    // Sequences are ordered by their KV length, longest first (counting sort on
    // 128-key tiles); each sequence's row tiles stay contiguous, last tile first,
    // so the CTAs reading the same K/V run together and share it through L2.
    for (int b = lo; b < hi; ++b) {
        int32_t n;
        bool bad;
        if (!prefill_seq(p, b, &n, &bad)) continue;
        const int32_t L = __ldg(p.context_lens + b);
        const int nt = min(kBuckets - 1, (L + kTileN - 1) / kTileN);
        atomicAdd(&hist[kBuckets - 1 - nt], (n + ppt - 1) / ppt);
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
        const int nt = min(kBuckets - 1, (L + kTileN - 1) / kTileN);
        const int nqt = (n + ppt - 1) / ppt;
        const int pos = atomicAdd(&hist[kBuckets - 1 - nt], nqt);
        for (int k = 0; k < nqt; ++k)
            if (pos + k < p.max_pairs) p.plan_pairs[pos + k] = make_int2(b, nqt - 1 - k);
    }
    if (tid == 0) p.plan_count[0] = (int32_t)min(total, (long long)p.max_pairs);
}

// ---------------------------------------------------------------------------
// main kernel
// ---------------------------------------------------------------------------

// Block ids of the (up to 8) TMA boxes of KV tile t of an item: box i covers
// keys t*128 + i*box_tokens; boxes past the item's keys or with an invalid
// block id get -1.  Warp-collective (the block-table window lives in lanes).
__device__ __forceinline__ int tile_boxes(const Params &p, const Item &it, const int32_t *bt_row, int t, int lane,
                                          int &win, int &win_val, int (&blk_of_box)[8]) {
    const int BS = p.block_size;
    const int nbox = kTileN / p.box_tokens;
    const int kv0 = t * kTileN;
    int nload = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        blk_of_box[i] = -1;
        if (i >= nbox) continue;
        const int ks = kv0 + i * p.box_tokens;
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
    return nload;
}

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
    prefill_attention_kernel(const Params p, const __grid_constant__ CUtensorMap kmap,
                             const __grid_constant__ CUtensorMap vmap) {
    using L = Smem<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 128-byte-swizzled tiles need 1024-byte-aligned shared addresses
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint64_t *q_full = bars + 0;   // Q of the item is in tensor memory (8 softmax warps)
    uint64_t *q_empty = bars + 1;  // the item's last S product is done
    uint64_t *k_full = bars + 2;   // [kKStages]
    uint64_t *k_empty = bars + 5;  // [kKStages]
    uint64_t *v_full = bars + 8;   // [kVStages]
    uint64_t *v_empty = bars + 11; // [kVStages]
    uint64_t *s_full = bars + 14;  // [2]
    uint64_t *s_free = bars + 16;  // [2]
    uint64_t *p_full = bars + 18;
    uint64_t *p_empty = bars + 19;
    uint64_t *o_full = bars + 20;
    uint64_t *o_free = bars + 21;
    uint64_t *x_full = bars + 22;  // [2]: partial row maxima exchanged, by tile parity
    uint64_t *l_full = bars + 24;  // partial row sums exchanged (once per item)
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(bars + 25);
    int *abort_flag = reinterpret_cast<int *>(bars + 26);
    float *xmax = reinterpret_cast<float *>(smem + L::kXmax);
    float *xsum = reinterpret_cast<float *>(smem + L::kXsum);
    uint8_t *sK = smem + L::k;
    uint8_t *sV = smem + L::v;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kDBlocks = D / 64;            // 64-element (128-byte) column blocks
    constexpr int kBlockBytes = kTileN * 128;   // one column block of a 128-row K or V tile

    if (threadIdx.x == 0) {
        mbar_init(q_full, kSoftmaxWarps);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], kSoftmaxWarps);
            mbar_init(&x_full[s], kSoftmaxWarps);
        }
        mbar_init(p_full, kSoftmaxWarps);
        mbar_init(p_empty, 1);
        mbar_init(o_full, 1);
        mbar_init(o_free, kSoftmaxWarps);
        mbar_init(l_full, kSoftmaxWarps);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kKProducerWarp && lane == 0) {
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

    if (warp == kKProducerWarp || warp == kVProducerWarp) {
        // ============================ TMA producers ============================
        const bool is_k = warp == kKProducerWarp;
        const int nstages = is_k ? kKStages : kVStages;
        uint64_t *full = is_k ? k_full : v_full;
        uint64_t *empty = is_k ? k_empty : v_empty;
        uint8_t *ring = is_k ? sK : sV;
        const CUtensorMap *map = is_k ? &kmap : &vmap;
        uint32_t kv_iter = 0;
        const int BS = p.block_size;
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) continue;
            const Item it = load_item<G>(p, idx);
            const int32_t *bt_row = p.block_tables + (size_t)it.b * p.max_blocks_per_seq;
            int win = -1, win_val = -1;
            for (int t = 0; t < it.ntiles; ++t, ++kv_iter) {
                const int s = (int)(kv_iter % nstages);
                NPV_WAIT(&empty[s], ((kv_iter / nstages) & 1) ^ 1);
                int blk_of_box[8];
                const int nload = tile_boxes(p, it, bt_row, t, lane, win, win_val, blk_of_box);
                if (lane == 0) {
                    const uint32_t bytes = (uint32_t)(nload * p.box_tokens * 128 * kDBlocks);
                    uint8_t *dst = ring + s * L::kKV;
                    if (bytes)
                        mbar_arrive_expect_tx(&full[s], bytes);
                    else
                        mbar_arrive(&full[s]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (blk_of_box[i] < 0) continue;
                        const int ks = t * kTileN + i * p.box_tokens;
                        const int slot_row = blk_of_box[i] * BS + ks % BS;
                        for (int db = 0; db < kDBlocks; ++db)
                            tc::tma_load_3d(dst + db * kBlockBytes + i * p.box_tokens * 128, map, db * 64, it.h,
                                            slot_row, &full[s]);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================ MMA issuer ============================
        constexpr uint32_t idesc_s = tc::idesc_bf16_f32(kTileM, kTileN, 0, 0);
        constexpr uint32_t idesc_o = tc::idesc_bf16_f32(kTileM, D, 0, 1);
        const uint32_t k_addr = smem_addr(sK), v_addr = smem_addr(sV);
        uint32_t kv_iter = 0, item_iter = 0;
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) continue;
            const Item it = load_item<G>(p, idx);
            NPV_WAIT(q_full, item_iter & 1);
            tc::fence_after_sync();
            for (int t = 0; t <= it.ntiles; ++t) {
                if (t < it.ntiles) {
                    // ---- S[t % 2] = Q K_t^T  (Q from tensor memory)
                    const uint32_t T = kv_iter + t;
                    const int s = T & 1;                 // S buffer
                    const int ks = (int)(T % kKStages);  // K stage
                    NPV_WAIT(&k_full[ks], (T / kKStages) & 1);
                    NPV_WAIT(&s_free[s], ((T >> 1) & 1) ^ 1);
                    tc::fence_after_sync();
                    if (lane == 0) {
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t off = (k >> 2) * kBlockBytes + (k & 3) * 32;
                            tc::mma_bf16_ts(tmem + s * kTileN, tmem + kTmemQ + k * 8,
                                            tc::smem_desc_sw128(k_addr + ks * L::kKV + off, 16, 1024), idesc_s,
                                            k > 0);
                        }
                        tc::mma_commit(&s_full[s]);
                        tc::mma_commit(&k_empty[ks]);
                        if (t == it.ntiles - 1) tc::mma_commit(q_empty);
                    }
                    __syncwarp();
                }
                if (t > 0) {
                    // ---- O (+)= P_{t-1} V_{t-1}  (P from tensor memory)
                    const int tp = t - 1;
                    const uint32_t T = kv_iter + tp;
                    const int s = (int)(T % kVStages);  // V stage
                    NPV_WAIT(p_full, T & 1);
                    NPV_WAIT(&v_full[s], (T / kVStages) & 1);
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
                            const uint32_t voff = k * 16 * 128;
                            tc::mma_bf16_ts(tmem + kTmemO, tmem + kTmemP + k * 8,
                                            tc::smem_desc_sw128(v_addr + s * L::kKV + voff, kBlockBytes, 1024),
                                            idesc_o, tp > 0 || k > 0);
                        }
                        tc::mma_commit(&v_empty[s]);
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
        // ======== softmax: warpgroup wg (warps 4 wg .. 4 wg + 3) owns key columns [64 wg, 64 wg + 64) ========
        const int wg = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int kc0 = wg * kHalf;    // first key column of this warpgroup
        const int oc0 = wg * (D / 2);  // first O column (and first Q element) of this warpgroup
        uint32_t kv_iter = 0, item_iter = 0;
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) continue;
            const Item it = load_item<G>(p, idx);
            const int pos = row / G, jh = row % G;
            const bool valid_row = pos < it.npos;
            const int lim = valid_row ? (it.L - it.n + it.p0 + pos) : (it.L - 1);
            const int lim_min = it.L - it.n + it.p0;  // smallest limit among the tile's rows
            {
                // ---- Q row -> tensor memory: this warpgroup's half of the row's D elements
                uint32_t qw[D / 4];
                if (valid_row) {
                    const uint16_t *qrow =
                        p.q + ((int64_t)(it.row0 + it.p0 + pos) * p.num_q_heads + it.h * G + jh) * D + oc0;
#pragma unroll
                    for (int v = 0; v < D / 16; ++v) {
                        const uint4 x = ld_nc_v4(qrow + v * 8);
                        qw[v * 4 + 0] = x.x;
                        qw[v * 4 + 1] = x.y;
                        qw[v * 4 + 2] = x.z;
                        qw[v * 4 + 3] = x.w;
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < D / 4; ++v) qw[v] = 0u;
                }
                NPV_WAIT(q_empty, (item_iter & 1) ^ 1);  // the previous item's S products are done
                tc::fence_after_sync();
                if constexpr (D == 128) {
                    tc::tmem_st32(tmem + lane_off + kTmemQ + wg * 32, qw);
                } else {
                    tc::tmem_st16(tmem + lane_off + kTmemQ + wg * 16, qw);
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(q_full);
            }
            float m = -INFINITY, l = 0.f;
            for (int t = 0; t < it.ntiles; ++t) {
                const uint32_t T = kv_iter + t;
                const int sb = T & 1;
                NPV_WAIT(&s_full[sb], (T >> 1) & 1);
                tc::fence_after_sync();
                float sv[kHalf];
                {
                    uint32_t raw[kHalf / 32][32];
#pragma unroll
                    for (int c = 0; c < kHalf / 32; ++c)
                        tc::tmem_ld32(tmem + lane_off + sb * kTileN + kc0 + c * 32, raw[c]);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < kHalf / 32; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(raw[c][e]);
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[sb]);
                const int kv0 = t * kTileN + kc0;
                if (kv0 + kHalf - 1 > lim_min) {
#pragma unroll
                    for (int c = 0; c < kHalf; ++c)
                        if (kv0 + c > lim) sv[c] = -INFINITY;
                }
                float mx8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx8[e] = sv[e];
#pragma unroll
                for (int c = 8; c < kHalf; c += 8)
#pragma unroll
                    for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], sv[c + e]);
                const float pmax = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
                // full-row max: swap partial maxima with the other warpgroup
                xmax[(sb * 2 + wg) * kTileM + row] = pmax;
                __syncwarp();
                if (lane == 0) mbar_arrive(&x_full[sb]);
                NPV_WAIT(&x_full[sb], (T >> 1) & 1);
                const float omax = xmax[(sb * 2 + (1 - wg)) * kTileM + row];
                const float m_tile = fmaxf(pmax, omax) * p.scale_log2;
                if (t == 0) {
                    m = m_tile;
                } else {
                    const float m_new = fmaxf(m, m_tile);
                    const bool need = m_new > m + kRescaleThreshold;  // the same in both warpgroups
                    if (__any_sync(0xffffffffu, need)) {
                        // the previous P.V must have landed before O is rescaled
                        NPV_WAIT(p_empty, (T - 1) & 1);
                        tc::fence_after_sync();
                        const float alpha = need ? fast_exp2(m - m_new) : 1.0f;
                        // this warpgroup's half of O, 32 columns at a time
#pragma unroll
                        for (int c = 0; c < D / 64; ++c) {
                            uint32_t raw[32];
                            const uint32_t ta = tmem + lane_off + kTmemO + oc0 + c * 32;
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
                // probabilities of this warpgroup's 64 keys, packed to bf16 pairs, into P's
                // columns [32 wg, 32 wg + 32) of tensor memory
                float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                uint32_t pk[kHalf / 2];
#pragma unroll
                for (int c = 0; c < kHalf; c += 2) {
                    const float p0v = fast_exp2(fmaf(sv[c], p.scale_log2, -m));
                    const float p1v = fast_exp2(fmaf(sv[c + 1], p.scale_log2, -m));
                    ls8[(c / 2) & 7] += p0v + p1v;
                    pk[c / 2] = pack_bf16x2(p0v, p1v);
                }
                l += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
                if (T > 0) NPV_WAIT(p_empty, (T - 1) & 1);  // the previous P.V has read P
                tc::fence_after_sync();
                tc::tmem_st32(tmem + lane_off + kTmemP + wg * (kHalf / 2), pk);
                tc::tmem_wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full);
            }
            // ---- epilogue: full row sum from the two partial sums, then O / l -> bf16
            xsum[wg * kTileM + row] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(l_full);
            NPV_WAIT(l_full, item_iter & 1);
            NPV_WAIT(o_full, item_iter & 1);
            tc::fence_after_sync();
            {
                const float lo = xsum[(1 - wg) * kTileM + row];
                uint32_t raw[D / 64][32];
#pragma unroll
                for (int c = 0; c < D / 64; ++c) tc::tmem_ld32(tmem + lane_off + kTmemO + oc0 + c * 32, raw[c]);
                tc::tmem_wait_ld();
                const float inv = 1.0f / (l + lo);
                uint16_t *orow =
                    p.out + ((int64_t)(it.row0 + it.p0 + pos) * p.num_q_heads + it.h * G + jh) * D + oc0;
                if (valid_row) {
#pragma unroll
                    for (int c = 0; c < D / 64; ++c)
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(raw[c][v * 8 + e]) * inv;
                            st_global_v4(orow + c * 32 + v * 8, pack8(f));
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
