// Chunked-prefill varlen causal attention over the paged cache on the tcgen05
// tensor cores.
//
// What it computes ("nano-vllm" README, Features: Chunked Prefill and Prefix
// Caching, Tutorial Mode chapter 3 on the causal mask; "Nano-vLLM Architecture
// and Performance", Key Features 1): for sequence b with n_b new rows that
// are already stored at positions L_b - n_b .. L_b - 1, row i attends to keys
// 0 .. L_b - n_b + i of the sequence's paged K/V, query head h reading KV head
// h / g, scale 1/sqrt(D) by default.  This kernel takes the sequences with
// more query rows than the split-KV decode kernel's tile holds (n_b > 16 / g,
// or 8 / g when the call's bound on n_b allows the lighter decode variant);
// shorter ones (decode rows, speculative-decode verification) go to the
// decode kernel in the same call.
//
// How (B200 design):
//   * Q tiles: 128 MMA rows pack 128/g positions x the g query heads of one
//     GQA group, so every K/V tile loaded feeds all g heads (row r = position *
//     g + head).  A work item is (sequence, KV head, pair of consecutive Q
//     tiles A and B): both Q tiles share every K/V tile the CTA loads, which
//     halves the K/V traffic from L2 against one Q tile per item.
//   * A one-CTA plan kernel lists the (sequence, pair) entries: sequences
//     counting-sorted by KV length, longest first, each sequence's pairs
//     contiguous (so the items that read the same K/V run at the same time and
//     share it through L2).  The persistent main kernel (one CTA per SM) takes
//     items (entry, KV head) from that list in snake order.
//   * Warp roles: warp 0 owns tensor memory and issues tcgen05.mma from one
//     thread; warp 1 issues the TMA loads of the K tiles (128 keys) through a
//     2-stage ring, warp 2 those of the V tiles through a 3-stage ring (block
//     ids from the block table a 32-entry window at a time, one TMA box per
//     block piece); warp 3 loads each item's two Q tiles.  Softmax warpgroup j
//     (warps 4-7 for A, 8-11 for B) owns Q tile j: its S buffer, running (max,
//     sum) and O accumulator, and writes its tile's output rows.  The first
//     warpgroup gives registers to the softmax warpgroups (setmaxnreg) so that
//     a softmax thread holds a whole 128-key row of S.
//   * Per KV tile t the MMA thread issues O_A += P_A(t) V_t, S_A(t+1), O_B +=
//     P_B(t) V_t, S_B(t+1): while softmax warpgroup A works on its tile the
//     tensor pipe runs B's products, and the other way round.
//   * Measured on B200: one tcgen05.mma M128 x N128 x K16 runs 64 cycles, but
//     the issuing thread, on a sub-partition shared with two busy softmax
//     warps, spends ~120 cycles per MMA instruction (traced in this kernel):
//     the single issuer paces the kernel, not the loads, the barrier hops
//     (~110 cycles), the tensor pipe or `ex2`.  One issuer per Q tile was
//     slower: the two tiles' products interleave in the tensor pipe and the
//     softmax warpgroups stop alternating with them.
//   * Operands: S = Q K^T reads Q and K from shared memory (K-major, 128-byte
//     swizzle); P V reads P from tensor memory, where the softmax writes it as
//     bf16 pairs over the first 64 columns of its own S buffer, and V from
//     shared memory (MN-major).  Tensor memory (512 columns): S_A, S_B (128
//     fp32 columns each), O_A, O_B (D columns each, at 256 and 384).
//   * The softmax keeps a per-row running max in the log2 domain and rescales
//     its O accumulator only when the max grows by more than 2^8 (otherwise the
//     stale max is kept; the final division by the row sum corrects it exactly
//     in real arithmetic).  V rows past the context of the last tile are zeroed
//     before the P.V product so unwritten cache slots never meet it; rows of a
//     tile past its positions attend like its first row and are not stored.
#pragma once

#include "npv_device.cuh"
#include "npv_tcgen05.cuh"

namespace npv {
namespace prefill {

constexpr int kTileM = 128;   // query rows per Q tile (MMA M); an item holds two Q tiles
constexpr int kTileN = 128;   // keys per KV tile (MMA N of S, K of P.V)
constexpr int kKStages = 2;   // K ring depth (a K stage is free once both S = Q K^T products are done)
constexpr int kVStages = 3;   // V ring depth (a V stage is free once both O += P V products are done)
constexpr int kThreads = 384;  // MMA, K producer, V producer, Q producer, 2 softmax warpgroups
constexpr int kMmaWarp = 0;
constexpr int kKProducerWarp = 1;
constexpr int kVProducerWarp = 2;
constexpr int kQProducerWarp = 3;
constexpr int kFirstSoftmaxWarp = 4;
constexpr int kSoftmaxWarps = 8;
constexpr int kTmemCols = 512;
constexpr int kTmemO = 2 * kTileN;  // S_A, S_B at [0, 256); O_A at [256, 256 + D), O_B at [384, 384 + D)
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
    int32_t *plan_count;  // [1]: number of (sequence, pair of Q tiles) entries
    int2 *plan_pairs;     // [max_pairs]: (sequence, index of the pair of Q tiles), longest first
    int32_t max_pairs;
    int32_t decode_rows_max;  // sequences with at most this many query rows run on the decode kernel
};

// Shared-memory layout (bytes from a 1024-aligned base): barriers, then the two
// Q tiles of an item and the K and V rings (2 x 32 + 2 + 3 stages of 32 KB at
// D = 128: 225 KB in all).
template <int D>
struct Smem {
    static constexpr int kHeader = 1024;
    static constexpr int kKV = kTileN * D * 2;
    static constexpr int kQ = kTileM * D * 2;
    static constexpr int q = kHeader;
    static constexpr int k = q + 2 * kQ;
    static constexpr int v = k + kKStages * kKV;
    static constexpr int total = v + kVStages * kKV;
};

// Per-item quantities every warp role derives the same way.  An item is a
// (sequence, KV head, pair of Q tiles): Q tile A holds positions p0 .. p0 + ppt - 1,
// Q tile B the next ppt positions (ppt = 128 / g positions x g heads = 128 MMA
// rows each); both read the same K/V tiles, loaded once.
struct Item {
    int32_t b, qt, h;
    int32_t row0;    // first packed query row of the sequence
    int32_t n;       // query rows of the sequence
    int32_t L;       // context length (new rows included)
    int32_t p0;      // first position of Q tile A (relative to the new rows)
    int32_t npos_a;  // positions in Q tile A
    int32_t npos_b;  // positions in Q tile B (0 .. ppt)
    int32_t kv_end;  // keys the item needs: [0, kv_end)
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
    it.p0 = it.qt * 2 * ppt;
    it.npos_a = min(ppt, it.n - it.p0);
    it.npos_b = max(0, min(ppt, it.n - it.p0 - ppt));
    it.kv_end = min(it.L, it.L - it.n + it.p0 + it.npos_a + it.npos_b);
    it.ntiles = (it.kv_end + kTileN - 1) / kTileN;
    return it;
}

// Item index of round r for this CTA (snake order over the sorted list).
__device__ __forceinline__ long long item_index(long long r) {
    const long long G = gridDim.x;
    return r * G + ((r & 1) ? (G - 1 - blockIdx.x) : blockIdx.x);
}

// A sequence runs on this kernel when it has more query rows than the decode
// kernel's warp-level tile takes (n_b > decode_rows_max: 16 / g or 8 / g).
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
    if (n <= p.decode_rows_max) return false;
    const int32_t L = __ldg(p.context_lens + b);
    if (L < n || (long long)L > (long long)p.max_blocks_per_seq * p.block_size) {
        *bad = true;
        return false;
    }
    return true;
}

// ---------------------------------------------------------------------------
// plan: list the (sequence, pair of Q tiles) items, longest KV range first
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(1024) prefill_plan_kernel(const Params p, int head_dim) {
    __shared__ int hist[kBuckets];
    __shared__ long long scratch[40];
    grid_dependency_wait();
    constexpr int ppt = 2 * (kTileM / G);  // positions per item (two Q tiles)
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
    // 128-key tiles); each sequence's pairs of Q tiles stay contiguous, last first,
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
    if (tid == 0) {
        // cu_seqlens_q must run from 0 to total_q; a list of entries longer than
        // the plan can hold means ranges overlap (some entry decreased).  Either
        // way the call's rows are not a partition of q: report it.  The plan is
        // clamped, so no access leaves the workspace.
        if (__ldg(p.cu_seqlens_q) != 0 || __ldg(p.cu_seqlens_q + p.num_seqs) != p.total_q ||
            total > (long long)p.max_pairs)
            report_error(NPV_DEVERR_QUERY_LENS);
        p.plan_count[0] = (int32_t)min(total, (long long)p.max_pairs);
    }
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

// Wait for the phase of `bar` with parity `parity`.  The fast path is a
// single try_wait; the slow path also watches the CTA's abort flag (set by a
// warp that gave up) and the time limit.  The outcome is made warp-uniform.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    bool ok = mbar_try_wait(bar, parity);
    if (!ok) {
        const uint64_t t0 = global_timer_ns();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(bar, parity)) {
                ok = true;
                break;
            }
            if ((it & 15u) == 0) {
                if (*abort_flag) break;
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                    report_error(NPV_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}

// A wait that gives up leaves the warp's loops for `label`, where the warp
// first settles what it has in flight, then meets the others at `finish`.
#define NPV_WAIT_OR(bar, parity, label)                               \
    do {                                                              \
        if (!wait_or_abort((bar), (parity), abort_flag)) goto label; \
    } while (0)
#define NPV_WAIT(bar, parity) NPV_WAIT_OR(bar, parity, finish)

__device__ __forceinline__ void setmaxnreg_dec56() { asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory"); }
__device__ __forceinline__ void setmaxnreg_inc224() { asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory"); }

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_attention_kernel(const Params p, const __grid_constant__ CUtensorMap qmap,
                             const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
    using L = Smem<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 128-byte-swizzled tiles need 1024-byte-aligned shared addresses
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
    uint64_t *q_full = bars + 0;   // both Q tiles landed (TMA)
    uint64_t *q_empty = bars + 1;  // the item's last S products are done
    uint64_t *k_full = bars + 2;   // [kKStages]
    uint64_t *k_empty = k_full + kKStages;
    uint64_t *v_full = k_empty + kKStages;  // [kVStages]
    uint64_t *v_empty = v_full + kVStages;
    uint64_t *s_full = v_empty + kVStages;  // [2]: S of Q tile j (A = 0, B = 1) is ready
    uint64_t *p_full = s_full + 2;          // [2]: P of Q tile j written over its S (4 warps)
    uint64_t *o_full = p_full + 2;          // [2]: the item's last P.V product of Q tile j is done
    uint64_t *o_free = o_full + 2;          // both O accumulators read out (8 softmax warps)
    uint64_t *mma_drain = o_free + 1;       // every tcgen05.mma issued so far is done (exit path)
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(mma_drain + 1);
    int *abort_flag = reinterpret_cast<int *>(mma_drain + 2);
    uint8_t *sQ = smem + L::q;
    uint8_t *sK = smem + L::k;
    uint8_t *sV = smem + L::v;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kDBlocks = D / 64;           // 64-element (128-byte) column blocks
    constexpr int kBlockBytes = kTileN * 128;  // one column block of a 128-row Q, K or V tile
    constexpr int ppt = kTileM / G;            // positions per Q tile

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            mbar_init(&s_full[j], 1);
            mbar_init(&p_full[j], kSoftmaxWarps / 2);
            mbar_init(&o_full[j], 1);
        }
        mbar_init(o_free, kSoftmaxWarps);
        mbar_init(mma_drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kQProducerWarp && lane == 0) {
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

    if (warp == kQProducerWarp) {
        // ============================ Q tiles (TMA) ============================
        setmaxnreg_dec56();
        uint32_t item_iter = 0;
        bool q_filled = false;  // the last Q tiles' copy, waited for before the CTA ends
        uint32_t q_parity = 0;
        for (long long r = 0; r < rounds; ++r, ++item_iter) {
            const long long idx = item_index(r);
            if (idx >= n_items) break;
            const Item it = load_item<G>(p, idx);
            NPV_WAIT_OR(q_empty, (item_iter & 1) ^ 1, q_exit);  // the previous item's S products are done
            q_filled = true;
            q_parity = item_iter & 1;
            if (lane == 0) {
                mbar_arrive_expect_tx(q_full, (uint32_t)(2 * kTileM * D * 2));
                // rows (position, head) of each tile: box {64 elements, G heads, 128 / G positions};
                // tile B's rows past the last query row read the map's zero fill
                for (int j = 0; j < 2; ++j)
                    for (int db = 0; db < kDBlocks; ++db)
                        tc::tma_load_3d(sQ + j * L::kQ + db * kBlockBytes, &qmap, db * 64, it.h * G,
                                        it.row0 + it.p0 + j * ppt, q_full);
            }
            __syncwarp();
        }
    q_exit:
        // the shared memory of a CTA must outlive every copy into it, also when a
        // wait gave up and the loop was left early (bounded: a copy always lands)
        if (q_filled) mbar_wait(q_full, q_parity);
    } else if (warp == kKProducerWarp || warp == kVProducerWarp) {
        // ============================ K / V tiles (TMA) ============================
        setmaxnreg_dec56();
        const bool is_k = warp == kKProducerWarp;
        const int nstages = is_k ? kKStages : kVStages;
        uint64_t *full = is_k ? k_full : v_full;
        uint64_t *empty = is_k ? k_empty : v_empty;
        uint8_t *ring = is_k ? sK : sV;
        const CUtensorMap *map = is_k ? &kmap : &vmap;
        uint32_t kv_iter = 0;
        const int BS = p.block_size;
        uint32_t filled = 0, filled_parity = 0;  // per stage: ever filled, parity of its last fill
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) break;
            const Item it = load_item<G>(p, idx);
            const int32_t *bt_row = p.block_tables + (size_t)it.b * p.max_blocks_per_seq;
            int win = -1, win_val = -1;
            for (int t = 0; t < it.ntiles; ++t, ++kv_iter) {
                const int s = (int)(kv_iter % nstages);
                NPV_WAIT_OR(&empty[s], ((kv_iter / nstages) & 1) ^ 1, kv_exit);
                int blk_of_box[8];
                const int nload = tile_boxes(p, it, bt_row, t, lane, win, win_val, blk_of_box);
                filled |= 1u << s;
                filled_parity = (filled_parity & ~(1u << s)) | (((kv_iter / nstages) & 1u) << s);
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
    kv_exit:
        for (int st = 0; st < nstages; ++st)
            if (filled & (1u << st)) mbar_wait(&full[st], (filled_parity >> st) & 1u);
    } else if (warp == kMmaWarp) {
        // ============================ MMA issuer ============================
        setmaxnreg_dec56();
        // Per KV tile t of an item, in this order: PV_A(t), S_A(t+1), PV_B(t),
        // S_B(t+1).  S_j(t+1) overwrites the columns P_j(t) occupies, which
        // PV_j(t), issued before it by this thread, reads (tcgen05.mma ops of one
        // thread run in order).  While softmax warpgroup A works on tile t the
        // tensor pipe runs B's products, and the other way round.
        constexpr uint32_t idesc_s = tc::idesc_bf16_f32(kTileM, kTileN, 0, 0);
        constexpr uint32_t idesc_o = tc::idesc_bf16_f32(kTileM, D, 0, 1);
        const uint64_t qdesc = tc::smem_desc_sw128(smem_addr(sQ), 16, 1024);
        const uint64_t kdesc = tc::smem_desc_sw128(smem_addr(sK), 16, 1024);
        const uint64_t vdesc = tc::smem_desc_sw128(smem_addr(sV), kBlockBytes, 1024);
        uint32_t kv_iter = 0, item_iter = 0;
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) break;
            const Item it = load_item<G>(p, idx);
            NPV_WAIT_OR(q_full, item_iter & 1, mma_exit);
            for (int t = -1; t < it.ntiles; ++t) {
                const int tn = t + 1;  // the tile whose S products follow
                const uint32_t Tn = kv_iter + tn;
                const int ks = (int)(Tn % kKStages);
                for (int j = 0; j < 2; ++j) {
                    if (t >= 0) {
                        // ---- O_j (+)= P_j(t) V_t (P from tensor memory, over S_j)
                        const uint32_t T = kv_iter + t;
                        const int vs = (int)(T % kVStages);
                        NPV_WAIT_OR(&p_full[j], T & 1, mma_exit);
                        if (j == 0) {
                            NPV_WAIT_OR(&v_full[vs], (T / kVStages) & 1, mma_exit);
                            if (t == 0) NPV_WAIT_OR(o_free, (item_iter & 1) ^ 1, mma_exit);
                        }
                        const int valid = min(kTileN, it.kv_end - t * kTileN);
                        const int ksteps = (valid + 15) / 16;
                        if (j == 0 && valid < ksteps * 16) {
                            // zero the V rows of the last K step that lie past the context
                            uint8_t *vsm = sV + vs * L::kKV;
                            const int nrows = ksteps * 16 - valid;
                            for (int e = lane; e < nrows * 8 * kDBlocks; e += 32) {
                                const int db = e / (nrows * 8);
                                const int rr = valid + (e % (nrows * 8)) / 8;
                                const int ch = e % 8;
                                *reinterpret_cast<uint4 *>(vsm + db * kBlockBytes + rr * 128 + ch * 16) =
                                    make_uint4(0, 0, 0, 0);
                            }
                            tc::fence_proxy_async_smem();
                            __syncwarp();
                        }
                        tc::fence_after_sync();
                        if (lane == 0) {
                            const uint32_t d = tmem + kTmemO + j * 128;
                            const uint32_t a = tmem + j * kTileN;
                            const uint64_t vd = vdesc + (uint64_t)((vs * L::kKV) >> 4);
#pragma unroll
                            for (int k = 0; k < kTileN / 16; ++k)
                                if (k < ksteps)
                                    tc::mma_bf16_ts(d, a + k * 8, vd + (uint64_t)(k * 128), idesc_o, t > 0 || k > 0);
                            if (j == 1) tc::mma_commit(&v_empty[vs]);
                            if (t == it.ntiles - 1) tc::mma_commit(&o_full[j]);
                        }
                        __syncwarp();
                    }
                    if (tn < it.ntiles) {
                        // ---- S_j(tn) = Q_j K_tn^T into S_j's columns
                        if (j == 0) NPV_WAIT_OR(&k_full[ks], (Tn / kKStages) & 1, mma_exit);
                        tc::fence_after_sync();
                        if (lane == 0) {
                            const uint32_t d = tmem + j * kTileN;
                            const uint64_t qd = qdesc + (uint64_t)((j * L::kQ) >> 4);
                            const uint64_t kd = kdesc + (uint64_t)((ks * L::kKV) >> 4);
#pragma unroll
                            for (int k = 0; k < D / 16; ++k) {
                                const uint64_t off = (uint64_t)(((k >> 2) * kBlockBytes + (k & 3) * 32) >> 4);
                                tc::mma_bf16_ss(d, qd + off, kd + off, idesc_s, k > 0);
                            }
                            tc::mma_commit(&s_full[j]);
                            if (j == 1) {
                                tc::mma_commit(&k_empty[ks]);
                                if (tn == it.ntiles - 1) tc::mma_commit(q_empty);
                            }
                        }
                        __syncwarp();
                    }
                }
            }
            kv_iter += it.ntiles;
            ++item_iter;
        }
    mma_exit:
        // tensor-core operations still reading shared memory or writing tensor memory
        if (lane == 0) {
            tc::mma_commit(mma_drain);
            mbar_wait(mma_drain, 0);
        }
        __syncwarp();
    } else if (warp >= kFirstSoftmaxWarp) {
        // ==== softmax: warpgroup j (warps 4 + 4 j .. 7 + 4 j) owns Q tile j of every item ====
        // Registers: the launch gives every thread 168; the first warpgroup (MMA,
        // producers) drops to 56 so that a softmax thread can hold a whole
        // 128-key S row: 128 x 56 + 256 x 224 = 384 x 168.
        setmaxnreg_inc224();
        const int j = (warp - kFirstSoftmaxWarp) >> 2;
        const int row = (warp & 3) * 32 + lane;  // warp % 4 selects the TMEM lane quarter
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_cols = tmem + lane_off + j * kTileN;   // S_j, then P_j over its first 64 columns
        const uint32_t o_cols = tmem + lane_off + kTmemO + j * 128;
        const float sl2 = p.scale_log2;
        uint32_t kv_iter = 0, item_iter = 0;
        for (long long r = 0; r < rounds; ++r) {
            const long long idx = item_index(r);
            if (idx >= n_items) break;
            const Item it = load_item<G>(p, idx);
            const int pos = row / G, jh = row % G;
            const int p0 = it.p0 + j * ppt;  // first position of this Q tile
            const int npos = j == 0 ? it.npos_a : it.npos_b;
            const bool valid_row = pos < npos;
            // rows past the tile's positions attend like its first row (their output is
            // dropped); no row's keys reach past the item's last key
            const int lim_min = min(it.L - it.n + p0, it.kv_end - 1);
            const int lim = min(valid_row ? (it.L - it.n + p0 + pos) : lim_min, it.kv_end - 1);
            float m = -INFINITY, l = 0.f;
            for (int t = 0; t < it.ntiles; ++t) {
                const uint32_t T = kv_iter + t;
                NPV_WAIT(&s_full[j], T & 1);
                tc::fence_after_sync();
                float sv[kTileN];
                {
                    uint32_t raw[kTileN / 32][32];
#pragma unroll
                    for (int c = 0; c < kTileN / 32; ++c) tc::tmem_ld32(s_cols + c * 32, raw[c]);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < kTileN / 32; ++c)
#pragma unroll
                        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(raw[c][e]);
                }
                const int kv0 = t * kTileN;
                if (kv0 + kTileN - 1 > lim_min) {
#pragma unroll
                    for (int c = 0; c < kTileN; ++c)
                        if (kv0 + c > lim) sv[c] = -INFINITY;
                }
                float mx8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx8[e] = sv[e];
#pragma unroll
                for (int c = 8; c < kTileN; c += 8)
#pragma unroll
                    for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], sv[c + e]);
                const float m_tile = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                           fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) *
                                     sl2;
                // lazy rescale: the running max moves only when it grows by more than
                // 2^kRescaleThreshold; O_j is then rescaled after P is written
                float alpha = 1.0f;
                bool rescale = false;
                if (t == 0) {
                    m = m_tile;
                } else {
                    const float m_new = fmaxf(m, m_tile);
                    const bool need = m_new > m + kRescaleThreshold;
                    rescale = __any_sync(0xffffffffu, need);
                    if (need) {
                        alpha = fast_exp2(m - m_new);
                        l *= alpha;
                        m = m_new;
                    }
                }
                // a row with every key so far masked keeps m = -inf: its probabilities are 0
                const float m_use = (m == -INFINITY) ? 0.f : m;
                float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < kTileN; ++c) {
                    sv[c] = fast_exp2(fmaf(sv[c], sl2, -m_use));  // in place: S -> P
                    ls8[c & 7] += sv[c];
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(sv[h * 64 + 2 * c], sv[h * 64 + 2 * c + 1]);
                    tc::tmem_st32(s_cols + h * 32, pk);
                }
                l += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
                if (rescale) {
                    // O_j: its last P.V (PV_j(t-1)) finished before S_j(t), issued after
                    // it, completed; the next one waits for p_full below
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t raw[32];
                        const uint32_t ta = o_cols + c * 32;
                        tc::tmem_ld32(ta, raw);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
                        tc::tmem_st32(ta, raw);
                    }
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[j]);
            }
            // ---- epilogue: O_j / l -> bf16 rows of this Q tile
            NPV_WAIT(&o_full[j], item_iter & 1);
            tc::fence_after_sync();
            {
                const float inv = 1.0f / l;
                uint16_t *orow = p.out + ((int64_t)(it.row0 + p0 + pos) * p.num_q_heads + it.h * G + jh) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r32[32];
                    tc::tmem_ld32(o_cols + c * 32, r32);
                    tc::tmem_wait_ld();
                    if (valid_row) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r32[v * 8 + e]) * inv;
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
#undef NPV_WAIT_OR

}  // namespace prefill
}  // namespace npv
