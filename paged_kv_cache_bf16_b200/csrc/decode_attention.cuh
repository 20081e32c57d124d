// Paged grouped-query decode attention with split-KV and a merge kernel.
//
// What it computes ("nano-vllm" README, X-Ray Mode; "Nano-vLLM Architecture and
// Performance", Key Features 2 and 4): for every sequence b and query head h,
// softmax(scale * q[b,h] . K_b^T) V_b over the context_lens[b] tokens that
// sequence b's block table points at, with query head h reading KV head
// h / (Hq / Hkv).
//
// How (B200 design):
//   * Work unit = (sequence, group of HC KV heads).  Each unit's tokens are cut
//     into 16-token chunks; a chunk of one KV head group is contiguous in the
//     [num_blocks, block_size, Hkv, D] cache (block_size is a multiple of 16, so
//     a chunk never crosses a block).
//   * A persistent grid of one CTA per SM splits the flattened list of all
//     chunks of all units into equal contiguous ranges (token-balanced split-KV:
//     ragged context lengths cost no imbalance).  A unit wholly inside one CTA's
//     range is finished in that CTA; a unit cut by a range boundary leaves
//     (max, sum, unnormalised output) partials that the merge kernel combines.
//   * Inside a CTA a producer warp streams chunks of K and V with bulk
//     asynchronous copies (TMA engine, untiled) into a ring of shared-memory
//     stages guarded by mbarriers; it looks block ids up in the block table a
//     32-entry window at a time.  HC consumer warps each own one KV head and
//     all g query heads that share it, so every K/V row read from HBM feeds g
//     query heads.
//   * A consumer warp runs both products of a chunk on the warp-level tensor
//     cores (mma.sync m16n8k16, bf16 in, fp32 accumulate), with the chunk's 16
//     tokens as the MMA's M and the query rows sharing the warp's KV head as
//     its N: the g heads of a GQA group times the sequence's n query rows
//     (n = 1 for decode; up to 16 / g for speculative-decode verification or a
//     short chunk), in one or two 8-column tiles, unused columns zero.
//     S^T = K Q^T takes D / 16 MMAs per tile; after the online softmax (log2
//     domain, running max and sum per row) and a bf16 rounding, movmatrix
//     transposes the accumulator into the B operand of O^T += V^T P^T (D / 16
//     MMAs per tile), so P never leaves registers.  Lanes read K and V rows
//     from shared memory with 16-byte loads: the head dimension inside a K
//     fragment follows a fixed permutation shared by Q (the dot product does
//     not depend on it) so the loads are contiguous, and V is transposed into
//     A fragments with byte permutes.  A row's causal limit is L - n + i for
//     its query row i.
#pragma once

#include "npv_device.cuh"

namespace npv {
namespace decode {

constexpr int kChunk = 16;  // tokens per pipeline stage
constexpr int kMaxConsumerWarps = 8;
constexpr int kMaxStages = 8;
constexpr int kStageBudgetBytes = 192 * 1024;
constexpr int kHeaderBytes = 1024;
constexpr int kTileRows = 16;              // most query rows per KV head: two 8-column MMA tiles
constexpr float kRescaleThreshold = 8.0f;  // log2 units a row max may grow before O is rescaled

enum : int32_t { kFlagFirst = 1, kFlagLast = 2, kFlagSkip = 4, kFlagNewToken = 8 };

// Failure-detection test hook (npv_debug_inject_decode_timeout), off unless the
// host sets it: every CTA's producer leaves its first stage unfilled, and the
// consumers wait for a stage at most kDebugWaitNs, so their wait certainly gives
// up, records NPV_DEVERR_TIMEOUT and ends the kernel through its exit path.
__device__ unsigned int g_debug_timeout;
constexpr uint64_t kDebugWaitNs = 1000000ull;

struct StageInfo {
    int32_t unit;     // (sequence, head group) index
    int32_t n_valid;  // live tokens in the chunk (1..16)
    int32_t flags;
    int32_t slot;  // partial slot written at kFlagLast, or -1 for a finished unit
    int32_t tok0;  // position of the chunk's first token in its sequence
};

struct Params {
    uint16_t *out;  // [rows, Hq, D]
    const uint16_t *q;
    int64_t q_row_stride;  // elements between query rows
    const uint16_t *k_cache;
    const uint16_t *v_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *cu_seqlens_q;  // non-null: mixed batch; sequences with 1..max_rows query rows run here
    int32_t total_q;              // rows of q and out in a mixed batch
    int32_t max_rows;             // most query rows of a sequence on this path (1 without cu_seqlens_q)
    int32_t rows_per_head;        // RP: query-row slots per KV head in a partial slot (g * max_rows)
    int32_t sole_path;            // mixed batch served by this kernel alone: a sequence of more than
                                  // max_rows rows, or a malformed range, is reported here
    int32_t max_blocks_per_seq;
    int32_t num_seqs;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t num_blocks;
    int32_t block_size;
    int32_t heads_per_cta;    // HC: KV heads per unit = consumer warps
    int32_t num_head_groups;  // Hkv / HC
    int32_t num_stages;
    float scale_log2;  // softmax scale * log2(e)
    // fused store (decode only): token b's key/value rows go to slot slot_mapping[b]
    // before its sequence's last chunk is read; null when the call stores nothing
    const uint16_t *key;
    const uint16_t *value;
    int64_t key_stride;    // elements between tokens
    int64_t value_stride;
    const int32_t *slot_mapping;
    // workspace
    float2 *part_ml;  // [grid][2][HC][RP]: (running max, sum) of a partial unit's rows
    float *part_o;    // [grid][2][HC][RP][D]: unnormalised output of a partial unit's rows
};

// Query rows of sequence b on this path: 1 in a decode call; in a mixed batch
// n_b when 1 <= n_b <= max_rows, else 0 (no rows, a malformed range, or a
// sequence the prefill kernel serves).
__device__ __forceinline__ int32_t path_rows(const Params &p, int32_t b) {
    if (p.cu_seqlens_q == nullptr) return 1;
    const int32_t cb = __ldg(p.cu_seqlens_q + b), ce = __ldg(p.cu_seqlens_q + b + 1);
    const int32_t n = ce - cb;
    if (cb < 0 || ce > p.total_q || n < 1 || n > p.max_rows) return 0;
    return n;
}

// Chunks of work for sequence b on this path (0 for an empty, invalid or
// foreign sequence; the merge kernel writes those rows or reports them).
__device__ __forceinline__ int32_t seq_chunks(const Params &p, int32_t b) {
    const int32_t n = path_rows(p, b);
    if (n == 0) return 0;
    const int32_t L = __ldg(p.context_lens + b);
    if (L < n || (long long)L > (long long)p.max_blocks_per_seq * p.block_size) return 0;
    return (L + kChunk - 1) / kChunk;
}

__device__ __forceinline__ int64_t query_row(const Params &p, int32_t b) {
    return p.cu_seqlens_q != nullptr ? (int64_t)__ldg(p.cu_seqlens_q + b) : (int64_t)b;
}

// In a mixed batch that this kernel serves alone (the caller's bound on the
// query rows fits its tile), sequence b with no rows on this path is either
// empty, malformed (NPV_DEVERR_QUERY_LENS) or longer than the bound: its rows
// are written as zeros and NPV_DEVERR_QUERY_LENS is reported.
__device__ __forceinline__ void reject_foreign_rows(const Params &p, int32_t b, int head_dim) {
    const int32_t cb = __ldg(p.cu_seqlens_q + b), ce = __ldg(p.cu_seqlens_q + b + 1);
    if (cb < 0 || ce < cb || ce > p.total_q) {
        report_error(NPV_DEVERR_QUERY_LENS);
        return;
    }
    if (ce - cb <= p.max_rows) return;  // empty
    report_error(NPV_DEVERR_QUERY_LENS);
    uint4 *o = reinterpret_cast<uint4 *>(p.out + (int64_t)cb * p.num_q_heads * head_dim);
    const int64_t nvec = (int64_t)(ce - cb) * p.num_q_heads * head_dim / 8;
    for (int64_t i = 0; i < nvec; ++i) o[i] = make_uint4(0, 0, 0, 0);
}

// Exclusive prefix sum over the block; returns the exclusive value and sets *total.
__device__ __forceinline__ long long block_exclusive_scan(long long v, long long *scratch, long long *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
    long long incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long run = 0;
        for (int w = 0; w < nwarps; ++w) {
            const long long t = scratch[w];
            scratch[w] = run;
            run += t;
        }
        scratch[nwarps] = run;
    }
    __syncthreads();
    *total = scratch[nwarps];
    return scratch[warp] + incl - v;
}

// The contiguous range [c0, c1) of the flattened chunk list that CTA blockIdx.x of a
// gridDim.x-CTA grid owns, and the unit holding chunk c0 with its chunk range
// [s_first, e_first).  Every thread of the block must call this.
struct Schedule {
    long long total, c0, c1, u_first, s_first, e_first;
};

__device__ __forceinline__ Schedule compute_schedule(const Params &p, long long *sched, long long *scratch) {
    const int NHG = p.num_head_groups;
    const long long U = (long long)p.num_seqs * NHG;
    const long long per = (U + blockDim.x - 1) / blockDim.x;
    const long long lo = min(U, (long long)threadIdx.x * per);
    const long long hi = min(U, lo + per);
    long long mine = 0;
    for (long long u = lo; u < hi; ++u) mine += seq_chunks(p, (int32_t)(u / NHG));
    Schedule sc;
    const long long excl = block_exclusive_scan(mine, scratch, &sc.total);
    sc.c0 = (long long)blockIdx.x * sc.total / gridDim.x;
    sc.c1 = (long long)(blockIdx.x + 1) * sc.total / gridDim.x;
    if (sc.c0 < sc.c1 && mine > 0 && excl <= sc.c0 && sc.c0 < excl + mine) {
        long long acc = excl;
        for (long long u = lo; u < hi; ++u) {
            const long long n = seq_chunks(p, (int32_t)(u / NHG));
            if (sc.c0 < acc + n) {
                sched[0] = u;
                sched[1] = acc;
                sched[2] = acc + n;
                break;
            }
            acc += n;
        }
    }
    __syncthreads();
    if (sc.c0 < sc.c1) {
        sc.u_first = sched[0];
        sc.s_first = sched[1];
        sc.e_first = sched[2];
    } else {
        sc.u_first = -1;
        sc.s_first = sc.e_first = 0;
    }
    return sc;
}

// Fused store of token b's key/value rows for KV heads [h0, h0 + nh) into slot
// slot_mapping[b] (a negative slot stores nothing), by the threads `lane` of `nthreads`.
__device__ __forceinline__ void store_token_rows(const Params &p, int32_t b, int h0, int nh, int D, int lane,
                                                 int nthreads) {
    const int32_t slot = __ldg(p.slot_mapping + b);
    if (slot < 0) return;
    if ((long long)slot >= (long long)p.num_blocks * p.block_size) {
        if (lane == 0) report_error(NPV_DEVERR_SLOT);
        return;
    }
    const int64_t dst = ((int64_t)slot * p.num_kv_heads + h0) * D;
    const uint16_t *ks = p.key + (int64_t)b * p.key_stride + (int64_t)h0 * D;
    const uint16_t *vs = p.value + (int64_t)b * p.value_stride + (int64_t)h0 * D;
    uint16_t *kc = const_cast<uint16_t *>(p.k_cache) + dst;
    uint16_t *vc = const_cast<uint16_t *>(p.v_cache) + dst;
    for (int v = lane; v < nh * D / 8; v += nthreads) {
        st_global_v4(kc + v * 8, ld_nc_v4(ks + v * 8));
        st_global_v4(vc + v * 8, ld_nc_v4(vs + v * 8));
    }
}

// D[16 x 8] += A[16 x 16] B[16 x 8]: bf16 inputs, fp32 accumulators, one warp.
// Fragments follow the PTX ISA's m16n8k16 layout: lane = 4 * group + t holds
// A rows group and group + 8, columns 2t, 2t + 1 (a0, a1) and 2t + 8, 2t + 9
// (a2, a3); B column group, rows 2t, 2t + 1 (b0) and 2t + 8, 2t + 9 (b1);
// D rows group (d0, d1) and group + 8 (d2, d3), columns 2t, 2t + 1.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void swap_if(uint4 &a, uint4 &b, bool c) {
    const uint4 x = a, y = b;
    a = c ? y : x;
    b = c ? x : y;
}

__device__ __forceinline__ uint32_t word(const uint4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// Transpose of an 8 x 8 matrix of 16-bit elements held one 32-bit pair per lane
// (lane 4 r + c holds row r, columns 2c, 2c + 1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// NR: tiles of 8 query rows per KV head (1: g * n <= 8, as in every decode call;
// 2: up to 16 rows, for the short sequences of a prefill call).
template <int D, int G, int NR>
__global__ void __launch_bounds__((kMaxConsumerWarps + 1) * 32, 1) decode_split_kernel(const Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty_bar = full_bar + kMaxStages;
    StageInfo *info = reinterpret_cast<StageInfo *>(empty_bar + kMaxStages);
    long long *sched = reinterpret_cast<long long *>(info + kMaxStages);  // [0..7]
    long long *scan_scratch = sched + 8;                                  // [kMaxConsumerWarps + 2]

    const int HC = p.heads_per_cta;
    const int NS = p.num_stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_elems = HC * D;  // one token of one head group
    const int stage_elems = kChunk * row_elems;
    uint16_t *stage_k = reinterpret_cast<uint16_t *>(smem + kHeaderBytes);
    uint16_t *stage_v = stage_k + (size_t)NS * stage_elems;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], HC);
        }
        fence_barrier_init();
    }
    grid_dependency_wait();

    // ---- schedule: which contiguous range of the flattened chunk list is ours
    const int NHG = p.num_head_groups;
    const Schedule sc = compute_schedule(p, sched, scan_scratch);
    // the merge kernel may now be scheduled; it waits for this grid before
    // reading any partial
    grid_launch_dependents();
    if (sc.c0 >= sc.c1) return;
    const long long c0 = sc.c0, c1 = sc.c1;
    const long long u_first = sc.u_first;
    const long long s_first = sc.s_first;

    const bool debug_timeout = *reinterpret_cast<volatile unsigned int *>(&g_debug_timeout) != 0;
    if (warp == HC) {
        // ===================== producer warp =====================
        bool drop = debug_timeout;  // leave the first stage unfilled (test hook)
        long long remaining = c1 - c0;
        long long u = u_first;
        long long k = c0 - s_first;
        int stage = 0;
        uint32_t eparity = 1;
        bool first_seg = true;
        uint32_t issued = 0, issued_parity = 0;  // per stage: ever filled, parity of its last fill
        const int Hkv = p.num_kv_heads;
        const int BS = p.block_size;
        bool abort = false;
        while (remaining > 0 && !abort) {
            const int32_t b = (int32_t)(u / NHG);
            const int32_t hg = (int32_t)(u % NHG);
            const int32_t nC = seq_chunks(p, b);
            if (k >= nC) {
                ++u;
                k = 0;
                continue;
            }
            const int32_t L = __ldg(p.context_lens + b);
            const long long seg_len = min((long long)nC - k, remaining);
            const bool complete = (k == 0) && (seg_len == nC);
            const int32_t slot = complete ? -1 : 2 * (int32_t)blockIdx.x + (first_seg ? 0 : 1);
            const int32_t *bt_row = p.block_tables + (size_t)b * p.max_blocks_per_seq;
            int bt_win = -1, bt_val = -1;
            for (long long i = 0; i < seg_len; ++i, ++k) {
                const int32_t t0 = (int32_t)k * kChunk;
                const int32_t n_valid = min(kChunk, L - t0);
                const int32_t li = t0 / BS;
                const int32_t win = li >> 5;
                if (win != bt_win) {
                    const int idx = (win << 5) + lane;
                    bt_val = idx < p.max_blocks_per_seq ? __ldg(bt_row + idx) : -1;
                    bt_win = win;
                }
                const int32_t blk = __shfl_sync(0xffffffffu, bt_val, li & 31);
                const bool valid = blk >= 0 && blk < p.num_blocks;
                if (!mbar_wait(&empty_bar[stage], eparity)) {
                    abort = true;
                    break;
                }
                if (drop) {
                    // test hook: no copy and no arrival, so this stage never fills
                    drop = false;
                    if (++stage == NS) {
                        stage = 0;
                        eparity ^= 1;
                    }
                    continue;
                }
                if (lane == 0) {
                    int32_t flags = (i == 0 ? kFlagFirst : 0) | (i == seg_len - 1 ? kFlagLast : 0);
                    // a fused store: this segment ends with the unit's last chunk, which
                    // holds the new token (the consumers store and substitute it)
                    if (i == 0 && p.key != nullptr && k + seg_len == nC) flags |= kFlagNewToken;
                    if (!valid) {
                        flags |= kFlagSkip;
                        report_error(NPV_DEVERR_BLOCK_ID);
                    }
                    info[stage] = StageInfo{(int32_t)u, n_valid, flags, slot, t0};
                    if (valid)
                        mbar_arrive_expect_tx(&full_bar[stage], (uint32_t)(2 * n_valid * row_elems * 2));
                    else
                        mbar_arrive(&full_bar[stage]);
                }
                __syncwarp();
                if (valid) {
                    const int64_t tok0 = (int64_t)blk * BS + (t0 % BS);
                    uint16_t *dk = stage_k + (size_t)stage * stage_elems;
                    uint16_t *dv = stage_v + (size_t)stage * stage_elems;
                    if (NHG == 1) {
                        if (lane == 0) {
                            const uint32_t bytes = (uint32_t)(n_valid * row_elems * 2);
                            bulk_copy_g2s(dk, p.k_cache + tok0 * row_elems, bytes, &full_bar[stage]);
                            bulk_copy_g2s(dv, p.v_cache + tok0 * row_elems, bytes, &full_bar[stage]);
                        }
                    } else {
                        const int t = lane & 15;
                        if (t < n_valid) {
                            const int64_t src = ((tok0 + t) * Hkv + (int64_t)hg * HC) * D;
                            const uint32_t bytes = (uint32_t)(row_elems * 2);
                            if (lane < 16)
                                bulk_copy_g2s(dk + t * row_elems, p.k_cache + src, bytes, &full_bar[stage]);
                            else
                                bulk_copy_g2s(dv + t * row_elems, p.v_cache + src, bytes, &full_bar[stage]);
                        }
                    }
                }
                issued |= 1u << stage;
                issued_parity = (issued_parity & ~(1u << stage)) | ((eparity ^ 1u) << stage);
                if (++stage == NS) {
                    stage = 0;
                    eparity ^= 1;
                }
            }
            remaining -= seg_len;
            first_seg = false;
            ++u;
            k = 0;
        }
        // never leave with copies in flight into this CTA's shared memory
        for (int st = 0; st < NS; ++st)
            if (issued & (1u << st)) mbar_wait(&full_bar[st], (issued_parity >> st) & 1u);
        return;
    }

    // ===================== consumer warps (one KV head each) =====================
    // Per 16-token chunk, with the chunk's tokens as MMA rows and the query rows
    // as MMA columns (NR tiles of 8):
    //   S^T = K Q^T       (D / 16 k-steps per 8 query rows)
    //   O^T += V^T P^T    (D / 16 tiles of 16 output dims per 8 query rows)
    // The S^T accumulator of lane (group, t) holds query rows 2t, 2t + 1 at
    // tokens group and group + 8; after the softmax, each bf16 pair of it is one
    // lane's share of an 8 x 8 block of P^T, and movmatrix's transpose turns the
    // two blocks into the B fragment of P^T.
    constexpr int KJ = D / 32;   // 16-byte K vectors a lane reads per token row
    constexpr int VH = D / 64;   // 16-byte V vectors a lane reads per token row
    constexpr int MT = D / 16;   // 16-dim tiles of the output
    const int gq = lane >> 2, tq = lane & 3;
    const uint32_t tok_bytes = (uint32_t)(row_elems * 2);
    const uint32_t stage_bytes = (uint32_t)(stage_elems * 2);
    // K fragment: tokens gq and gq + 8, vector j holding dims 32 j + 8 tq .. + 7 (a
    // fixed permutation of the head dim inside each k-step pair, shared by Q).
    // Lanes with odd gq read the two vectors of a pair in the other order, so a
    // quarter-warp's loads hit distinct banks, and swap them back in registers.
    const uint32_t k_lane = smem_addr(stage_k) + (uint32_t)(warp * D * 2) + (uint32_t)gq * tok_bytes + 16u * tq;
    const bool k_odd = KJ > 1 && (gq & 1);
    // V fragment: tokens 2 tq, 2 tq + 1, 2 tq + 8, 2 tq + 9 at dims (D / 8) gq .. + D / 8 - 1;
    // output tile mt's rows gq and gq + 8 are dims (D / 8) gq + mt and + D / 16 + mt.
    const uint32_t v_lane = smem_addr(stage_v) + (uint32_t)(warp * D * 2) + (uint32_t)(2 * tq) * tok_bytes +
                            (uint32_t)(2 * (D / 8) * gq);
    const bool v_odd = VH > 1 && (tq & 1);

    uint4 qf[NR][KJ];  // query row 8 nr + gq, vectors as K's
    float o[NR][MT][4];
    float m_run[NR][2], l_run[NR][2];
    int32_t lim[NR][2];
    int32_t b = 0, hg = 0, R = 0, lim_min = 0;
    int64_t row0 = 0;
    // fused store: this lane's 8-element slices of the new token's K and V rows
    uint4 new_k = make_uint4(0, 0, 0, 0), new_v = make_uint4(0, 0, 0, 0);
    int32_t new_slot = -1;
    int stage = 0;
    uint32_t fparity = 0;
    const float sl2 = p.scale_log2;
    const long long nchunks = c1 - c0;
    const uint64_t wait_ns = debug_timeout ? kDebugWaitNs : kWaitLimitNs;
    for (long long it = 0; it < nchunks; ++it) {
        if (!mbar_wait(&full_bar[stage], fparity, wait_ns)) break;
        const StageInfo inf = info[stage];
        if (inf.flags & kFlagFirst) {
            b = inf.unit / NHG;
            hg = inf.unit % NHG;
            const int32_t n = path_rows(p, b);
            const int32_t L = __ldg(p.context_lens + b);
            R = G * n;
            row0 = query_row(p, b);
            lim_min = L - n;
#pragma unroll
            for (int nr = 0; nr < NR; ++nr) {
                const int r = 8 * nr + gq;
                if (r < R) {
                    const uint16_t *qrow = p.q + (row0 + r / G) * p.q_row_stride +
                                           ((int64_t)(hg * HC + warp) * G + r % G) * D + 8 * tq;
#pragma unroll
                    for (int j = 0; j < KJ; ++j) qf[nr][j] = ld_nc_v4(qrow + 32 * j);
                } else {
#pragma unroll
                    for (int j = 0; j < KJ; ++j) qf[nr][j] = make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    // row i of the sequence sees keys 0 .. L - n + i; rows past R (never
                    // stored) attend like the unit's last row
                    const int rr = 8 * nr + 2 * tq + u;
                    lim[nr][u] = rr < R ? L - n + rr / G : L - 1;
                    m_run[nr][u] = -INFINITY;
                    l_run[nr][u] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < MT; ++i) o[nr][i][0] = o[nr][i][1] = o[nr][i][2] = o[nr][i][3] = 0.f;
            }
            new_slot = -1;
            if (inf.flags & kFlagNewToken) {
                // fetch now; used when the segment's last chunk arrives
                const int32_t slot = __ldg(p.slot_mapping + b);
                if (slot >= 0 && (long long)slot < (long long)p.num_blocks * p.block_size) {
                    new_slot = slot;
                    if (lane < D / 8) {
                        const int64_t h = (int64_t)(hg * HC + warp) * D + lane * 8;
                        new_k = ld_nc_v4(p.key + (int64_t)b * p.key_stride + h);
                        new_v = ld_nc_v4(p.value + (int64_t)b * p.value_stride + h);
                    }
                } else if (slot >= 0 && lane == 0) {
                    report_error(NPV_DEVERR_SLOT);
                }
            }
        }
        if ((inf.flags & kFlagLast) && new_slot >= 0) {
            // the unit's last chunk: put the new token into the stage (its cache
            // slot may not hold it yet) and into the cache
            if (lane < D / 8) {
                const uint32_t off = (uint32_t)((((inf.n_valid - 1) * HC + warp) * D + lane * 8) * 2);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_addr(stage_k) + stage * stage_bytes +
                                                                            off),
                             "r"(new_k.x), "r"(new_k.y), "r"(new_k.z), "r"(new_k.w)
                             : "memory");
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_addr(stage_v) + stage * stage_bytes +
                                                                            off),
                             "r"(new_v.x), "r"(new_v.y), "r"(new_v.z), "r"(new_v.w)
                             : "memory");
                const int64_t dst = ((int64_t)new_slot * p.num_kv_heads + hg * HC + warp) * D + lane * 8;
                st_global_v4(const_cast<uint16_t *>(p.k_cache) + dst, new_k);
                st_global_v4(const_cast<uint16_t *>(p.v_cache) + dst, new_v);
            }
            __syncwarp();
        }
        if (!(inf.flags & kFlagSkip)) {
            const int nr_live = R > 8 ? NR : 1;  // warp-uniform
            // ---- S^T = K Q^T
            const uint32_t ks = k_lane + stage * stage_bytes;
            uint4 kv[2][KJ];
#pragma unroll
            for (int mh = 0; mh < 2; ++mh)
#pragma unroll
                for (int j = 0; j < KJ; ++j)
                    kv[mh][j] = ld_shared_v4(ks + (uint32_t)(mh * 8) * tok_bytes + (uint32_t)((64 * j) ^ (k_odd ? 64 : 0)));
            if (KJ > 1) {
#pragma unroll
                for (int mh = 0; mh < 2; ++mh)
#pragma unroll
                    for (int j = 0; j < KJ; j += 2) swap_if(kv[mh][j], kv[mh][j + 1], k_odd);
            }
            float x[NR][4];
#pragma unroll
            for (int nr = 0; nr < NR; ++nr) {
                x[nr][0] = x[nr][1] = x[nr][2] = x[nr][3] = 0.f;
                if (nr < nr_live) {
                    // vector j, elements 0-3: k-step 2 j; elements 4-7: k-step 2 j + 1
#pragma unroll
                    for (int j = 0; j < KJ; ++j) {
                        mma_16816(x[nr], kv[0][j].x, kv[1][j].x, kv[0][j].y, kv[1][j].y, qf[nr][j].x, qf[nr][j].y);
                        mma_16816(x[nr], kv[0][j].z, kv[1][j].z, kv[0][j].w, kv[1][j].w, qf[nr][j].z, qf[nr][j].w);
                    }
                }
            }
            // ---- online softmax (log2 domain) per query row; x[nr][c]: row 8 nr + 2 tq + (c & 1),
            // token gq + 8 (c >> 1)
            const bool masked = inf.n_valid < kChunk || inf.tok0 + kChunk - 1 > lim_min;
            uint32_t pb[NR][2];
#pragma unroll
            for (int nr = 0; nr < NR; ++nr) {
                pb[nr][0] = pb[nr][1] = 0u;
                if (nr >= nr_live) continue;
#pragma unroll
                for (int c = 0; c < 4; ++c) x[nr][c] *= sl2;
                if (masked) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int tok = gq + 8 * (c >> 1);
                        if (tok >= inf.n_valid || inf.tok0 + tok > lim[nr][c & 1]) x[nr][c] = -INFINITY;
                    }
                }
                float mx[2] = {fmaxf(x[nr][0], x[nr][2]), fmaxf(x[nr][1], x[nr][3])};
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], 4));
                    mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], 8));
                    mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], 16));
                }
                // lazy rescale: a row's reference max moves only when the row max
                // grows by more than kRescaleThreshold; the final division by the
                // row sum makes the result independent of the reference
                const float n0 = fmaxf(m_run[nr][0], mx[0]), n1 = fmaxf(m_run[nr][1], mx[1]);
                const bool need0 = n0 > m_run[nr][0] + kRescaleThreshold;
                const bool need1 = n1 > m_run[nr][1] + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need0 || need1)) {
                    const float a0 = need0 ? fast_exp2(m_run[nr][0] - n0) : 1.f;
                    const float a1 = need1 ? fast_exp2(m_run[nr][1] - n1) : 1.f;
                    if (need0) m_run[nr][0] = n0;
                    if (need1) m_run[nr][1] = n1;
                    l_run[nr][0] *= a0;
                    l_run[nr][1] *= a1;
#pragma unroll
                    for (int i = 0; i < MT; ++i) {
                        o[nr][i][0] *= a0;
                        o[nr][i][2] *= a0;
                        o[nr][i][1] *= a1;
                        o[nr][i][3] *= a1;
                    }
                }
                // a row with every key so far masked keeps m = -inf: its probabilities are 0
                const float u0 = m_run[nr][0] == -INFINITY ? 0.f : m_run[nr][0];
                const float u1 = m_run[nr][1] == -INFINITY ? 0.f : m_run[nr][1];
                // (token gq, rows 2tq, 2tq+1) and (token gq + 8, ...): one lane's share of
                // the two 8 x 8 blocks of P^T; transposed, the B fragment of P^T
                const uint32_t w0 = pack_bf16x2(fast_exp2(x[nr][0] - u0), fast_exp2(x[nr][1] - u1));
                const uint32_t w1 = pack_bf16x2(fast_exp2(x[nr][2] - u0), fast_exp2(x[nr][3] - u1));
                // the row sums add the bf16-rounded probabilities the P V product uses
                l_run[nr][0] += bf16lo_to_f32(w0) + bf16lo_to_f32(w1);
                l_run[nr][1] += bf16hi_to_f32(w0) + bf16hi_to_f32(w1);
                pb[nr][0] = movmatrix_trans(w0);
                pb[nr][1] = movmatrix_trans(w1);
            }
            // ---- O^T += V^T P^T
            const uint32_t vs = v_lane + stage * stage_bytes;
            uint4 vv[4][VH];
#pragma unroll
            for (int d4 = 0; d4 < 4; ++d4)
#pragma unroll
                for (int h = 0; h < VH; ++h)
                    vv[d4][h] = ld_shared_v4(vs + (uint32_t)((d4 & 1) + 8 * (d4 >> 1)) * tok_bytes +
                                             (uint32_t)((16 * h) ^ (v_odd ? 16 : 0)));
            if (VH > 1) {
#pragma unroll
                for (int d4 = 0; d4 < 4; ++d4) swap_if(vv[d4][0], vv[d4][VH - 1], v_odd);
            }
            if (inf.n_valid < kChunk) {
                // rows past the chunk's tokens hold stale bytes: zero them (P is 0 there)
#pragma unroll
                for (int d4 = 0; d4 < 4; ++d4)
                    if (2 * tq + (d4 & 1) + 8 * (d4 >> 1) >= inf.n_valid)
#pragma unroll
                        for (int h = 0; h < VH; ++h) vv[d4][h] = make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                // A = V^T tile mt: rows (dims) e0 = mt and e1 = D / 16 + mt of this lane's
                // slice, columns (tokens) 2 tq, 2 tq + 1 and 2 tq + 8, 2 tq + 9
                const int e0 = mt, e1 = D / 16 + mt;
                const uint32_t s0 = (e0 & 1) ? 0x7632u : 0x5410u, s1 = (e1 & 1) ? 0x7632u : 0x5410u;
                const uint32_t a0 = __byte_perm(word(vv[0][e0 >> 3], (e0 & 7) >> 1), word(vv[1][e0 >> 3], (e0 & 7) >> 1), s0);
                const uint32_t a1 = __byte_perm(word(vv[0][e1 >> 3], (e1 & 7) >> 1), word(vv[1][e1 >> 3], (e1 & 7) >> 1), s1);
                const uint32_t a2 = __byte_perm(word(vv[2][e0 >> 3], (e0 & 7) >> 1), word(vv[3][e0 >> 3], (e0 & 7) >> 1), s0);
                const uint32_t a3 = __byte_perm(word(vv[2][e1 >> 3], (e1 & 7) >> 1), word(vv[3][e1 >> 3], (e1 & 7) >> 1), s1);
#pragma unroll
                for (int nr = 0; nr < NR; ++nr)
                    if (nr < nr_live) mma_16816(o[nr][mt], a0, a1, a2, a3, pb[nr][0], pb[nr][1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);
        if (++stage == NS) {
            stage = 0;
            fparity ^= 1;
        }
        if (inf.flags & kFlagLast) {
            // ---- total the row sums over the row's 8 lanes (one per token pair); write
            // out or a partial.  This lane holds dims (D / 8) gq + e of query rows
            // 8 nr + 2 tq + u: o[nr][e][u] for e < D / 16, o[nr][e - D / 16][2 + u] above.
#pragma unroll
            for (int nr = 0; nr < NR; ++nr) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    float lt = l_run[nr][u];
                    lt += __shfl_xor_sync(0xffffffffu, lt, 4);
                    lt += __shfl_xor_sync(0xffffffffu, lt, 8);
                    lt += __shfl_xor_sync(0xffffffffu, lt, 16);
                    const int r = 8 * nr + 2 * tq + u;
                    if (r >= R) continue;
                    float f[D / 8];
#pragma unroll
                    for (int e = 0; e < D / 8; ++e) f[e] = e < D / 16 ? o[nr][e][u] : o[nr][e - D / 16][2 + u];
                    if (inf.slot < 0) {
                        uint16_t *orow = p.out +
                                         ((row0 + r / G) * p.num_q_heads + (int64_t)(hg * HC + warp) * G + r % G) * D +
                                         (D / 8) * gq;
                        const float inv = 1.0f / lt;
#pragma unroll
                        for (int v = 0; v < D / 64; ++v) {
                            float w[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) w[e] = f[8 * v + e] * inv;
                            st_global_v4(orow + 8 * v, pack8(w));
                        }
                    } else {
                        const size_t pr = ((size_t)inf.slot * HC + warp) * p.rows_per_head + r;
                        float4 *po = reinterpret_cast<float4 *>(p.part_o + pr * D + (D / 8) * gq);
#pragma unroll
                        for (int v = 0; v < D / 32; ++v) po[v] = make_float4(f[4 * v], f[4 * v + 1], f[4 * v + 2], f[4 * v + 3]);
                        if (gq == 0) p.part_ml[pr] = make_float2(m_run[nr][u], lt);
                    }
                }
            }
        }
    }
}

// Finish what the split kernel left: combine the partials of every unit that
// was cut by a CTA boundary (merge CTA c takes the unit that starts before
// split CTA c's range and ends inside it), and write zero rows (reporting
// invalid lengths) for sequences the split kernel had no chunks for.  The grid
// has the split kernel's size.  Everything that does not read the split
// kernel's output runs before griddepcontrol.wait, overlapping the split
// kernel's tail; every CTA waits before it exits.  Each thread's (row, 4
// columns) item is two rounds of dependent loads (the partial maxima, then
// the weighted sums), so the CTA is wide to keep many items' loads in flight:
// a unit holds HC * g * n * D / 4 items (512 for 8 KV heads of 2 decode rows at
// D = 128, 2,048 for 8 verification rows).  512 threads still fit on an SM
// beside a split-kernel CTA, so the merge's schedule runs during the split
// kernel's tail; 1,024 do not, and pay off only for multi-row units.
template <int kThreadsM>
__global__ void __launch_bounds__(kThreadsM) decode_merge_kernel(const Params p, int head_dim) {
    __shared__ long long sched[4];
    __shared__ long long scratch[kThreadsM / 32 + 1];
    const int D = head_dim;
    const long long c = blockIdx.x;
    const long long G = gridDim.x;
    const int HC = p.heads_per_cta;
    const int g = p.num_q_heads / p.num_kv_heads;
    const int RP = p.rows_per_head;
    const int NHG = p.num_head_groups;

    const Schedule sc = compute_schedule(p, sched, scratch);

    // (0) with no prefill kernel in the call, its check that cu_seqlens_q runs
    // from 0 to total_q is made here
    if (p.sole_path && c == 0 && threadIdx.x == 0 &&
        (__ldg(p.cu_seqlens_q) != 0 || __ldg(p.cu_seqlens_q + p.num_seqs) != p.total_q))
        report_error(NPV_DEVERR_QUERY_LENS);

    // (1) rows of this path's sequences with no chunks
    for (long long b = c + G * threadIdx.x; b < p.num_seqs; b += G * blockDim.x) {
        const int32_t n = path_rows(p, (int32_t)b);
        if (n == 0) {
            // other sequences belong to the prefill kernel, which also reports
            // malformed cu_seqlens_q, unless this call runs no prefill kernel
            if (p.sole_path) reject_foreign_rows(p, (int32_t)b, D);
            continue;
        }
        const int32_t L = __ldg(p.context_lens + b);
        const bool bad = L < 0 || (long long)L > (long long)p.max_blocks_per_seq * p.block_size ||
                         (p.cu_seqlens_q != nullptr && L < n);
        if (bad) report_error(NPV_DEVERR_CONTEXT_LEN);
        if (L < n || bad) {
            uint4 *orow = reinterpret_cast<uint4 *>(p.out + query_row(p, (int32_t)b) * (int64_t)p.num_q_heads * D);
            for (int i = 0; i < n * p.num_q_heads * D / 8; ++i) orow[i] = make_uint4(0, 0, 0, 0);
            // a fused store still writes this sequence's token
            if (p.key != nullptr) store_token_rows(p, (int32_t)b, 0, p.num_kv_heads, D, 0, 1);
        }
    }

    // (2) the unit that starts before this CTA's range and ends inside it
    const bool work = sc.c0 < sc.c1 && sc.s_first < sc.c0 && sc.e_first <= sc.c1;
    const long long N = sc.total, u = sc.u_first, S = sc.s_first;
    const long long ca = work ? ((S + 1) * G - 1) / N : 0;  // split CTA holding the unit's first chunk
    const int sa = (work && S == ca * N / G) ? 0 : 1;
    grid_dependency_wait();
    if (!work) return;
    const int32_t b = (int32_t)(u / NHG), hg = (int32_t)(u % NHG);
    const int R = g * path_rows(p, b);
    const int64_t row0 = query_row(p, b);
    for (int idx = threadIdx.x; idx < HC * R * D / 4; idx += blockDim.x) {
        const int hl = idx / (R * D / 4), rem = idx % (R * D / 4);
        const int r = rem / (D / 4), d4 = (rem % (D / 4)) * 4;
        const long long pr = (long long)hl * RP + r;  // row within a partial slot
        float M = p.part_ml[(2 * ca + sa) * HC * RP + pr].x;
        for (long long cc = ca + 1; cc <= c; ++cc) {
            if (cc * N / G == (cc + 1) * N / G) continue;  // empty range
            M = fmaxf(M, p.part_ml[(2 * cc) * HC * RP + pr].x);
        }
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f, lsum = 0.f;
        for (long long cc = ca; cc <= c; ++cc) {
            long long slot;
            if (cc == ca) {
                slot = 2 * ca + sa;
            } else {
                if (cc * N / G == (cc + 1) * N / G) continue;
                slot = 2 * cc;
            }
            const float2 ml = p.part_ml[slot * HC * RP + pr];
            // a partial whose rows saw only masked keys has m = -inf and weight 0
            const float w = fast_exp2(ml.x - M);
            const float4 ov = *reinterpret_cast<const float4 *>(p.part_o + (slot * HC * RP + pr) * D + d4);
            lsum = fmaf(w, ml.y, lsum);
            acc0 = fmaf(w, ov.x, acc0);
            acc1 = fmaf(w, ov.y, acc1);
            acc2 = fmaf(w, ov.z, acc2);
            acc3 = fmaf(w, ov.w, acc3);
        }
        const float inv = 1.0f / lsum;
        uint2 packed = make_uint2(pack_bf16x2(acc0 * inv, acc1 * inv), pack_bf16x2(acc2 * inv, acc3 * inv));
        uint16_t *orow = p.out + ((row0 + r / g) * p.num_q_heads + (int64_t)(hg * HC + hl) * g + r % g) * D;
        *reinterpret_cast<uint2 *>(orow + d4) = packed;
    }
}

}  // namespace decode
}  // namespace npv
