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
//   * A consumer warp reads 16-byte rows from shared memory (D/8 lanes per row,
//     conflict-free), forms partial dot products, reduce-scatters them across
//     the row's lanes so that each lane ends with one token's score per head,
//     and runs an fp32 online softmax in the log2 domain (scale * log2 e is
//     folded into q).  Probabilities pass through a per-warp shared buffer to
//     the P.V step, which accumulates an 8-element slice of the output per lane.
#pragma once

#include "npv_device.cuh"

namespace npv {
namespace decode {

constexpr int kChunk = 16;  // tokens per pipeline stage
constexpr int kMaxConsumerWarps = 8;
constexpr int kMaxStages = 8;
constexpr int kStageBudgetBytes = 192 * 1024;
constexpr int kHeaderBytes = 1024;

enum : int32_t { kFlagFirst = 1, kFlagLast = 2, kFlagSkip = 4, kFlagNewToken = 8 };

struct StageInfo {
    int32_t unit;     // (sequence, head group) index
    int32_t n_valid;  // live tokens in the chunk (1..16)
    int32_t flags;
    int32_t slot;  // partial slot written at kFlagLast, or -1 for a finished unit
};

struct Params {
    uint16_t *out;  // [rows, Hq, D]
    const uint16_t *q;
    int64_t q_row_stride;  // elements between query rows
    const uint16_t *k_cache;
    const uint16_t *v_cache;
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *cu_seqlens_q;  // non-null: mixed batch; only sequences with one query row run here
    int32_t total_q;              // rows of q and out in a mixed batch
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
    float2 *part_ml;  // [grid][2][HC*g]: (running max, sum) of a partial unit
    float *part_o;    // [grid][2][HC*g][D]: unnormalised output of a partial unit
};

// Chunks of work for sequence b on this path (0 for an empty, invalid or
// multi-row sequence; the merge kernel writes those rows or reports them).
__device__ __forceinline__ int32_t seq_chunks(const Params &p, int32_t b) {
    const int32_t L = __ldg(p.context_lens + b);
    if (p.cu_seqlens_q != nullptr) {
        const int32_t cb = __ldg(p.cu_seqlens_q + b), ce = __ldg(p.cu_seqlens_q + b + 1);
        if (ce - cb != 1 || cb < 0 || ce > p.total_q) return 0;
    }
    if (L <= 0 || (long long)L > (long long)p.max_blocks_per_seq * p.block_size) return 0;
    return (L + kChunk - 1) / kChunk;
}

__device__ __forceinline__ int64_t query_row(const Params &p, int32_t b) {
    return p.cu_seqlens_q != nullptr ? (int64_t)__ldg(p.cu_seqlens_q + b) : (int64_t)b;
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

template <int D, int G>
struct Shape {
    static constexpr int LPR = D / 8;          // lanes per 16-byte-vector row
    static constexpr int RPL = 32 / LPR;       // rows per warp-wide load
    static constexpr int NI = kChunk / RPL;    // warp-wide loads per stage
    static constexpr int LOG_NI = NI == 8 ? 3 : (NI == 4 ? 2 : 1);
};

// Consumer warps (= KV heads) per CTA: 8, or 4 when g = 8 so that the larger
// per-thread state (8 query heads) fits in registers.
__host__ __device__ constexpr int max_heads_per_cta(int g) { return g >= 8 ? 4 : kMaxConsumerWarps; }

template <int D, int G>
__global__ void __launch_bounds__((max_heads_per_cta(G) + 1) * 32, 1) decode_split_kernel(const Params p) {
    using S = Shape<D, G>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty_bar = full_bar + kMaxStages;
    StageInfo *info = reinterpret_cast<StageInfo *>(empty_bar + kMaxStages);
    long long *sched = reinterpret_cast<long long *>(info + kMaxStages);  // [0..7]
    long long *scan_scratch = sched + 8;                                  // [kMaxConsumerWarps + 2]
    float *pbuf = reinterpret_cast<float *>(smem + kHeaderBytes);         // [HC][kChunk][G]

    const int HC = p.heads_per_cta;
    const int NS = p.num_stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pbuf_bytes = ((HC * kChunk * G * 4) + 1023) & ~1023;
    const int row_elems = HC * D;  // one token of one head group
    const int stage_elems = kChunk * row_elems;
    uint16_t *stage_k = reinterpret_cast<uint16_t *>(smem + kHeaderBytes + pbuf_bytes);
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

    if (warp == HC) {
        // ===================== producer warp =====================
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
                if (lane == 0) {
                    int32_t flags = (i == 0 ? kFlagFirst : 0) | (i == seg_len - 1 ? kFlagLast : 0);
                    // a fused store: this segment ends with the unit's last chunk, which
                    // holds the new token (the consumers store and substitute it)
                    if (i == 0 && p.key != nullptr && k + seg_len == nC) flags |= kFlagNewToken;
                    if (!valid) {
                        flags |= kFlagSkip;
                        report_error(NPV_DEVERR_BLOCK_ID);
                    }
                    info[stage] = StageInfo{(int32_t)u, n_valid, flags, slot};
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
    constexpr int LPR = S::LPR, RPL = S::RPL, NI = S::NI;
    const int rg = lane / LPR;   // which row of a warp-wide load this lane reads
    const int sub = lane % LPR;  // which 8-element slice of the row
    const int HCG = HC * G;
    float *my_p = pbuf + warp * (kChunk * G);
    const uint32_t k_lane = smem_addr(stage_k) + (uint32_t)((warp * D + sub * 8) * 2);
    const uint32_t v_lane = smem_addr(stage_v) + (uint32_t)((warp * D + sub * 8) * 2);
    const uint32_t tok_bytes = (uint32_t)(row_elems * 2);
    const uint32_t stage_bytes = (uint32_t)(stage_elems * 2);

    float qf[G][8], o[G][8], m_run[G], l_run[G];
    int32_t b = 0, hg = 0;
    // fused store: this lane's 8-element slices of the new token's K and V rows
    uint4 new_k = make_uint4(0, 0, 0, 0), new_v = make_uint4(0, 0, 0, 0);
    int32_t new_slot = -1;
    int stage = 0;
    uint32_t fparity = 0;
    const long long nchunks = c1 - c0;
    for (long long it = 0; it < nchunks; ++it) {
        if (!mbar_wait(&full_bar[stage], fparity)) break;
        const StageInfo inf = info[stage];
        if (inf.flags & kFlagFirst) {
            b = inf.unit / NHG;
            hg = inf.unit % NHG;
            const uint16_t *qrow = p.q + query_row(p, b) * p.q_row_stride +
                                   ((int64_t)(hg * HC + warp) * G) * D + sub * 8;
#pragma unroll
            for (int j = 0; j < G; ++j) {
                float f[8];
                unpack8(ld_nc_v4(qrow + j * D), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    qf[j][e] = f[e] * p.scale_log2;
                    o[j][e] = 0.f;
                }
                m_run[j] = -INFINITY;
                l_run[j] = 0.f;
            }
            new_slot = -1;
            if (inf.flags & kFlagNewToken) {
                // fetch now; used when the segment's last chunk arrives
                const int32_t slot = __ldg(p.slot_mapping + b);
                if (slot >= 0 && (long long)slot < (long long)p.num_blocks * p.block_size) {
                    new_slot = slot;
                    const int64_t h = (int64_t)(hg * HC + warp) * D + sub * 8;
                    new_k = ld_nc_v4(p.key + (int64_t)b * p.key_stride + h);
                    new_v = ld_nc_v4(p.value + (int64_t)b * p.value_stride + h);
                } else if (slot >= 0 && lane == 0) {
                    report_error(NPV_DEVERR_SLOT);
                }
            }
        }
        if ((inf.flags & kFlagLast) && new_slot >= 0) {
            // the unit's last chunk: put the new token into the stage (its cache
            // slot may not hold it yet) and into the cache
            const int tl = inf.n_valid - 1;
            if (rg == 0) {
                const uint32_t off = (uint32_t)(((tl * HC + warp) * D + sub * 8) * 2);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_addr(stage_k) + stage * stage_bytes +
                                                                            off),
                             "r"(new_k.x), "r"(new_k.y), "r"(new_k.z), "r"(new_k.w)
                             : "memory");
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_addr(stage_v) + stage * stage_bytes +
                                                                            off),
                             "r"(new_v.x), "r"(new_v.y), "r"(new_v.z), "r"(new_v.w)
                             : "memory");
                const int64_t dst = ((int64_t)new_slot * p.num_kv_heads + hg * HC + warp) * D + sub * 8;
                st_global_v4(const_cast<uint16_t *>(p.k_cache) + dst, new_k);
                st_global_v4(const_cast<uint16_t *>(p.v_cache) + dst, new_v);
            }
            __syncwarp();
        }
        if (!(inf.flags & kFlagSkip)) {
            const bool full = inf.n_valid == kChunk;
            const uint32_t kst = k_lane + stage * stage_bytes;
            const uint32_t vst = v_lane + stage * stage_bytes;
            // ---- scores: partial dot products of this lane's 8 dims
            float acc[NI][G];
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                float kf[8];
                unpack8(ld_shared_v4(kst + (uint32_t)(i * RPL + rg) * tok_bytes), kf);
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    // even and odd dims accumulate in the two halves of a pair
                    float2 a = fmul2(make_float2(qf[j][0], qf[j][1]), make_float2(kf[0], kf[1]));
#pragma unroll
                    for (int e = 2; e < 8; e += 2)
                        a = ffma2(make_float2(qf[j][e], qf[j][e + 1]), make_float2(kf[e], kf[e + 1]), a);
                    acc[i][j] = a.x + a.y;
                }
            }
            // ---- reduce-scatter over the row's lanes: halve the token list at
            // each step, keeping the half selected by this lane's bit
#pragma unroll
            for (int step = 0; step < S::LOG_NI; ++step) {
                const int n = NI >> (step + 1);
                const int mask = LPR >> (step + 1);
                const bool upper = (sub & mask) != 0;
#pragma unroll
                for (int i = 0; i < n; ++i) {
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const float send = upper ? acc[i][j] : acc[i + n][j];
                        const float keep = upper ? acc[i + n][j] : acc[i][j];
                        acc[i][j] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
                    }
                }
            }
            float s[G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                float v = acc[0][j];
#pragma unroll
                for (int mask = (LPR >> (S::LOG_NI + 1)); mask >= 1; mask >>= 1)
                    v += __shfl_xor_sync(0xffffffffu, v, mask);
                s[j] = v;
            }
            // this lane now holds the score of token (sub >> 1) * RPL + rg
            const int my_tok = (sub >> 1) * RPL + rg;
            if (!full && my_tok >= inf.n_valid) {
#pragma unroll
                for (int j = 0; j < G; ++j) s[j] = -INFINITY;
            }
            // ---- online softmax (log2 domain); the running max is warp-uniform
            float pj[G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                float mx = s[j];
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                if (mx > m_run[j]) {
                    const float alpha = fast_exp2(m_run[j] - mx);
                    l_run[j] *= alpha;
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[j][e] *= alpha;
                    m_run[j] = mx;
                }
                pj[j] = fast_exp2(s[j] - m_run[j]);
                l_run[j] += pj[j];
            }
            __syncwarp();
            if ((lane & 1) == 0) {
#pragma unroll
                for (int j = 0; j < G; ++j) my_p[my_tok * G + j] = pj[j];
            }
            __syncwarp();
            // ---- o += p . V over this lane's tokens and 8 dims
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const int tok = i * RPL + rg;
                if (full || tok < inf.n_valid) {
                    float vf[8];
                    unpack8(ld_shared_v4(vst + (uint32_t)tok * tok_bytes), vf);
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const float pv = my_p[tok * G + j];
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float2 r = ffma2(make_float2(pv, pv), make_float2(vf[e], vf[e + 1]),
                                                   make_float2(o[j][e], o[j][e + 1]));
                            o[j][e] = r.x;
                            o[j][e + 1] = r.y;
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);
        if (++stage == NS) {
            stage = 0;
            fparity ^= 1;
        }
        if (inf.flags & kFlagLast) {
            // ---- combine the row groups, total the sums, write out or a partial
#pragma unroll
            for (int mask = LPR; mask < 32; mask <<= 1) {
#pragma unroll
                for (int j = 0; j < G; ++j)
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[j][e] += __shfl_xor_sync(0xffffffffu, o[j][e], mask);
            }
            float lt[G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                float v = l_run[j];
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                lt[j] = v;
            }
            if (inf.slot < 0) {
                if (rg == 0) {
                    uint16_t *orow = p.out + query_row(p, b) * (int64_t)p.num_q_heads * D +
                                     ((int64_t)(hg * HC + warp) * G) * D + sub * 8;
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const float inv = 1.0f / lt[j];
                        float r[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) r[e] = o[j][e] * inv;
                        st_global_v4(orow + j * D, pack8(r));
                    }
                }
            } else {
                if (rg == 0) {
                    float *po = p.part_o + ((size_t)inf.slot * HCG + warp * G) * D + sub * 8;
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        reinterpret_cast<float4 *>(po + j * D)[0] = make_float4(o[j][0], o[j][1], o[j][2], o[j][3]);
                        reinterpret_cast<float4 *>(po + j * D)[1] = make_float4(o[j][4], o[j][5], o[j][6], o[j][7]);
                    }
                }
                if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < G; ++j)
                        p.part_ml[(size_t)inf.slot * HCG + warp * G + j] = make_float2(m_run[j], lt[j]);
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
// kernel's tail; every CTA waits before it exits.
__global__ void __launch_bounds__(256) decode_merge_kernel(const Params p, int head_dim) {
    __shared__ long long sched[4];
    __shared__ long long scratch[16];
    const int D = head_dim;
    const long long c = blockIdx.x;
    const long long G = gridDim.x;
    const int HC = p.heads_per_cta;
    const int g = p.num_q_heads / p.num_kv_heads;
    const int HCG = HC * g;
    const int NHG = p.num_head_groups;

    const Schedule sc = compute_schedule(p, sched, scratch);

    // (1) rows with no chunks on this path
    for (long long b = c + G * threadIdx.x; b < p.num_seqs; b += G * blockDim.x) {
        const int32_t L = __ldg(p.context_lens + b);
        if (p.cu_seqlens_q != nullptr) {
            const int32_t cb = __ldg(p.cu_seqlens_q + b), ce = __ldg(p.cu_seqlens_q + b + 1);
            // multi-row sequences belong to the prefill kernel, which also
            // reports malformed cu_seqlens_q
            if (ce - cb != 1 || cb < 0 || ce > p.total_q) continue;
        }
        const bool bad = L < 0 || (long long)L > (long long)p.max_blocks_per_seq * p.block_size ||
                         (p.cu_seqlens_q != nullptr && L < 1);
        if (bad) report_error(NPV_DEVERR_CONTEXT_LEN);
        if (L <= 0 || bad) {
            uint4 *orow = reinterpret_cast<uint4 *>(p.out + query_row(p, (int32_t)b) * (int64_t)p.num_q_heads * D);
            for (int i = 0; i < p.num_q_heads * D / 8; ++i) orow[i] = make_uint4(0, 0, 0, 0);
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
    uint16_t *orow = p.out + query_row(p, b) * (int64_t)p.num_q_heads * D + (int64_t)hg * HCG * D;
    for (int idx = threadIdx.x; idx < HCG * D / 4; idx += blockDim.x) {
        const int h = idx / (D / 4), d4 = (idx % (D / 4)) * 4;
        float M = p.part_ml[(2 * ca + sa) * HCG + h].x;
        for (long long cc = ca + 1; cc <= c; ++cc) {
            if (cc * N / G == (cc + 1) * N / G) continue;  // empty range
            M = fmaxf(M, p.part_ml[(2 * cc) * HCG + h].x);
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
            const float2 ml = p.part_ml[slot * HCG + h];
            const float w = fast_exp2(ml.x - M);
            const float4 ov = *reinterpret_cast<const float4 *>(p.part_o + (slot * HCG + h) * D + d4);
            lsum = fmaf(w, ml.y, lsum);
            acc0 = fmaf(w, ov.x, acc0);
            acc1 = fmaf(w, ov.y, acc1);
            acc2 = fmaf(w, ov.z, acc2);
            acc3 = fmaf(w, ov.w, acc3);
        }
        const float inv = 1.0f / lsum;
        uint2 packed = make_uint2(pack_bf16x2(acc0 * inv, acc1 * inv), pack_bf16x2(acc2 * inv, acc3 * inv));
        *reinterpret_cast<uint2 *>(orow + (int64_t)h * D + d4) = packed;
    }
}

}  // namespace decode
}  // namespace npv
