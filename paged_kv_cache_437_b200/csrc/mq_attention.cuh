// Multi-query paged attention on the 5th-generation tensor cores (tcgen05).
//
// What is computed ("LLM Inference: KV Cache, Batching & Scheduling",
// cariara.com, section "Chunked prefill": a prompt is fed in fixed-size
// chunks, e.g. 512 tokens, interleaved with other requests' decode steps):
// query i (0-based) of a chunk of n tokens whose sequence has context c after
// the chunk's append attends, for every query head, to positions
// 0 .. c - n + i of that sequence's paged cache -- causal inside the chunk,
// everything before it.
//
// Kernel design (B200):
//  * Work unit = (source, KV head, block of `tpb` consecutive query sources):
//    a source is a chunk's sequence (its tokens are the queries) or a
//    sharing group (its members' decode queries over their common prefix).
//    The rows are the tpb sources x the G query heads that share the KV head
//    (tpb * G <= 128): one 128-row tile.  Every K/V tile of the unit's range
//    is loaded once for all of them, so a chunk reads each K/V position once
//    per row block instead of once per query token.
//  * S = Q K^T (both operands in shared memory: 128-byte swizzled tiles
//    straight from TMA) and, per 64-position half h of the tile,
//    O_h += P_h V_h with P_h read from tensor memory, as tcgen05.mma
//    (kind::f16, M = 128) with fp32 accumulators in tensor memory: S
//    double-buffered (2 x 128 columns; P is written over its own scores),
//    O_0 and O_1 (D columns each).
//  * Warp roles in a 352-thread CTA: warps 0-7 the softmax (warp w: the rows
//    of TMEM lane quarter w % 4, the positions of half w / 4 of each tile,
//    with a running max and sum of its own; the two halves of a row meet in
//    the epilogue); warp 8 the unit scheduler and the TMA loads of Q and K;
//    warp 10 the TMA loads of V; warp 9 allocates TMEM and one of its threads
//    issues every MMA.  All hand-offs are mbarriers; every wait is bounded
//    (time-out -> error word, orderly teardown).
//  * Persistent grid (one CTA per SM); units are taken from a global counter
//    in order of decreasing causal length within each source.
//  * Online softmax in the log2 domain with a lazy rescale: the running
//    reference max only moves when the tile max exceeds it by more than 2^8,
//    so P stays <= 256 (exact enough in 16 bits) and O in TMEM is almost
//    never rescaled.  Positions past a row's causal limit get -inf before the
//    exponential; V rows past the context are zeroed in shared memory before
//    the P V product (0 * NaN would otherwise leak a poisoned slot).
#pragma once

#include "decode.cuh"

namespace pkv {

constexpr int kMqRows = 128;      // MMA M: query rows of one unit
constexpr int kMqTile = 128;      // KV positions per tile (N of Q K^T, K of P V)
constexpr int kMqSoftmaxWarps = 8;  // two per 32-row quarter: one per 64-column half of S
constexpr int kMqProducerWarp = 8;   // units, Q and K tiles
constexpr int kMqMmaWarp = 9;
constexpr int kMqVProducerWarp = 10; // V tiles
constexpr int kMqThreads = 352;   // warps 0-7 softmax, 8 K producer, 9 MMA, 10 V producer
constexpr int kMqKStages = 2;     // K tiles in flight
constexpr int kMqVStages = 2;     // V tiles in flight
constexpr float kMqRescaleLog2 = 8.0f;
constexpr int kMqMaxSeqs = 4096;  // per-sequence unit prefix kept in shared memory

enum MqMode : int {
    kMqPrefill = 0,  // chunks of query tokens, causal limits, normalized output
    kMqPrefix = 1,   // decode queries of a sharing group over its common prefix, fp32 partials
};

struct MqArgs {
    int mode;
    uint16_t *out;                 // prefill: [T][Hq][D]
    const int32_t *block_tables;   // [B][MB]
    const int32_t *query_start;    // prefill: [B + 1]
    const int32_t *context_lens;   // prefill: [B], after the chunk's append
    // shared-prefix groups: members of group g are sequences
    // group_start[g] .. group_start[g+1]-1; the group's common blocks are read
    // through row group_ref[g] of the table, up to position group_len[g];
    // member s attends to its first shared[s] positions there
    const int32_t *group_start, *group_ref, *group_len, *shared;
    float *part_o, *part_m, *part_l;  // prefix: [B][Hq][D], [B][Hq], [B][Hq] (log2-domain max)
    int nsrc;                      // sources of units: sequences (prefill) or groups (prefix)
    int64_t mb;                    // MB
    int64_t nb;                    // NB
    int B, T, Hq, Hkv, G, bs, tpb;
    float scale_log2;              // |scale| * log2(e)
    int negate_q;                  // scale < 0: the score product negates Q
    int *unit_counter;             // zero at launch (written by the expansion kernel)
    int pool_rows;                 // rows of the pools' TMA view; this row reads zeros
    unsigned *err;
    uint64_t wait_limit_ns;
    int inject_no_issue;           // testing: issue no copies so that waits run out
};

// Shared-memory plan (from a 1024-aligned base): Q tile, K ring, V ring,
// then the exchange buffer, barriers, small state and the per-sequence unit
// prefix.  P never touches shared memory: it is written to tensor memory over
// its own scores and read from there by the P V product.
template <int D>
struct MqSmem {
    static constexpr int kTileBytes = kMqTile * D * 2;   // K or V tile; Q (128 rows) too
    static constexpr int kHalf = kMqTile * 128;          // one 128-byte column half of a tile
    static constexpr int q = 0;
    static constexpr int k = q + kTileBytes;
    static constexpr int v = k + kMqKStages * kTileBytes;
    static constexpr int xbuf = v + kMqVStages * kTileBytes;  // [2 parity][2 halves][128 rows] f32
    static constexpr int bars = xbuf + 2 * 2 * kMqRows * 4;
    // barrier indices
    static constexpr int kQFull = 0, kQEmpty = 1, kKFull = 2, kKEmpty = kKFull + kMqKStages,
                         kVFull = kKEmpty + kMqKStages, kVEmpty = kVFull + kMqVStages, kSFull = kVEmpty + kMqVStages,
                         kPFull = kSFull + 2, kODone = kPFull + 2, kUnitFull = kODone + 1,
                         kUnitEmpty = kUnitFull + 2, kDrain = kUnitEmpty + 2, kXch = kDrain + 1,
                         kNumBars = kXch + 4;
    static constexpr int misc = bars + kNumBars * 8;     // [0..1] unit slots, [2] TMEM base, [3] abort
    static constexpr int prefix = misc + 32;
    static constexpr int bytes(int B) { return prefix + (B + 1) * 4 + 1024; }  // + base re-alignment
};

// A unit: rows = `tpb` consecutive query sources (chunk tokens, or members
// of a sharing group) x the G heads of KV head kvh; K/V positions
// [0, lim_max) read through table row trow; z0 = index of the unit's first
// source in q's [sources][Hq][D] view.
struct MqUnit {
    int s, rb, kvh, nt, ctx, n, q0, lim_max, trow;
};

// Units of source s (0 for sources this kernel does not handle).
__device__ __forceinline__ int mq_units_of(int s, const MqArgs &a) {
    if (a.mode == kMqPrefix) {
        const int gs = __ldg(a.group_start + s), ge = __ldg(a.group_start + s + 1);
        // an invalid or empty group has no reference (its members share nothing)
        if (gs < 0 || ge > a.B || ge <= gs || __ldg(a.group_len + s) <= 0)
            return 0;
        return ((ge - gs + a.tpb - 1) / a.tpb) * a.Hkv;
    }
    const int q0 = __ldg(a.query_start + s);
    const int n = __ldg(a.query_start + s + 1) - q0;
    const int c = __ldg(a.context_lens + s);
    // decode tokens (n == 1) and inconsistent lengths are not this kernel's
    if (n < 2 || c < n || (int64_t)c > a.mb * a.bs)
        return 0;
    return ((n + a.tpb - 1) / a.tpb) * a.Hkv;
}

__device__ __forceinline__ MqUnit mq_unit(int u, const int *prefix, const MqArgs &a) {
    MqUnit U;
    U.s = upper_bound_i(prefix, a.nsrc + 1, u) - 1;
    if (a.mode == kMqPrefix) {
        U.q0 = __ldg(a.group_start + U.s);
        U.n = __ldg(a.group_start + U.s + 1) - U.q0;
        U.ctx = __ldg(a.group_len + U.s);
        U.trow = __ldg(a.group_ref + U.s);
    } else {
        U.q0 = __ldg(a.query_start + U.s);
        U.n = __ldg(a.query_start + U.s + 1) - U.q0;
        U.ctx = __ldg(a.context_lens + U.s);
        U.trow = U.s;
    }
    const int nrb = (U.n + a.tpb - 1) / a.tpb;
    const int idx = u - prefix[U.s];
    U.rb = nrb - 1 - idx / a.Hkv;  // the longest causal ranges first
    U.kvh = idx - (idx / a.Hkv) * a.Hkv;
    U.lim_max = a.mode == kMqPrefix ? U.ctx : U.ctx - U.n + min(U.n, (U.rb + 1) * a.tpb);
    U.nt = (U.lim_max + kMqTile - 1) / kMqTile;
    return U;
}

// 2^x on the FMA and integer pipes, for part of the softmax exponentials so
// that they do not all queue on the SFU (16 results per clock per SM): x =
// n + f with n = round(x) (by the 1.5 * 2^23 add), f in [-1/2, 1/2]; 2^f by a
// degree-4 polynomial (least-squares fit on Chebyshev nodes of [-1/2, 1/2],
// relative error < 8e-6, coefficients from csrc/gen_exp2_poly.py); 2^n added
// to the exponent field.  Arguments below -126 give 0.
__device__ __forceinline__ float exp2_poly(float x) {
    const float xc = fmaxf(x, -126.f);
    const float t = xc + 12582912.f;
    const float f = xc - (t - 12582912.f);
    float p = fmaf(f, 0.00927829f, 0.05586502f);
    p = fmaf(p, f, 0.24030896f);
    p = fmaf(p, f, 0.69312954f);
    p = fmaf(p, f, 0.99999785f);
    const float r = __int_as_float(__float_as_int(p) + ((__float_as_int(t) - 0x4B400000) << 23));
    return x < -126.f ? 0.f : r;
}

__global__ void exp2_poly_test_kernel(const float *__restrict__ x, float *__restrict__ y, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        y[i] = exp2_poly(x[i]);
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, A and B
// both f16 or both bf16, A K-major, B K-major (b_mn = 0) or MN-major (1), N x
// M = n x 128, optional negation of A.
__host__ __device__ constexpr uint32_t mq_idesc(bool bf16, int n, bool negate_a, bool b_mn) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((negate_a ? 1u : 0u) << 13) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kMqRows >> 4) << 24);
}

// Bounded wait that also gives up when another role has aborted; a time-out
// records the error and raises the abort flag.  Each try_wait may wait in
// the instruction for a short, hardware-chosen time; the clock and the abort
// flag are checked between tries.  (Waits with a 20 us suspend-time hint
// instead were ~4% slower on the chunked-prefill row: 111-112 vs 107 us.)
__device__ __forceinline__ bool mq_wait(uint32_t bar, uint32_t parity, const MqArgs &a, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag)
            return false;
        if (global_timer_ns() - t0 > a.wait_limit_ns) {
            *abort_flag = 1;
            atomicOr(a.err, kErrTimeout);
            return false;
        }
    }
    return true;
}

// POLY: of every 8 pairs of a row's probabilities, POLY are computed with
// exp2_poly and the rest with the SFU's exp2.
template <int D, bool BF16, int POLY = 0>
__global__ void __launch_bounds__(kMqThreads, 1)
    mq_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const MqArgs a) {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    using L = MqSmem<D>;
    constexpr int KS = kMqKStages, VS = kMqVStages;
    constexpr int NH = D / 64;              // 128-byte column halves of a row
    constexpr int kTileBytes = L::kTileBytes;
    constexpr int kHalf = L::kHalf;
    constexpr uint32_t kTmemCols = 512;     // S0 | S1 | O_0 | O_1 (one O per 64-position half)
    constexpr uint32_t kColO = 256;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + L::q, sK = base + L::k, sV = base + L::v;
    auto bar = [&](int i) { return base + (uint32_t)(L::bars + i * 8); };
    volatile int *misc = reinterpret_cast<volatile int *>(gbase + L::misc);
    int *prefix = reinterpret_cast<int *>(gbase + L::prefix);
    volatile int *abort_flag = misc + 3;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows_used = a.tpb * a.G;

    if (threadIdx.x == 0) {
        mbar_init(bar(L::kQFull), 1);
        mbar_init(bar(L::kQEmpty), 1);
        for (int i = 0; i < KS; ++i) {
            mbar_init(bar(L::kKFull + i), 1);
            mbar_init(bar(L::kKEmpty + i), 1);
        }
        for (int i = 0; i < VS; ++i) {
            mbar_init(bar(L::kVFull + i), 1);
            mbar_init(bar(L::kVEmpty + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(L::kSFull + i), 1);
            mbar_init(bar(L::kUnitFull + i), 1);
            mbar_init(bar(L::kUnitEmpty + i), 2 + kMqSoftmaxWarps);  // MMA thread, V producer, softmax warps
        }
        for (int i = 0; i < 2; ++i)
            mbar_init(bar(L::kPFull + i), kMqSoftmaxWarps);  // P of tiles of this parity: one arrival per softmax warp
        for (int i = 0; i < 4; ++i)
            mbar_init(bar(L::kXch + i), 2);  // the two warps of a 32-row quarter
        mbar_init(bar(L::kODone), 1);
        mbar_init(bar(L::kDrain), 1);
        misc[3] = 0;
        fence_mbar_init();
    }
    if ((warp == kMqProducerWarp || warp == kMqVProducerWarp) && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    // Q rows past tpb * G are never written by the TMA: keep them zero
    for (int i = threadIdx.x; i < (kMqRows - rows_used) * 8 * NH; i += blockDim.x) {
        const int r = rows_used + i / (8 * NH), rest = i % (8 * NH), h = rest / 8, c = rest % 8;
        *reinterpret_cast<uint4 *>(gbase + L::q + h * kHalf + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    if (warp == kMqMmaWarp) {
        tmem_alloc(base + L::misc + 8, kTmemCols);
        tmem_relinquish();
    }

    // every read of an input (and every write of out) comes after this
    griddep_wait();
    griddep_launch_dependents();

    // ---- per-sequence unit counts and their prefix sums (block-wide scan)
    {
        const int nthr = blockDim.x;
        const int per = (a.nsrc + nthr - 1) / nthr;
        const int beg = min(a.nsrc, (int)threadIdx.x * per), end = min(a.nsrc, beg + per);
        int local = 0;
        for (int s = beg; s < end; ++s)
            local += mq_units_of(s, a);
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(FULL, incl, o);
            if (lane >= o)
                incl += v;
        }
        __shared__ int warp_tot[kMqThreads / 32];
        if (lane == 31)
            warp_tot[warp] = incl;
        __syncthreads();
        int run = 0;
        for (int w = 0; w < warp; ++w)
            run += warp_tot[w];
        run += incl - local;
        for (int s = beg; s < end; ++s) {
            prefix[s] = run;
            run += mq_units_of(s, a);
        }
        if (threadIdx.x == 0) {
            int tot = 0;
            for (int w = 0; w < kMqThreads / 32; ++w)
                tot += warp_tot[w];
            prefix[a.nsrc] = tot;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[2];
    const int total = prefix[a.nsrc];

    if (total > 0 && (warp == kMqProducerWarp || warp == kMqVProducerWarp)) {
        // ================= producers: units + Q + K tiles (warp 8), V tiles (warp 10)
        // Two warps so that the two tensors' copies are issued in parallel; each
        // walks the same units.  Per tile, lane l < 8 * NH issues the box of
        // 16 positions l % 8 in column half l / 8.
        const bool is_k = warp == kMqProducerWarp;
        int k = 0;
        uint32_t jg = 0;
        int q_issued = -1;                 // last unit whose Q copy was issued
        int t_last[KS > VS ? KS : VS];     // last use index with copies issued, per stage
        for (int i = 0; i < (KS > VS ? KS : VS); ++i)
            t_last[i] = -1;
        const int NS = is_k ? KS : VS;
        const uint32_t ring = is_k ? sK : sV;
        const CUtensorMap *tm = is_k ? &tmK : &tmV;
        const int full0 = is_k ? L::kKFull : L::kVFull, empty0 = is_k ? L::kKEmpty : L::kVEmpty;
        bool ok = true;
        while (ok) {
            const int slot = k & 1;
            int u = 0;
            if (is_k) {
                if (lane == 0)
                    u = atomicAdd(a.unit_counter, 1);
                u = __shfl_sync(FULL, u, 0);
                ok = __all_sync(FULL, mq_wait(bar(L::kUnitEmpty + slot), ((k >> 1) & 1) ^ 1, a, abort_flag));
                if (!ok)
                    break;
                if (lane == 0) {
                    misc[slot] = u < total ? u : -1;
                    mbar_arrive(bar(L::kUnitFull + slot));
                }
                if (u >= total)
                    break;
            } else {
                ok = __all_sync(FULL, mq_wait(bar(L::kUnitFull + slot), (k >> 1) & 1, a, abort_flag));
                if (!ok)
                    break;
                u = misc[slot];
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(L::kUnitEmpty + slot));
                if (u < 0)
                    break;
            }
            const MqUnit U = mq_unit(u, prefix, a);
            if (is_k) {
                ok = __all_sync(FULL, mq_wait(bar(L::kQEmpty), (k & 1) ^ 1, a, abort_flag));
                if (!ok)
                    break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(L::kQFull), (uint32_t)(NH * rows_used * 128));
                    if (!a.inject_no_issue) {
#pragma unroll
                        for (int h = 0; h < NH; ++h)
                            tma_load_3d(sQ + h * kHalf, &tmQ, h * 64, U.kvh * a.G, U.q0 + U.rb * a.tpb,
                                        bar(L::kQFull));
                        q_issued = k;
                    }
                }
            }
            const int32_t *trow = a.block_tables + (size_t)U.trow * a.mb;
            const int nblk = (U.ctx + a.bs - 1) / a.bs;
            // The unit's table entries, 32 at a time: lane i holds entry
            // cur_base + i; the next 32 are loaded one window ahead so that a
            // tile never waits for its table entries.
            auto load_win = [&](int b) { return b + lane < nblk ? __ldg(trow + b + lane) : -1; };
            int cur_base = 0, cur_val = load_win(0);
            int nxt_base = 32, nxt_val = load_win(32);
            // lane l: the pool row of box l % 8 (16 positions) of tile j;
            // positions past the range (and bad table entries) read zeros
            auto box_row = [&](int j) {
                const int b0 = j * kMqTile / a.bs, b1 = min(nblk - 1, (j * kMqTile + kMqTile - 1) / a.bs);
                if (b0 < cur_base || b1 >= cur_base + 32) {
                    if (b0 == nxt_base) {
                        cur_base = nxt_base;
                        cur_val = nxt_val;
                    } else {
                        cur_base = b0;
                        cur_val = load_win(b0);
                    }
                    nxt_base = cur_base + 32;
                    nxt_val = load_win(nxt_base);
                }
                const int pos = j * kMqTile + (lane & 7) * 16;
                const int blk = __shfl_sync(FULL, cur_val, min(31, max(0, pos / a.bs - cur_base)));
                int y = a.pool_rows;
                if (pos < U.ctx) {
                    if (blk < 0 || (int64_t)blk >= a.nb) {
                        if (is_k && lane < 8)
                            atomicOr(a.err, kErrTable);
                    } else {
                        y = (blk * a.Hkv + U.kvh) * a.bs + pos % a.bs;
                    }
                }
                return y;
            };
            for (int j = 0; j < U.nt && ok; ++j) {
                const uint32_t tg = jg + j;
                const int y = box_row(j);
                const int st = (int)(tg % NS);
                ok = __all_sync(FULL, mq_wait(bar(empty0 + st), ((tg / NS) & 1) ^ 1, a, abort_flag));
                if (!ok)
                    break;
                if (lane == 0)
                    mbar_arrive_expect_tx(bar(full0 + st), kTileBytes);
                __syncwarp();
                if (lane < 8 * NH && !a.inject_no_issue) {
                    const int h = lane >> 3;
                    tma_load_2d(ring + st * kTileBytes + h * kHalf + (lane & 7) * 2048, tm, h * 64, y, bar(full0 + st));
                }
                if (!a.inject_no_issue)
                    t_last[st] = (int)(tg / NS);
            }
            jg += U.nt;
            ++k;
        }
        // copies still in flight land before the CTA may exit (bounded)
        if (lane == 0) {
            if (q_issued >= 0)
                mbar_wait_bounded(bar(L::kQFull), q_issued & 1, a.wait_limit_ns);
            for (int i = 0; i < NS; ++i)
                if (t_last[i] >= 0)
                    mbar_wait_bounded(bar(full0 + i), t_last[i] & 1, a.wait_limit_ns);
        }
        __syncwarp();
    } else if (total > 0 && warp == kMqMmaWarp) {
        // ================= MMA issuer (one thread) =================
        if (lane == 0) {
            const uint32_t idesc_s = mq_idesc(BF16, kMqTile, a.negate_q != 0, false);
            const uint32_t idesc_o = mq_idesc(BF16, D, false, true);
            int k = 0;
            uint32_t jg = 0;
            bool ok = true, issued = false;
            auto issue_pv = [&](uint32_t jp, bool first) {
                const int vt = (int)(jp % VS);
                if (!mq_wait(bar(L::kPFull + (jp & 1)), (jp >> 1) & 1, a, abort_flag) ||
                    !mq_wait(bar(L::kVFull + vt), (jp / VS) & 1, a, abort_flag))
                    return false;
                tc_fence_after();
                // O_h += P_h V_h for the two 64-position halves h of the tile:
                // each softmax half keeps its own running max, so each has its
                // own accumulator (combined once per unit in the epilogue).
                // P_h sits in tensor memory over the first 32 columns of the
                // half's scores (16-bit pairs, one row per lane); a k-step of
                // 16 positions is 8 columns.
                const uint32_t p_cols = tmem + (jp & 1) * kMqTile;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int ks = 0; ks < kMqTile / 32; ++ks) {
                        const uint64_t bd =
                            smem_desc_sw128(sV + vt * kTileBytes + h * (kMqTile / 2) * 128 + ks * 2048, kHalf, 1024);
                        tc_mma_ts(tmem + kColO + h * D, p_cols + h * (kMqTile / 2) + ks * 8, bd, idesc_o,
                                  (first && ks == 0) ? 0u : 1u);
                    }
                tc_commit(bar(L::kODone));
                tc_commit(bar(L::kVEmpty + vt));
                return true;
            };
            while (ok) {
                const int slot = k & 1;
                ok = mq_wait(bar(L::kUnitFull + slot), (k >> 1) & 1, a, abort_flag);
                if (!ok)
                    break;
                const int u = misc[slot];
                mbar_arrive(bar(L::kUnitEmpty + slot));
                if (u < 0)
                    break;
                const MqUnit U = mq_unit(u, prefix, a);
                ok = mq_wait(bar(L::kQFull), k & 1, a, abort_flag);
                if (!ok)
                    break;
                for (int j = 0; j < U.nt; ++j, ++jg) {
                    const int st = (int)(jg % KS);
                    // (the score buffer of tile jg held P of tile jg - 2: the
                    // P V that read it was issued before this S, and tcgen05
                    // MMAs issued by one thread execute in issue order)
                    ok = mq_wait(bar(L::kKFull + st), (jg / KS) & 1, a, abort_flag);
                    if (!ok)
                        break;
                    tc_fence_after();
                    const uint32_t d = tmem + (jg & 1) * kMqTile;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
                        tc_mma_ss(d, smem_desc_sw128(sQ + off, 16, 1024),
                                  smem_desc_sw128(sK + st * kTileBytes + off, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit(bar(L::kSFull + (jg & 1)));
                    tc_commit(bar(L::kKEmpty + st));
                    if (j == U.nt - 1)
                        tc_commit(bar(L::kQEmpty));
                    if (j >= 1 && !(ok = issue_pv(jg - 1, j == 1)))
                        break;
                }
                if (!ok)
                    break;
                ok = issue_pv(jg - 1, U.nt == 1);
                ++k;
            }
            // every MMA issued so far completes before TMEM is released
            if (issued) {
                tc_commit(bar(L::kDrain));
                mbar_wait_bounded(bar(L::kDrain), 0, a.wait_limit_ns);
            }
        }
        __syncwarp();
    } else if (total > 0 && warp < kMqSoftmaxWarps) {
        // ================= softmax + epilogue =================
        // warp w owns rows 32 (w % 4) .. +31 (its TMEM lane quarter) and
        // half hc = w / 4 of each tile's 128 positions (64 hc .. 64 hc + 63):
        // an online softmax of its own over those positions (own running max
        // and sum) into its own accumulator O_hc.  The two halves of a row
        // meet once per unit, in the epilogue, through shared memory.
        const int q4 = warp & 3, hc = warp >> 2;
        const int r = q4 * 32 + lane;  // row = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        constexpr int HC = kMqTile / 2;  // positions per warp per tile
        constexpr int OC = D / 2;        // output columns each warp writes
        const uint32_t col_o = kColO + hc * D;  // this warp's accumulator
        const int t = r / a.G, hj = r - (r / a.G) * a.G;
        float *xb = reinterpret_cast<float *>(gbase + L::xbuf);
        uint32_t xc = 0;  // exchanges done with the partner warp
        // this warp's value for its rows -> the partner's (bounded wait)
        auto exchange = [&](float mine, float &theirs) {
            const int par = (int)(xc & 1);
            reinterpret_cast<volatile float *>(xb)[(par * 2 + hc) * kMqRows + r] = mine;
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(L::kXch + q4));
            const bool okx = __all_sync(FULL, mq_wait(bar(L::kXch + q4), xc & 1, a, abort_flag));
            ++xc;
            theirs = reinterpret_cast<volatile float *>(xb)[(par * 2 + (hc ^ 1)) * kMqRows + r];
            return okx;
        };
        int k = 0;
        uint32_t jg = 0;
        bool ok = true;
        while (ok) {
            const int slot = k & 1;
            ok = __all_sync(FULL, mq_wait(bar(L::kUnitFull + slot), (k >> 1) & 1, a, abort_flag));
            if (!ok)
                break;
            const int u = misc[slot];
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(L::kUnitEmpty + slot));
            if (u < 0)
                break;
            const MqUnit U = mq_unit(u, prefix, a);
            const int tok = U.rb * a.tpb + t;  // the row's source within the unit's (chunk token / member)
            const bool valid = r < rows_used && tok < U.n;
            int lim = U.lim_max;
            if (valid)
                lim = a.mode == kMqPrefix ? min(__ldg(a.shared + U.q0 + tok), U.lim_max) : U.ctx - U.n + tok + 1;
            // V rows at positions >= ctx are unwritten (or poisoned) slots:
            // this thread zeroes column half hc of row r of the tile's V stage
            // (0 * NaN would leak through P V)
            auto zero_v_tail = [&](int j) {
                const int pos0 = j * kMqTile;
                if (pos0 + kMqTile <= U.ctx)
                    return true;
                const int vt = (int)(jg % VS);
                if (!__all_sync(FULL, mq_wait(bar(L::kVFull + vt), (jg / VS) & 1, a, abort_flag)))
                    return false;
                if (pos0 + r >= U.ctx && hc < NH) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t addr = sV + vt * kTileBytes + hc * kHalf + r * 128 + c * 16;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
                    }
                }
                return true;
            };
            // a quarter whose 32 rows are all padding does no softmax work
            // (its rows of P and O are never read back); its warps still take
            // part in every hand-off and zero their share of the V rows
            const bool warp_active = __any_sync(FULL, valid);
            float m_ref = -INFINITY, l = 0.f;  // this half's running max (log2) and sum
            for (int j = 0; j < U.nt; ++j, ++jg) {
                ok = __all_sync(FULL, mq_wait(bar(L::kSFull + (jg & 1)), (jg >> 1) & 1, a, abort_flag));
                if (!ok)
                    break;
                tc_fence_after();
                // (S_j complete means P V of tile j - 2 is done: the arrival
                // below lands in the phase of tile j of this parity's P_full)
                const bool ragged = (j + 1) * kMqTile > U.ctx;
                if (!warp_active) {
                    if (!(ok = zero_v_tail(j)))
                        break;
                    if (ragged)
                        fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(bar(L::kPFull + (jg & 1)));
                    continue;
                }
                uint32_t sv[HC];
#pragma unroll
                for (int c = 0; c < HC / 32; ++c)
                    tmem_ld32(lane_base + (jg & 1) * kMqTile + hc * HC + c * 32,
                              *reinterpret_cast<uint32_t(*)[32]>(sv + c * 32));
                tmem_wait_ld();
                const int pos0 = j * kMqTile + hc * HC;
                if (pos0 + HC > lim) {
#pragma unroll
                    for (int i = 0; i < HC; ++i)
                        if (pos0 + i >= lim)
                            sv[i] = __float_as_uint(-INFINITY);
                }
                // row max: eight independent chains of three-input maxima
                float mxc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mxc[i] = fmaxf(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
#pragma unroll
                for (int i = 16; i < HC; i += 2)
                    mxc[(i >> 1) & 7] = fmax3(mxc[(i >> 1) & 7], __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
                const float mx = fmaxf(fmax3(mxc[0], mxc[1], mxc[2]), fmax3(mxc[3], fmax3(mxc[4], mxc[5], mxc[6]), mxc[7])) *
                                 a.scale_log2;
                const float m_new = fmaxf(m_ref, mx);
                const bool need = m_new > m_ref + kMqRescaleLog2;
                float alpha = 1.f;
                if (need) {
                    alpha = exp2f(m_ref - m_new);
                    l *= alpha;
                    m_ref = m_new;
                }
                const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;  // a half masked so far: P = 0
                // exponent arguments and row sums on packed fp32 pairs (one
                // instruction per two elements)
                uint32_t pk[HC / 2];
                const uint64_t c2 = f32x2_pack(a.scale_log2, a.scale_log2), nm2 = f32x2_pack(neg_m, neg_m);
                uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int i = 0; i < HC / 2; ++i) {
                    const float2 x = f32x2_unpack(
                        f32x2_fma(f32x2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), c2, nm2));
                    const bool poly = (i & 7) < POLY;
                    const float p0 = poly ? exp2_poly(x.x) : exp2f(x.x);
                    const float p1 = poly ? exp2_poly(x.y) : exp2f(x.y);
                    rs2[i & 3] = f32x2_add(rs2[i & 3], f32x2_pack(p0, p1));
                    pk[i] = pack2<BF16>(p0, p1);
                }
                const float2 r01 = f32x2_unpack(f32x2_add(rs2[0], rs2[1]));
                const float2 r23 = f32x2_unpack(f32x2_add(rs2[2], rs2[3]));
                l += (r01.x + r01.y) + (r23.x + r23.y);
                // O_done of the previous tile is waited at every tile (before
                // the rescale when there is one, else just before P_full's
                // arrival): S_j complete means P V of tile jg - 2 is done, and
                // P V of tile jg needs this warp's arrival, so the barrier is
                // within one phase of the one waited for, as its parity test
                // needs; the epilogue's wait for the last tile relies on it
                bool o_prev = jg == 0;
                if (j > 0 && __any_sync(FULL, need)) {
                    // the reference max moved: O_hc is rescaled once the
                    // previous tile's P V is in it
                    ok = __all_sync(FULL, mq_wait(bar(L::kODone), (jg - 1) & 1, a, abort_flag));
                    if (!ok)
                        break;
                    o_prev = true;
                    tc_fence_after();
                    {
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(lane_base + col_o + c * 32, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                            tmem_st32(lane_base + col_o + c * 32, o);
                        }
                        tmem_wait_st();
                    }
                }
                // P_hc -> tensor memory over this warp's own (already read)
                // scores: positions 64 hc .. 64 hc + 63 of row r as 32
                // columns of 16-bit pairs from column 64 hc of the buffer
                tmem_st32(lane_base + (jg & 1) * kMqTile + hc * HC, *reinterpret_cast<uint32_t(*)[32]>(pk));
                tmem_wait_st();
                if (!(ok = zero_v_tail(j)))
                    break;
                if (ragged)
                    fence_proxy_async_smem();
                if (!o_prev && !(ok = __all_sync(FULL, mq_wait(bar(L::kODone), (jg - 1) & 1, a, abort_flag))))
                    break;
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(L::kPFull + (jg & 1)));
            }
            if (!ok)
                break;
            // ---- epilogue: the two halves of each row combined,
            //   M = max(m_0, m_1), f_h = 2^(m_h - M) (0 for an empty half),
            //   out = (f_0 O_0 + f_1 O_1) / (f_0 l_0 + f_1 l_1);
            // this warp writes output columns OC hc .. OC hc + OC - 1
            if (!warp_active) {
                ++k;
                continue;
            }
            // O holds every tile once the last P V is done (the one before it
            // was waited at the last tile)
            ok = __all_sync(FULL, mq_wait(bar(L::kODone), (jg - 1) & 1, a, abort_flag));
            if (!ok)
                break;
            float m_o, l_o;
            if (!(ok = exchange(m_ref, m_o)) || !(ok = exchange(l, l_o)))
                break;
            const float m0 = hc == 0 ? m_ref : m_o, m1 = hc == 0 ? m_o : m_ref;
            const float l0 = hc == 0 ? l : l_o, l1 = hc == 0 ? l_o : l;
            const float M = fmaxf(m0, m1);
            const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M);
            const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
            const float l_row = f0 * l0 + f1 * l1;
            tc_fence_after();
            const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
            const size_t orow_idx = (size_t)(U.q0 + (valid ? tok : 0)) * a.Hq + U.kvh * a.G + hj;
            uint16_t *orow = a.out + orow_idx * D + hc * OC;
            if (a.mode == kMqPrefix && valid && hc == 0) {
                a.part_m[orow_idx] = M;
                a.part_l[orow_idx] = l_row;
            }
#pragma unroll
            for (int c = 0; c < OC / 32; ++c) {
                uint32_t o0[32], o1[32];
                tmem_ld32(lane_base + kColO + hc * OC + c * 32, o0);
                tmem_ld32(lane_base + kColO + D + hc * OC + c * 32, o1);
                tmem_wait_ld();
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    v[i] = f0 * __uint_as_float(o0[i]) + f1 * __uint_as_float(o1[i]);
                if (a.mode == kMqPrefix) {
                    // unnormalized fp32 partial, relative to 2^M
                    if (valid) {
                        float4 *dst = reinterpret_cast<float4 *>(a.part_o + orow_idx * D + hc * OC + c * 32);
#pragma unroll
                        for (int v4 = 0; v4 < 8; ++v4)
                            dst[v4] = make_float4(v[4 * v4], v[4 * v4 + 1], v[4 * v4 + 2], v[4 * v4 + 3]);
                    }
                } else if (valid) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = pack2<BF16>(v[v4 * 8 + 0] * inv, v[v4 * 8 + 1] * inv);
                        w.y = pack2<BF16>(v[v4 * 8 + 2] * inv, v[v4 * 8 + 3] * inv);
                        w.z = pack2<BF16>(v[v4 * 8 + 4] * inv, v[v4 * 8 + 5] * inv);
                        w.w = pack2<BF16>(v[v4 * 8 + 6] * inv, v[v4 * 8 + 7] * inv);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + v4 * 8) = w;
                    }
                }
            }
            tc_fence_before();
            ++k;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMqMmaWarp)
        tmem_dealloc(tmem, kTmemCols);
}

}  // namespace pkv

namespace pkv {

// Preparation of a shared-prefix decode step: one warp per sequence.  The
// sequence's group (binary search of group_start, staged in shared memory);
// the group's reference (the first member with the largest claim, each
// claim in whole blocks and cut so that the member's last position -- this
// step's token -- stays in its own blocks); the sequence's effective shared
// length (its claim, cut at the first table entry that differs from the
// reference's: 32 entries compared per round); its remaining (suffix)
// length and table offset for the decode kernel; and (every member, the same
// values) the group's reference row and KV range.  A claim that does not hold
// only shrinks the shared part, so the result stays exact.  An invalid
// group_start shares nothing and is reported.
__global__ void __launch_bounds__(256) cascade_prep_kernel(
    const int32_t *__restrict__ group_start, int NG, const int32_t *__restrict__ claimed,
    const int32_t *__restrict__ context_lens, const int32_t *__restrict__ block_tables, int64_t mb, int bs,
    int B, int32_t *group_ref, int32_t *group_len, int32_t *shared, int32_t *suffix_len, int32_t *table_off,
    int *mq_counter, unsigned *err) {
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ int gs_s[];  // group_start[0 .. NG]
    griddep_wait();
    griddep_launch_dependents();
    if (blockIdx.x == 0 && threadIdx.x == 0)
        *mq_counter = 0;
    for (int i = threadIdx.x; i <= NG; i += blockDim.x)
        gs_s[i] = __ldg(group_start + i);
    __syncthreads();
    // group_start must run from 0 to B without decreasing; otherwise nothing
    // is shared (every group length 0) and the fault is reported
    int bad = 0;
    for (int i = threadIdx.x; i <= NG; i += blockDim.x)
        bad |= (i == 0 && gs_s[0] != 0) || (i == NG && gs_s[NG] != B) || (i < NG && gs_s[i + 1] < gs_s[i]);
    if (__syncthreads_or(bad)) {
        if (threadIdx.x == 0)
            atomicOr(err, kErrContext);
        for (int i = threadIdx.x; i < NG; i += blockDim.x)
            group_len[i] = 0;
        for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < B; s += gridDim.x * blockDim.x) {
            const int c = __ldg(context_lens + s);
            const int64_t cap = mb * bs;
            shared[s] = 0;
            suffix_len[s] = c < 0 ? 0 : ((int64_t)c > cap ? (int)cap : c);
            table_off[s] = 0;
        }
        return;
    }
    const int lane = threadIdx.x & 31;
    const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (m >= B)
        return;
    const int64_t cap = mb * bs;
    auto ctx_of = [&](int s) {
        const int c = __ldg(context_lens + s);
        return c < 0 ? 0 : ((int64_t)c > cap ? (int)cap : c);
    };
    // claim in whole blocks, the sequence's last position kept private
    auto claim_blocks = [&](int s) {
        const int c = ctx_of(s);
        const int cl = __ldg(claimed + s);
        return (c < 1 || cl <= 0) ? 0 : min(cl, c - 1) / bs;
    };
    const int ctx = ctx_of(m);
    {
        const int c = __ldg(context_lens + m);
        if (lane == 0 && (c < 0 || (int64_t)c > cap))
            atomicOr(err, kErrContext);
    }
    int e = 0;  // shared blocks of m
    // the group holding m: the last g with group_start[g] <= m
    int lo = 0, hi = NG + 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (gs_s[mid] <= m)
            lo = mid + 1;
        else
            hi = mid;
    }
    const int g = lo - 1;  // valid: group_start runs from 0 to B
    {
        const int gs = gs_s[g], ge = gs_s[g + 1];
        {
            int best = -1, best_c = -1;
            for (int q = gs + lane; q < ge; q += 32) {
                const int c = claim_blocks(q);
                if (c > best_c) {
                    best_c = c;
                    best = q;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const int oc = __shfl_xor_sync(FULL, best_c, o), om = __shfl_xor_sync(FULL, best, o);
                if (oc > best_c || (oc == best_c && om >= 0 && (best < 0 || om < best))) {
                    best_c = oc;
                    best = om;
                }
            }
            const int ref = best;
            const int cb = min(claim_blocks(m), best_c);
            const int32_t *tm = block_tables + (size_t)m * mb, *tr = block_tables + (size_t)ref * mb;
            while (e < cb) {
                const int i = e + lane;
                const bool eq = i >= cb || __ldg(tm + i) == __ldg(tr + i);
                const unsigned diff = __ballot_sync(FULL, !eq);
                if (diff) {
                    e += __ffs(diff) - 1;
                    break;
                }
                e = min(cb, e + 32);
            }
            if (lane == 0) {  // every member writes the same values
                group_ref[g] = ref;
                group_len[g] = best_c * bs;
            }
        }
    }
    if (lane == 0) {
        shared[m] = e * bs;
        suffix_len[m] = ctx - e * bs;
        table_off[m] = e;
    }
}

}  // namespace pkv
