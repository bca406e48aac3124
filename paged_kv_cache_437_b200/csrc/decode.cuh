// Paged decode attention for sm_100a: append kernel, decode kernel and the
// log-sum-exp merge kernel.
//
// What is computed ("LLM Inference: KV Cache, Batching & Scheduling",
// cariara.com, sections "The KV cache" and "PagedAttention and vLLM"): for
// every sequence s and query head h, attention of q[s][h] over the keys and
// values of all cached positions 0..ctx-1, where position p lives in physical
// block block_tables[s][p / bs], row p % bs, of KV head h / G.
//
// Kernel design (B200):
//  * Work unit = (sequence, KV head, group of <= 16 query heads sharing it,
//    range of 16-token tiles).  The query heads of one KV head are the M rows
//    of an m16n8k16 tensor-core MMA, so every K/V tile is read from HBM once
//    for the whole GQA group.
//  * Persistent grid of CTAs made of independent warps.  Each warp owns a ring
//    of `stages` shared-memory stages; lane 0 issues TMA tile loads
//    (cp.async.bulk.tensor, 128-byte swizzle) of the next tiles' K and V,
//    completion tracked by one mbarrier per stage, while the warp computes on
//    the oldest stage.  The block-table indirection is resolved 32 entries at
//    a time with one coalesced load and warp shuffles.
//  * Scores S = Q K^T and O += P V with ldmatrix fragments (conflict-free
//    thanks to the swizzle) and fp32 accumulation; the S accumulator layout is
//    reused directly as the A operand of the P V product.  Online softmax in
//    the log2 domain (scale * log2(e) folded into one multiply, exp2f).
//  * Three schedules: one unit per (sequence, KV head group) ("direct"),
//    fixed P-token partitions with a log-sum-exp merge ("partition"), and a
//    work-balanced split in which every warp gets the same number of tiles of
//    the flattened (sequence, head group, tile) sequence ("balanced"); split
//    pieces are merged by log-sum-exp in a second kernel.
//  * Every reduction runs in logical-position order, so results do not
//    depend on which physical blocks hold the data.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>
#include <cstdint>

#include "ptx.cuh"

namespace pkv {

constexpr int kTileTokens = 16;                        // tokens per MMA k-step / TMA box rows
constexpr int kBoxCols = 64;                           // 16-bit elements per box row (128 B)
constexpr int kBoxBytes = kBoxCols * 2 * kTileTokens;  // 2048
constexpr int kMaxRows = 16;                           // max query heads per unit (MMA N, 1 or 2 n-tiles)
constexpr uint64_t kWaitLimitNs = 2000000000ull;       // 2 s bound on every wait

// device error word bits
constexpr unsigned kErrTable = 1u;    // block-table entry outside [0, NB)
constexpr unsigned kErrContext = 2u;  // context length < 0 or > MB * bs
constexpr unsigned kErrSlot = 4u;     // append slot outside the pool
constexpr unsigned kErrTimeout = 8u;  // a bounded wait gave up

enum DecodeMode : int { kModeDirect = 0, kModePartition = 1, kModeBalanced = 2 };

struct DecodeArgs {
    const uint16_t *q;             // [B][Hq][D]
    uint16_t *out;                 // [B][Hq][D]
    const int32_t *block_tables;   // [B][MB]
    const int32_t *context_lens;   // [B]
    int64_t mb;                    // MB
    int64_t nb;                    // NB
    int B, Hq, Hkv, G, n_hg, npairs, bs;  // n_hg = ceil(G / heads per unit)
    float scale_log2;              // scale * log2(e)
    int mode;
    int part_tiles;                // partition mode: tiles per partition
    int S;                         // partition mode: partitions per sequence (layout)
    float *part_o;                 // partials (see the workspace layout on the host)
    float *part_m;
    float *part_l;
    int32_t *prefix_out;           // balanced: tile prefix for the merge kernel
    // balanced: one counter per (sequence, head group), zero at launch; the
    // warp that finishes the last piece of a split row merges it (no merge
    // kernel).  Null: the merge kernel does it.
    int *fold_cnt;
    // balanced: every (sequence, head group) with work weighs its tiles plus
    // unit_cost virtual tiles at the end of its range (nothing is computed
    // there), so that a warp given many short units gets fewer tiles: a unit
    // costs a query load, a resume and an epilogue beside its tiles
    int unit_cost;
    int total_warps;
    int stages;
    unsigned *err;
    uint64_t wait_limit_ns;        // bound on every mbarrier wait
    int inject_no_issue;           // testing: issue no copies so that waits run out
    // fused append (pkv_append_decode_attention), all null otherwise: token s
    // is sequence s's new token, at position context_lens[s] - 1, slot slots[s]
    const uint16_t *k_new;         // [B][Hkv][D]
    const uint16_t *v_new;
    const int64_t *slots;          // [B], < 0: no append for that sequence
    uint16_t *k_cache, *v_cache;   // the pools, for the generic-store append
    int64_t pool_slots;            // NB * bs
    // E4M3 pools: one fp32 scale per (slot, KV head), [NB][Hkv][bs]
    const float *k_scales, *v_scales;
    // chunked prefill: "sequence" s reads block-table row table_rows[s]
    // (several query tokens of one sequence share its row); null = row s
    const int32_t *table_rows;
    // shared-prefix cascade (16-bit MMA path): sequence s starts
    // table_offset[s] entries into its table row (its positions before that
    // were attended by the shared-prefix kernel), and a unit that starts a
    // row with table_offset[s] > 0 resumes from that kernel's fp32 partial
    // (init_o [B][Hq][D] relative to 2^init_m, init_l; log2 domain); null = none
    const int32_t *table_offset;
    const float *init_o, *init_m, *init_l;
};

struct SmemLayout {
    int prefix_off, ctx_off, bar_off, ring_off, total;
};

__host__ __device__ inline int align_up_int(int x, int a) { return (x + a - 1) / a * a; }

// Bytes of one pipeline stage: a 16-token K tile and V tile (16-bit), or
// for the E4M3 cache the 1-byte tiles plus their 16 K and 16 V row scales.
__host__ __device__ inline int decode_stage_bytes(int D, bool fp8) {
    return fp8 ? 2 * kTileTokens * D + 2 * kTileTokens * 4 : 2 * kTileTokens * D * 2;
}

// Per-warp region (1024-aligned, for the swizzle): its ring of stages; for
// E4M3 the stages' code tiles come first (2*16*D bytes each, so every tile
// stays aligned to its swizzle span) and their scales after them.
// CUDA-core variant: per warp the unit's query rows in fp32 ([8][D + 8], the
// two column halves 16 bytes apart) and one tile's probabilities ([16][8]).
__host__ __device__ inline int decode_fma_bytes(int D) { return 8 * (D + 8) * 4 + kTileTokens * 8 * 4; }

__host__ __device__ inline int decode_warp_bytes(int D, int stages, bool fp8, bool fma = false) {
    return align_up_int(stages * decode_stage_bytes(D, fp8) + (fma ? decode_fma_bytes(D) : 0), 1024);
}

// Byte offset inside a 16-row E4M3 tile as the TMA wrote it: rows of D bytes
// with the 16-byte chunks XOR-swizzled by address bits 7.. (128-byte swizzle
// for D = 128, 64-byte swizzle for D = 64).
template <int D>
__device__ __forceinline__ uint32_t e4m3_swz(uint32_t off) {
    return D == 128 ? off ^ (((off >> 7) & 7u) << 4) : off ^ (((off >> 7) & 3u) << 4);
}

__host__ __device__ inline SmemLayout decode_smem_layout(int B, int warps, int stages, int D,
                                                         bool need_prefix, bool fp8 = false, bool fma = false) {
    SmemLayout L;
    const int prefix_bytes = need_prefix ? (B + 1) * 4 : 0;
    const int ctx_bytes = need_prefix ? B * 4 : 0;
    L.prefix_off = 0;
    L.ctx_off = prefix_bytes;
    L.bar_off = align_up_int(prefix_bytes + ctx_bytes, 16);
    L.ring_off = align_up_int(L.bar_off + warps * stages * 8, 1024);
    // + 1024: the dynamic smem base is re-aligned to 1024 B at run time
    L.total = L.ring_off + warps * decode_warp_bytes(D, stages, fp8, fma) + 1024;
    return L;
}

__device__ __forceinline__ int ceil_div_i(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int clamp_ctx(int c, const DecodeArgs &a) {
    const int64_t cap = a.mb * a.bs;
    if (c < 0 || c > cap) {
        atomicOr(a.err, kErrContext);
        return c < 0 ? 0 : (int)cap;
    }
    return c;
}

// first index i in [0, n) with a[i] > x, n if none (a non-decreasing)
__device__ __forceinline__ int upper_bound_i(const int *a, int n, long long x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((long long)a[mid] <= x)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

// ------------------------------------------------------------- work walker

struct Seg {
    int seq, pair, t0, t1, ctx, dest;  // dest < 0: final output, else partial index
    int trow;                          // block-table row of the sequence
    int toff;                          // entries of that row to skip
};

struct Walker {
    long long u;    // direct / partition: next unit; balanced: current position
    long long lo, hi;
    int seq, pair, t;
};

__device__ __forceinline__ long long range_lo(long long w, long long T, long long W) {
    return w * T / W;
}

__device__ __forceinline__ void walker_init(Walker &w, const DecodeArgs &a, const int *prefix,
                                            int gw) {
    w.u = gw;
    w.lo = w.hi = 0;
    w.seq = w.pair = w.t = 0;
    if (a.mode == kModeBalanced) {
        const long long T = (long long)prefix[a.B] * a.npairs;
        w.lo = range_lo(gw, T, a.total_warps);
        w.hi = range_lo(gw + 1, T, a.total_warps);
        w.u = w.lo;
        if (w.lo < w.hi) {
            // the range may start in a pair's virtual tail: the walker skips it
            int s = upper_bound_i(prefix, a.B + 1, w.lo / a.npairs) - 1;
            const int ws = prefix[s + 1] - prefix[s];
            const long long r = w.lo - (long long)prefix[s] * a.npairs;
            w.seq = s;
            w.pair = (int)(r / ws);
            w.t = (int)(r % ws);
        }
    }
}

// balanced: from the end of a pair's span to the start of the next pair with work
__device__ __forceinline__ void walker_next_pair(Walker &w, const DecodeArgs &a, const int *prefix) {
    w.t = 0;
    if (++w.pair == a.npairs) {
        w.pair = 0;
        ++w.seq;
        while (w.seq < a.B && prefix[w.seq + 1] == prefix[w.seq])
            ++w.seq;
    }
}

__device__ __forceinline__ bool walker_next_raw(Walker &w, Seg &sg, const DecodeArgs &a,
                                                const int *prefix, const int *ctxs, int gw);

__device__ __forceinline__ bool walker_next(Walker &w, Seg &sg, const DecodeArgs &a,
                                            const int *prefix, const int *ctxs, int gw) {
    const bool has = walker_next_raw(w, sg, a, prefix, ctxs, gw);
    if (has) {
        sg.trow = a.table_rows ? __ldg(a.table_rows + sg.seq) : sg.seq;
        sg.toff = a.table_offset ? __ldg(a.table_offset + sg.seq) : 0;
    }
    return has;
}

__device__ __forceinline__ bool walker_next_raw(Walker &w, Seg &sg, const DecodeArgs &a,
                                                const int *prefix, const int *ctxs, int gw) {
    if (a.mode == kModeDirect) {
        if (w.u >= (long long)a.B * a.npairs)
            return false;
        sg.seq = (int)(w.u / a.npairs);
        sg.pair = (int)(w.u % a.npairs);
        sg.ctx = clamp_ctx(__ldg(a.context_lens + sg.seq), a);
        sg.t0 = 0;
        sg.t1 = ceil_div_i(sg.ctx, kTileTokens);
        sg.dest = -1;
        w.u += a.total_warps;
        return true;
    }
    if (a.mode == kModePartition) {
        if (w.u >= (long long)prefix[a.B] * a.npairs)
            return false;
        const long long qidx = w.u / a.npairs;
        sg.pair = (int)(w.u % a.npairs);
        const int s = upper_bound_i(prefix, a.B + 1, qidx) - 1;
        const int j = (int)(qidx - prefix[s]);
        const int nparts = prefix[s + 1] - prefix[s];
        sg.seq = s;
        sg.ctx = ctxs[s];
        const int nt = ceil_div_i(sg.ctx, kTileTokens);
        sg.t0 = j * a.part_tiles;
        sg.t1 = min(nt, sg.t0 + a.part_tiles);
        sg.dest = nparts == 1 ? -1 : j;
        w.u += a.total_warps;
        return true;
    }
    // balanced: pair p of sequence s spans ws = nt + unit_cost positions of
    // the flattened order, its nt real tiles first
    for (;;) {
        if (w.u >= w.hi)
            return false;
        const int ws = prefix[w.seq + 1] - prefix[w.seq];
        const int nt = ws - a.unit_cost;
        if (w.t >= nt) {
            // a range that starts in a pair's virtual tail: step over it
            w.u += ws - w.t;
            walker_next_pair(w, a, prefix);
            continue;
        }
        sg.seq = w.seq;
        sg.pair = w.pair;
        sg.ctx = ctxs[w.seq];
        sg.t0 = w.t;
        sg.t1 = (int)min((long long)nt, (long long)w.t + (w.hi - w.u));
        const long long pair_start = (long long)prefix[w.seq] * a.npairs + (long long)w.pair * ws;
        const bool complete = (sg.t0 == 0 && sg.t1 == nt);
        sg.dest = complete ? -1 : 2 * gw + (pair_start < w.lo ? 0 : 1);
        w.u += sg.t1 - sg.t0;
        w.t = sg.t1;
        if (w.t == nt) {
            w.u += ws - nt;
            walker_next_pair(w, a, prefix);
        }
        return true;
    }
}

// ------------------------------------------------------------- conversions

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (BF16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    } else {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
}

// Two 16-bit values (low half first) -> two floats (exact).
template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t w) {
    if constexpr (BF16) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    } else {
        __half2 h = *reinterpret_cast<__half2 *>(&w);
        return __half22float2(h);
    }
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts_f4(uint32_t addr, float x, float y, float z, float w) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(x), "f"(y), "f"(z), "f"(w) : "memory");
}

// ------------------------------------------------------------- merging split rows
// (used by the merge kernel and by the decode kernel's last piece of a row)

struct MergeArgs {
    uint16_t *out;
    const int32_t *context_lens;
    const int32_t *prefix;   // balanced: tile prefix written by the decode kernel
    const float *part_o, *part_m, *part_l;
    int64_t mb;
    int B, Hq, G, n_hg, npairs, bs;
    int hpu;                 // query heads per decode unit (8 or 16)
    int mode, part_tiles, S, total_warps;
    int unit_cost;           // balanced: virtual tiles per pair (decode kernel's)
};

// Balanced: where pair `pair` of sequence `seq` sits in the flattened order:
// its first position a0 and its real tiles nt (0: no work), the pair's span
// being nt + unit_cost positions.
__device__ __forceinline__ void pair_span(const int32_t *prefix, int seq, int pair, int npairs, int unit_cost,
                                          long long &a0, int &nt) {
    const int ws = prefix[seq + 1] - prefix[seq];
    nt = ws > 0 ? ws - unit_cost : 0;
    a0 = (long long)prefix[seq] * npairs + (long long)pair * ws;
}
// Balanced mode: prefix[B + 1] holds an upper bound on the pieces per row;
// partition mode: S is the bound.

constexpr int kMergeThreads = 128;
constexpr int kMergeWideThreads = 512;  // one row per CTA, many pieces per row

template <int NTH>
__device__ __forceinline__ float block_reduce(float v, bool is_max, float *red) {
    constexpr unsigned FULL = 0xffffffffu;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float x = __shfl_xor_sync(FULL, v, o);
        v = is_max ? fmaxf(v, x) : v + x;
    }
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0)
        red[warp] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < NTH / 32; ++w)
        r = is_max ? fmaxf(r, red[w]) : r + red[w];
    __syncthreads();
    return r;
}

// Where the pieces of one query head's split context are.
struct MergeRow {
    int seq, h, g;
    long long count;   // pieces; <= 1 means nothing to merge
    long long first;   // balanced: first warp
    long long a0, T;   // balanced: flattened start of the pair, total tiles
};

__device__ __forceinline__ MergeRow merge_row(const MergeArgs &a, long long row) {
    MergeRow r;
    r.seq = (int)(row / a.Hq);
    r.h = (int)(row - (long long)r.seq * a.Hq);
    const int kvh = r.h / a.G;
    const int hl = r.h - kvh * a.G;
    const int hg = hl / a.hpu;
    r.g = hl - hg * a.hpu;
    const int pair = kvh * a.n_hg + hg;
    r.first = 0;
    r.a0 = 0;
    r.T = 1;
    if (a.mode == kModePartition) {
        int c = a.context_lens[r.seq];
        const int64_t cap = a.mb * a.bs;
        c = c < 0 ? 0 : (c > cap ? (int)cap : c);
        const int nt = (c + kTileTokens - 1) / kTileTokens;
        r.count = (nt + a.part_tiles - 1) / a.part_tiles;  // <= 1: written by the decode kernel
    } else {
        int nt;
        pair_span(a.prefix, r.seq, pair, a.npairs, a.unit_cost, r.a0, nt);
        r.count = 0;
        if (nt > 0) {
            r.T = (long long)a.prefix[a.B] * a.npairs;
            const long long W = a.total_warps;
            r.first = ((r.a0 + 1) * W + r.T - 1) / r.T - 1;                 // warp holding a0
            const long long last = ((r.a0 + nt) * W + r.T - 1) / r.T - 1;  // warp holding a0+nt-1
            r.count = last - r.first + 1;  // 1: the pair sat in one warp, already final
        }
    }
    return r;
}

// Partial row of piece k, or -1 (a warp whose range is empty).
__device__ __forceinline__ long long merge_piece(const MergeArgs &a, const MergeRow &r, long long k) {
    if (a.mode == kModePartition)
        return ((long long)r.seq * a.Hq + r.h) * a.S + k;
    const long long w = r.first + k;
    if (r.T >= a.total_warps) {
        // no warp has an empty range: the first piece is the first warp's
        // last segment (slot 1), every later piece its warp's first (slot 0)
        return (2 * w + (k == 0 ? 1 : 0)) * kMaxRows + r.g;
    }
    const long long lo = w * r.T / a.total_warps;
    const long long hi = (w + 1) * r.T / a.total_warps;
    if (lo >= hi)
        return -1;
    return (2 * w + (r.a0 < lo ? 0 : 1)) * kMaxRows + r.g;
}

template <int D, bool BF16>
__device__ __forceinline__ void store_row(const MergeArgs &a, const MergeRow &r, int c, const float *v,
                                          int n) {
    uint32_t *dst = reinterpret_cast<uint32_t *>(a.out + ((size_t)r.seq * a.Hq + r.h) * D + c);
    for (int i = 0; i < n / 2; ++i)
        dst[i] = pack2<BF16>(v[2 * i], v[2 * i + 1]);
}

// All `rows` query heads of one split (sequence, head group) merged by one
// warp at once: the heads share their pieces (the same warps computed them),
// and a piece's rows are contiguous (partial row base + g).  Lane l takes head
// g = l / (32 / rp) (rp = rows rounded up to a power of two) and D / (32 / rp)
// of its columns, 16 at a time.  First pass: each head's M over the pieces;
// second: weights 2^(m_k - M) and the weighted sums.  Every load of a pass
// is independent, so the merge costs two or three memory round trips instead
// of one per piece batch per head.
constexpr int kPairMergeMaxPieces = 16;

template <int D, bool BF16>
__device__ __forceinline__ void merge_pair_warp(const MergeArgs &a, const MergeRow &r0, int rows) {
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int CH = 16;  // columns per lane per pass
    const int lane = threadIdx.x & 31;
    int rp = 1;
    while (rp < rows)
        rp <<= 1;
    const int lpr = 32 / rp;          // lanes per head
    const int g = lane / lpr;
    const int cpl = D / lpr;          // columns per lane (>= 4)
    const int c_lane = (lane - g * lpr) * cpl;
    const bool on = g < rows;
    const int n = (int)r0.count;
    // piece k's partial row base (of head 0 of the group), -1 for an empty piece
    long long base[kPairMergeMaxPieces];
#pragma unroll
    for (int k = 0; k < kPairMergeMaxPieces; ++k)
        base[k] = k < n ? merge_piece(a, r0, k) - r0.g : -1;
    float mk[kPairMergeMaxPieces];
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kPairMergeMaxPieces; ++k) {
        mk[k] = (on && base[k] >= 0) ? a.part_m[base[k] + g] : -INFINITY;
        M = fmaxf(M, mk[k]);
    }
    float L = 0.f;
#pragma unroll
    for (int k = 0; k < kPairMergeMaxPieces; ++k) {
        mk[k] = mk[k] == -INFINITY ? 0.f : exp2f(mk[k] - M);  // the piece's weight
        if (mk[k] != 0.f)
            L = fmaf(mk[k], a.part_l[base[k] + g], L);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    MergeRow rg = r0;
    rg.h = r0.h + g;
    for (int c0 = 0; c0 < cpl; c0 += CH) {
        const int nc = cpl - c0 < CH ? cpl - c0 : CH;  // 4, 8 or 16
        float acc[CH];
#pragma unroll
        for (int i = 0; i < CH; ++i)
            acc[i] = 0.f;
#pragma unroll
        for (int k = 0; k < kPairMergeMaxPieces; ++k) {
            if (mk[k] == 0.f)
                continue;
            const float4 *src = reinterpret_cast<const float4 *>(a.part_o + (base[k] + g) * D + c_lane + c0);
#pragma unroll
            for (int i = 0; i < CH / 4; ++i) {
                if (4 * i < nc) {
                    const float4 x = src[i];
                    acc[4 * i] = fmaf(mk[k], x.x, acc[4 * i]);
                    acc[4 * i + 1] = fmaf(mk[k], x.y, acc[4 * i + 1]);
                    acc[4 * i + 2] = fmaf(mk[k], x.z, acc[4 * i + 2]);
                    acc[4 * i + 3] = fmaf(mk[k], x.w, acc[4 * i + 3]);
                }
            }
        }
        if (on) {
#pragma unroll
            for (int i = 0; i < CH; ++i)
                acc[i] *= inv;
            store_row<D, BF16>(a, rg, c_lane + c0, acc, nc);
        }
    }
    __syncwarp(FULL);
}

constexpr int kWarpPieces = 64;  // rows with at most this many pieces: one warp each

// One warp merges one row, kWarpBatch pieces at a time (rescaled online
// across batches).  A piece's output row does not depend on its weight, so
// each batch issues every load at once: lane j < kWarpBatch fetches piece
// j's (m, l), every lane its D/32 columns of all the batch's outputs; the
// reductions are shuffles.  One memory round trip per batch.
constexpr int kWarpBatch = 16;

template <int D, bool BF16, int kWarpBatch = kWarpBatch>
__device__ __forceinline__ void merge_row_warp(const MergeArgs &a, const MergeRow &r) {
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int VEC = D / 32;
    const int lane = threadIdx.x & 31;
    float M = -INFINITY, L = 0.f;
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i)
        acc[i] = 0.f;
    for (long long k0 = 0; k0 < r.count; k0 += kWarpBatch) {
        const long long kl = k0 + lane;
        const long long rl = (lane < kWarpBatch && kl < r.count) ? merge_piece(a, r, kl) : -1;
        const float ml = rl >= 0 ? a.part_m[rl] : -INFINITY;
        const float ll = rl >= 0 ? a.part_l[rl] : 0.f;
        float v[kWarpBatch][VEC];
#pragma unroll
        for (int j = 0; j < kWarpBatch; ++j) {
            const long long rr = __shfl_sync(FULL, rl, j);
#pragma unroll
            for (int i = 0; i < VEC; ++i)
                v[j][i] = 0.f;
            if (rr >= 0) {  // an empty piece (-1) has no row
                const float *p = a.part_o + rr * D + lane * VEC;
                if constexpr (VEC == 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(p);
                    v[j][0] = x.x;
                    v[j][1 % VEC] = x.y;
                    v[j][2 % VEC] = x.z;
                    v[j][3 % VEC] = x.w;
                } else {
                    const float2 x = *reinterpret_cast<const float2 *>(p);
                    v[j][0] = x.x;
                    v[j][1 % VEC] = x.y;
                }
            }
        }
        float cm = ml;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            cm = fmaxf(cm, __shfl_xor_sync(FULL, cm, o));
        const float mnew = fmaxf(M, cm);
        const float rescale = M == -INFINITY ? 0.f : exp2f(M - mnew);
        const float w = ml == -INFINITY ? 0.f : exp2f(ml - mnew);
        float lsum = w * ll;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            lsum += __shfl_xor_sync(FULL, lsum, o);
        L = L * rescale + lsum;
        M = mnew;
#pragma unroll
        for (int i = 0; i < VEC; ++i)
            acc[i] *= rescale;
#pragma unroll
        for (int j = 0; j < kWarpBatch; ++j) {
            const float wj = __shfl_sync(FULL, w, j);
#pragma unroll
            for (int i = 0; i < VEC; ++i)
                acc[i] = wj != 0.f ? fmaf(wj, v[j][i], acc[i]) : acc[i];
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int i = 0; i < VEC; ++i)
        acc[i] *= inv;
    store_row<D, BF16>(a, r, lane * VEC, acc, VEC);
}

// ------------------------------------------------------------- decode kernel

// BF16: q / out are bf16 (else f16).  FP8: the pools hold E4M3 codes with one
// fp32 scale per (slot, KV head); tiles are converted exactly to f16 in
// shared memory and the MMAs run in f16 (a bf16 query is converted to f16,
// exact in f16's normal range); K scales multiply the scores, V scales the
// probabilities.
// CAS: the shared-prefix cascade (table offsets, resume from a partial);
// compiled separately so that the plain decode is unchanged by it.
template <int D, bool BF16, int NT, bool FP8 = false, bool FMA = false, bool CAS = false>
__global__ void __launch_bounds__(256) paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV,
                                                           const DecodeArgs a) {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(!FMA || (!FP8 && NT == 1), "the CUDA-core variant: 16-bit pools, 8 heads per unit");
    static_assert(!CAS || (!FP8 && !FMA), "the cascade resumes 16-bit MMA accumulators");
    constexpr int kTile = kTileTokens * D * 2;  // bytes of one 16-bit K (or V) tile
    constexpr int kMT = D / 16;                 // k-steps of Q K^T == 16-row d tiles of P V
    constexpr int HPU = 8 * NT;                 // query heads per unit (MMA N)
    constexpr bool MMA_BF16 = FP8 ? false : BF16;
    // stage stride: the E4M3 stages hold only the code tiles (scales apart)
    constexpr int kStage = FP8 ? 2 * kTileTokens * D : 2 * kTile;
    constexpr int KW8 = FP8 ? D / 16 : 1;  // E4M3: words of one K row a lane reads
    constexpr int VW8 = FP8 ? D / 32 : 1;  // E4M3: words of one V row a lane reads
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    const int warps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * warps + warp;
    const bool need_prefix = a.mode != kModeDirect;
    const SmemLayout L = decode_smem_layout(a.B, warps, a.stages, D, need_prefix, FP8, FMA);
    int *prefix = reinterpret_cast<int *>(smem_raw + L.prefix_off);
    int *ctxs = reinterpret_cast<int *>(smem_raw + L.ctx_off);
    const uint32_t smem_base = smem_addr(smem_raw);
    const uint32_t bar_base = smem_base + L.bar_off + warp * a.stages * 8;
    const uint32_t warp_base = ((smem_base + L.ring_off + 1023u) & ~1023u) +
                               (uint32_t)(warp * decode_warp_bytes(D, a.stages, FP8, FMA));
    const uint32_t ring_base = warp_base;
    // E4M3: per stage 16 K scales then 16 V scales, after all the code tiles
    const uint32_t scale_base = ring_base + a.stages * kStage;
    // CUDA-core variant: query rows and probabilities, after the stages
    constexpr int kQS = D + 8;  // fp32 row stride of the staged query rows
    constexpr int FD = D / 32;  // output columns per lane
    const uint32_t fq_base = ring_base + a.stages * kStage;
    const uint32_t fp_base = fq_base + 8 * kQS * 4;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (lane == 0) {
        for (int s = 0; s < a.stages; ++s)
            mbar_init(bar_base + s * 8, 1);
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    // everything above overlaps the previous kernel (the append); every read
    // of an input comes after this point
    griddep_wait();
    griddep_launch_dependents();

    // ---- schedule prologue: per-sequence unit counts and their prefix sums
    if (need_prefix) {
        const int nthreads = blockDim.x;
        const int per = (a.B + nthreads - 1) / nthreads;
        const int beg = min(a.B, threadIdx.x * per);
        const int end = min(a.B, beg + per);
        int local = 0;
        for (int s = beg; s < end; ++s) {
            const int c = clamp_ctx(__ldg(a.context_lens + s), a);
            ctxs[s] = c;
            const int nt = ceil_div_i(c, kTileTokens);
            local += a.mode == kModeBalanced ? (nt > 0 ? nt + a.unit_cost : 0) : ceil_div_i(nt, a.part_tiles);
        }
        // block-wide exclusive scan of `local`
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(FULL, incl, o);
            if (lane >= o)
                incl += v;
        }
        __shared__ int warp_tot[32];
        if (lane == 31)
            warp_tot[warp] = incl;
        __syncthreads();
        int base = 0;
        for (int w = 0; w < warp; ++w)
            base += warp_tot[w];
        int run = base + incl - local;
        for (int s = beg; s < end; ++s) {
            prefix[s] = run;
            const int nt = ceil_div_i(ctxs[s], kTileTokens);
            run += a.mode == kModeBalanced ? (nt > 0 ? nt + a.unit_cost : 0) : ceil_div_i(nt, a.part_tiles);
        }
        if (threadIdx.x == 0) {
            int tot = 0;
            for (int w = 0; w < warps; ++w)
                tot += warp_tot[w];
            prefix[a.B] = tot;
        }
    }
    __syncthreads();

    if (need_prefix) {
        // sequences with no context: their output rows are all zero
        for (int s = blockIdx.x; s < a.B; s += gridDim.x) {
            if (ctxs[s] != 0)
                continue;
            if (CAS && __ldg(a.table_offset + s) > 0) {
                // nothing after the shared prefix: its partial, normalized
                uint32_t *o = reinterpret_cast<uint32_t *>(a.out + (size_t)s * a.Hq * D);
                for (int i = threadIdx.x; i < a.Hq * D / 2; i += blockDim.x) {
                    const size_t row = (size_t)s * a.Hq + (2 * i) / D;
                    const float l = __ldg(a.init_l + row);
                    const float inv = l > 0.f ? 1.f / l : 0.f;
                    const float2 v = __ldg(reinterpret_cast<const float2 *>(a.init_o + row * D) + (i % (D / 2)));
                    o[i] = pack2<BF16>(v.x * inv, v.y * inv);
                }
                continue;
            }
            uint4 *o = reinterpret_cast<uint4 *>(a.out + (size_t)s * a.Hq * D);
            const int n = a.Hq * D / 8;
            for (int i = threadIdx.x; i < n; i += blockDim.x)
                o[i] = make_uint4(0, 0, 0, 0);
        }
        if (a.mode == kModeBalanced && blockIdx.x == 0) {
            // the merge kernel reads the schedule back, plus an upper bound
            // on the pieces any (sequence, head group) is split into
            __shared__ int s_ntmax;
            if (threadIdx.x == 0)
                s_ntmax = 0;
            __syncthreads();
            int ntmax = 0;
            for (int i = threadIdx.x; i <= a.B; i += blockDim.x) {
                a.prefix_out[i] = prefix[i];
                if (i < a.B)
                    ntmax = max(ntmax, prefix[i + 1] - prefix[i]);
            }
            atomicMax(&s_ntmax, ntmax);
            __syncthreads();
            if (threadIdx.x == 0) {
                // nt consecutive tiles touch at most ceil(nt * W / T) + 1 warps
                // (empty-range warps in between included)
                const long long T = max((long long)prefix[a.B] * a.npairs, 1LL);
                const long long W = a.total_warps;
                const long long bound = ((long long)s_ntmax * W + T - 1) / T + 1;
                a.prefix_out[a.B + 1] = (int)min(bound, (long long)INT_MAX);
            }
        }
    }

    const int c4 = lane & 3;   // thread-in-quad (MMA column pair)
    const int g8 = lane >> 2;  // quad index (MMA row)

    // ---- producer state (whole warp runs it; lane 0 issues the copies)
    Walker pw;
    Seg ps;
    walker_init(pw, a, prefix, gw);
    bool p_has = walker_next(pw, ps, a, prefix, ctxs, gw);
    while (p_has && ps.t0 >= ps.t1)
        p_has = walker_next(pw, ps, a, prefix, ctxs, gw);
    if (a.inject_no_issue)
        p_has = false;
    int p_t = p_has ? ps.t0 : 0;
    int tb_seq = -1, tb_base = 0, tb_val = 0;  // lane i caches table entry tb_base + i
    int nx_seq = -1, nx_base = 0, nx_val = 0;  // the same, prefetched for the next unit
    int issued = 0;

    // Start loading the first 32 table entries of the unit after the current
    // one, so that entering it does not stall the warp on a dependent load.
    auto prefetch_next_chunk = [&]() {
        Walker tmp = pw;
        Seg ns;
        bool has = walker_next(tmp, ns, a, prefix, ctxs, gw);
        while (has && ns.t0 >= ns.t1)
            has = walker_next(tmp, ns, a, prefix, ctxs, gw);
        nx_seq = -1;
        if (has) {
            const int lb = ns.t0 * kTileTokens / a.bs;
            const int nblk = ceil_div_i(ns.ctx, a.bs);
            nx_seq = ns.seq;
            nx_base = lb;
            nx_val = (lb + lane < nblk) ? __ldg(a.block_tables + (size_t)ns.trow * a.mb + (CAS ? ns.toff : 0) + lb + lane) : 0;
        }
    };
    // set when the producer enters a unit; the prefetch for the unit after it
    // is issued once this unit's own first chunk is in hand
    bool want_prefetch = p_has;

    auto issue = [&](int stage) {
        const int pos0 = p_t * kTileTokens;
        const int lb = pos0 / a.bs;
        const int row0 = pos0 - lb * a.bs;
        if (ps.seq != tb_seq || lb < tb_base || lb >= tb_base + 32) {
            tb_seq = ps.seq;
            tb_base = lb;
            if (ps.seq == nx_seq && lb == nx_base) {
                tb_val = nx_val;
                nx_seq = -1;
            } else {
                const int nblk = ceil_div_i(ps.ctx, a.bs);
                tb_val = (lb + lane < nblk) ? __ldg(a.block_tables + (size_t)ps.trow * a.mb + (CAS ? ps.toff : 0) + lb + lane) : 0;
            }
        }
        if (want_prefetch) {
            want_prefetch = false;
            prefetch_next_chunk();
        }
        int blk = __shfl_sync(FULL, tb_val, lb - tb_base);
        if (blk < 0 || (int64_t)blk >= a.nb) {
            if (lane == 0)
                atomicOr(a.err, kErrTable);
            blk = 0;  // read a valid block; the result is flagged as wrong
        }
        const int kvh = ps.pair / a.n_hg;
        const int y = (blk * a.Hkv + kvh) * a.bs + row0;
        if (lane == 0) {
            const uint32_t bar = bar_base + stage * 8;
            const uint32_t kdst = ring_base + stage * kStage;
            if constexpr (FP8) {
                // 1-byte tiles (one swizzled box of 16 rows x D bytes each)
                // and the tile's 16 K and 16 V scales (64 contiguous bytes each)
                const uint32_t sdst = scale_base + stage * (4 * kTileTokens * 2);
                mbar_arrive_expect_tx(bar, kStage + 2 * kTileTokens * 4);
                tma_load_2d(kdst, &tmK, 0, y, bar);
                tma_load_2d(kdst + kTileTokens * D, &tmV, 0, y, bar);
                bulk_load(sdst, a.k_scales + y, kTileTokens * 4, bar);
                bulk_load(sdst + kTileTokens * 4, a.v_scales + y, kTileTokens * 4, bar);
            } else {
                mbar_arrive_expect_tx(bar, 2 * kTile);
#pragma unroll
                for (int h = 0; h < D / kBoxCols; ++h) {
                    tma_load_2d(kdst + h * kBoxBytes, &tmK, h * kBoxCols, y, bar);
                    tma_load_2d(kdst + kTile + h * kBoxBytes, &tmV, h * kBoxCols, y, bar);
                }
            }
        }
        ++issued;
        if (++p_t >= ps.t1) {
            do {
                p_has = walker_next(pw, ps, a, prefix, ctxs, gw);
            } while (p_has && ps.t0 >= ps.t1);
            p_t = p_has ? ps.t0 : 0;
            want_prefetch = p_has;
        }
    };

    for (int s = 0; s < a.stages && p_has; ++s)
        issue(s);

    // ---- consumer
    // Per 16-token tile, with the tokens as the M rows of the MMA:
    //   S^T[16 tok][HPU heads] = K[16 tok][D] * Q^T[D][HPU]         (kMT k-steps)
    //   O^T[D][HPU]          += V^T[D][16 tok] * P^T[16 tok][HPU]   (kMT m-tiles)
    // P^T comes out of the first product in accumulator layout; one movmatrix
    // per 8x8 block turns it into the B operand of the second.
    Walker cw;
    Seg cs;
    walker_init(cw, a, prefix, gw);
    uint32_t phases = 0;
    int stage = 0;
    int consumed = 0;
    bool failed = false;

    while (!failed && walker_next(cw, cs, a, prefix, ctxs, gw)) {
        const int kvh = cs.pair / a.n_hg;
        const int hg = cs.pair - kvh * a.n_hg;
        const int h0 = kvh * a.G + hg * HPU;
        const int rows = min(HPU, a.G - hg * HPU);

        // Q^T as the B operand (k = head dim, n = query head)
        uint32_t qb[NT][kMT][2];
#pragma unroll
        for (int nt = 0; nt < (FMA ? 0 : NT); ++nt) {
            const int head = nt * 8 + g8;
            const bool valid = head < rows;
            const uint32_t *qr =
                reinterpret_cast<const uint32_t *>(a.q + ((size_t)cs.seq * a.Hq + h0 + (valid ? head : 0)) * D);
#pragma unroll
            for (int ks = 0; ks < kMT; ++ks) {
                if constexpr (FP8) {
                    // the E4M3 path takes the head dim in a permuted order
                    // (the same for K): k-step ks, pair j of lane c4 is
                    // d = c4 * D/4 + 4 ks + 2 j, +1 -- a dot product does not
                    // depend on the order of its terms
                    const uint2 v = valid ? __ldg(reinterpret_cast<const uint2 *>(qr) + (c4 * (D / 16) + ks))
                                          : make_uint2(0u, 0u);
                    qb[nt][ks][0] = v.x;
                    qb[nt][ks][1] = v.y;
                } else {
                    qb[nt][ks][0] = valid ? __ldg(qr + ks * 8 + c4) : 0u;
                    qb[nt][ks][1] = valid ? __ldg(qr + ks * 8 + 4 + c4) : 0u;
                }
                if constexpr (FP8 && BF16) {
                    // the f16 MMA of the E4M3 path: bf16 pairs -> f16 pairs
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const uint32_t w = qb[nt][ks][j];
                        __half2 h2 = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
                        qb[nt][ks][j] = *reinterpret_cast<uint32_t *>(&h2);
                    }
                }
            }
        }

        if constexpr (FMA) {
            // the unit's query rows as fp32 in shared memory (zeros past
            // `rows`); column c of head h at h * kQS + c (+4 in the upper half)
            __syncwarp();  // the previous unit is done reading them
            for (int i = lane; i < D; i += 32) {  // 8 heads x D/8 chunks of 8
                const int h = i / (D / 8), c = (i - h * (D / 8)) * 8;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (h < rows)
                    v = __ldg(reinterpret_cast<const uint4 *>(a.q + ((size_t)cs.seq * a.Hq + h0 + h) * D + c));
                const float2 f0 = unpack2<BF16>(v.x), f1 = unpack2<BF16>(v.y);
                const float2 f2 = unpack2<BF16>(v.z), f3 = unpack2<BF16>(v.w);
                const uint32_t dst = fq_base + (uint32_t)(h * kQS + c + (c >= D / 2 ? 4 : 0)) * 4;
                sts_f4(dst, f0.x, f0.y, f1.x, f1.y);
                sts_f4(dst + 16, f2.x, f2.y, f3.x, f3.y);
            }
            __syncwarp();
        }

        {
            // pull the next unit's query rows into L2 while this one runs
            Walker nw = cw;
            Seg ns;
            if (walker_next(nw, ns, a, prefix, ctxs, gw)) {
                const int nk = ns.pair / a.n_hg;
                const int nh = ns.pair - nk * a.n_hg;
                const int nrows = min(HPU, a.G - nh * HPU);
                const char *base = reinterpret_cast<const char *>(
                    a.q + ((size_t)ns.seq * a.Hq + nk * a.G + nh * HPU) * D);
                if (lane * 128 < nrows * D * 2)
                    prefetch_l2(base + lane * 128);
            }
        }

        // Fused append: this unit holds its sequence's last position.  The
        // new token's row (one 8-byte piece per lane) and slot are loaded here,
        // together with Q, and first used at the last tile.
        const bool has_new = !FP8 && a.k_new != nullptr && cs.t1 > cs.t0 && cs.t1 * kTileTokens >= cs.ctx;
        int64_t new_slot = -1;
        uint2 kn2 = make_uint2(0, 0), vn2 = make_uint2(0, 0);
        if (has_new) {
            new_slot = __ldg(a.slots + cs.seq);
            if (lane < D / 4) {
                const size_t src = ((size_t)cs.seq * a.Hkv + kvh) * D;
                kn2 = __ldg(reinterpret_cast<const uint2 *>(a.k_new + src) + lane);
                vn2 = __ldg(reinterpret_cast<const uint2 *>(a.v_new + src) + lane);
            }
        }

        float o[NT][kMT][4];
        float m_run[NT][2], l_run[NT][2];
        // CUDA-core variant: heads x this lane's FD columns, per-head state
        float of[FMA ? 8 : 1][FMA ? FD : 1], mf[FMA ? 8 : 1], lf[FMA ? 8 : 1];
        if constexpr (FMA) {
#pragma unroll
            for (int h = 0; h < 8; ++h) {
#pragma unroll
                for (int j = 0; j < FD; ++j)
                    of[h][j] = 0.f;
                mf[h] = -INFINITY;
                lf[h] = 0.f;
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt)
                o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
            m_run[nt][0] = m_run[nt][1] = -INFINITY;
            l_run[nt][0] = l_run[nt][1] = 0.f;
        }

        if constexpr (CAS) {
            if (cs.t0 == 0 && cs.toff > 0) {
                // the row's positions before its own blocks were attended by
                // the shared-prefix kernel: resume from its partial.  Lane
                // (g8, c4) holds heads 2c4, 2c4+1 of each n-tile at d = 16 mt +
                // g8 (+8); the sum l is kept once per head (lane g8 == 0).
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int head = nt * 8 + 2 * c4 + j;
                        if (head < rows) {
                            const size_t row = (size_t)cs.seq * a.Hq + h0 + head;
                            m_run[nt][j] = __ldg(a.init_m + row);
                            l_run[nt][j] = g8 == 0 ? __ldg(a.init_l + row) : 0.f;
                            const float *po = a.init_o + row * D;
#pragma unroll
                            for (int mt = 0; mt < kMT; ++mt) {
                                o[nt][mt][j] = __ldg(po + 16 * mt + g8);
                                o[nt][mt][2 + j] = __ldg(po + 16 * mt + g8 + 8);
                            }
                        }
                    }
                }
            }
        }

        for (int t = cs.t0; t < cs.t1; ++t) {
            const uint32_t bar = bar_base + stage * 8;
            // every lane must agree, or the warp-collective code below diverges
            const bool ok = __all_sync(FULL, mbar_wait_bounded(bar, (phases >> stage) & 1u, a.wait_limit_ns));
            if (!ok) {
                if (lane == 0)
                    atomicOr(a.err, kErrTimeout);
                failed = true;
                break;
            }
            phases ^= 1u << stage;
            uint32_t kb = ring_base + stage * kStage;
            uint32_t vb = kb + kTile;
            const int nvalid = min(kTileTokens, cs.ctx - t * kTileTokens);
            float sk_lo = 1.f, sk_hi = 1.f, sv_lo = 1.f, sv_hi = 1.f;
            // E4M3: this lane's code words, taken straight into registers.
            // K (A operand of S^T, rows = tokens): rows g8 and g8+8, bytes
            // [c4 D/4, c4 D/4 + D/4) -- word ks is k-step ks of the permuted
            // head dim.  V (A operand of O^T, rows = head dim): tokens 2c4,
            // 2c4+1, 2c4+8, 2c4+9, bytes [g8 D/8, g8 D/8 + D/8) -- byte b is
            // output row d = g8 D/8 + b, i.e. m-tile b/2, row g8 + 8 (b%2).
            uint32_t kw[2][KW8], vw[4][VW8];
            if constexpr (FP8) {
                const uint32_t k8 = kb, v8 = kb + kTileTokens * D;
                const uint32_t scl = scale_base + stage * (4 * kTileTokens * 2);
#pragma unroll
                for (int r = 0; r < 2; ++r) {
#pragma unroll
                    for (int i = 0; i < KW8 / 4; ++i)
                        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(kw[r][4 * i]), "=r"(kw[r][4 * i + 1]), "=r"(kw[r][4 * i + 2]),
                                       "=r"(kw[r][4 * i + 3])
                                     : "r"(k8 + e4m3_swz<D>((g8 + 8 * r) * D + c4 * (D / 4) + 16 * i)));
                }
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int tok = 2 * c4 + (r & 1) + 8 * (r >> 1);
                    const uint32_t addr = v8 + e4m3_swz<D>(tok * D + g8 * (D / 8));
                    if constexpr (VW8 == 4)
                        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(vw[r][0]), "=r"(vw[r][1]), "=r"(vw[r][2]), "=r"(vw[r][3])
                                     : "r"(addr));
                    else
                        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(vw[r][0]), "=r"(vw[r][1]) : "r"(addr));
                }
                float f[4];
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f[0]) : "r"(scl + g8 * 4));
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f[1]) : "r"(scl + (g8 + 8) * 4));
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f[2]) : "r"(scl + kTileTokens * 4 + g8 * 4));
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f[3]) : "r"(scl + kTileTokens * 4 + (g8 + 8) * 4));
                sk_lo = f[0];
                sk_hi = f[1];
                // a position past the context may hold any scale (even NaN):
                // its probability is 0 and must stay 0 after the V scale
                sv_lo = g8 < nvalid ? f[2] : 0.f;
                sv_hi = g8 + 8 < nvalid ? f[3] : 0.f;
                __syncwarp();
                // everything is in registers: the stage goes back to the producer now
                ++consumed;
                if (p_has) {
                    if (lane == 0)
                        fence_proxy_async_smem();
                    issue(stage);
                }
                if (++stage == a.stages)
                    stage = 0;
            }
            if (has_new && t == cs.t1 - 1 && new_slot >= 0) {
                if (new_slot >= a.pool_slots) {
                    if (lane == 0)
                        atomicOr(a.err, kErrSlot);
                } else if (hg == 0 && lane < D / 4) {
                    // the append proper: the new row to its cache slot
                    const int64_t blk = new_slot / a.bs;
                    const int64_t row = new_slot - blk * a.bs;
                    const size_t dst = ((size_t)(blk * a.Hkv + kvh) * a.bs + row) * D;
                    reinterpret_cast<uint2 *>(a.k_cache + dst)[lane] = kn2;
                    reinterpret_cast<uint2 *>(a.v_cache + dst)[lane] = vn2;
                }
            }
            if (has_new && t == cs.t1 - 1 && new_slot >= 0 && new_slot < a.pool_slots) {
                // the new token's row of this tile, in the 128-byte swizzle
                const int r = cs.ctx - 1 - t * kTileTokens;
                if (lane < D / 4) {
                    const int chunk = lane >> 1;  // 16-byte chunk of the row
                    const uint32_t off = (chunk >> 3) * kBoxBytes + r * 128 +
                                         ((uint32_t)((chunk & 7) ^ (r & 7)) << 4) + (lane & 1) * 8;
                    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(kb + off), "r"(kn2.x), "r"(kn2.y)
                                 : "memory");
                    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(vb + off), "r"(vn2.x), "r"(vn2.y)
                                 : "memory");
                }
                __syncwarp();
            }

            if constexpr (FMA) {
                // CUDA-core variant.  Scores: lane (token tt, column half hf)
                // forms the partial dot products of its token's K row half
                // with every head's query row half; one shuffle adds the halves.
                const int tt = lane & 15, hf = lane >> 4;
                float s[8];
#pragma unroll
                for (int h = 0; h < 8; ++h)
                    s[h] = 0.f;
#pragma unroll
                for (int c = 0; c < D / 16; ++c) {
                    const int chunk = hf * (D / 16) + c;  // 16-byte chunk of the K row
                    uint32_t kw4[4];
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(kw4[0]), "=r"(kw4[1]), "=r"(kw4[2]), "=r"(kw4[3])
                                 : "r"(kb + (chunk >> 3) * kBoxBytes + tt * 128 +
                                       ((uint32_t)((chunk & 7) ^ (tt & 7)) << 4)));
                    float kf[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f2 = unpack2<BF16>(kw4[j]);
                        kf[2 * j] = f2.x;
                        kf[2 * j + 1] = f2.y;
                    }
                    const uint32_t qa = fq_base + (uint32_t)(8 * chunk + 4 * hf) * 4;
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        if (h < rows) {
                            const float4 q0 = lds_f4(qa + h * kQS * 4), q1 = lds_f4(qa + h * kQS * 4 + 16);
                            float acc = s[h];
                            acc = fmaf(kf[0], q0.x, acc);
                            acc = fmaf(kf[1], q0.y, acc);
                            acc = fmaf(kf[2], q0.z, acc);
                            acc = fmaf(kf[3], q0.w, acc);
                            acc = fmaf(kf[4], q1.x, acc);
                            acc = fmaf(kf[5], q1.y, acc);
                            acc = fmaf(kf[6], q1.z, acc);
                            s[h] = fmaf(kf[7], q1.w, acc);
                        }
                    }
                }
                // online softmax per head over the tile's 16 tokens (log2 domain)
                const bool tv = tt < nvalid;
                float ph[8];
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    ph[h] = 0.f;
                    if (h < rows) {
                        const float sh = s[h] + __shfl_xor_sync(FULL, s[h], 16);
                        const float x = tv ? sh * a.scale_log2 : -INFINITY;
                        float mx = x;
#pragma unroll
                        for (int off = 1; off < 16; off <<= 1)
                            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, off));
                        const float mn = fmaxf(mf[h], mx);
                        if (mn > mf[h]) {  // uniform: every lane holds the same max
                            const float al = exp2f(mf[h] - mn);
                            lf[h] *= al;
#pragma unroll
                            for (int j = 0; j < FD; ++j)
                                of[h][j] *= al;
                            mf[h] = mn;
                        }
                        ph[h] = exp2f(x - mn);
                        lf[h] += ph[h];
                    }
                }
                if (hf == 0) {
                    sts_f4(fp_base + tt * 32, ph[0], ph[1], ph[2], ph[3]);
                    sts_f4(fp_base + tt * 32 + 16, ph[4], ph[5], ph[6], ph[7]);
                }
                __syncwarp();
                // O += P V: lane owns columns [FD lane, FD lane + FD) of every
                // head; only tokens inside the context are read
                const int d0 = lane * FD;
                const int vchunk = d0 >> 3;
#pragma unroll
                for (int u = 0; u < kTileTokens; ++u) {
                    if (u < nvalid) {
                        const uint32_t addr = vb + (vchunk >> 3) * kBoxBytes + u * 128 +
                                              ((uint32_t)((vchunk & 7) ^ (u & 7)) << 4) + (uint32_t)(d0 & 7) * 2;
                        float vf[FD];
                        if constexpr (FD == 4) {
                            uint32_t w0, w1;
                            asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(addr));
                            const float2 v0 = unpack2<BF16>(w0), v1 = unpack2<BF16>(w1);
                            vf[0] = v0.x;
                            vf[1] = v0.y;
                            vf[2 % FD] = v1.x;
                            vf[3 % FD] = v1.y;
                        } else {
                            uint32_t w0;
                            asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w0) : "r"(addr));
                            const float2 v0 = unpack2<BF16>(w0);
                            vf[0] = v0.x;
                            vf[1 % FD] = v0.y;
                        }
                        const float4 p0 = lds_f4(fp_base + u * 32), p1 = lds_f4(fp_base + u * 32 + 16);
                        const float pp[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            if (h < rows) {
#pragma unroll
                                for (int j = 0; j < FD; ++j)
                                    of[h][j] = fmaf(pp[h], vf[j], of[h][j]);
                            }
                        }
                    }
                }
                __syncwarp();  // the probabilities are rewritten by the next tile
            } else {
                // S^T = K Q^T, as two independent accumulation chains (even
                // and odd k-steps) added at the end: half the dependent MMAs
                float sc[NT][4], sc2[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                    sc2[nt][0] = sc2[nt][1] = sc2[nt][2] = sc2[nt][3] = 0.f;
                }
#pragma unroll
                for (int ks = 0; ks < kMT; ++ks) {
                    const int mi = lane >> 3;
                    const int tok = (lane & 7) + 8 * (mi & 1);
                    const int chunk = 2 * ks + (mi >> 1);
                    const uint32_t addr = kb + (chunk >> 3) * kBoxBytes + tok * 128 +
                                          ((uint32_t)((chunk & 7) ^ (tok & 7)) << 4);
                    uint32_t ka[4];
                    if constexpr (FP8) {
                        ka[0] = e4m3x2_to_f16x2((uint16_t)(kw[0][ks] & 0xffffu));
                        ka[1] = e4m3x2_to_f16x2((uint16_t)(kw[1][ks] & 0xffffu));
                        ka[2] = e4m3x2_to_f16x2((uint16_t)(kw[0][ks] >> 16));
                        ka[3] = e4m3x2_to_f16x2((uint16_t)(kw[1][ks] >> 16));
                    } else {
                        ldmatrix_x4(addr, ka[0], ka[1], ka[2], ka[3]);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816<MMA_BF16>((ks & 1) ? sc2[nt] : sc[nt], ka, qb[nt][ks][0], qb[nt][ks][1]);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        sc[nt][j] += sc2[nt][j];
                }

                // online softmax per query head (one column of S^T), log2 domain;
                // this thread holds tokens g8, g8+8 of heads 2*c4, 2*c4+1
                const bool v_lo = g8 < nvalid;
                const bool v_hi = g8 + 8 < nvalid;
                uint32_t pb[NT][2];
                float x[NT][4];
                bool up = false;  // some score above its head's running max
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    x[nt][0] = v_lo ? sc[nt][0] * (sk_lo * a.scale_log2) : -INFINITY;
                    x[nt][1] = v_lo ? sc[nt][1] * (sk_lo * a.scale_log2) : -INFINITY;
                    x[nt][2] = v_hi ? sc[nt][2] * (sk_hi * a.scale_log2) : -INFINITY;
                    x[nt][3] = v_hi ? sc[nt][3] * (sk_hi * a.scale_log2) : -INFINITY;
                    up |= (fmaxf(x[nt][0], x[nt][2]) > m_run[nt][0]) | (fmaxf(x[nt][1], x[nt][3]) > m_run[nt][1]);
                }
                // Only when some head's max grows (every first tile, rarely
                // afterwards) are the maxima reduced across the 8 token rows and
                // the accumulators rescaled; otherwise the running max stands
                // and every rescale factor would be exactly 1.
                if (__any_sync(FULL, up)) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float mx0 = fmaxf(x[nt][0], x[nt][2]), mx1 = fmaxf(x[nt][1], x[nt][3]);
#pragma unroll
                        for (int off = 4; off < 32; off <<= 1) {
                            mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, off));
                            mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, off));
                        }
                        const float mn0 = fmaxf(m_run[nt][0], mx0);
                        const float mn1 = fmaxf(m_run[nt][1], mx1);
                        const float al0 = exp2f(m_run[nt][0] - mn0);
                        const float al1 = exp2f(m_run[nt][1] - mn1);
                        m_run[nt][0] = mn0;
                        m_run[nt][1] = mn1;
                        l_run[nt][0] *= al0;
                        l_run[nt][1] *= al1;
#pragma unroll
                        for (int mt = 0; mt < kMT; ++mt) {
                            o[nt][mt][0] *= al0;
                            o[nt][mt][2] *= al0;
                            o[nt][mt][1] *= al1;
                            o[nt][mt][3] *= al1;
                        }
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float p0 = exp2f(x[nt][0] - m_run[nt][0]), p2 = exp2f(x[nt][2] - m_run[nt][0]);
                    const float p1 = exp2f(x[nt][1] - m_run[nt][1]), p3 = exp2f(x[nt][3] - m_run[nt][1]);
                    l_run[nt][0] += p0 + p2;
                    l_run[nt][1] += p1 + p3;
                    // (E4M3: the V row scales multiply the probabilities here; l
                    // keeps the unscaled sums)
                    pb[nt][0] = movmatrix_trans(pack2<MMA_BF16>(p0 * sv_lo, p1 * sv_lo));  // tokens 0-7
                    pb[nt][1] = movmatrix_trans(pack2<MMA_BF16>(p2 * sv_hi, p3 * sv_hi));  // tokens 8-15
                }

                // O^T += V^T P^T.  Positions past the context may hold anything
                // (even NaN): zero their V so that 0 * V stays 0 in the MMA.
                uint32_t m01 = 0xffffffffu, m23 = 0xffffffffu;
                if (nvalid < kTileTokens) {
                    m01 = (2 * c4 < nvalid ? 0x0000ffffu : 0u) | (2 * c4 + 1 < nvalid ? 0xffff0000u : 0u);
                    m23 = (2 * c4 + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c4 + 9 < nvalid ? 0xffff0000u : 0u);
                }
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    const int mi = lane >> 3;
                    const int tok = (lane & 7) + 8 * (mi >> 1);
                    const int chunk = 2 * mt + (mi & 1);
                    const uint32_t addr = vb + (chunk >> 3) * kBoxBytes + tok * 128 +
                                          ((uint32_t)((chunk & 7) ^ (tok & 7)) << 4);
                    uint32_t va[4];
                    if constexpr (FP8) {
                        // pair the codes of two consecutive tokens for one d:
                        // bytes 2(mt%2) and 2(mt%2)+1 of word mt/2 are rows g8 and g8+8
                        const int wi = mt >> 1;
                        const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
                        const uint32_t p01 = __byte_perm(vw[0][wi], vw[1][wi], sel);
                        const uint32_t p23 = __byte_perm(vw[2][wi], vw[3][wi], sel);
                        va[0] = e4m3x2_to_f16x2((uint16_t)(p01 & 0xffffu));
                        va[1] = e4m3x2_to_f16x2((uint16_t)(p01 >> 16));
                        va[2] = e4m3x2_to_f16x2((uint16_t)(p23 & 0xffffu));
                        va[3] = e4m3x2_to_f16x2((uint16_t)(p23 >> 16));
                    } else {
                        ldmatrix_x4_trans(addr, va[0], va[1], va[2], va[3]);
                    }
                    if (nvalid < kTileTokens) {  // only a ragged tile has positions to mask
                        va[0] &= m01;
                        va[1] &= m01;
                        va[2] &= m23;
                        va[3] &= m23;
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816<MMA_BF16>(o[nt][mt], va, pb[nt][0], pb[nt][1]);
                }

            }
            if constexpr (!FP8) {
                // stage consumed: hand it back to the producer for a later tile
                __syncwarp();
                ++consumed;
                if (p_has) {
                    if (lane == 0)
                        fence_proxy_async_smem();
                    issue(stage);
                }
                if (++stage == a.stages)
                    stage = 0;
            }
        }
        if (failed)
            break;

        if constexpr (FMA) {
            // per-head sums over one column half's 16 token lanes (the other
            // half holds the same values)
            const int d0 = lane * FD;
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                if (h < rows) {
                    float l = lf[h];
#pragma unroll
                    for (int off = 1; off < 16; off <<= 1)
                        l += __shfl_xor_sync(FULL, l, off);
                    if (cs.dest < 0) {
                        const float inv = l > 0.f ? 1.f / l : 0.f;
                        uint16_t *dst = a.out + ((size_t)cs.seq * a.Hq + h0 + h) * D + d0;
                        if constexpr (FD == 4)
                            *reinterpret_cast<uint2 *>(dst) = make_uint2(
                                pack2<BF16>(of[h][0] * inv, of[h][1 % FD] * inv),
                                pack2<BF16>(of[h][2 % FD] * inv, of[h][3 % FD] * inv));
                        else
                            *reinterpret_cast<uint32_t *>(dst) = pack2<BF16>(of[h][0] * inv, of[h][1 % FD] * inv);
                    } else {
                        const size_t row = a.mode == kModePartition
                                               ? ((size_t)cs.seq * a.Hq + h0 + h) * a.S + cs.dest
                                               : (size_t)cs.dest * kMaxRows + h;
                        float *dst = a.part_o + row * D + d0;
                        if constexpr (FD == 4)
                            *reinterpret_cast<float4 *>(dst) =
                                make_float4(of[h][0], of[h][1 % FD], of[h][2 % FD], of[h][3 % FD]);
                        else
                            *reinterpret_cast<float2 *>(dst) = make_float2(of[h][0], of[h][1 % FD]);
                        if (lane == 0) {
                            a.part_m[row] = mf[h];
                            a.part_l[row] = l;
                        }
                    }
                }
            }
        } else {
            // ---- epilogue: per-head sums over the 16 token rows (lanes with the same c4)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1)
                        l_run[nt][j] += __shfl_xor_sync(FULL, l_run[nt][j], off);
                }
            }
            // Accumulator 8x8 blocks are (d rows) x (head columns); movmatrix
            // turns each into (head rows) x (d columns): lane (g8, c4) then owns
            // head g8, d = 16*mt + 8*half + 2*c4 and the next one.
            if (FP8 && cs.dest < 0) {
                // permuted head dim: lane (g8, c4) holds heads 2c4, 2c4+1 at
                // d = g8 D/8 + 2 mt (row g8 of m-tile mt) and d + 1 (row g8+8),
                // i.e. D/8 consecutive elements of each of its two heads
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int head = nt * 8 + 2 * c4 + j;
                        const float inv = l_run[nt][j] > 0.f ? 1.f / l_run[nt][j] : 0.f;
                        uint32_t wv[kMT];
#pragma unroll
                        for (int mt = 0; mt < kMT; ++mt)
                            wv[mt] = pack2<BF16>(o[nt][mt][j] * inv, o[nt][mt][2 + j] * inv);
                        if (head < rows) {
                            uint4 *dst = reinterpret_cast<uint4 *>(a.out + ((size_t)cs.seq * a.Hq + h0 + head) * D +
                                                                   g8 * (D / 8));
#pragma unroll
                            for (int i = 0; i < kMT / 4; ++i)
                                dst[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
                        }
                    }
                }
            } else if (FP8) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int head = nt * 8 + 2 * c4 + j;
                        if (head < rows) {
                            const size_t row = a.mode == kModePartition
                                                   ? ((size_t)cs.seq * a.Hq + h0 + head) * a.S + cs.dest
                                                   : (size_t)cs.dest * kMaxRows + head;
                            float4 *dst = reinterpret_cast<float4 *>(a.part_o + row * D + g8 * (D / 8));
#pragma unroll
                            for (int i = 0; i < kMT / 2; ++i)
                                dst[i] = make_float4(o[nt][2 * i][j], o[nt][2 * i][2 + j], o[nt][2 * i + 1][j],
                                                     o[nt][2 * i + 1][2 + j]);
                            if (g8 == 0) {
                                a.part_m[row] = m_run[nt][j];
                                a.part_l[row] = l_run[nt][j];
                            }
                        }
                    }
                }
            } else if (cs.dest < 0) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float inv0 = l_run[nt][0] > 0.f ? 1.f / l_run[nt][0] : 0.f;
                    const float inv1 = l_run[nt][1] > 0.f ? 1.f / l_run[nt][1] : 0.f;
                    const int head = nt * 8 + g8;
                    uint32_t *dst = reinterpret_cast<uint32_t *>(
                        a.out + ((size_t)cs.seq * a.Hq + h0 + (head < rows ? head : 0)) * D);
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        const uint32_t b0 = movmatrix_trans(pack2<BF16>(o[nt][mt][0] * inv0, o[nt][mt][1] * inv1));
                        const uint32_t b1 = movmatrix_trans(pack2<BF16>(o[nt][mt][2] * inv0, o[nt][mt][3] * inv1));
                        if (head < rows) {
                            dst[mt * 8 + c4] = b0;
                            dst[mt * 8 + 4 + c4] = b1;
                        }
                    }
                }
            } else {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int head = nt * 8 + g8;
                    size_t row;
                    if (a.mode == kModePartition)
                        row = ((size_t)cs.seq * a.Hq + h0 + head) * a.S + cs.dest;
                    else
                        row = (size_t)cs.dest * kMaxRows + head;
                    float *dst = a.part_o + row * D;
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            // transpose the fp32 block as two 16-bit halves
                            const uint32_t xb = __float_as_uint(o[nt][mt][2 * half]);
                            const uint32_t yb = __float_as_uint(o[nt][mt][2 * half + 1]);
                            const uint32_t hi = movmatrix_trans((xb >> 16) | (yb & 0xffff0000u));
                            const uint32_t lo = movmatrix_trans((xb & 0xffffu) | (yb << 16));
                            const float e0 = __uint_as_float((hi << 16) | (lo & 0xffffu));
                            const float e1 = __uint_as_float((hi & 0xffff0000u) | (lo >> 16));
                            if (head < rows)
                                *reinterpret_cast<float2 *>(dst + mt * 16 + half * 8 + 2 * c4) = make_float2(e0, e1);
                        }
                    }
                    // column state: lanes 0-3 hold heads 2*c4, 2*c4+1 of this n-tile
                    if (g8 == 0) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int hc = nt * 8 + 2 * c4 + j;
                            if (hc < rows) {
                                const size_t r = a.mode == kModePartition
                                                     ? ((size_t)cs.seq * a.Hq + h0 + hc) * a.S + cs.dest
                                                     : (size_t)cs.dest * kMaxRows + hc;
                                a.part_m[r] = m_run[nt][j];
                                a.part_l[r] = l_run[nt][j];
                            }
                        }
                    }
                }
            }
        }

        if (a.fold_cnt != nullptr && cs.dest >= 0) {
            // A piece of a split (sequence, head group): count it, and the
            // warp that completes the count merges the group's rows -- the
            // merge kernel's work, done where the last piece lands.  Every
            // piece is visible before it is counted (fence, then atomic).
            __threadfence();
            __syncwarp();
            int is_last = 0;
            if (lane == 0) {
                long long a0;
                int ntu;
                pair_span(prefix, cs.seq, cs.pair, a.npairs, a.unit_cost, a0, ntu);
                const long long T = (long long)prefix[a.B] * a.npairs;
                const long long W = a.total_warps;
                const long long first = ((a0 + 1) * W + T - 1) / T - 1;
                const long long last = ((a0 + ntu) * W + T - 1) / T - 1;
                // warps whose range meets the pair's tiles; with fewer tiles
                // than warps each range holds at most one tile
                const long long expected = T >= W ? last - first + 1 : ntu;
                is_last = atomicAdd(a.fold_cnt + (size_t)cs.seq * a.npairs + cs.pair, 1) == expected - 1;
            }
            is_last = __shfl_sync(FULL, is_last, 0);
            if (is_last) {
                __threadfence();
                MergeArgs ma;
                ma.out = a.out;
                ma.context_lens = a.context_lens;
                ma.prefix = prefix;
                ma.part_o = a.part_o;
                ma.part_m = a.part_m;
                ma.part_l = a.part_l;
                ma.mb = a.mb;
                ma.B = a.B;
                ma.Hq = a.Hq;
                ma.G = a.G;
                ma.n_hg = a.n_hg;
                ma.npairs = a.npairs;
                ma.bs = a.bs;
                ma.hpu = HPU;
                ma.mode = a.mode;
                ma.part_tiles = a.part_tiles;
                ma.S = a.S;
                ma.total_warps = a.total_warps;
                ma.unit_cost = a.unit_cost;
                const MergeRow m0 = merge_row(ma, (long long)cs.seq * a.Hq + h0);
                if (rows > 1 && m0.count <= kPairMergeMaxPieces) {
                    merge_pair_warp<D, BF16>(ma, m0, rows);  // every head at once
                } else {
                    for (int g = 0; g < rows; ++g) {
                        const MergeRow mr = merge_row(ma, (long long)cs.seq * a.Hq + h0 + g);
                        if (mr.count > 1)  // small batches: few registers beside the decode loop's
                            merge_row_warp<D, BF16, 4>(ma, mr);
                    }
                }
            }
        }
    }

    if (failed) {
        // a wait timed out: let every copy still in flight land before the
        // CTA's shared memory goes away, each wait again bounded
        for (int k = consumed; k < issued; ++k) {
            const int st = k % a.stages;
            mbar_wait_bounded(bar_base + st * 8, (phases >> st) & 1u, a.wait_limit_ns);
            phases ^= 1u << st;
        }
    }
}

// Zero the decode kernel's per-row piece counters of this call.  Launched as
// a programmatic dependent: it waits for the previous kernel in the stream
// (which may still count with them) and lets the decode kernel's prologue
// start at once.
__global__ void __launch_bounds__(256) fold_zero_kernel(int *__restrict__ cnt, int n) {
    griddep_launch_dependents();
    griddep_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        cnt[i] = 0;
}

// ------------------------------------------------------------- merge kernel

// The whole CTA merges one row with many pieces, GROUPS * kCtaBatch pieces
// per batch (rescaled online across batches): thread (grp, col) owns one
// 16-byte column slice of pieces grp, grp + GROUPS, ...; its outputs, and the
// (m, l) of piece threadIdx.x, are loaded at once, then the weights go
// through shared memory.
constexpr int kCtaBatch = 8;

template <int D, bool BF16, int NTH>
__device__ __forceinline__ void merge_row_cta(const MergeArgs &a, const MergeRow &r, float *red, float *s_w,
                                              float *s_l, float4 *s_acc) {
    constexpr int COLS = D / 4;
    constexpr int GROUPS = NTH / COLS;
    constexpr int BATCH = GROUPS * kCtaBatch;  // <= NTH
    static_assert(BATCH <= NTH, "one (m, l) per thread");
    const int col = threadIdx.x % COLS;
    const int grp = threadIdx.x / COLS;
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long k0 = 0; k0 < r.count; k0 += BATCH) {
        const int kn = (int)min((long long)BATCH, r.count - k0);
        float m = -INFINITY;
        if (threadIdx.x < kn) {
            const long long rr = merge_piece(a, r, k0 + threadIdx.x);
            m = rr >= 0 ? a.part_m[rr] : -INFINITY;
            s_l[threadIdx.x] = rr >= 0 ? a.part_l[rr] : 0.f;
        }
        float4 v[kCtaBatch];
#pragma unroll
        for (int q = 0; q < kCtaBatch; ++q) {
            const int i = grp + q * GROUPS;
            const long long rr = i < kn ? merge_piece(a, r, k0 + i) : -1;
            v[q] = rr >= 0 ? *reinterpret_cast<const float4 *>(a.part_o + rr * D + col * 4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (threadIdx.x < BATCH)
            s_w[threadIdx.x] = m;
        const float cmax = block_reduce<NTH>(m, true, red);  // also orders the s_* writes
        const float mnew = fmaxf(M, cmax);
        const float rescale = M == -INFINITY ? 0.f : exp2f(M - mnew);
        float lsum = 0.f;
        if (threadIdx.x < kn) {
            const float w = m == -INFINITY ? 0.f : exp2f(m - mnew);
            s_w[threadIdx.x] = w;
            lsum = w * s_l[threadIdx.x];
        }
        lsum = block_reduce<NTH>(lsum, false, red);  // also orders the weights
        L = L * rescale + lsum;
        M = mnew;
        acc.x *= rescale;
        acc.y *= rescale;
        acc.z *= rescale;
        acc.w *= rescale;
#pragma unroll
        for (int q = 0; q < kCtaBatch; ++q) {
            const int i = grp + q * GROUPS;
            const float w = i < kn ? s_w[i] : 0.f;
            if (w != 0.f) {
                acc.x = fmaf(w, v[q].x, acc.x);
                acc.y = fmaf(w, v[q].y, acc.y);
                acc.z = fmaf(w, v[q].z, acc.z);
                acc.w = fmaf(w, v[q].w, acc.w);
            }
        }
        __syncthreads();  // s_w / s_l are rewritten by the next batch
    }
    s_acc[threadIdx.x] = acc;
    __syncthreads();
    if (threadIdx.x < COLS) {
        float4 t = s_acc[threadIdx.x];
#pragma unroll
        for (int q = 1; q < GROUPS; ++q) {
            const float4 u = s_acc[threadIdx.x + q * COLS];
            t.x += u.x;
            t.y += u.y;
            t.z += u.z;
            t.w += u.w;
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const float vv[4] = {t.x * inv, t.y * inv, t.z * inv, t.w * inv};
        store_row<D, BF16>(a, r, threadIdx.x * 4, vv, 4);
    }
    __syncthreads();
}

// Combine the partial results (o_j unnormalised, m_j in the log2 domain, l_j)
// of the pieces each query head's context was split into:
//   M = max m_j,  L = sum l_j 2^(m_j - M),  out = sum o_j 2^(m_j - M) / L.
// Pieces with m = -inf (no positions) weigh 0.  Each CTA takes four
// consecutive (sequence, query head) rows, grid-stride: one warp per row when
// every row has few pieces, else the four rows one after another with the
// whole CTA.  The work is latency-bound (dependent round trips), so every
// batch of pieces issues all its loads at once and many rows stay in flight.
// NTH = 512 (one row per CTA) serves fixed partitions with many pieces per
// row: 128 pieces per round trip.  Launched as a programmatic dependent of
// the decode kernel, so its launch overlaps the decode tail.
template <int D, bool BF16, int NTH = kMergeThreads>
__global__ void __launch_bounds__(NTH) lse_merge_kernel(const MergeArgs a) {
    __shared__ float red[NTH / 32];
    __shared__ float s_w[NTH];
    __shared__ float s_l[NTH];
    __shared__ float4 s_acc[NTH];
    griddep_wait();
    constexpr int ROWS = NTH / 32;
    const int warp = threadIdx.x >> 5;
    const long long rows_total = (long long)a.B * a.Hq;
    const int bound = a.mode == kModePartition ? a.S : a.prefix[a.B + 1];
    if (bound <= kWarpPieces) {
        // few pieces per row: one warp per row, four rows per CTA
        const long long groups = (rows_total + ROWS - 1) / ROWS;
        for (long long grp = blockIdx.x; grp < groups; grp += gridDim.x) {
            const long long row = grp * ROWS + warp;
            if (row < rows_total) {
                const MergeRow r = merge_row(a, row);
                if (r.count > 1)
                    merge_row_warp<D, BF16>(a, r);
            }
        }
    } else {
        // many pieces per row: the whole CTA on one row
        for (long long row = blockIdx.x; row < rows_total; row += gridDim.x) {
            const MergeRow r = merge_row(a, row);
            if (r.count > 1)
                merge_row_cta<D, BF16, NTH>(a, r, red, s_w, s_l, s_acc);
        }
    }
}

// ------------------------------------------------------------- append kernel

// cache[slot / bs][h][slot % bs][:] = new[t][h][:], 16 bytes per thread.
__global__ void __launch_bounds__(256) append_kernel(const uint4 *__restrict__ k_new,
                                                     const uint4 *__restrict__ v_new,
                                                     const int64_t *__restrict__ slots, int64_t T,
                                                     int Hkv, int chunks, int bs, int64_t nb,
                                                     uint4 *__restrict__ k_cache,
                                                     uint4 *__restrict__ v_cache, unsigned *err) {
    griddep_launch_dependents();
    const int64_t per_tok = (int64_t)Hkv * chunks;
    const int64_t total = T * per_tok;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_tok;
        const int64_t rem = i - t * per_tok;
        const int64_t h = rem / chunks;
        const int64_t ch = rem - h * chunks;
        const int64_t slot = __ldg(slots + t);
        if (slot < 0)
            continue;  // padding token
        const int64_t blk = slot / bs;
        const int64_t row = slot - blk * bs;
        if (blk >= nb) {
            atomicOr(err, kErrSlot);
            continue;
        }
        const int64_t dst = ((blk * Hkv + h) * bs + row) * chunks + ch;
        k_cache[dst] = __ldg(k_new + i);
        v_cache[dst] = __ldg(v_new + i);
    }
}

// ------------------------------------------------------------- E4M3 append

// One warp per (token, KV head, K|V) row: amax over the row by shuffles,
// scale = amax / 448 (1 if amax == 0) and y = x / scale as correctly rounded
// fp32 divisions, codes by round-to-nearest-even with saturation; the codes
// go to cache[slot / bs][h][slot % bs][:] and the scale beside them.
template <int D, bool BF16IN>
__global__ void __launch_bounds__(256) append_e4m3_kernel(const uint16_t *__restrict__ k_new,
                                                          const uint16_t *__restrict__ v_new,
                                                          const int64_t *__restrict__ slots, int64_t T, int Hkv,
                                                          int bs, int64_t nb, uint8_t *__restrict__ k8,
                                                          float *__restrict__ ks, uint8_t *__restrict__ v8,
                                                          float *__restrict__ vs, unsigned *err) {
    constexpr int E = D / 32;  // elements per lane (4 or 2)
    constexpr unsigned FULL = 0xffffffffu;
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t rows = T * Hkv * 2;
    for (int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; w < rows;
         w += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int which = (int)(w & 1);  // 0: K, 1: V
        const int64_t th = w >> 1;       // token * Hkv + head
        const int64_t t = th / Hkv;
        const int64_t h = th - t * Hkv;
        const int64_t slot = __ldg(slots + t);
        if (slot < 0)
            continue;
        const int64_t blk = slot / bs;
        if (blk >= nb) {
            if (lane == 0 && which == 0)
                atomicOr(err, kErrSlot);
            continue;
        }
        const uint16_t *src = (which ? v_new : k_new) + th * D + lane * E;
        float x[E];
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const uint32_t b = __ldg(src + i);
            x[i] = BF16IN ? __uint_as_float(b << 16) : __half2float(__ushort_as_half((unsigned short)b));
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < E; ++i)
            amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
        const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < E; i += 2) {
            const uint16_t c = f32x2_to_e4m3x2(__fdiv_rn(x[i], scale), __fdiv_rn(x[i + 1], scale));
            packed |= (uint32_t)c << (8 * i);
        }
        const int64_t r = (blk * Hkv + h) * bs + (slot - blk * bs);
        uint8_t *dst = (which ? v8 : k8) + r * D + lane * E;
        if constexpr (E == 4)
            *reinterpret_cast<uint32_t *>(dst) = packed;
        else
            *reinterpret_cast<uint16_t *>(dst) = (uint16_t)packed;
        if (lane == 0)
            (which ? vs : ks)[r] = scale;
    }
}

// ------------------------------------------------------------- block copy

// Copy-on-write: whole blocks src -> dst in both pools, 16 bytes per thread.
// A block is `chunks` 16-byte pieces, contiguous.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const int32_t *__restrict__ pairs, int64_t n,
                                                          int64_t chunks, int64_t nb,
                                                          uint4 *__restrict__ k_cache,
                                                          uint4 *__restrict__ v_cache, unsigned *err) {
    const int64_t total = n * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t p = i / chunks;
        const int64_t c = i - p * chunks;
        const int64_t src = __ldg(pairs + 2 * p), dst = __ldg(pairs + 2 * p + 1);
        if (src < 0 || src >= nb || dst < 0 || dst >= nb) {
            atomicOr(err, kErrSlot);
            continue;
        }
        k_cache[dst * chunks + c] = k_cache[src * chunks + c];
        v_cache[dst * chunks + c] = v_cache[src * chunks + c];
    }
}

// ------------------------------------------------------------- chunked prefill

// Query token j of sequence s (chunk of n tokens, context ctx after the
// chunk's append) attends to positions 0 .. ctx - n + i: a decode of length
// ctx - n + i + 1 over row s of the block table.
__global__ void __launch_bounds__(256) prefill_expand_kernel(const int32_t *__restrict__ query_start,
                                                             const int32_t *__restrict__ context_lens,
                                                             int B, int T, int64_t cap,
                                                             int32_t *__restrict__ lens,
                                                             int32_t *__restrict__ rows, int *mq_counter,
                                                             unsigned *err) {
    // with the multi-query kernel enabled (mq_counter != null), chunks of two
    // or more tokens are its work: their tokens get length 0 here (a zero
    // row from the decode kernel, overwritten by the multi-query kernel,
    // which runs after it in the stream) and its unit counter starts at 0
    if (mq_counter && blockIdx.x == 0 && threadIdx.x == 0)
        *mq_counter = 0;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < T; j += gridDim.x * blockDim.x) {
        int lo = 0, hi = B + 1;  // first index with query_start > j
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(query_start + mid) <= j)
                lo = mid + 1;
            else
                hi = mid;
        }
        const int s = max(0, min(B - 1, lo - 1));
        const int q0 = __ldg(query_start + s);
        const int n = __ldg(query_start + s + 1) - q0;
        const int c = __ldg(context_lens + s);
        int len = c - n + (j - q0) + 1;
        if (n <= 0 || c < n || c > cap || j < q0 || j >= q0 + n) {
            atomicOr(err, kErrContext);
            len = 0;
        } else if (mq_counter && n >= 2) {
            len = 0;
        }
        lens[j] = len;
        rows[j] = s;
    }
}

}  // namespace pkv
