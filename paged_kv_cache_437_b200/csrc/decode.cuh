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

#include <cstdint>

#include "ptx.cuh"

namespace pkv {

constexpr int kTileTokens = 16;                        // tokens per MMA k-step / TMA box rows
constexpr int kBoxCols = 64;                           // 16-bit elements per box row (128 B)
constexpr int kBoxBytes = kBoxCols * 2 * kTileTokens;  // 2048
constexpr int kMaxRows = 16;                           // query heads per unit (MMA M)
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
    int B, Hq, Hkv, G, n_hg, npairs, bs;
    float scale_log2;              // scale * log2(e)
    int mode;
    int part_tiles;                // partition mode: tiles per partition
    int S;                         // partition mode: partitions per sequence (layout)
    float *part_o;                 // partials (see the workspace layout on the host)
    float *part_m;
    float *part_l;
    int32_t *prefix_out;           // balanced: tile prefix for the merge kernel
    int total_warps;
    int stages;
    unsigned *err;
    uint64_t wait_limit_ns;        // bound on every mbarrier wait
    int inject_no_issue;           // testing: issue no copies so that waits run out
};

struct SmemLayout {
    int prefix_off, ctx_off, bar_off, ring_off, total;
};

__host__ __device__ inline int align_up_int(int x, int a) { return (x + a - 1) / a * a; }

__host__ __device__ inline SmemLayout decode_smem_layout(int B, int warps, int stages, int D,
                                                         bool need_prefix) {
    SmemLayout L;
    const int tile = kTileTokens * D * 2;
    const int prefix_bytes = need_prefix ? (B + 1) * 4 : 0;
    const int ctx_bytes = need_prefix ? B * 4 : 0;
    L.prefix_off = 0;
    L.ctx_off = prefix_bytes;
    L.bar_off = align_up_int(prefix_bytes + ctx_bytes, 16);
    L.ring_off = align_up_int(L.bar_off + warps * stages * 8, 1024);
    // + 1024: the dynamic smem base is re-aligned to 1024 B at run time
    L.total = L.ring_off + warps * stages * 2 * tile + 1024;
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
            int s = upper_bound_i(prefix, a.B + 1, w.lo / a.npairs) - 1;
            const int nt = prefix[s + 1] - prefix[s];
            const long long r = w.lo - (long long)prefix[s] * a.npairs;
            w.seq = s;
            w.pair = (int)(r / nt);
            w.t = (int)(r % nt);
        }
    }
}

__device__ __forceinline__ bool walker_next(Walker &w, Seg &sg, const DecodeArgs &a,
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
    // balanced
    if (w.u >= w.hi)
        return false;
    const int nt = prefix[w.seq + 1] - prefix[w.seq];
    sg.seq = w.seq;
    sg.pair = w.pair;
    sg.ctx = ctxs[w.seq];
    sg.t0 = w.t;
    sg.t1 = (int)min((long long)nt, (long long)w.t + (w.hi - w.u));
    const long long pair_start = (long long)prefix[w.seq] * a.npairs + (long long)w.pair * nt;
    const bool complete = (sg.t0 == 0 && sg.t1 == nt);
    sg.dest = complete ? -1 : 2 * gw + (pair_start < w.lo ? 0 : 1);
    w.u += sg.t1 - sg.t0;
    w.t = sg.t1;
    if (w.t == nt) {
        w.t = 0;
        if (++w.pair == a.npairs) {
            w.pair = 0;
            ++w.seq;
            while (w.seq < a.B && prefix[w.seq + 1] == prefix[w.seq])
                ++w.seq;
        }
    }
    return true;
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

// ------------------------------------------------------------- decode kernel

template <int D, bool BF16, bool TWO>
__global__ void __launch_bounds__(256) paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV,
                                                           const DecodeArgs a) {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    constexpr int kTile = kTileTokens * D * 2;  // bytes of one K (or V) tile
    constexpr int kKSteps = D / 16;
    constexpr int kNTiles = D / 8;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    const int warps = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * warps + warp;
    const bool need_prefix = a.mode != kModeDirect;
    const SmemLayout L = decode_smem_layout(a.B, warps, a.stages, D, need_prefix);
    int *prefix = reinterpret_cast<int *>(smem_raw + L.prefix_off);
    int *ctxs = reinterpret_cast<int *>(smem_raw + L.ctx_off);
    const uint32_t smem_base = smem_addr(smem_raw);
    const uint32_t bar_base = smem_base + L.bar_off + warp * a.stages * 8;
    const uint32_t ring_base = ((smem_base + L.ring_off + 1023u) & ~1023u) +
                               (uint32_t)(warp * a.stages * 2 * kTile);

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
            local += a.mode == kModeBalanced ? nt : ceil_div_i(nt, a.part_tiles);
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
            run += a.mode == kModeBalanced ? nt : ceil_div_i(nt, a.part_tiles);
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
            uint4 *o = reinterpret_cast<uint4 *>(a.out + (size_t)s * a.Hq * D);
            const int n = a.Hq * D / 8;
            for (int i = threadIdx.x; i < n; i += blockDim.x)
                o[i] = make_uint4(0, 0, 0, 0);
        }
        if (a.mode == kModeBalanced && blockIdx.x == 0) {
            for (int i = threadIdx.x; i <= a.B; i += blockDim.x)
                a.prefix_out[i] = prefix[i];
        }
    }

    const int c4 = lane & 3;   // thread-in-quad
    const int g8 = lane >> 2;  // quad index (MMA row / column group)

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
    int issued = 0;

    auto issue = [&](int stage) {
        const int pos0 = p_t * kTileTokens;
        const int lb = pos0 / a.bs;
        const int row0 = pos0 - lb * a.bs;
        if (ps.seq != tb_seq || lb < tb_base || lb >= tb_base + 32) {
            tb_seq = ps.seq;
            tb_base = lb;
            const int nblk = ceil_div_i(ps.ctx, a.bs);
            tb_val = (lb + lane < nblk) ? __ldg(a.block_tables + (size_t)ps.seq * a.mb + lb + lane) : 0;
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
            const uint32_t kdst = ring_base + stage * 2 * kTile;
            mbar_arrive_expect_tx(bar, 2 * kTile);
#pragma unroll
            for (int h = 0; h < D / kBoxCols; ++h) {
                tma_load_2d(kdst + h * kBoxBytes, &tmK, h * kBoxCols, y, bar);
                tma_load_2d(kdst + kTile + h * kBoxBytes, &tmV, h * kBoxCols, y, bar);
            }
        }
        ++issued;
        if (++p_t >= ps.t1) {
            do {
                p_has = walker_next(pw, ps, a, prefix, ctxs, gw);
            } while (p_has && ps.t0 >= ps.t1);
            p_t = p_has ? ps.t0 : 0;
        }
    };

    for (int s = 0; s < a.stages && p_has; ++s)
        issue(s);

    // ---- consumer
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
        const int h0 = kvh * a.G + hg * kMaxRows;
        const int rows = min(kMaxRows, a.G - hg * kMaxRows);

        // Q fragments (A operand, rows = query heads, k = head dim)
        uint32_t qa[kKSteps][4];
        {
            const uint32_t *qlo = reinterpret_cast<const uint32_t *>(a.q + ((size_t)cs.seq * a.Hq + h0 + g8) * D);
            const uint32_t *qhi = reinterpret_cast<const uint32_t *>(a.q + ((size_t)cs.seq * a.Hq + h0 + g8 + 8) * D);
            const bool vlo = g8 < rows;
            const bool vhi = TWO && (g8 + 8 < rows);
#pragma unroll
            for (int ks = 0; ks < kKSteps; ++ks) {
                qa[ks][0] = vlo ? __ldg(qlo + ks * 8 + c4) : 0u;
                qa[ks][2] = vlo ? __ldg(qlo + ks * 8 + 4 + c4) : 0u;
                qa[ks][1] = vhi ? __ldg(qhi + ks * 8 + c4) : 0u;
                qa[ks][3] = vhi ? __ldg(qhi + ks * 8 + 4 + c4) : 0u;
            }
        }

        float o[kNTiles][4];
#pragma unroll
        for (int j = 0; j < kNTiles; ++j)
            o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        float m_lo = -INFINITY, l_lo = 0.f, m_hi = -INFINITY, l_hi = 0.f;

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
            const uint32_t kb = ring_base + stage * 2 * kTile;
            const uint32_t vb = kb + kTile;
            const int nvalid = min(kTileTokens, cs.ctx - t * kTileTokens);

            // S^T tile: rows = query heads, columns = 16 tokens (two n-tiles of 8)
            float sc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
            for (int kc = 0; kc < D / 32; ++kc) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int row = nt * 8 + (lane & 7);
                    const int chunk = kc * 4 + (lane >> 3);
                    const uint32_t addr = kb + (chunk >> 3) * kBoxBytes + row * 128 +
                                          ((uint32_t)((chunk & 7) ^ (row & 7)) << 4);
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(addr, b0, b1, b2, b3);
                    mma_16816<BF16>(sc[nt], qa[2 * kc], b0, b1);
                    mma_16816<BF16>(sc[nt], qa[2 * kc + 1], b2, b3);
                }
            }

            // online softmax (log2 domain)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tok = nt * 8 + 2 * c4 + (i & 1);
                    const float v = sc[nt][i] * a.scale_log2;
                    sc[nt][i] = tok < nvalid ? v : -INFINITY;
                }
            }
            float mx = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
            const float mnew = fmaxf(m_lo, mx);
            const float alpha = exp2f(m_lo - mnew);
            m_lo = mnew;
            float p00 = exp2f(sc[0][0] - mnew), p01 = exp2f(sc[0][1] - mnew);
            float p10 = exp2f(sc[1][0] - mnew), p11 = exp2f(sc[1][1] - mnew);
            l_lo = l_lo * alpha + ((p00 + p01) + (p10 + p11));
            float alpha_hi = 1.f, q00 = 0.f, q01 = 0.f, q10 = 0.f, q11 = 0.f;
            if constexpr (TWO) {
                float mh = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
                mh = fmaxf(mh, __shfl_xor_sync(FULL, mh, 1));
                mh = fmaxf(mh, __shfl_xor_sync(FULL, mh, 2));
                const float mnh = fmaxf(m_hi, mh);
                alpha_hi = exp2f(m_hi - mnh);
                m_hi = mnh;
                q00 = exp2f(sc[0][2] - mnh);
                q01 = exp2f(sc[0][3] - mnh);
                q10 = exp2f(sc[1][2] - mnh);
                q11 = exp2f(sc[1][3] - mnh);
                l_hi = l_hi * alpha_hi + ((q00 + q01) + (q10 + q11));
            }
#pragma unroll
            for (int j = 0; j < kNTiles; ++j) {
                o[j][0] *= alpha;
                o[j][1] *= alpha;
                if constexpr (TWO) {
                    o[j][2] *= alpha_hi;
                    o[j][3] *= alpha_hi;
                }
            }
            uint32_t pa[4];
            pa[0] = pack2<BF16>(p00, p01);
            pa[1] = TWO ? pack2<BF16>(q00, q01) : 0u;
            pa[2] = pack2<BF16>(p10, p11);
            pa[3] = TWO ? pack2<BF16>(q10, q11) : 0u;

            // positions past the context may hold anything (even NaN): zero
            // their V so that 0 * V stays 0 in the MMA
            uint32_t m01 = 0xffffffffu, m23 = 0xffffffffu;
            if (nvalid < kTileTokens) {
                m01 = (2 * c4 < nvalid ? 0x0000ffffu : 0u) | (2 * c4 + 1 < nvalid ? 0xffff0000u : 0u);
                m23 = (2 * c4 + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c4 + 9 < nvalid ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int jj = 0; jj < D / 16; ++jj) {
                const int mi = lane >> 3;
                const int tok = (lane & 7) + 8 * (mi & 1);
                const int chunk = 2 * jj + (mi >> 1);
                const uint32_t addr = vb + (chunk >> 3) * kBoxBytes + tok * 128 +
                                      ((uint32_t)((chunk & 7) ^ (tok & 7)) << 4);
                uint32_t v0, v1, v2, v3;
                ldmatrix_x4_trans(addr, v0, v1, v2, v3);
                mma_16816<BF16>(o[2 * jj], pa, v0 & m01, v1 & m23);
                mma_16816<BF16>(o[2 * jj + 1], pa, v2 & m01, v3 & m23);
            }

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
        if (failed)
            break;

        // ---- epilogue: final output (normalised) or a partial (m, l, o)
        l_lo += __shfl_xor_sync(FULL, l_lo, 1);
        l_lo += __shfl_xor_sync(FULL, l_lo, 2);
        if constexpr (TWO) {
            l_hi += __shfl_xor_sync(FULL, l_hi, 1);
            l_hi += __shfl_xor_sync(FULL, l_hi, 2);
        }
        if (cs.dest < 0) {
            const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f;
            const float inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
            if (g8 < rows) {
                uint32_t *dst = reinterpret_cast<uint32_t *>(a.out + ((size_t)cs.seq * a.Hq + h0 + g8) * D);
#pragma unroll
                for (int j = 0; j < kNTiles; ++j)
                    dst[j * 4 + c4] = pack2<BF16>(o[j][0] * inv_lo, o[j][1] * inv_lo);
            }
            if (TWO && g8 + 8 < rows) {
                uint32_t *dst = reinterpret_cast<uint32_t *>(a.out + ((size_t)cs.seq * a.Hq + h0 + g8 + 8) * D);
#pragma unroll
                for (int j = 0; j < kNTiles; ++j)
                    dst[j * 4 + c4] = pack2<BF16>(o[j][2] * inv_hi, o[j][3] * inv_hi);
            }
        } else {
            for (int half = 0; half < (TWO ? 2 : 1); ++half) {
                const int g = g8 + 8 * half;
                if (g >= rows)
                    continue;
                size_t row;
                if (a.mode == kModePartition)
                    row = ((size_t)cs.seq * a.Hq + h0 + g) * a.S + cs.dest;
                else
                    row = (size_t)cs.dest * kMaxRows + g;
                float2 *dst = reinterpret_cast<float2 *>(a.part_o + row * D);
#pragma unroll
                for (int j = 0; j < kNTiles; ++j)
                    dst[j * 4 + c4] = half ? make_float2(o[j][2], o[j][3]) : make_float2(o[j][0], o[j][1]);
                if (c4 == 0) {
                    a.part_m[row] = half ? m_hi : m_lo;
                    a.part_l[row] = half ? l_hi : l_lo;
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

// ------------------------------------------------------------- merge kernel

struct MergeArgs {
    uint16_t *out;
    const int32_t *context_lens;
    const int32_t *prefix;   // balanced: tile prefix written by the decode kernel
    const float *part_o, *part_m, *part_l;
    int64_t mb;
    int B, Hq, G, n_hg, npairs, bs, D;
    int mode, part_tiles, S, total_warps;
    unsigned *err;
};

constexpr int kMergeChunk = 64;

// One CTA per (sequence, KV-head group): combine the partial results of the
// pieces the context was split into.  M = max m_j, L = sum l_j 2^(m_j - M),
// out = sum o_j 2^(m_j - M) / L.  Pieces with m = -inf weigh 0.
template <bool BF16>
__global__ void __launch_bounds__(256) lse_merge_kernel(const MergeArgs a) {
    const int seq = blockIdx.x / a.npairs;
    const int pair = blockIdx.x - seq * a.npairs;
    const int kvh = pair / a.n_hg;
    const int hg = pair - kvh * a.n_hg;
    const int h0 = kvh * a.G + hg * kMaxRows;
    const int rows = min(kMaxRows, a.G - hg * kMaxRows);

    long long first = 0, count = 0;       // partition: j in [0, count)
    long long a0 = 0, T = 0;              // balanced
    if (a.mode == kModePartition) {
        int c = a.context_lens[seq];
        const int64_t cap = a.mb * a.bs;
        c = c < 0 ? 0 : (c > cap ? (int)cap : c);
        const int nt = (c + kTileTokens - 1) / kTileTokens;
        count = (nt + a.part_tiles - 1) / a.part_tiles;
        if (count <= 1)
            return;  // written directly by the decode kernel (or all-zero)
    } else {
        const int nt = a.prefix[seq + 1] - a.prefix[seq];
        if (nt == 0)
            return;
        T = (long long)a.prefix[a.B] * a.npairs;
        a0 = (long long)a.prefix[seq] * a.npairs + (long long)pair * nt;
        const long long b0 = a0 + nt;
        const long long W = a.total_warps;
        first = ((a0 + 1) * W + T - 1) / T - 1;        // warp holding index a0
        const long long last = (b0 * W + T - 1) / T - 1;  // warp holding index b0 - 1
        if (first == last)
            return;  // the whole pair sat in one warp: already final
        count = last - first + 1;
    }

    __shared__ float s_m[kMaxRows], s_inv[kMaxRows];
    __shared__ float s_w[kMaxRows][kMergeChunk];
    __shared__ long long s_row[kMergeChunk];  // partial row base (row index * 16 or per-head)
    __shared__ int s_ok[kMergeChunk];

    // row index of piece k for head row g
    auto piece_row = [&](long long k, int g, bool &ok) -> long long {
        ok = true;
        if (a.mode == kModePartition)
            return ((long long)seq * a.Hq + h0 + g) * a.S + k;
        const long long w = first + k;
        const long long lo = w * T / a.total_warps;
        const long long hi = (w + 1) * T / a.total_warps;
        if (lo >= hi) {
            ok = false;
            return 0;
        }
        const long long slot = 2 * w + (a0 < lo ? 0 : 1);
        return slot * kMaxRows + g;
    };

    // pass 1: per-row max and normaliser
    if (threadIdx.x < rows) {
        const int g = threadIdx.x;
        float M = -INFINITY;
        for (long long k = 0; k < count; ++k) {
            bool ok;
            const long long r = piece_row(k, g, ok);
            if (ok)
                M = fmaxf(M, a.part_m[r]);
        }
        float Lsum = 0.f;
        if (M != -INFINITY) {
            for (long long k = 0; k < count; ++k) {
                bool ok;
                const long long r = piece_row(k, g, ok);
                if (ok && a.part_m[r] != -INFINITY)
                    Lsum += a.part_l[r] * exp2f(a.part_m[r] - M);
            }
        }
        s_m[g] = M;
        s_inv[g] = Lsum > 0.f ? 1.f / Lsum : 0.f;
    }
    __syncthreads();

    // pass 2: weighted sum of the partial outputs, chunk by chunk.  Each
    // thread owns up to kMaxPer pairs of consecutive d (rows <= 16, D <= 128,
    // 256 threads).
    constexpr int kMaxPer = 4;
    const int D = a.D;
    const int per_row = D / 2;
    const int n_elem = rows * per_row;
    float acc[kMaxPer][2];
#pragma unroll
    for (int e = 0; e < kMaxPer; ++e)
        acc[e][0] = acc[e][1] = 0.f;
    for (long long k0 = 0; k0 < count; k0 += kMergeChunk) {
        const int kn = (int)min((long long)kMergeChunk, count - k0);
        for (int i = threadIdx.x; i < rows * kn; i += blockDim.x) {
            const int g = i / kn, k = i - g * kn;
            bool ok;
            const long long r = piece_row(k0 + k, g, ok);
            float w = 0.f;
            if (ok && s_m[g] != -INFINITY && a.part_m[r] != -INFINITY)
                w = exp2f(a.part_m[r] - s_m[g]) * s_inv[g];
            s_w[g][k] = w;
            if (g == 0) {
                s_row[k] = ok ? r : -1;
                s_ok[k] = ok;
            }
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < kMaxPer; ++e) {
            const int idx = threadIdx.x + e * blockDim.x;
            if (idx < n_elem) {
                const int g = idx / per_row;
                const int d = (idx - g * per_row) * 2;
                float x0 = acc[e][0], x1 = acc[e][1];
                for (int k = 0; k < kn; ++k) {
                    if (!s_ok[k])
                        continue;
                    const float w = s_w[g][k];
                    // rows of the other heads: +g*S (partition layout) or +g (slots)
                    const long long r = a.mode == kModePartition ? s_row[k] + (long long)g * a.S
                                                                 : s_row[k] + g;
                    const float2 v = *reinterpret_cast<const float2 *>(a.part_o + r * D + d);
                    x0 += w * v.x;
                    x1 += w * v.y;
                }
                acc[e][0] = x0;
                acc[e][1] = x1;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int e = 0; e < kMaxPer; ++e) {
        const int idx = threadIdx.x + e * blockDim.x;
        if (idx < n_elem) {
            const int g = idx / per_row;
            const int d = (idx - g * per_row) * 2;
            uint32_t *dst = reinterpret_cast<uint32_t *>(a.out + ((size_t)seq * a.Hq + h0 + g) * D + d);
            *dst = pack2<BF16>(acc[e][0], acc[e][1]);
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

}  // namespace pkv
