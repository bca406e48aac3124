// C ABI of the device calls: argument validation, TMA tensor maps, launch
// planning and the split-context workspace layout.  Every kernel lives in
// decode.cuh (one translation unit so that the device error word is shared).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <algorithm>
#include <mutex>
#include <utility>
#include <tuple>
#include <vector>

#include "decode.cuh"
#include "mq_attention.cuh"
#include "pkv.h"

namespace pkv {

__device__ unsigned g_error_word = 0;

namespace {

constexpr int kMaxSmemPerCta = 226 * 1024;  // 227 KB opt-in limit minus static smem

// testing hook state (pkv_test_inject_wait_timeout)
int g_inject_no_issue = 0;
uint64_t g_wait_limit_ns = kWaitLimitNs;

int env_int(const char *name, int dflt) {
    const char *v = std::getenv(name);
    if (!v || !*v)
        return dflt;
    return std::atoi(v);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool cache_ok(const pkv_cache &c) {
    return c.data && aligned16(c.data) && (c.dtype == PKV_F16 || c.dtype == PKV_BF16) &&
           c.num_blocks > 0 && c.block_size > 0 && c.num_kv_heads > 0 && c.head_dim > 0;
}

bool cache_ok_e4m3(const pkv_cache &c) {
    return c.data && aligned16(c.data) && c.dtype == PKV_E4M3 && c.scales && aligned16(c.scales) &&
           c.num_blocks > 0 && c.block_size > 0 && c.num_kv_heads > 0 && c.head_dim > 0;
}

bool same_shape(const pkv_cache &a, const pkv_cache &b) {
    return a.dtype == b.dtype && a.num_blocks == b.num_blocks && a.block_size == b.block_size &&
           a.num_kv_heads == b.num_kv_heads && a.head_dim == b.head_dim;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Remember a failed runtime call for pkv_last_cuda_error().
bool cuda_ok(cudaError_t e) {
    if (e != cudaSuccess) {
        g_last_cuda_error = e;
        return false;
    }
    return true;
}

unsigned *error_word() {
    static unsigned *ptr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    if (!ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess)
            return nullptr;
        ptr[dev] = static_cast<unsigned *>(p);
    }
    return ptr[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool make_pool_map_uncached(CUtensorMap *map, const pkv_cache &c);

// Tensor maps are plain host encodings of (pointer, shape); a decode loop
// over the same pool reuses them.
bool make_pool_map(CUtensorMap *map, const pkv_cache &c) {
    struct Entry {
        void *data;
        int dtype;
        int64_t nb, bs, hkv, d;
        CUtensorMap map;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const Entry &e : cache)
            if (e.data == c.data && e.dtype == c.dtype && e.nb == c.num_blocks && e.bs == c.block_size &&
                e.hkv == c.num_kv_heads && e.d == c.head_dim) {
                *map = e.map;
                return true;
            }
    }
    if (!make_pool_map_uncached(map, c))
        return false;
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() >= 32)
        cache.erase(cache.begin());
    cache.push_back(Entry{c.data, (int)c.dtype, c.num_blocks, c.block_size, c.num_kv_heads, c.head_dim, *map});
    return true;
}

// The pool viewed as a 2-D tensor: rows = NB * Hkv * bs, columns = D; one TMA
// box = 16 rows x 64 columns (128 bytes per row), 128-byte swizzle.
bool make_pool_map_uncached(CUtensorMap *map, const pkv_cache &c) {
    auto fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)c.head_dim,
                          (cuuint64_t)(c.num_blocks * c.num_kv_heads * c.block_size)};
    cuuint32_t estr[2] = {1, 1};
    if (c.dtype == PKV_E4M3) {
        // E4M3 codes: one box = 16 rows x D bytes, swizzled over the row
        // width (128-byte swizzle for D = 128, 64-byte for D = 64) so that
        // the kernel's per-lane row reads are free of bank conflicts
        cuuint64_t strides[1] = {(cuuint64_t)c.head_dim};
        cuuint32_t box[2] = {(cuuint32_t)c.head_dim, (cuuint32_t)kTileTokens};
        const CUtensorMapSwizzle sw = c.head_dim == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
        CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, c.data, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        return r == CUDA_SUCCESS;
    }
    cuuint64_t strides[1] = {(cuuint64_t)c.head_dim * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBoxCols, (cuuint32_t)kTileTokens};
    CUtensorMapDataType dt =
        c.dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUresult r = fn(map, dt, 2, c.data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The query rows of a chunked-prefill call, q [T][Hq][D], as a 3-D tensor
// (columns, heads, tokens); one box = 64 columns x G heads x tpb tokens
// (128-byte swizzle), i.e. the rows (token, head of the group) of one unit
// of the multi-query kernel, one 128-byte column half at a time.
bool make_q_map(CUtensorMap *map, const void *q, int64_t T, int64_t Hq, int64_t D, int G, int tpb, bool bf16) {
    auto fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)(Hq * D * 2)};
    cuuint32_t box[3] = {64u, (cuuint32_t)G, (cuuint32_t)tpb};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                    const_cast<void *>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct Plan {
    int mode = kModeDirect;
    int warps = 4;
    int stages = 3;
    int ctas = 0;
    int total_warps = 0;
    int max_total_warps = 0;  // warps of the largest grid this shape may launch
    int part_tiles = 0;
    int S = 0;
    int smem = 0;
    int Hkv = 0, G = 0, n_hg = 0, npairs = 0;
    int nt = 1, hpu = 8;  // MMA column tiles and query heads per unit
    bool fma = false;     // CUDA-core variant (PKV_FMA=1, 16-bit pools only)
};

using DecodeKernel = void (*)(const CUtensorMap, const CUtensorMap, const DecodeArgs);

// NT = number of 8-head MMA column tiles per unit: 1 for G <= 8, else 2.
// bf16: q / out dtype; fp8: E4M3 pools; fma: the CUDA-core variant (16-bit
// pools, 8 heads per unit), kept to compare against the MMA kernel.
DecodeKernel pick_decode(int D, bool bf16, int nt, bool fp8 = false, bool fma = false, bool cas = false) {
    if (cas) {
        if (fp8 || fma)
            return nullptr;
#define PKV_PICK_CAS(DD, BB, NN) \
    if (D == DD && bf16 == BB && nt == NN) return paged_decode_kernel<DD, BB, NN, false, false, true>;
        PKV_PICK_CAS(64, false, 1)
        PKV_PICK_CAS(64, false, 2)
        PKV_PICK_CAS(64, true, 1)
        PKV_PICK_CAS(64, true, 2)
        PKV_PICK_CAS(128, false, 1)
        PKV_PICK_CAS(128, false, 2)
        PKV_PICK_CAS(128, true, 1)
        PKV_PICK_CAS(128, true, 2)
#undef PKV_PICK_CAS
        return nullptr;
    }
    if (fma) {
        if (fp8 || nt != 1)
            return nullptr;
        if (D == 64)
            return bf16 ? paged_decode_kernel<64, true, 1, false, true> : paged_decode_kernel<64, false, 1, false, true>;
        if (D == 128)
            return bf16 ? paged_decode_kernel<128, true, 1, false, true>
                        : paged_decode_kernel<128, false, 1, false, true>;
        return nullptr;
    }
#define PKV_PICK(DD, BB, NN, FF) \
    if (D == DD && bf16 == BB && nt == NN && fp8 == FF) return paged_decode_kernel<DD, BB, NN, FF>;
#define PKV_PICK_ALL(FF)          \
    PKV_PICK(64, false, 1, FF)    \
    PKV_PICK(64, false, 2, FF)    \
    PKV_PICK(64, true, 1, FF)     \
    PKV_PICK(64, true, 2, FF)     \
    PKV_PICK(128, false, 1, FF)   \
    PKV_PICK(128, false, 2, FF)   \
    PKV_PICK(128, true, 1, FF)    \
    PKV_PICK(128, true, 2, FF)
    PKV_PICK_ALL(false)
    PKV_PICK_ALL(true)
#undef PKV_PICK_ALL
#undef PKV_PICK
    return nullptr;
}

int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel in the stream is still running; it calls
// griddepcontrol.wait before reading anything that kernel may have written.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Decide schedule, CTA shape and grid.  PKV_ERR_INVALID if the shape cannot
// be run (shared memory), PKV_ERR_CUDA if the device cannot be queried.
pkv_status make_plan_uncached(Plan &p, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t max_ctx,
                              int32_t partition_tokens, bool have_workspace, bool bf16, bool for_launch,
                              bool fp8);

// Plans depend only on the shape, the device and two tuning variables; they
// are cached so that a steady decode loop pays no occupancy queries.
// Balanced schedules: virtual tiles weighed per (sequence, head group), the
// unit's fixed cost (query load, resume, epilogue) in tile-equivalents.  A
// batch of many one- and two-tile units (the suffixes left after a shared
// prefix) otherwise gives the warps that draw them several times the work of
// the warps that stream long units.  PKV_UNIT_COST overrides it (0..8).
constexpr int kMaxUnitCost = 8;
int unit_cost() {
    const int v = env_int("PKV_UNIT_COST", 3);
    return v < 0 ? 0 : (v > kMaxUnitCost ? kMaxUnitCost : v);
}

struct PlanKey {
    int dev, warps_env, stages_env, fma_env;
    int64_t B, Hq, Hkv, D, max_ctx;
    int32_t partition;
    bool ws, bf16, launch, fp8;
    bool operator==(const PlanKey &o) const {
        return dev == o.dev && warps_env == o.warps_env && stages_env == o.stages_env &&
               fma_env == o.fma_env && B == o.B &&
               Hq == o.Hq && Hkv == o.Hkv && D == o.D && max_ctx == o.max_ctx &&
               partition == o.partition && ws == o.ws && bf16 == o.bf16 && launch == o.launch &&
               fp8 == o.fp8;
    }
};

pkv_status make_plan(Plan &p, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t max_ctx,
                     int32_t partition_tokens, bool have_workspace, bool bf16, bool for_launch,
                     bool fp8 = false) {
    static std::mutex mu;
    static std::vector<std::pair<PlanKey, Plan>> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PKV_ERR_CUDA;
    const PlanKey key{dev, env_int("PKV_WARPS", 0), env_int("PKV_STAGES", 0), env_int("PKV_FMA", 0),
                      B, Hq, Hkv, D, max_ctx,
                      partition_tokens, have_workspace, bf16, for_launch, fp8};
    {
        std::lock_guard<std::mutex> lock(mu);
        for (auto &e : cache)
            if (e.first == key) {
                p = e.second;
                return PKV_OK;
            }
    }
    pkv_status st = make_plan_uncached(p, B, Hq, Hkv, D, max_ctx, partition_tokens, have_workspace, bf16,
                                       for_launch, fp8);
    if (st == PKV_OK) {
        std::lock_guard<std::mutex> lock(mu);
        if (cache.size() >= 64)
            cache.erase(cache.begin());
        cache.emplace_back(key, p);
    }
    return st;
}

pkv_status make_plan_uncached(Plan &p, int64_t B, int64_t Hq, int64_t Hkv, int64_t D, int64_t max_ctx,
                              int32_t partition_tokens, bool have_workspace, bool bf16, bool for_launch,
                              bool fp8) {
    p.Hkv = (int)Hkv;
    p.G = (int)(Hq / Hkv);
    // the CUDA-core variant is a measurement aid for the choice of the MMA
    // (same pipeline and schedules, FFMA arithmetic); 16-bit pools only
    p.fma = !fp8 && env_int("PKV_FMA", 0) == 1;
    p.nt = (p.G > 8 && !p.fma) ? 2 : 1;
    p.hpu = 8 * p.nt;
    p.n_hg = (p.G + p.hpu - 1) / p.hpu;
    p.npairs = (int)Hkv * p.n_hg;
    // CTA shape, from measurements on B200 (two 8 KB stages per warp):
    //  * large batches (>= 128 sequences, continuous-batching mixes) switch
    //    units often and hide that latency best with 12 warps per SM (two
    //    6-warp CTAs);
    //  * otherwise one 8-warp CTA per SM.
    //  * E4M3 pools: two 6-warp CTAs per SM everywhere (the conversions
    //    lengthen each tile's instruction chain; more warps hide it).
    const int dflt_warps = ((partition_tokens <= 0 && B >= 128) || fp8) ? 6 : 8;
    p.warps = env_int("PKV_WARPS", dflt_warps);
    // E4M3 stages are half the bytes: twice as many keep as much in flight
    p.stages = env_int("PKV_STAGES", fp8 ? 4 : 2);
    if (p.warps < 1 || p.warps > 8)
        p.warps = 8;
    if (p.stages < 2 || p.stages > 16)
        p.stages = 3;
    if (partition_tokens > 0) {
        p.mode = kModePartition;
        p.part_tiles = partition_tokens / kTileTokens;
        p.S = (int)ceil_div64(max_ctx, partition_tokens);
        if (p.S < 1)
            p.S = 1;
    } else if (partition_tokens == PKV_PARTITION_AUTO && have_workspace) {
        p.mode = kModeBalanced;
    } else {
        p.mode = kModeDirect;
    }
    const bool need_prefix = p.mode != kModeDirect;
    // the on-chip schedule keeps per-sequence tile counts in int32
    if (need_prefix && B * (ceil_div64(max_ctx, kTileTokens) + kMaxUnitCost) * p.npairs >= (int64_t(1) << 31))
        return PKV_ERR_INVALID;
    for (;;) {
        SmemLayout L = decode_smem_layout((int)B, p.warps, p.stages, (int)D, need_prefix, fp8, p.fma);
        p.smem = L.total;
        if (p.smem <= kMaxSmemPerCta)
            break;
        if (p.stages > 2)
            --p.stages;
        else if (p.warps > 1)
            --p.warps;
        else
            return PKV_ERR_INVALID;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PKV_ERR_CUDA;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int per_sm = 1;
    DecodeKernel k = pick_decode((int)D, bf16, p.nt, fp8, p.fma);
    if (!k)
        return PKV_ERR_INVALID;
    // The attribute is per-kernel state shared by every cached plan: set the
    // ceiling, never a plan's own size (a smaller plan would otherwise lower
    // it under a larger one).  It only permits; occupancy uses p.smem.
    if (!cuda_ok(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemPerCta)))
        return PKV_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, p.warps * 32, p.smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t max_ctas = (int64_t)sms * per_sm;
    p.max_total_warps = (int)(max_ctas * p.warps);
    int64_t want = max_ctas;
    if (for_launch) {
        const int64_t tiles_upper = ceil_div64(max_ctx, kTileTokens);
        int64_t units;
        if (p.mode == kModeDirect)
            units = B * p.npairs;
        else if (p.mode == kModePartition)
            units = B * p.npairs * p.S;
        else
            units = ceil_div64(B * p.npairs * tiles_upper, 4);  // >= ~4 tiles per warp
        if (p.mode == kModePartition) {
            // equal-sized units taken round-robin: the makespan is
            // ceil(units / warps) units; keep the smallest makespan the grid
            // allows with the fewest warps (less contention for the same time)
            const int64_t max_w = max_ctas * p.warps;
            const int64_t rounds = ceil_div64(units, max_w);
            units = ceil_div64(units, rounds);
        }
        want = std::min<int64_t>(max_ctas, std::max<int64_t>(1, ceil_div64(units, p.warps)));
    }
    p.ctas = (int)want;
    p.total_warps = p.ctas * p.warps;
    return PKV_OK;
}

// Workspace layout.
//  partition: part_o [B][Hq][S][D] f32 | part_m [B][Hq][S] f32 | part_l [B][Hq][S] f32
//  balanced:  prefix [B+1] i32 + pieces bound (256-aligned) | part_m [2W][16] | part_l [2W][16] | part_o [2W][16][D]
//             | piece counters [B][npairs] i32, with W = the largest warp count a launch may use.
struct WsLayout {
    size_t prefix = 0, m = 0, l = 0, o = 0, cnt = 0, total = 0;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(const Plan &p, int64_t B, int64_t Hq, int64_t D, int64_t max_warps) {
    WsLayout w;
    if (p.mode == kModePartition) {
        const size_t rows = (size_t)B * Hq * p.S;
        w.o = 0;
        w.m = align256(rows * D * 4);
        w.l = align256(w.m + rows * 4);
        w.total = align256(w.l + rows * 4);
    } else if (p.mode == kModeBalanced) {
        const size_t slots = (size_t)2 * max_warps;
        w.prefix = 0;
        w.m = align256((size_t)(B + 2) * 4);
        w.l = align256(w.m + slots * kMaxRows * 4);
        w.o = align256(w.l + slots * kMaxRows * 4);
        w.cnt = align256(w.o + slots * kMaxRows * D * 4);  // piece counters [B][npairs]
        w.total = align256(w.cnt + (size_t)B * p.npairs * 4);
    }
    return w;
}

// Launch the multi-query kernel.  Prefill: every chunk of two or more tokens
// (the expansion kernel has zeroed its unit counter and given those tokens
// no decode work).  Prefix: every sharing group's common prefix (the cascade
// preparation kernel has zeroed the counter and filled the group arrays).
// One CTA per SM, programmatic stream serialisation.
pkv_status mq_launch(MqArgs a, const void *q, int64_t nz, const pkv_cache &kc, const pkv_cache &vc, float scale,
                     pkv_stream stream) {
    const int64_t Hkv = kc.num_kv_heads, D = kc.head_dim;
    a.Hkv = (int)Hkv;
    a.G = (int)(a.Hq / Hkv);
    a.tpb = kMqRows / a.G;
    a.nb = kc.num_blocks;
    a.bs = (int)kc.block_size;
    a.scale_log2 = std::fabs(scale) * 1.4426950408889634f;
    a.negate_q = scale < 0.0f ? 1 : 0;
    a.pool_rows = (int)(kc.num_blocks * Hkv * kc.block_size);
    a.wait_limit_ns = g_wait_limit_ns;
    a.inject_no_issue = g_inject_no_issue;
    const bool bf16 = kc.dtype == PKV_BF16;
    CUtensorMap tmQ, tmK, tmV;
    if (!make_q_map(&tmQ, q, nz, a.Hq, D, a.G, a.tpb, bf16) || !make_pool_map(&tmK, kc) || !make_pool_map(&tmV, vc))
        return PKV_ERR_CUDA;
    void (*k)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const MqArgs) = nullptr;
    int smem = 0;
    // PKV_MQ_POLY=n (1..3): n of every 8 probability pairs by the FMA-pipe exp2
    const int poly = env_int("PKV_MQ_POLY", 0);
    if (D == 128) {
        if (poly == 1)
            k = bf16 ? mq_attention_kernel<128, true, 1> : mq_attention_kernel<128, false, 1>;
        else if (poly == 2)
            k = bf16 ? mq_attention_kernel<128, true, 2> : mq_attention_kernel<128, false, 2>;
        else if (poly == 3)
            k = bf16 ? mq_attention_kernel<128, true, 3> : mq_attention_kernel<128, false, 3>;
        else
            k = bf16 ? mq_attention_kernel<128, true> : mq_attention_kernel<128, false>;
        smem = MqSmem<128>::bytes(a.nsrc);
    } else {
        k = bf16 ? mq_attention_kernel<64, true> : mq_attention_kernel<64, false>;
        smem = MqSmem<64>::bytes(a.nsrc);
    }
    // one CTA per SM: a second one would only wait for the first's TMEM
    smem = std::max(smem, kMaxSmemPerCta / 2 + 1024);
    if (smem > kMaxSmemPerCta)
        return PKV_ERR_INVALID;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return PKV_ERR_CUDA;
    {
        // shared-memory ceiling and SM count, once per (device, kernel)
        static std::mutex mu;
        static std::vector<std::tuple<int, const void *, int>> done;
        std::lock_guard<std::mutex> lock(mu);
        bool found = false;
        for (auto &e : done)
            if (std::get<0>(e) == dev && std::get<1>(e) == (const void *)k) {
                sms = std::get<2>(e);
                found = true;
            }
        if (!found) {
            if (!cuda_ok(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemPerCta)))
                return PKV_ERR_CUDA;
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            done.emplace_back(dev, (const void *)k, sms);
        }
    }
    if (!cuda_ok(launch_dependent(k, dim3(sms), dim3(kMqThreads), smem, (cudaStream_t)stream, tmQ, tmK, tmV, a)))
        return PKV_ERR_CUDA;
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

pkv_status pkv_append(const void *k_new, const void *v_new, const int64_t *slot_mapping,
                      int64_t num_tokens, pkv_cache k_cache, pkv_cache v_cache, pkv_stream stream) {
    if (num_tokens < 0)
        return PKV_ERR_INVALID;
    if (!cache_ok(k_cache) || !cache_ok(v_cache) || !same_shape(k_cache, v_cache))
        return PKV_ERR_INVALID;
    if (k_cache.head_dim % 8 != 0)
        return PKV_ERR_INVALID;
    if (num_tokens == 0)
        return PKV_OK;
    if (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PKV_ERR_INVALID;
    unsigned *err = error_word();
    if (!err)
        return PKV_ERR_CUDA;
    const int chunks = (int)(k_cache.head_dim / 8);
    const int64_t total = num_tokens * k_cache.num_kv_heads * chunks;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 148 * 32)
        blocks = 148 * 32;
    append_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slot_mapping,
        num_tokens, (int)k_cache.num_kv_heads, chunks, (int)k_cache.block_size,
        k_cache.num_blocks, static_cast<uint4 *>(k_cache.data), static_cast<uint4 *>(v_cache.data),
        err);
    return cuda_ok(cudaGetLastError()) ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_copy_blocks(pkv_cache k_cache, pkv_cache v_cache, const int32_t *pairs, int64_t num_pairs,
                           pkv_stream stream) {
    if (num_pairs < 0 || !cache_ok(k_cache) || !cache_ok(v_cache) || !same_shape(k_cache, v_cache))
        return PKV_ERR_INVALID;
    if (num_pairs == 0)
        return PKV_OK;
    if (!pairs || (reinterpret_cast<uintptr_t>(pairs) & 7u))
        return PKV_ERR_INVALID;
    const int64_t block_bytes = k_cache.num_kv_heads * k_cache.block_size * k_cache.head_dim * 2;
    if (block_bytes % 16)
        return PKV_ERR_INVALID;
    unsigned *err = error_word();
    if (!err)
        return PKV_ERR_CUDA;
    const int64_t chunks = block_bytes / 16;
    const int64_t total = num_pairs * chunks;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 148 * 32)
        blocks = 148 * 32;
    copy_blocks_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
        pairs, num_pairs, chunks, k_cache.num_blocks, static_cast<uint4 *>(k_cache.data),
        static_cast<uint4 *>(v_cache.data), err);
    return cuda_ok(cudaGetLastError()) ? PKV_OK : PKV_ERR_CUDA;
}

size_t pkv_decode_workspace_bytes(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                  int64_t head_dim, int64_t max_context_len,
                                  int32_t partition_tokens) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
        (head_dim != 64 && head_dim != 128) || max_context_len < 0)
        return 0;
    if (partition_tokens == PKV_PARTITION_NONE)
        return 0;
    if (partition_tokens < 0 || partition_tokens % kTileTokens)
        return 0;
    // the largest of the layouts a 16-bit or an E4M3 launch of this shape may use
    size_t best = 0;
    for (int fp8 = 0; fp8 < 2; ++fp8) {
        Plan p;
        if (make_plan(p, num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                      partition_tokens, true, false, false, fp8 != 0) != PKV_OK)
            return 0;
        best = std::max(best, ws_layout(p, num_seqs, num_q_heads, head_dim, p.max_total_warps).total);
    }
    return best;
}

}  // extern "C"

namespace {

struct FusedAppend {
    const void *k_new, *v_new;
    const int64_t *slots;
};

// Shared-prefix cascade inputs of the decode kernel (see DecodeArgs).
struct CascadeIn {
    const int32_t *table_offset;
    const float *init_o, *init_m, *init_l;
};

pkv_status decode_impl(const void *q, int64_t num_seqs, int64_t num_q_heads, pkv_cache k_cache,
                       pkv_cache v_cache, const int32_t *block_tables, int64_t max_blocks_per_seq,
                       const int32_t *context_lens, float scale, void *out, void *workspace,
                       size_t workspace_bytes, int32_t partition_tokens, pkv_stream stream,
                       const FusedAppend *fa, const int32_t *table_rows = nullptr,
                       pkv_dtype q_dtype = PKV_F16, const CascadeIn *cas = nullptr) {
    if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0)
        return PKV_ERR_INVALID;
    const bool fp8 = k_cache.dtype == PKV_E4M3;
    if (fp8) {
        if (!cache_ok_e4m3(k_cache) || !cache_ok_e4m3(v_cache) || !same_shape(k_cache, v_cache) || fa ||
            (q_dtype != PKV_F16 && q_dtype != PKV_BF16))
            return PKV_ERR_INVALID;
    } else {
        if (!cache_ok(k_cache) || !cache_ok(v_cache) || !same_shape(k_cache, v_cache))
            return PKV_ERR_INVALID;
        q_dtype = k_cache.dtype;
    }
    const int64_t Hkv = k_cache.num_kv_heads, D = k_cache.head_dim, bs = k_cache.block_size;
    if (num_q_heads % Hkv != 0 || (D != 64 && D != 128) || bs % kTileTokens != 0)
        return PKV_ERR_INVALID;
    if (!std::isfinite(scale))
        return PKV_ERR_INVALID;
    if (partition_tokens < PKV_PARTITION_NONE ||
        (partition_tokens > 0 && partition_tokens % kTileTokens != 0))
        return PKV_ERR_INVALID;
    // TMA coordinates are 32-bit; the row count of the pool view must fit
    if (k_cache.num_blocks * Hkv * bs >= (int64_t(1) << 31))
        return PKV_ERR_INVALID;
    if (max_blocks_per_seq * bs >= (int64_t(1) << 30) || num_seqs >= (int64_t(1) << 24) ||
        num_q_heads * D >= (int64_t(1) << 24))
        return PKV_ERR_INVALID;
    if (num_seqs == 0)
        return PKV_OK;
    if (!q || !out || !block_tables || !context_lens || !aligned16(q) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u))
        return PKV_ERR_INVALID;
    const bool bf16 = q_dtype == PKV_BF16;
    const int64_t max_ctx = max_blocks_per_seq * bs;
    const bool have_ws = workspace != nullptr;
    if (have_ws && !aligned16(workspace))
        return PKV_ERR_INVALID;
    if (partition_tokens > 0 && !have_ws)
        return PKV_ERR_INVALID;

    Plan p;
    pkv_status ps = make_plan(p, num_seqs, num_q_heads, Hkv, D, max_ctx, partition_tokens, have_ws,
                              bf16, true, fp8);
    if (ps == PKV_ERR_INVALID && partition_tokens == PKV_PARTITION_AUTO) {
        // AUTO with a batch too large for the on-chip schedule: one pass per unit
        ps = make_plan(p, num_seqs, num_q_heads, Hkv, D, max_ctx, PKV_PARTITION_NONE, false, bf16, true,
                       fp8);
    }
    if (ps != PKV_OK)
        return ps;
    WsLayout wl;
    if (p.mode != kModeDirect) {
        wl = ws_layout(p, num_seqs, num_q_heads, D, p.max_total_warps);
        if (workspace_bytes < wl.total)
            return PKV_ERR_INVALID;
    }
    unsigned *err = error_word();
    if (!err)
        return PKV_ERR_CUDA;

    CUtensorMap tmK, tmV;
    if (!make_pool_map(&tmK, k_cache) || !make_pool_map(&tmV, v_cache))
        return PKV_ERR_CUDA;

    DecodeArgs a;
    a.q = static_cast<const uint16_t *>(q);
    a.out = static_cast<uint16_t *>(out);
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.mb = max_blocks_per_seq;
    a.nb = k_cache.num_blocks;
    a.B = (int)num_seqs;
    a.Hq = (int)num_q_heads;
    a.Hkv = (int)Hkv;
    a.G = p.G;
    a.n_hg = p.n_hg;
    a.npairs = p.npairs;
    a.bs = (int)bs;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.mode = p.mode;
    a.part_tiles = p.part_tiles;
    a.S = p.S;
    char *ws = static_cast<char *>(workspace);
    a.part_o = have_ws ? reinterpret_cast<float *>(ws + wl.o) : nullptr;
    a.part_m = have_ws ? reinterpret_cast<float *>(ws + wl.m) : nullptr;
    a.part_l = have_ws ? reinterpret_cast<float *>(ws + wl.l) : nullptr;
    a.prefix_out = have_ws ? reinterpret_cast<int32_t *>(ws + wl.prefix) : nullptr;
    // Balanced schedules merge split rows in the decode kernel itself (the
    // warp finishing a (sequence, head group)'s last piece merges all its
    // heads at once), saving the merge kernel's launch, when rows are split
    // into few pieces: at most ~4 warps per (sequence, head group) on average.
    // Long rows split over many warps (one or two long sequences) keep the
    // merge kernel, which spreads them over the whole GPU.  PKV_FOLD_MERGE=0
    // / 1 forces it off / on.
    const int fold_env = env_int("PKV_FOLD_MERGE", -1);
    const bool fold = p.mode == kModeBalanced &&
                      (fold_env < 0 ? (int64_t)p.total_warps <= 4 * num_seqs * p.npairs : fold_env != 0);
    a.fold_cnt = fold ? reinterpret_cast<int *>(ws + wl.cnt) : nullptr;
    a.unit_cost = p.mode == kModeBalanced ? unit_cost() : 0;
    a.total_warps = p.total_warps;
    a.stages = p.stages;
    a.err = err;
    a.wait_limit_ns = g_wait_limit_ns;
    a.inject_no_issue = g_inject_no_issue;
    a.k_new = fa ? static_cast<const uint16_t *>(fa->k_new) : nullptr;
    a.v_new = fa ? static_cast<const uint16_t *>(fa->v_new) : nullptr;
    a.slots = fa ? fa->slots : nullptr;
    a.k_cache = static_cast<uint16_t *>(k_cache.data);
    a.v_cache = static_cast<uint16_t *>(v_cache.data);
    a.pool_slots = k_cache.num_blocks * bs;
    a.table_rows = table_rows;
    a.table_offset = cas ? cas->table_offset : nullptr;
    a.init_o = cas ? cas->init_o : nullptr;
    a.init_m = cas ? cas->init_m : nullptr;
    a.init_l = cas ? cas->init_l : nullptr;
    if (cas && (fp8 || p.fma))
        return PKV_ERR_INVALID;  // the cascade resumes 16-bit MMA accumulators only
    a.k_scales = k_cache.scales;
    a.v_scales = v_cache.scales;

    DecodeKernel k = pick_decode((int)D, bf16, p.nt, fp8, p.fma, cas != nullptr);
    if (!k)
        return PKV_ERR_INVALID;
    if (fold) {
        const int n = (int)(num_seqs * p.npairs);
        if (!cuda_ok(launch_dependent(fold_zero_kernel, dim3((unsigned)std::min(148, (n + 255) / 256)), dim3(256), 0,
                                      (cudaStream_t)stream, a.fold_cnt, n)))
            return PKV_ERR_CUDA;
    }
    if (cas) {
        // the cascade instantiation shares the plan of the plain kernel; give
        // it the same shared-memory ceiling once per device
        static std::mutex mu;
        static std::vector<std::pair<int, DecodeKernel>> done;
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess)
            return PKV_ERR_CUDA;
        std::lock_guard<std::mutex> lock(mu);
        if (std::find(done.begin(), done.end(), std::make_pair(dev, k)) == done.end()) {
            if (!cuda_ok(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemPerCta)))
                return PKV_ERR_CUDA;
            done.emplace_back(dev, k);
        }
    }
    if (!cuda_ok(launch_dependent(k, dim3(p.ctas), dim3(p.warps * 32), p.smem, (cudaStream_t)stream, tmK,
                                  tmV, a)))
        return PKV_ERR_CUDA;

    const bool merge = (p.mode == kModeBalanced && !fold) || (p.mode == kModePartition && p.S > 1);
    if (merge) {
        MergeArgs m;
        m.out = a.out;
        m.context_lens = context_lens;
        m.prefix = a.prefix_out;
        m.part_o = a.part_o;
        m.part_m = a.part_m;
        m.part_l = a.part_l;
        m.mb = max_blocks_per_seq;
        m.B = a.B;
        m.Hq = a.Hq;
        m.G = a.G;
        m.n_hg = a.n_hg;
        m.npairs = a.npairs;
        m.bs = a.bs;
        m.hpu = p.hpu;
        m.mode = p.mode;
        m.part_tiles = p.part_tiles;
        m.S = p.S;
        m.total_warps = p.total_warps;
        m.unit_cost = a.unit_cost;
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        // enough CTAs for one row each when rows have many pieces; with few
        // pieces a CTA takes four rows and the rest exit at once.  Fixed
        // partitions with more pieces per row than one warp's chunk: one
        // 512-thread CTA per row.
        const bool wide = p.mode == kModePartition && p.S > kWarpPieces;
        const int64_t rows = num_seqs * num_q_heads;
        const unsigned grid = (unsigned)std::min<int64_t>(rows, (int64_t)sms * (wide ? 4 : 8));
        const dim3 block(wide ? kMergeWideThreads : kMergeThreads);
        void (*mk)(const MergeArgs) = nullptr;
        if (D == 128)
            mk = wide ? (bf16 ? lse_merge_kernel<128, true, kMergeWideThreads> : lse_merge_kernel<128, false, kMergeWideThreads>)
                      : (bf16 ? lse_merge_kernel<128, true> : lse_merge_kernel<128, false>);
        else
            mk = wide ? (bf16 ? lse_merge_kernel<64, true, kMergeWideThreads> : lse_merge_kernel<64, false, kMergeWideThreads>)
                      : (bf16 ? lse_merge_kernel<64, true> : lse_merge_kernel<64, false>);
        cudaError_t e = launch_dependent(mk, dim3(grid), block, 0, (cudaStream_t)stream, m);
        if (!cuda_ok(e))
            return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

}  // namespace

extern "C" {

pkv_status pkv_decode_attention(const void *q, int64_t num_seqs, int64_t num_q_heads,
                                pkv_cache k_cache, pkv_cache v_cache, const int32_t *block_tables,
                                int64_t max_blocks_per_seq, const int32_t *context_lens,
                                float scale, void *out, void *workspace, size_t workspace_bytes,
                                int32_t partition_tokens, pkv_stream stream) {
    return decode_impl(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables, max_blocks_per_seq,
                       context_lens, scale, out, workspace, workspace_bytes, partition_tokens, stream,
                       nullptr);
}

pkv_status pkv_append_decode_attention(const void *k_new, const void *v_new,
                                       const int64_t *slot_mapping, const void *q, int64_t num_seqs,
                                       int64_t num_q_heads, pkv_cache k_cache, pkv_cache v_cache,
                                       const int32_t *block_tables, int64_t max_blocks_per_seq,
                                       const int32_t *context_lens, float scale, void *out,
                                       void *workspace, size_t workspace_bytes,
                                       int32_t partition_tokens, pkv_stream stream) {
    if (num_seqs > 0 && (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new) ||
                         (reinterpret_cast<uintptr_t>(slot_mapping) & 7u)))
        return PKV_ERR_INVALID;
    const FusedAppend fa{k_new, v_new, slot_mapping};
    return decode_impl(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables, max_blocks_per_seq,
                       context_lens, scale, out, workspace, workspace_bytes, partition_tokens, stream,
                       &fa);
}

const char *pkv_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

size_t pkv_prefill_workspace_bytes(int64_t num_tokens, int64_t num_q_heads, int64_t num_kv_heads,
                                   int64_t head_dim, int64_t max_context_len) {
    if (num_tokens < 0)
        return 0;
    const size_t dec = pkv_decode_workspace_bytes(num_tokens, num_q_heads, num_kv_heads, head_dim,
                                                  max_context_len, PKV_PARTITION_AUTO);
    if (dec == 0 && num_tokens > 0)
        return 0;
    // per-token lengths and table rows, then the multi-query unit counter
    return align256((size_t)num_tokens * 8 + 4) + dec;
}

pkv_status pkv_prefill_attention(const void *q, int64_t num_tokens, int64_t num_seqs, int64_t num_q_heads,
                                 pkv_cache k_cache, pkv_cache v_cache, const int32_t *block_tables,
                                 int64_t max_blocks_per_seq, const int32_t *query_start,
                                 const int32_t *context_lens, float scale, void *out, void *workspace,
                                 size_t workspace_bytes, pkv_stream stream) {
    if (num_tokens < 0 || num_seqs < 0 || num_tokens >= (int64_t(1) << 24))
        return PKV_ERR_INVALID;
    if (num_tokens == 0)
        return PKV_OK;
    if (num_seqs == 0 || !query_start || !context_lens || !workspace || !aligned16(workspace) ||
        !cache_ok(k_cache) || (reinterpret_cast<uintptr_t>(query_start) & 3u))
        return PKV_ERR_INVALID;
    const size_t head = align256((size_t)num_tokens * 8 + 4);
    if (workspace_bytes < head)
        return PKV_ERR_INVALID;
    unsigned *err = error_word();
    if (!err)
        return PKV_ERR_CUDA;
    const int64_t Hkv = k_cache.num_kv_heads, D = k_cache.head_dim;
    const int64_t G = Hkv > 0 ? num_q_heads / Hkv : 0;
    // Chunks of two or more tokens run on the multi-query tensor-core kernel
    // (one K/V pass per block of tokens); decode tokens stay on the decode
    // kernel.  PKV_PREFILL_MQ=0 sends every token through the decode kernel.
    const bool mq = env_int("PKV_PREFILL_MQ", 1) != 0 && (D == 64 || D == 128) && G >= 1 && G <= kMqRows &&
                    num_q_heads % Hkv == 0 && scale != 0.0f && std::isfinite(scale) &&
                    num_seqs <= kMqMaxSeqs && q && out && aligned16(q) && aligned16(out) && block_tables &&
                    (reinterpret_cast<uintptr_t>(block_tables) & 3u) == 0 && same_shape(k_cache, v_cache) &&
                    cache_ok(v_cache) && k_cache.block_size % kTileTokens == 0 &&
                    k_cache.num_blocks * Hkv * k_cache.block_size < (int64_t(1) << 31) - 16 &&
                    max_blocks_per_seq > 0 && max_blocks_per_seq * k_cache.block_size < (int64_t(1) << 30);
    int32_t *lens = static_cast<int32_t *>(workspace);
    int32_t *rows = lens + num_tokens;
    int *counter = reinterpret_cast<int *>(rows + num_tokens);
    const int64_t blocks = std::min<int64_t>((num_tokens + 255) / 256, 148 * 8);
    prefill_expand_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
        query_start, context_lens, (int)num_seqs, (int)num_tokens, max_blocks_per_seq * k_cache.block_size,
        lens, rows, mq ? counter : nullptr, err);
    if (!cuda_ok(cudaGetLastError()))
        return PKV_ERR_CUDA;
    char *rest = static_cast<char *>(workspace) + head;
    pkv_status st = decode_impl(q, num_tokens, num_q_heads, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                lens, scale, out, workspace_bytes > head ? rest : nullptr, workspace_bytes - head,
                                PKV_PARTITION_AUTO, stream, nullptr, rows);
    if (st != PKV_OK || !mq)
        return st;
    MqArgs a = {};
    a.mode = kMqPrefill;
    a.out = static_cast<uint16_t *>(out);
    a.block_tables = block_tables;
    a.query_start = query_start;
    a.context_lens = context_lens;
    a.nsrc = (int)num_seqs;
    a.mb = max_blocks_per_seq;
    a.B = (int)num_seqs;
    a.T = (int)num_tokens;
    a.Hq = (int)num_q_heads;
    a.unit_counter = counter;
    a.err = err;
    return mq_launch(a, q, num_tokens, k_cache, v_cache, scale, stream);
}

// Workspace of pkv_append_decode_attention_shared_prefix:
//   group_ref [NG] | group_len [NG] | shared [B] | suffix_len [B] | table_off [B] | counter  (256-aligned)
//   part_o [B][Hq][D] f32 | part_m [B][Hq] | part_l [B][Hq]                                  (each 256-aligned)
//   then the decode kernel's AUTO workspace.
struct CascadeWs {
    size_t ref = 0, len = 0, shared = 0, suffix = 0, toff = 0, counter = 0, o = 0, m = 0, l = 0, dec = 0, total = 0;
};

static CascadeWs cascade_ws(int64_t B, int64_t Hq, int64_t D, int64_t NG, size_t dec_bytes) {
    CascadeWs w;
    w.ref = 0;
    w.len = w.ref + NG * 4;
    w.shared = w.len + NG * 4;
    w.suffix = w.shared + B * 4;
    w.toff = w.suffix + B * 4;
    w.counter = w.toff + B * 4;
    w.o = align256(w.counter + 4);
    w.m = align256(w.o + (size_t)B * Hq * D * 4);
    w.l = align256(w.m + (size_t)B * Hq * 4);
    w.dec = align256(w.l + (size_t)B * Hq * 4);
    w.total = w.dec + dec_bytes;
    return w;
}

size_t pkv_shared_prefix_workspace_bytes(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                         int64_t head_dim, int64_t max_context_len, int64_t num_groups) {
    if (num_seqs < 0 || num_groups < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
        (head_dim != 64 && head_dim != 128) || max_context_len < 0)
        return 0;
    const size_t dec = pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                                  PKV_PARTITION_AUTO);
    return cascade_ws(num_seqs, num_q_heads, head_dim, num_groups, dec).total;
}

pkv_status pkv_append_decode_attention_shared_prefix(
    const void *k_new, const void *v_new, const int64_t *slot_mapping, const void *q, int64_t num_seqs,
    int64_t num_q_heads, pkv_cache k_cache, pkv_cache v_cache, const int32_t *block_tables,
    int64_t max_blocks_per_seq, const int32_t *context_lens, const int32_t *group_start, int64_t num_groups,
    const int32_t *shared_lens, float scale, void *out, void *workspace, size_t workspace_bytes,
    pkv_stream stream) {
    const bool append = k_new || v_new || slot_mapping;
    if (append && num_seqs > 0 &&
        (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new) ||
         (reinterpret_cast<uintptr_t>(slot_mapping) & 7u)))
        return PKV_ERR_INVALID;
    if (num_seqs < 0 || num_groups < 0 || num_groups > kMqMaxSeqs || num_q_heads <= 0)
        return PKV_ERR_INVALID;
    if (!cache_ok(k_cache) || !cache_ok(v_cache) || !same_shape(k_cache, v_cache))
        return PKV_ERR_INVALID;
    const int64_t Hkv = k_cache.num_kv_heads, D = k_cache.head_dim;
    if (num_q_heads % Hkv != 0 || num_q_heads / Hkv > kMqRows || (D != 64 && D != 128) || !std::isfinite(scale))
        return PKV_ERR_INVALID;
    if (num_seqs == 0)
        return PKV_OK;
    if (num_groups > 0 && (!group_start || !shared_lens || (reinterpret_cast<uintptr_t>(group_start) & 3u) ||
                           (reinterpret_cast<uintptr_t>(shared_lens) & 3u)))
        return PKV_ERR_INVALID;
    if (!workspace || !aligned16(workspace) || !block_tables || !context_lens || !q || !aligned16(q))
        return PKV_ERR_INVALID;
    const size_t dec = pkv_decode_workspace_bytes(num_seqs, num_q_heads, Hkv, D, max_blocks_per_seq * k_cache.block_size,
                                                  PKV_PARTITION_AUTO);
    const CascadeWs wl = cascade_ws(num_seqs, num_q_heads, D, num_groups, dec);
    if (workspace_bytes < wl.total)
        return PKV_ERR_INVALID;
    char *ws = static_cast<char *>(workspace);
    const FusedAppend fa{k_new, v_new, slot_mapping};
    if (num_groups == 0 || scale == 0.0f) {
        // nothing shared (or a degenerate scale): the plain decode step
        return decode_impl(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables, max_blocks_per_seq,
                           context_lens, scale, out, dec ? ws + wl.dec : nullptr, dec, PKV_PARTITION_AUTO, stream,
                           append ? &fa : nullptr);
    }
    unsigned *err = error_word();
    if (!err)
        return PKV_ERR_CUDA;
    int32_t *g_ref = reinterpret_cast<int32_t *>(ws + wl.ref);
    int32_t *g_len = reinterpret_cast<int32_t *>(ws + wl.len);
    int32_t *shared = reinterpret_cast<int32_t *>(ws + wl.shared);
    int32_t *suffix = reinterpret_cast<int32_t *>(ws + wl.suffix);
    int32_t *toff = reinterpret_cast<int32_t *>(ws + wl.toff);
    int *counter = reinterpret_cast<int *>(ws + wl.counter);
    float *po = reinterpret_cast<float *>(ws + wl.o);
    float *pm = reinterpret_cast<float *>(ws + wl.m);
    float *pl = reinterpret_cast<float *>(ws + wl.l);
    // a programmatic dependent like the kernels after it (it waits for the
    // previous kernel before reading anything)
    if (!cuda_ok(launch_dependent(cascade_prep_kernel, dim3((unsigned)((num_seqs + 7) / 8)), dim3(256),
                                  (size_t)(num_groups + 1) * 4, (cudaStream_t)stream, group_start, (int)num_groups,
                                  shared_lens, context_lens, block_tables, max_blocks_per_seq,
                                  (int)k_cache.block_size, (int)num_seqs, g_ref, g_len, shared, suffix, toff, counter,
                                  err)))
        return PKV_ERR_CUDA;
    MqArgs a = {};
    a.mode = kMqPrefix;
    a.out = nullptr;
    a.block_tables = block_tables;
    a.group_start = group_start;
    a.group_ref = g_ref;
    a.group_len = g_len;
    a.shared = shared;
    a.part_o = po;
    a.part_m = pm;
    a.part_l = pl;
    a.nsrc = (int)num_groups;
    a.mb = max_blocks_per_seq;
    a.B = (int)num_seqs;
    a.T = (int)num_seqs;
    a.Hq = (int)num_q_heads;
    a.unit_counter = counter;
    a.err = err;
    pkv_status st = mq_launch(a, q, num_seqs, k_cache, v_cache, scale, stream);
    if (st != PKV_OK)
        return st;
    const CascadeIn cas{toff, po, pm, pl};
    return decode_impl(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables, max_blocks_per_seq, suffix, scale,
                       out, dec ? ws + wl.dec : nullptr, dec, PKV_PARTITION_AUTO, stream, append ? &fa : nullptr,
                       nullptr, PKV_F16, &cas);
}

pkv_status pkv_decode_attention_e4m3(const void *q, pkv_dtype q_dtype, int64_t num_seqs, int64_t num_q_heads,
                                     pkv_cache k_cache, pkv_cache v_cache, const int32_t *block_tables,
                                     int64_t max_blocks_per_seq, const int32_t *context_lens, float scale,
                                     void *out, void *workspace, size_t workspace_bytes,
                                     int32_t partition_tokens, pkv_stream stream) {
    if (k_cache.dtype != PKV_E4M3 || v_cache.dtype != PKV_E4M3)
        return PKV_ERR_INVALID;
    return decode_impl(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables, max_blocks_per_seq,
                       context_lens, scale, out, workspace, workspace_bytes, partition_tokens, stream, nullptr,
                       nullptr, q_dtype);
}

pkv_status pkv_append_e4m3(const void *k_new, const void *v_new, pkv_dtype new_dtype,
                           const int64_t *slot_mapping, int64_t num_tokens, pkv_cache k_cache,
                           pkv_cache v_cache, pkv_stream stream) {
    if (num_tokens < 0 || (new_dtype != PKV_F16 && new_dtype != PKV_BF16))
        return PKV_ERR_INVALID;
    if (!cache_ok_e4m3(k_cache) || !cache_ok_e4m3(v_cache) || !same_shape(k_cache, v_cache))
        return PKV_ERR_INVALID;
    const int64_t D = k_cache.head_dim;
    if (D != 64 && D != 128)
        return PKV_ERR_INVALID;
    if (num_tokens == 0)
        return PKV_OK;
    if (!k_new || !v_new || !slot_mapping || !aligned16(k_new) || !aligned16(v_new) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PKV_ERR_INVALID;
    unsigned *err = error_word();
    if (!err)
        return PKV_ERR_CUDA;
    const int64_t rows = num_tokens * k_cache.num_kv_heads * 2;
    const int64_t blocks = std::min<int64_t>((rows * 32 + 255) / 256, 148 * 16);
    auto args = std::make_tuple(static_cast<const uint16_t *>(k_new), static_cast<const uint16_t *>(v_new),
                                slot_mapping, num_tokens, (int)k_cache.num_kv_heads, (int)k_cache.block_size,
                                k_cache.num_blocks, static_cast<uint8_t *>(k_cache.data), k_cache.scales,
                                static_cast<uint8_t *>(v_cache.data), v_cache.scales, err);
    const bool bf = new_dtype == PKV_BF16;
    cudaStream_t st = (cudaStream_t)stream;
    std::apply(
        [&](auto... xs) {
            if (D == 128 && bf)
                append_e4m3_kernel<128, true><<<(unsigned)blocks, 256, 0, st>>>(xs...);
            else if (D == 128)
                append_e4m3_kernel<128, false><<<(unsigned)blocks, 256, 0, st>>>(xs...);
            else if (bf)
                append_e4m3_kernel<64, true><<<(unsigned)blocks, 256, 0, st>>>(xs...);
            else
                append_e4m3_kernel<64, false><<<(unsigned)blocks, 256, 0, st>>>(xs...);
        },
        args);
    return cuda_ok(cudaGetLastError()) ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_get_last_error(void) {
    if (!cuda_ok(cudaDeviceSynchronize()))
        return PKV_ERR_CUDA;
    unsigned *err = error_word();
    if (!err)
        return PKV_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, err, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (v != 0) {
        const unsigned zero = 0;
        cudaMemcpy(err, &zero, sizeof zero, cudaMemcpyHostToDevice);
        return (v & kErrTimeout) ? PKV_ERR_TIMEOUT : PKV_ERR_DEVICE_CHECK;
    }
    return PKV_OK;
}

pkv_status pkv_test_exp2_poly(const float *x, float *y, int64_t n, pkv_stream stream) {
    if (n < 0 || (n > 0 && (!x || !y)))
        return PKV_ERR_INVALID;
    if (n == 0)
        return PKV_OK;
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 8);
    exp2_poly_test_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(x, y, n);
    return cuda_ok(cudaGetLastError()) ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_test_inject_wait_timeout(int32_t enable, int64_t wait_limit_ns) {
    if (enable) {
        if (wait_limit_ns < 1000000)
            wait_limit_ns = 1000000;
        if (wait_limit_ns > (int64_t)kWaitLimitNs)
            wait_limit_ns = (int64_t)kWaitLimitNs;
        g_inject_no_issue = 1;
        g_wait_limit_ns = (uint64_t)wait_limit_ns;
    } else {
        g_inject_no_issue = 0;
        g_wait_limit_ns = kWaitLimitNs;
    }
    return PKV_OK;
}


}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention without any device allocation by the caller or by us.
//
// Some callers cannot allocate device memory: a plugin or custom-operator
// interface that only receives device pointers for its inputs and outputs,
// or a serving loop that bans cudaMalloc after start-up (it can synchronise
// the device, fail under pressure or fragment memory mid-run).  For them the
// split-context scratch lives in this fixed file-scope array instead of a
// caller-provided workspace.  Every GPU that loads the library keeps it for
// the life of the process, so its size is kept modest.
static __device__ __align__(256) unsigned char g_static_scratch[PKV_STATIC_SCRATCH_BYTES];

namespace {

// In host code `g_static_scratch` names a host-side shadow, not device
// memory: the device address has to be asked for, once per device, with that
// device current.  Returns nullptr if the runtime cannot provide it.
void *static_scratch_device_ptr() {
    static void *addr[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess)
            return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" pkv_status pkv_decode_attention_static_scratch(
    const void *q, int64_t num_seqs, int64_t num_q_heads, pkv_cache k_cache, pkv_cache v_cache,
    const int32_t *block_tables, int64_t max_blocks_per_seq, const int32_t *context_lens, float scale,
    void *out, int32_t partition_tokens, pkv_stream stream) {
    if (partition_tokens == PKV_PARTITION_NONE)
        return pkv_decode_attention(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables,
                                    max_blocks_per_seq, context_lens, scale, out, nullptr, 0,
                                    partition_tokens, stream);
    if (num_seqs == 0)
        return pkv_decode_attention(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables,
                                    max_blocks_per_seq, context_lens, scale, out, nullptr, 0,
                                    partition_tokens, stream);
    if (!cache_ok(k_cache) || max_blocks_per_seq <= 0)
        return PKV_ERR_INVALID;
    const size_t need = pkv_decode_workspace_bytes(
        num_seqs, num_q_heads, k_cache.num_kv_heads, k_cache.head_dim,
        max_blocks_per_seq * k_cache.block_size, partition_tokens);
    if (need == 0) {
        // AUTO on a batch too large for the on-chip schedule: the regular
        // entry point then runs one pass per unit with no scratch at all, and
        // so does this one (an invalid shape is refused there just the same)
        if (partition_tokens == PKV_PARTITION_AUTO)
            return pkv_decode_attention(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables,
                                        max_blocks_per_seq, context_lens, scale, out, nullptr, 0,
                                        partition_tokens, stream);
        return PKV_ERR_INVALID;  // shape rejected (or no device to size it on)
    }
    if (need > (size_t)PKV_STATIC_SCRATCH_BYTES)
        return PKV_ERR_SCRATCH_TOO_SMALL;
    void *scratch = static_scratch_device_ptr();
    if (!scratch)
        return PKV_ERR_CUDA;
    return pkv_decode_attention(q, num_seqs, num_q_heads, k_cache, v_cache, block_tables,
                                max_blocks_per_seq, context_lens, scale, out, scratch,
                                (size_t)PKV_STATIC_SCRATCH_BYTES, partition_tokens, stream);
}
