// api.cu -- host side of the C ABI declared in include/gemm_bf16.h: argument validation,
// tile-plan choice, tensor-map encoding, the alignment pre-pass and the kernel launches.
// Every step of the computation runs in the kernels of gemm_kernel.cuh; this file only
// prepares and enqueues them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <array>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gemm_bf16.h"
#include "gemm_kernel.cuh"

using namespace pw;

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;
constexpr int kGroupM = 8;

std::atomic<int> g_plan_override{-1};
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

struct DevInfo {
    bool init = false;
    int sms = 0;
    int major = 0;
    int minor = 0;
};

std::mutex g_dev_mu;
std::array<DevInfo, kMaxDevices> g_dev;

bool device_info(int dev, DevInfo& out) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo& d = g_dev[dev];
    if (!d.init) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return false;
        d.init = true;
    }
    out = d;
    return true;
}

// Stream-ordered pool of the library's per-call workspace (alignment pre-pass copies, split-K
// partial sums and counters), one per device.  Its release threshold is unlimited: memory freed
// at the end of a call stays in the pool for the next call on any stream instead of going back
// to the driver at the next synchronisation, so steady-state calls map no new pages.  The pool
// holds the largest workspace seen so far until the process exits.
std::mutex g_pool_mu;
std::array<cudaMemPool_t, kMaxDevices> g_pool{};

gemm_status_t workspace_pool(int dev, cudaMemPool_t* out) {
    if (dev < 0 || dev >= kMaxDevices) return GEMM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_pool_mu);
    if (g_pool[dev] == nullptr) {
        cudaMemPoolProps props;
        std::memset(&props, 0, sizeof props);
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return GEMM_ERR_CUDA;
        uint64_t keep = UINT64_MAX;
        if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return GEMM_ERR_CUDA;
        }
        g_pool[dev] = pool;
    }
    *out = g_pool[dev];
    return GEMM_OK;
}

// One request, in the batched form (batch == 1 for the plain GEMM).
struct Req {
    int batch, M, N, K;
    const void* A;
    long long lda;
    const void* B;
    long long ldb, stride_b;
    bool b_mn;  // B stored K x N (N-major) instead of N x K (K-major)
    void* C;
    long long ldc, stride_c;
    int out;  // OUT_F32 / OUT_BF16
    float alpha, beta;
    cudaStream_t stream;
};

struct PlanDesc {
    int cg, bn, nsub, stages, bk;  // CTAs per tile, MMA N, N sub-tiles per tile, ring stages, K per stage
    int ares;                      // A resident in shared memory (needs M <= 128*cg, K <= 512)
    double rate;                   // TFLOP/s with every SM busy (B200, 8192^3 bf16); 0: never auto
};
constexpr int kNumPlans = 9;
constexpr PlanDesc kPlans[kNumPlans] = {
    {1, 128, 1, 6, 64, 0, 880.0},   // 0: 128x128, one CTA
    {1, 256, 1, 4, 64, 0, 1190.0},  // 1: 128x256, one CTA
    {2, 256, 1, 6, 64, 0, 1250.0},  // 2: 256x256, 2-CTA cluster
    {2, 128, 1, 8, 64, 0, 790.0},   // 3: 256x128, 2-CTA cluster
    {2, 256, 2, 4, 64, 0, 1400.0},  // 4: 256x512, 2-CTA cluster, two 256-column MMA sub-tiles
    {2, 128, 1, 8, 64, 1, 0.0},     // 5: 256x128, 2-CTA cluster, A resident (M <= 256, K <= 512)
    {1, 128, 1, 4, 64, 1, 0.0},     // 6: 128x128, one CTA, A resident (M <= 128, K <= 512)
    {2, 256, 1, 4, 64, 1, 0.0},     // 7: 256x256, 2-CTA cluster, A resident (M <= 256, K <= 512)
    {1, 64, 1, 8, 64, 0, 590.0},    // 8: 128x64, one CTA (twice the tiles of plan 0 on thin shapes)
};

// Batch entries packed side by side into one tile by plan `pd` (1 = no packing): needs the
// N-major (batched) B operand, N a multiple of the 64-column box and dividing the tile width.
int pack_factor(const PlanDesc& pd, bool b_mn, int N) {
    const int tile_n = pd.bn * pd.nsub;
    if (!b_mn || N <= 0 || N % 64 != 0 || tile_n % N != 0 || tile_n == N) return 1;
    return tile_n / N;
}

inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

// Failure-detection test hook: with GEMM_BF16_TEST_STALL_LOADS=1 the kernel's producer issues
// no loads, so the MMA thread's first bounded wait expires and the kernel reports a timeout
// through gemm_bf16_device_status.  Nothing faults; the context stays usable.
bool test_stall_requested() {
    const char* e = std::getenv("GEMM_BF16_TEST_STALL_LOADS");
    return e && e[0] == '1';
}

// m-blocks per raster group; GEMM_BF16_GROUP_M (1..64) overrides the default for tuning sweeps.
int group_m() {
    const char* e = std::getenv("GEMM_BF16_GROUP_M");
    if (e) {
        const int v = std::atoi(e);
        if (v >= 1 && v <= 64) return v;
    }
    return kGroupM;
}
inline long long round_up(long long a, long long b) { return cdiv(a, b) * b; }
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

gemm_status_t validate(const Req& r) {
    if (r.batch < 0 || r.M < 0 || r.N < 0 || r.K < 0) return GEMM_ERR_INVALID_ARG;
    if (r.out != OUT_F32 && r.out != OUT_BF16) return GEMM_ERR_INVALID_ARG;
    const long long minA = r.K > 1 ? r.K : 1;
    const long long minB = r.b_mn ? (r.N > 1 ? r.N : 1) : (r.K > 1 ? r.K : 1);
    const long long minC = r.N > 1 ? r.N : 1;
    if (r.lda < minA || r.ldb < minB || r.ldc < minC) return GEMM_ERR_INVALID_ARG;
    if (r.stride_b < 0 || r.stride_c < 0) return GEMM_ERR_INVALID_ARG;
    if (r.batch == 0 || r.M == 0 || r.N == 0) return GEMM_OK;
    const uintptr_t es = r.out == OUT_F32 ? 4 : 2;
    if (r.C == nullptr || !aligned(r.C, es)) return GEMM_ERR_INVALID_ARG;
    if (r.batch > 1 && r.stride_c < (long long)(r.M - 1) * r.ldc + r.N) return GEMM_ERR_INVALID_ARG;
    if (r.K > 0 && r.alpha != 0.0f) {
        if (r.A == nullptr || r.B == nullptr) return GEMM_ERR_INVALID_ARG;
        if (!aligned(r.A, 2) || !aligned(r.B, 2)) return GEMM_ERR_INVALID_ARG;
    }
    return GEMM_OK;
}

gemm_status_t encode_3d(CUtensorMap* m, const void* base, bool f32, uint64_t d0, uint64_t d1,
                        uint64_t d2, uint64_t s1_bytes, uint64_t s2_bytes, uint32_t b0, uint32_t b1,
                        CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GEMM_ERR_CUDA;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1_bytes, s2_bytes};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult res = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return res == CUDA_SUCCESS ? GEMM_OK : GEMM_ERR_CUDA;
}

// The automatic choice minimises the modelled time of plan_time() below over the streaming
// plans (rate > 0): large tiles move fewer operand bytes per FLOP, small tiles quantise better
// on small grids.

// Split-K limits: at most kMaxSplits slices of K, each at least kMinSplitKBlocks k-blocks long
// (the smem ring needs a few blocks to fill), and a split must beat the unsplit choice by 10%.
constexpr int kMaxSplits = 8;
constexpr int kMinSplitKBlocks = 8;
// Operand bytes one CTA pulls through TMA per second when its tiles are not compute-bound
// (measured on B200 with few, deep tiles: 8192x256x4096, 1024x1024x8192).
constexpr double kCtaOperandBytesPerSec = 140e9;
// Split-K cost per unit, measured on B200: a fixed part (counter, fences, the longer fixup
// epilogue), the write of the unit's fp32 partial sums and the last unit's read of the others.
constexpr double kSplitFixedSec = 4e-6;
constexpr double kSplitWriteBytesPerSec = 45e9;
constexpr double kSplitReadBytesPerSec = 90e9;
// Fixed cost of one launch that the waves do not cover: pipeline fill, the exposed epilogue of
// the last tiles and teardown.  Fitted on B200 to single-wave shapes (2048^3, 8192x512x4096,
// 8192x256x4096, 127x8191x2048), where 2-CTA tiles pay more (the leader waits for both CTAs'
// loads) and plan 1 beats plan 2 by 13 % although their waves model equal.
constexpr double kLaunchFixedSecOneCta = 3e-6;
constexpr double kLaunchFixedSecCtaPair = 6e-6;
// Split-K arrival counters per CTA and tile: one per epilogue warp.
constexpr int kSplitCountersPerCta = 4;

// Can plan `i` serve this request?
bool plan_serves(int i, const Req& r) {
    const PlanDesc& pd = kPlans[i];
    if (pd.ares) return r.M <= 128 * pd.cg && r.K <= 8 * pd.bk;
    return true;
}

// Output tiles of plan `pd` for the request.
long long plan_tiles(const PlanDesc& pd, const Req& r) {
    const long long tm = 128LL * pd.cg, tn = (long long)pd.bn * pd.nsub;
    const int pk = pack_factor(pd, r.b_mn, r.N);
    return pk > 1 ? cdiv(r.M, tm) * cdiv(r.batch, pk) : cdiv(r.M, tm) * cdiv(r.N, tn) * r.batch;
}

// Modelled time (s) of streaming plan `i` with K cut into `splits` slices: waves of work units,
// each bound by the plan's per-cluster tensor rate or by its CTAs' operand streaming, a fixed
// cost per launch, and, when split, each unit's partial-sum write and the last unit's read of
// the other slices.
double plan_time(int i, const Req& r, int sms, int splits) {
    const PlanDesc& pd = kPlans[i];
    const long long tm = 128LL * pd.cg, tn = (long long)pd.bn * pd.nsub;
    const long long slots = sms / pd.cg;
    const long long kb = cdiv(cdiv(r.K, pd.bk), splits);  // k-blocks per unit
    const double unit_k = (double)(kb * pd.bk);
    const double compute = 2.0 * (double)(tm * tn) * unit_k / (pd.rate * 1e12 / (double)slots);
    const double stream = (double)(tm + tn) * unit_k * 2.0 / (pd.cg * kCtaOperandBytesPerSec);
    double t = (double)cdiv(plan_tiles(pd, r) * splits, slots) * (compute > stream ? compute : stream) +
               (pd.cg == 2 ? kLaunchFixedSecCtaPair : kLaunchFixedSecOneCta);
    if (splits > 1) {
        const double partial = 128.0 * (double)tn * 4.0;  // bytes per CTA and unit
        t += kSplitFixedSec + partial / kSplitWriteBytesPerSec + (splits - 1) * partial / kSplitReadBytesPerSec;
    }
    return t;
}

// Split counts the kernel takes for plan `pd`: every slice non-empty and the same length
// except the last.
bool split_valid(const PlanDesc& pd, const Req& r, int splits) {
    if (splits == 1) return true;
    if (pd.ares || splits < 1 || splits > kMaxSplits) return false;
    const long long kb = cdiv(r.K, pd.bk);
    return cdiv(kb, cdiv(kb, splits)) == splits;
}

// GEMM_BF16_SPLIT_K=s (1..8) forces s slices of K wherever the plan takes it (tests, tuning);
// unset or 0 leaves the choice to the model.
int forced_splits() {
    const char* e = std::getenv("GEMM_BF16_SPLIT_K");
    if (e) {
        const int v = std::atoi(e);
        if (v >= 1 && v <= kMaxSplits) return v;
    }
    return 0;
}

struct Choice {
    int plan;
    int splits;
};

// Plan and K split for a request on a device with `sms` SMs (auto unless overridden); without
// `allow_split` the best unsplit plan.
Choice choose(const Req& r, int sms, bool allow_split) {
    const int fs = allow_split ? forced_splits() : 1;
    const int forced = g_plan_override.load();
    int only = -1;  // the one plan to consider, or -1 for every streaming plan
    if (forced >= 0 && plan_serves(forced, r)) {
        if (kPlans[forced].ares) return {forced, 1};
        only = forced;
    } else if (r.b_mn && r.K <= 1024 && pack_factor(kPlans[2], r.b_mn, r.N) > 1) {
        // Shared-W batched shapes with short K are bound by streaming X and Y through HBM: a
        // 256x256 tile holding several batch entries side by side, with W resident in shared
        // memory when it fits (read once per CTA instead of once per tile from L2), measured
        // fastest (RecSys 2048 x (256x512 . 512x128): plan 7 81.7 us, plan 2 84.5 us).
        if (plan_serves(7, r)) return {7, 1};
        only = 2;
    }
    // Unsplit plans first; a split must then beat the best of them by 10 %.
    Choice best{only >= 0 ? only : 0, 1};
    double best_t = 0.0;
    bool have = false;
    for (int i = 0; i < kNumPlans; ++i) {
        const PlanDesc& pd = kPlans[i];
        if (only >= 0 ? i != only : pd.rate <= 0.0) continue;
        const int s = fs > 0 && split_valid(pd, r, fs) ? fs : 1;
        const double t = plan_time(i, r, sms, s);
        if (!have || t < best_t * 0.999) best = {i, s}, best_t = t, have = true;
    }
    if (fs > 0 || !allow_split) return best;
    const double split_bar = best_t * 0.90;
    for (int i = 0; i < kNumPlans; ++i) {
        const PlanDesc& pd = kPlans[i];
        if (only >= 0 ? i != only : pd.rate <= 0.0) continue;
        long long smax = cdiv(r.K, pd.bk) / kMinSplitKBlocks;
        if (smax > kMaxSplits) smax = kMaxSplits;
        for (int sp = 2; sp <= (int)smax; ++sp) {
            if (!split_valid(pd, r, sp)) continue;
            const double t = plan_time(i, r, sms, sp);
            if (t < split_bar && t < best_t * 0.999) best = {i, sp}, best_t = t;
        }
    }
    return best;
}

template <int CG, int BN, int NSUB, int STAGES, int BK, int B_MN, int OUT, int ARES>
gemm_status_t launch_persistent(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc,
                                const KParams& p, int dev, int sms, cudaStream_t stream) {
    using T = Tile<CG, BN, NSUB, STAGES, BK, B_MN, OUT, ARES>;
    auto kern = gemm_persistent<CG, BN, NSUB, STAGES, BK, B_MN, OUT, ARES>;
    static_assert(T::EPI_WARPS == kSplitCountersPerCta, "split-K counters sized per epilogue warp");
    static std::array<std::atomic<int>, kMaxDevices> attr_done{};
    static std::array<std::atomic<int>, kMaxDevices> max_clusters{};
    if (!attr_done[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM_ALLOC) !=
            cudaSuccess)
            return GEMM_ERR_CUDA;
        int clusters = sms / CG;
        if constexpr (CG == 2) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(sms, 1, 1);
            q.blockDim = dim3(T::THREADS, 1, 1);
            q.dynamicSmemBytes = T::SMEM_ALLOC;
            cudaLaunchAttribute qa[1];
            qa[0].id = cudaLaunchAttributeClusterDimension;
            qa[0].val.clusterDim.x = 2;
            qa[0].val.clusterDim.y = 1;
            qa[0].val.clusterDim.z = 1;
            q.attrs = qa;
            q.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &q) == cudaSuccess && n > 0 && n < clusters)
                clusters = n;
        }
        max_clusters[dev].store(clusters);
        attr_done[dev].store(1);
    }
    const long long units = (long long)p.tiles * (p.splits > 1 ? p.splits : 1);  // work units
    const int clusters = (int)(units < max_clusters[dev].load() ? units : max_clusters[dev].load());
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(clusters * CG, 1, 1);
    cfg.blockDim = dim3(T::THREADS, 1, 1);
    cfg.dynamicSmemBytes = T::SMEM_ALLOC;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[1];
    if constexpr (CG == 2) {
        attrs[0].id = cudaLaunchAttributeClusterDimension;
        attrs[0].val.clusterDim.x = 2;
        attrs[0].val.clusterDim.y = 1;
        attrs[0].val.clusterDim.z = 1;
        cfg.attrs = attrs;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kern, ma, mb, mc, p) == cudaSuccess ? GEMM_OK : GEMM_ERR_CUDA;
}

template <int CG, int BN, int NSUB, int STAGES, int BK, int ARES>
gemm_status_t launch_plan(bool b_mn, int out, const CUtensorMap& ma, const CUtensorMap& mb,
                          const CUtensorMap& mc, const KParams& p, int dev, int sms, cudaStream_t st) {
    if (b_mn) {
        if constexpr ((BN / CG) % 64 == 0) {
            return out == OUT_F32
                       ? launch_persistent<CG, BN, NSUB, STAGES, BK, 1, OUT_F32, ARES>(ma, mb, mc, p, dev, sms, st)
                       : launch_persistent<CG, BN, NSUB, STAGES, BK, 1, OUT_BF16, ARES>(ma, mb, mc, p, dev, sms, st);
        } else {
            return GEMM_ERR_UNSUPPORTED;
        }
    }
    return out == OUT_F32
               ? launch_persistent<CG, BN, NSUB, STAGES, BK, 0, OUT_F32, ARES>(ma, mb, mc, p, dev, sms, st)
               : launch_persistent<CG, BN, NSUB, STAGES, BK, 0, OUT_BF16, ARES>(ma, mb, mc, p, dev, sms, st);
}

gemm_status_t launch_by_plan(int plan, bool b_mn, int out, const CUtensorMap& ma, const CUtensorMap& mb,
                             const CUtensorMap& mc, const KParams& p, int dev, int sms, cudaStream_t st) {
    switch (plan) {
        case 0: return launch_plan<1, 128, 1, 6, 64, 0>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        case 1: return launch_plan<1, 256, 1, 4, 64, 0>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        case 2: return launch_plan<2, 256, 1, 6, 64, 0>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        case 3: return launch_plan<2, 128, 1, 8, 64, 0>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        case 4: return launch_plan<2, 256, 2, 4, 64, 0>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        case 5: return launch_plan<2, 128, 1, 8, 64, 1>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        case 6: return launch_plan<1, 128, 1, 4, 64, 1>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        case 7: return launch_plan<2, 256, 1, 4, 64, 1>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        case 8: return launch_plan<1, 64, 1, 8, 64, 0>(b_mn, out, ma, mb, mc, p, dev, sms, st);
        default: return GEMM_ERR_INVALID_ARG;
    }
}

gemm_status_t launch_scale(const Req& r) {
    const long long total = (long long)r.batch * r.M * r.N;
    const int threads = 256;
    long long blocks = cdiv(total, threads);
    if (blocks > 148LL * 32) blocks = 148LL * 32;
    if (r.out == OUT_F32)
        scale_c_kernel<float><<<(unsigned)blocks, threads, 0, r.stream>>>(
            static_cast<float*>(r.C), r.ldc, r.stride_c, r.batch, r.M, r.N, r.beta);
    else
        scale_c_kernel<uint16_t><<<(unsigned)blocks, threads, 0, r.stream>>>(
            static_cast<uint16_t*>(r.C), r.ldc, r.stride_c, r.batch, r.M, r.N, r.beta);
    return cudaGetLastError() == cudaSuccess ? GEMM_OK : GEMM_ERR_CUDA;
}

void launch_pad(const void* src, long long ld_src, long long bs_src, void* dst, long long ld_dst,
                long long bs_dst, int batch, int rows, int cols, cudaStream_t st) {
    const int threads = 128;
    int gx = (int)cdiv(cdiv(cols, 8), threads);
    if (gx > 8) gx = 8;
    int gy = rows < 4096 ? (rows > 0 ? rows : 1) : 4096;
    int gz = batch < 65535 ? batch : 65535;
    // extent of the source: from its first element to one past its last
    const uintptr_t lo = reinterpret_cast<uintptr_t>(src);
    const uintptr_t hi = lo + 2 * (uintptr_t)((long long)(batch - 1) * bs_src + (long long)(rows - 1) * ld_src + cols);
    pad_copy_kernel<<<dim3(gx, gy, gz), threads, 0, st>>>(
        static_cast<const uint16_t*>(src), ld_src, bs_src, static_cast<uint16_t*>(dst), ld_dst, bs_dst,
        batch, rows, cols, lo, hi);
}

gemm_status_t run(Req r) {
    gemm_status_t v = validate(r);
    if (v != GEMM_OK) return v;
    if (r.batch == 0 || r.M == 0 || r.N == 0) return GEMM_OK;
    if (r.batch == 1) {
        r.stride_b = r.b_mn ? (long long)r.K * r.ldb : (long long)r.N * r.ldb;
        r.stride_c = (long long)r.M * r.ldc;
    }
    if (r.K == 0 || r.alpha == 0.0f) return launch_scale(r);

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GEMM_ERR_CUDA;
    DevInfo di;
    if (!device_info(dev, di)) return GEMM_ERR_CUDA;
    if (di.major != 10 || di.minor != 0) return GEMM_ERR_UNSUPPORTED;

    // Operands TMA cannot read as given go through a padded, 16-byte aligned copy.
    const bool a_ok = aligned(r.A, 16) && (r.lda % 8) == 0;
    const long long b_rows = r.b_mn ? r.K : r.N;  // rows of the stored B matrix per batch
    const long long b_cols = r.b_mn ? r.N : r.K;
    const bool b_ok = aligned(r.B, 16) && (r.ldb % 8) == 0 &&
                      (r.batch == 1 || ((r.stride_b % 8) == 0 && r.stride_b >= b_rows * r.ldb));
    long long lda_p = r.lda, ldb_p = r.ldb, sb_p = r.stride_b;
    size_t ws_a = 0, ws_b = 0;
    if (!a_ok) {
        lda_p = round_up(r.K, 8);
        ws_a = (size_t)round_up((long long)r.M * lda_p * 2, 256);
    }
    if (!b_ok) {
        ldb_p = round_up(b_cols, 8);
        sb_p = b_rows * ldb_p;
        ws_b = (size_t)round_up(sb_p * 2 * r.batch, 256);
    }
    // Split-K partial sums (fp32, one 128 x tile_n slab per CTA, tile and slice) and the
    // per-(tile, CTA, epilogue warp) arrival counters, which must start at zero.
    const Choice ch = choose(r, di.sms, true);
    const int plan = ch.plan;
    const PlanDesc pd = kPlans[plan];
    const long long tiles_est = plan_tiles(pd, r);
    size_t ws_p = 0, ws_n = 0;
    if (ch.splits > 1) {
        ws_p = (size_t)tiles_est * pd.cg * ch.splits * 128 * pd.bn * pd.nsub * sizeof(float);
        ws_n = (size_t)round_up(tiles_est * pd.cg * kSplitCountersPerCta * (long long)sizeof(unsigned int), 256);
    }
    void* ws = nullptr;
    if (ws_a + ws_b + ws_p + ws_n) {
        cudaMemPool_t pool = nullptr;
        const gemm_status_t ps = workspace_pool(dev, &pool);
        if (ps != GEMM_OK) return ps;
        if (cudaMallocFromPoolAsync(&ws, ws_a + ws_b + ws_p + ws_n, pool, r.stream) != cudaSuccess)
            return GEMM_ERR_NO_MEMORY;
    }
    float* ws_partials = ch.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + ws_a + ws_b) : nullptr;
    unsigned int* ws_counters =
        ch.splits > 1 ? reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + ws_a + ws_b + ws_p) : nullptr;
    if (ws_n && cudaMemsetAsync(ws_counters, 0, ws_n, r.stream) != cudaSuccess) {
        cudaFreeAsync(ws, r.stream);
        return GEMM_ERR_CUDA;
    }
    const void* A = r.A;
    const void* B = r.B;
    if (!a_ok) {
        launch_pad(r.A, r.lda, 0, ws, lda_p, 0, 1, r.M, r.K, r.stream);
        A = ws;
    }
    if (!b_ok) {
        void* dst = static_cast<char*>(ws) + ws_a;
        launch_pad(r.B, r.ldb, r.stride_b, dst, ldb_p, sb_p, r.batch, (int)b_rows, (int)b_cols, r.stream);
        B = dst;
    }

    const int b_chunk = pd.bn * pd.nsub / pd.cg;  // B rows per CTA and stage
    const int es = r.out == OUT_F32 ? 4 : 2;
    const int stg_cols = r.out == OUT_F32 ? 32 : 64;
    const bool c_tma = aligned(r.C, 16) && ((r.ldc * es) % 16) == 0 &&
                       (r.batch == 1 || ((r.stride_c * es) % 16) == 0);

    CUtensorMap ma, mb, mc;
    std::memset(&mc, 0, sizeof mc);
    const CUtensorMapSwizzle ksw = pd.bk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    gemm_status_t st = encode_3d(&ma, A, false, (uint64_t)r.K, (uint64_t)r.M, 1, (uint64_t)lda_p * 2,
                                 (uint64_t)lda_p * 2 * (uint64_t)r.M, (uint32_t)pd.bk, 128, ksw);
    if (st == GEMM_OK) {
        if (!r.b_mn)
            st = encode_3d(&mb, B, false, (uint64_t)r.K, (uint64_t)r.N, (uint64_t)r.batch,
                           (uint64_t)ldb_p * 2, (uint64_t)sb_p * 2, (uint32_t)pd.bk, (uint32_t)b_chunk, ksw);
        else
            st = encode_3d(&mb, B, false, (uint64_t)r.N, (uint64_t)r.K, (uint64_t)r.batch,
                           (uint64_t)ldb_p * 2, (uint64_t)sb_p * 2, 64, (uint32_t)pd.bk);
    }
    if (st == GEMM_OK && c_tma)
        st = encode_3d(&mc, r.C, r.out == OUT_F32, (uint64_t)r.N, (uint64_t)r.M, (uint64_t)r.batch,
                       (uint64_t)r.ldc * es, (uint64_t)r.stride_c * es, (uint32_t)stg_cols, 32);
    if (st == GEMM_OK) {
        KParams p;
        std::memset(&p, 0, sizeof p);
        p.M = r.M;
        p.N = r.N;
        p.K = r.K;
        p.m_blocks = (int)cdiv(r.M, 128 * pd.cg);
        p.pack = pack_factor(pd, r.b_mn, r.N);
        p.batch_real = r.batch;
        if (p.pack > 1) {
            p.n_blocks = (int)cdiv(r.batch, p.pack);
            p.batch = 1;
        } else {
            p.n_blocks = (int)cdiv(r.N, pd.bn * pd.nsub);
            p.batch = r.batch;
        }
        p.tiles = p.m_blocks * p.n_blocks * p.batch;
        p.k_blocks = (int)cdiv(r.K, pd.bk);
        if (ch.splits > 1) {
            p.splits = ch.splits;
            p.kb_per_split = (int)cdiv(p.k_blocks, ch.splits);
            p.ws = ws_partials;
            p.counters = ws_counters;
        }
        p.group_m = group_m();
        p.alpha = r.alpha;
        p.beta = r.beta;
        p.C = r.C;
        p.ldc = r.ldc;
        p.stride_c = r.stride_c;
        p.c_tma = c_tma ? 1 : 0;
        // Whole chunks up to the last 16-byte-aligned column may use tensor stores; when the row
        // end itself is aligned, the clipped last chunk may too.
        p.n_store_tma = ((long long)r.N * es) % 16 == 0 ? (int)round_up(r.N, stg_cols) : r.N;
        p.c_read = r.beta != 0.0f ? 1 : 0;
        p.timeout_ns = g_timeout_ns.load();
        p.test_stall = test_stall_requested() ? 1 : 0;
        st = launch_by_plan(plan, r.b_mn, r.out, ma, mb, mc, p, dev, di.sms, r.stream);
    }
    if (ws) cudaFreeAsync(ws, r.stream);
    return st;
}

}  // namespace

// ------------------------------------------------------------------ allocation-free variant
// Scratch of gemm_bf16_noalloc: the padded copies of A and B written by the alignment pre-pass
// and read by the GEMM kernel.  Every device that loads this library holds it until the process
// exits.  In host code this name is only a host-side stand-in, never a device address: kernels
// are given the address that noalloc_scratch() obtains once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GEMM_BF16_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_scratch_mu;
std::array<void*, kMaxDevices> g_scratch_ptr{};

// Device address of the scratch on device `dev`, which must be the current device.  The first
// call per device asks the runtime for it; later calls reuse the cached value.
gemm_status_t noalloc_scratch(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return GEMM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return GEMM_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GEMM_OK;
}

// The gemm_bf16 path with the pre-pass copies placed in the static scratch.
gemm_status_t run_noalloc(Req r) {
    gemm_status_t v = validate(r);
    if (v != GEMM_OK) return v;
    if (r.batch == 0 || r.M == 0 || r.N == 0) return GEMM_OK;
    if (r.batch == 1) {
        r.stride_b = r.b_mn ? (long long)r.K * r.ldb : (long long)r.N * r.ldb;
        r.stride_c = (long long)r.M * r.ldc;
    }
    if (r.K == 0 || r.alpha == 0.0f) return launch_scale(r);

    const bool a_ok = aligned(r.A, 16) && (r.lda % 8) == 0;
    const long long b_rows = r.b_mn ? r.K : r.N;
    const long long b_cols = r.b_mn ? r.N : r.K;
    const bool b_ok = aligned(r.B, 16) && (r.ldb % 8) == 0 &&
                      (r.batch == 1 || ((r.stride_b % 8) == 0 && r.stride_b >= b_rows * r.ldb));
    long long lda_p = r.lda, ldb_p = r.ldb, sb_p = r.stride_b;
    long long ws_a = 0, ws_b = 0;
    if (!a_ok) {
        lda_p = round_up(r.K, 8);
        ws_a = round_up((long long)r.M * lda_p * 2, 256);
    }
    if (!b_ok) {
        ldb_p = round_up(b_cols, 8);
        sb_p = b_rows * ldb_p;
        ws_b = round_up(sb_p * 2 * r.batch, 256);
    }
    if (ws_a + ws_b > (long long)GEMM_BF16_NOALLOC_SCRATCH_BYTES) return GEMM_ERR_INVALID_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GEMM_ERR_CUDA;
    DevInfo di;
    if (!device_info(dev, di)) return GEMM_ERR_CUDA;
    if (di.major != 10 || di.minor != 0) return GEMM_ERR_UNSUPPORTED;

    const void* A = r.A;
    const void* B = r.B;
    if (ws_a + ws_b) {
        void* ws = nullptr;
        gemm_status_t s = noalloc_scratch(dev, &ws);
        if (s != GEMM_OK) return s;
        if (!a_ok) {
            launch_pad(r.A, r.lda, 0, ws, lda_p, 0, 1, r.M, r.K, r.stream);
            A = ws;
        }
        if (!b_ok) {
            void* dst = static_cast<char*>(ws) + ws_a;
            launch_pad(r.B, r.ldb, r.stride_b, dst, ldb_p, sb_p, r.batch, (int)b_rows, (int)b_cols,
                       r.stream);
            B = dst;
        }
    }

    const int plan = choose(r, di.sms, false).plan;
    const PlanDesc pd = kPlans[plan];
    const int b_chunk = pd.bn * pd.nsub / pd.cg;  // B rows per CTA and stage
    const int es = r.out == OUT_F32 ? 4 : 2;
    const int stg_cols = r.out == OUT_F32 ? 32 : 64;
    const bool c_tma = aligned(r.C, 16) && ((r.ldc * es) % 16) == 0 &&
                       (r.batch == 1 || ((r.stride_c * es) % 16) == 0);
    CUtensorMap ma, mb, mc;
    std::memset(&mc, 0, sizeof mc);
    const CUtensorMapSwizzle ksw = pd.bk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    gemm_status_t st = encode_3d(&ma, A, false, (uint64_t)r.K, (uint64_t)r.M, 1, (uint64_t)lda_p * 2,
                                 (uint64_t)lda_p * 2 * (uint64_t)r.M, (uint32_t)pd.bk, 128, ksw);
    if (st == GEMM_OK) {
        if (!r.b_mn)
            st = encode_3d(&mb, B, false, (uint64_t)r.K, (uint64_t)r.N, (uint64_t)r.batch,
                           (uint64_t)ldb_p * 2, (uint64_t)sb_p * 2, (uint32_t)pd.bk, (uint32_t)b_chunk, ksw);
        else
            st = encode_3d(&mb, B, false, (uint64_t)r.N, (uint64_t)r.K, (uint64_t)r.batch,
                           (uint64_t)ldb_p * 2, (uint64_t)sb_p * 2, 64, (uint32_t)pd.bk);
    }
    if (st == GEMM_OK && c_tma)
        st = encode_3d(&mc, r.C, r.out == OUT_F32, (uint64_t)r.N, (uint64_t)r.M, (uint64_t)r.batch,
                       (uint64_t)r.ldc * es, (uint64_t)r.stride_c * es, (uint32_t)stg_cols, 32);
    if (st != GEMM_OK) return st;
    KParams p;
    std::memset(&p, 0, sizeof p);
    p.M = r.M;
    p.N = r.N;
    p.K = r.K;
    p.m_blocks = (int)cdiv(r.M, 128 * pd.cg);
    p.pack = pack_factor(pd, r.b_mn, r.N);
    p.batch_real = r.batch;
    if (p.pack > 1) {
        p.n_blocks = (int)cdiv(r.batch, p.pack);
        p.batch = 1;
    } else {
        p.n_blocks = (int)cdiv(r.N, pd.bn * pd.nsub);
        p.batch = r.batch;
    }
    p.tiles = p.m_blocks * p.n_blocks * p.batch;
    p.k_blocks = (int)cdiv(r.K, pd.bk);
    p.group_m = group_m();
    p.alpha = r.alpha;
    p.beta = r.beta;
    p.C = r.C;
    p.ldc = r.ldc;
    p.stride_c = r.stride_c;
    p.c_tma = c_tma ? 1 : 0;
    p.n_store_tma = ((long long)r.N * es) % 16 == 0 ? (int)round_up(r.N, stg_cols) : r.N;
    p.c_read = r.beta != 0.0f ? 1 : 0;
    p.timeout_ns = g_timeout_ns.load();
    return launch_by_plan(plan, r.b_mn, r.out, ma, mb, mc, p, dev, di.sms, r.stream);
}

}  // namespace

extern "C" {

gemm_status_t gemm_bf16(int M, int N, int K, const void* A, int lda, const void* B, int ldb, void* C,
                        int ldc, gemm_out_t out_type, float alpha, float beta, cudaStream_t stream) {
    try {
        Req r{1, M, N, K, A, lda, B, ldb, 0, false, C, ldc, 0, (int)out_type, alpha, beta, stream};
        return run(r);
    } catch (...) {
        return GEMM_ERR_CUDA;
    }
}

gemm_status_t gemm_bf16_batched_shared_w(int batch, int M, int N, int K, const void* W, int ldw,
                                         const void* X, int ldx, long long stride_x, void* Y, int ldy,
                                         long long stride_y, gemm_out_t out_type, float alpha,
                                         float beta, cudaStream_t stream) {
    try {
        Req r{batch, M, N, K, W, ldw, X, ldx, stride_x, true, Y, ldy, stride_y, (int)out_type,
              alpha, beta, stream};
        return run(r);
    } catch (...) {
        return GEMM_ERR_CUDA;
    }
}

gemm_status_t gemm_bf16_noalloc(int M, int N, int K, const void* A, int lda, const void* B, int ldb,
                                void* C, int ldc, gemm_out_t out_type, float alpha, float beta,
                                cudaStream_t stream) {
    try {
        Req r{1, M, N, K, A, lda, B, ldb, 0, false, C, ldc, 0, (int)out_type, alpha, beta, stream};
        return run_noalloc(r);
    } catch (...) {
        return GEMM_ERR_CUDA;
    }
}

const char* gemm_bf16_status_string(gemm_status_t s) {
    switch (s) {
        case GEMM_OK: return "GEMM_OK";
        case GEMM_ERR_INVALID_ARG: return "GEMM_ERR_INVALID_ARG";
        case GEMM_ERR_UNSUPPORTED: return "GEMM_ERR_UNSUPPORTED";
        case GEMM_ERR_CUDA: return "GEMM_ERR_CUDA";
        case GEMM_ERR_TIMEOUT: return "GEMM_ERR_TIMEOUT";
        case GEMM_ERR_NO_MEMORY: return "GEMM_ERR_NO_MEMORY";
    }
    return "GEMM_ERR_UNKNOWN";
}

gemm_status_t gemm_bf16_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GEMM_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_pw_status, sizeof v) != cudaSuccess) return GEMM_ERR_CUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_pw_status, &zero, sizeof zero) != cudaSuccess) return GEMM_ERR_CUDA;
        return GEMM_ERR_TIMEOUT;
    }
    return GEMM_OK;
}

gemm_status_t gemm_bf16_set_plan(int plan) {
    if (plan < -1 || plan >= kNumPlans) return GEMM_ERR_INVALID_ARG;
    g_plan_override.store(plan);
    return GEMM_OK;
}

gemm_status_t gemm_bf16_set_wait_timeout_ns(unsigned long long ns) {
    g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : ns);
    return GEMM_OK;
}

int gemm_bf16_version(void) { return 100; }

}  // extern "C"
