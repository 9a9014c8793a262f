// api.cu -- host side of the C ABI declared in include/gemm_bf16.h: argument validation,
// tile-plan choice, tensor-map encoding (cached), the alignment pre-pass and the kernel
// launches.  Every step of the computation runs in the kernels of gemm_kernel.cuh and
// aux_kernels.cuh; this file only prepares and enqueues them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <array>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <cstdio>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "aux_kernels.cuh"
#include "gemm_bf16.h"
#include "launch.cuh"

using namespace pw;

// The library's device status word: bit i set = a bounded wait of kernel role i expired.
// Kernels of every plan reach it through the address stored in KParams::status.
static __device__ unsigned int g_pw_status;

namespace {

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;
// m-blocks per raster group: groups of 16 read 13 % fewer DRAM bytes than groups of 8 on the
// LLM up-projection (7.33 vs 8.43 GB per launch under ncu on B200) and timed faster there and on
// 8192^3 in the same call.
constexpr int kGroupM = 16;

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
    unsigned int* status = nullptr;  // device address of g_pw_status
    // Clusters of 2, 4 and 8 CTAs (one CTA per SM: the GEMM kernels' shared memory) that the
    // device holds at once; a cluster must sit inside one GPC, so this is below sms / size.
    int cluster_cap[3] = {0, 0, 0};
};

// Empty kernel with the GEMM kernels' footprint (one CTA per SM), for the cluster occupancy query.
__global__ void cluster_probe_kernel() {}
constexpr int kProbeSmemBytes = 200 * 1024;

// Clusters of `cdim` CTAs of one SM each that the device can hold at once (sms / cdim if the
// query fails).
int query_cluster_cap(int sms, int cdim) {
    static bool attr = cudaFuncSetAttribute(cluster_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kProbeSmemBytes) == cudaSuccess;
    int n = 0;
    if (attr) {
        cudaLaunchConfig_t q = {};
        q.gridDim = dim3((unsigned)cdim, 1, 1);
        q.blockDim = dim3(192, 1, 1);
        q.dynamicSmemBytes = kProbeSmemBytes;
        cudaLaunchAttribute qa[1];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = (unsigned)cdim;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        q.attrs = qa;
        q.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, cluster_probe_kernel, &q) != cudaSuccess) n = 0;
    }
    return n > 0 && n <= sms / cdim ? n : sms / cdim;
}

std::mutex g_dev_mu;
std::array<DevInfo, kMaxDevices> g_dev;

// Attributes of device `dev` (the current device) and the address of the status word on it.
bool device_info(int dev, DevInfo& out) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo& d = g_dev[dev];
    if (!d.init) {
        void* st = nullptr;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return false;
        if (d.major == 10 && d.minor == 0) {
            if (cudaGetSymbolAddress(&st, g_pw_status) != cudaSuccess || st == nullptr) return false;
            d.status = static_cast<unsigned int*>(st);
            for (int i = 0; i < 3; ++i) d.cluster_cap[i] = query_cluster_cap(d.sms, 2 << i);
        }
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

// A kernel configuration: tile plan, how K is cut, and the raster group.
struct Choice {
    int plan;
    int splits;       // global split-K slices (1: none)
    int csplit = 1;   // cluster split-K slices (1: none)
    int group_m = 0;  // m-blocks per raster group (0: the default)
    int sk = 0;       // 1: stream-K (the last, partial wave's tiles cut into K ranges over every cluster)
};

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
    int out;     // OUT_F32 / OUT_BF16 / OUT_F16
    int in_f16;  // A and B hold fp16 (1) or bf16 (0) values
    float alpha, beta;
    cudaStream_t stream;
    // Deduplicated shared-W form: B (X) holds n_x distinct entries and output item b uses entry
    // index[b] (device memory, `batch` ints); nullptr for the plain forms.
    const int* index = nullptr;
    int n_x = 0;
    int items = 0;  // planning copies of a deduplicated request: the output items (batch = n_x)
    // A configuration to run as is (the autotuner's candidates); nullptr: choose one.
    const Choice* force = nullptr;
};

// Device status bits beyond the kernels' bounded-wait roles (kStatus* in gemm_kernel.cuh).
constexpr unsigned int kStatusBadIndex = 8u;  // a deduplicated batch's index was out of range

struct PlanDesc {
    int cg, bn, nsub, stages, bk;  // CTAs per tile, MMA N, N sub-tiles per tile, ring stages, K per stage
    int ares;                      // A resident in shared memory (needs M <= 128*cg, K <= 512)
    double rate;                   // TFLOP/s with every SM busy (B200, 8192^3 bf16); 0: never auto
};
constexpr int kNumPlans = PW_NUM_PLANS;
constexpr PlanDesc kPlans[kNumPlans] = {
    {PW_PLAN0_ARGS, 880.0},   // 128x128, one CTA
    {PW_PLAN1_ARGS, 1190.0},  // 128x256, one CTA
    {PW_PLAN2_ARGS, 1250.0},  // 256x256, 2-CTA cluster
    {PW_PLAN3_ARGS, 790.0},   // 256x128, 2-CTA cluster
    {PW_PLAN4_ARGS, 1400.0},  // 256x512, 2-CTA cluster, two 256-column MMA sub-tiles
    {PW_PLAN5_ARGS, 0.0},     // 256x128, 2-CTA cluster, A resident (M <= 256, K <= 512)
    {PW_PLAN6_ARGS, 0.0},     // 128x128, one CTA, A resident (M <= 128, K <= 512)
    {PW_PLAN7_ARGS, 0.0},     // 256x256, 2-CTA cluster, A resident (M <= 256, K <= 512)
    {PW_PLAN8_ARGS, 590.0},   // 128x64, one CTA (twice the tiles of plan 0 on thin shapes)
};

gemm_status_t launch_by_plan(int plan, const LaunchArgs& a) {
    switch (plan) {
        case 0: return launch_plan0(a);
        case 1: return launch_plan1(a);
        case 2: return launch_plan2(a);
        case 3: return launch_plan3(a);
        case 4: return launch_plan4(a);
        case 5: return launch_plan5(a);
        case 6: return launch_plan6(a);
        case 7: return launch_plan7(a);
        case 8: return launch_plan8(a);
        default: return GEMM_ERR_INVALID_ARG;
    }
}

// Batch entries packed side by side into one tile by plan `pd` (1 = no packing): needs the
// N-major (batched) B operand, N a multiple of the 64-column box and dividing the tile width.
int pack_factor(const PlanDesc& pd, bool b_mn, int N) {
    const int tile_n = pd.bn * pd.nsub;
    if (!b_mn || N <= 0 || N % 64 != 0 || tile_n % N != 0 || tile_n == N) return 1;
    return tile_n / N;
}

inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
inline long long round_up(long long a, long long b) { return cdiv(a, b) * b; }
inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline int out_bytes(int out) { return out == OUT_F32 ? 4 : 2; }

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

gemm_status_t validate(const Req& r) {
    if (r.batch < 0 || r.M < 0 || r.N < 0 || r.K < 0) return GEMM_ERR_INVALID_ARG;
    if (r.index != nullptr && r.n_x < 0) return GEMM_ERR_INVALID_ARG;
    if (r.out != OUT_F32 && r.out != OUT_BF16 && r.out != OUT_F16) return GEMM_ERR_INVALID_ARG;
    const long long minA = r.K > 1 ? r.K : 1;
    const long long minB = r.b_mn ? (r.N > 1 ? r.N : 1) : (r.K > 1 ? r.K : 1);
    const long long minC = r.N > 1 ? r.N : 1;
    if (r.lda < minA || r.ldb < minB || r.ldc < minC) return GEMM_ERR_INVALID_ARG;
    if (r.stride_b < 0 || r.stride_c < 0) return GEMM_ERR_INVALID_ARG;
    if (r.batch == 0 || r.M == 0 || r.N == 0) return GEMM_OK;
    if (r.C == nullptr || !aligned(r.C, (uintptr_t)out_bytes(r.out))) return GEMM_ERR_INVALID_ARG;
    if (r.batch > 1 && r.stride_c < (long long)(r.M - 1) * r.ldc + r.N) return GEMM_ERR_INVALID_ARG;
    if (r.K > 0 && r.alpha != 0.0f) {
        if (r.A == nullptr || r.B == nullptr) return GEMM_ERR_INVALID_ARG;
        if (!aligned(r.A, 2) || !aligned(r.B, 2)) return GEMM_ERR_INVALID_ARG;
        if (r.index != nullptr && (r.n_x == 0 || !aligned(r.index, 4))) return GEMM_ERR_INVALID_ARG;
    }
    return GEMM_OK;
}

// ------------------------------------------------------------------ tensor-map cache
// An encoded CUtensorMap depends only on its arguments (base address, element type, extents,
// strides, box and swizzle), so repeated calls on the same buffers reuse the encoded maps
// instead of calling the driver three times per GEMM.  The cache holds at most kMapCacheMax
// maps and is emptied when it is full.
struct MapKey {
    uint64_t base;
    uint64_t dims[3];
    uint64_t strides[2];
    uint32_t box[2];
    int32_t dtype;
    int32_t swizzle;
    bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof *this) == 0; }
};
static_assert(sizeof(MapKey) == 64, "MapKey has no padding");

struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        const unsigned char* b = reinterpret_cast<const unsigned char*>(&k);
        uint64_t h = 1469598103934665603ull;  // FNV-1a
        for (size_t i = 0; i < sizeof k; ++i) h = (h ^ b[i]) * 1099511628211ull;
        return (size_t)h;
    }
};

constexpr size_t kMapCacheMax = 4096;

// L2 sector promotion of the TMA loads (build option PW_L2_PROMOTION: 0 none, 64, 128, 256 bytes).
#ifndef PW_L2_PROMOTION
#define PW_L2_PROMOTION 256
#endif
constexpr CUtensorMapL2promotion kL2Promotion =
    PW_L2_PROMOTION == 0 ? CU_TENSOR_MAP_L2_PROMOTION_NONE
    : PW_L2_PROMOTION == 64 ? CU_TENSOR_MAP_L2_PROMOTION_L2_64B
    : PW_L2_PROMOTION == 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                             : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;
std::atomic<unsigned long long> g_map_hits{0}, g_map_misses{0};

gemm_status_t encode_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, uint64_t d0,
                        uint64_t d1, uint64_t d2, uint64_t s1_bytes, uint64_t s2_bytes, uint32_t b0,
                        uint32_t b1, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    MapKey key;
    std::memset(&key, 0, sizeof key);
    key.base = reinterpret_cast<uint64_t>(base);
    key.dims[0] = d0, key.dims[1] = d1, key.dims[2] = d2;
    key.strides[0] = s1_bytes, key.strides[1] = s2_bytes;
    key.box[0] = b0, key.box[1] = b1;
    key.dtype = (int32_t)dtype;
    key.swizzle = (int32_t)swizzle;
    {
        std::lock_guard<std::mutex> lk(g_map_mu);
        auto it = g_maps.find(key);
        if (it != g_maps.end()) {
            *m = it->second;
            g_map_hits.fetch_add(1);
            return GEMM_OK;
        }
    }
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GEMM_ERR_CUDA;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1_bytes, s2_bytes};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult res = fn(m, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, kL2Promotion,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (res != CUDA_SUCCESS) return GEMM_ERR_CUDA;
    g_map_misses.fetch_add(1);
    std::lock_guard<std::mutex> lk(g_map_mu);
    if (g_maps.size() >= kMapCacheMax) g_maps.clear();
    g_maps.emplace(key, *m);
    return GEMM_OK;
}

CUtensorMapDataType out_dtype(int out) {
    return out == OUT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
           : out == OUT_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                            : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

// ------------------------------------------------------------------ plan choice
// The automatic choice minimises the modelled time of plan_time() below over the streaming
// plans (rate > 0): large tiles move fewer operand bytes per FLOP, small tiles quantise better
// on small grids.

// Split-K limits: at most kMaxSplits slices of K, each at least kMinSplitKBlocks k-blocks long
// (the smem ring needs a few blocks to fill), and a split must beat the unsplit choice by 10%.
constexpr int kMaxSplits = 8;
constexpr int kMinSplitKBlocks = 8;
// Operand bytes one CTA pulls through TMA per second when its tiles are not compute-bound
// (fitted on B200 to few, deep tiles: 8192x256x4096, 127x8191x2048, 512^2 x 8192, 1024^2 x 8192,
// 2048^2 x 8192, every streaming plan, unsplit and cut across a cluster).
constexpr double kCtaOperandBytesPerSec = 100e9;
// Time of a tile that its mainloop does not cover: the first loads' latency and the epilogue
// (the same fit).  A persistent launch pays it once (later tiles overlap their epilogue with
// the next mainloop); cluster split-K, whose CTAs hold one tile each, once per wave.
constexpr double kTileFixedSec = 10e-6;
// Split-K cost per unit, measured on B200: a fixed part (counter, fences, the longer fixup
// epilogue), the write of the unit's fp32 partial sums and the last unit's read of the others.
constexpr double kSplitFixedSec = 4e-6;
constexpr double kSplitWriteBytesPerSec = 45e9;
constexpr double kSplitReadBytesPerSec = 90e9;
// Fixed cost of one launch besides kTileFixedSec: launch latency, prologue and teardown.
// 2-CTA tiles pay more (the leader waits for both CTAs' loads; on B200 plan 1 beats plan 2 by
// 13 % on 2048^3 although their waves model equal).
constexpr double kLaunchFixedSecOneCta = 5e-6;
constexpr double kLaunchFixedSecCtaPair = 8e-6;
// Split-K arrival counters per CTA and tile: one per epilogue warp.
constexpr int kSplitCountersPerCta = 8;
// Cluster split-K: a tile's K slices run on the CTAs of one cluster (2, 4 or 8 CTAs) and their
// partial tiles are added through distributed shared memory.  Cost per wave beyond its slices'
// mainloop and kTileFixedSec: each CTA's read of the other slices' share of its part of the
// tile, at the per-warp rate distributed shared memory gives the reduction (fitted with the
// constants above).
constexpr double kClusterSplitBytesPerSec = 25e9;

// Can plan `i` serve this request?
bool plan_serves(int i, const Req& r) {
    const PlanDesc& pd = kPlans[i];
    if (pd.ares) return r.M <= 128 * pd.cg && r.K <= 8 * pd.bk;
    if (r.b_mn && (pd.bn / pd.cg) % 64 != 0) return false;
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
               (pd.cg == 2 ? kLaunchFixedSecCtaPair : kLaunchFixedSecOneCta) + kTileFixedSec;
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

// GEMM_BF16_STREAM_K=1 forces stream-K wherever it applies (tests, tuning); 0 forbids it; unset
// leaves the choice to the model.
int forced_stream_k() {
    const char* e = std::getenv("GEMM_BF16_STREAM_K");
    if (e && (e[0] == '0' || e[0] == '1') && e[1] == '\0') return e[0] == '1' ? 1 : 2;
    return 0;  // 0: unset, 1: forced, 2: forbidden
}

// Stream-K geometry of a plan for a request: the persistent grid's clusters, the tiles of the
// last, partial wave (computed as K ranges spread evenly over every cluster; the whole tiles
// come after them in the tile order) and a bound on the ranges one of those tiles is cut into
// (its partial-sum slots): a tile's kb consecutive k-blocks meet at most ceil((kb-1)/base) + 1
// ranges of at least `base` k-blocks each.  sk_tiles == 0: stream-K does not apply (at most one
// wave, whole waves only, or ranges shorter than kMinSplitKBlocks k-blocks).
struct SkGeom {
    int clusters = 0;
    int sk_tiles = 0;
    int max_parts = 0;
};
SkGeom sk_geometry(const PlanDesc& pd, const Req& r, int clusters) {
    SkGeom g;
    const long long tiles = plan_tiles(pd, r), kb = cdiv(r.K, pd.bk);
    if (pd.ares || clusters <= 0 || tiles <= clusters) return g;
    const long long sk = tiles % clusters;
    const long long total = sk * kb;
    if (sk == 0 || total < (long long)clusters * kMinSplitKBlocks) return g;
    const long long base = total / clusters;
    long long mp = cdiv(kb - 1, base) + 1;
    if (mp > clusters) mp = clusters;
    g.clusters = clusters;
    g.sk_tiles = (int)sk;
    g.max_parts = (int)mp;
    return g;
}
// Persistent clusters of a plan on the device (one CTA per SM; CTA pairs as the device places them).
int persistent_clusters(const PlanDesc& pd, int sms, const int* ccap) { return pd.cg == 2 ? ccap[0] : sms; }

// Plans whose kernels take cluster split-K: streaming tiles with one MMA sub-tile (the kernel's
// Tile::CSPLIT_OK), sliced over up to 8 CTAs per cluster (CTA pairs: up to 4 slices).
bool plan_csplit_ok(const PlanDesc& pd) { return pd.nsub == 1 && !pd.ares; }
int max_csplit(const PlanDesc& pd) { return 8 / pd.cg; }

// Modelled time (s) of plan `i` with cluster split-K over `cs` slices (CTAs or CTA pairs): the
// tiles' clusters run in waves of `cap` clusters (as many as the device holds at once), each
// slice streaming its K range; then the tile's fixed cost and the reduction.
double plan_time_csplit(int i, const Req& r, int sms, int cs, int cap) {
    const PlanDesc& pd = kPlans[i];
    const long long tm = 128LL * pd.cg, tn = (long long)pd.bn * pd.nsub;
    const long long kb = cdiv(cdiv(r.K, pd.bk), cs);
    const double unit_k = (double)(kb * pd.bk);
    const long long slots = sms / pd.cg;  // one CTA per SM
    const double compute = 2.0 * (double)(tm * tn) * unit_k / (pd.rate * 1e12 / (double)slots);
    const double stream = (double)(tm + tn) * unit_k * 2.0 / (pd.cg * kCtaOperandBytesPerSec);
    const long long waves = cdiv(plan_tiles(pd, r), cap > 0 ? cap : 1);
    const double xbytes = 128.0 * (double)tn * 4.0 * (double)(cs - 1) / (double)cs;
    return (double)waves * ((compute > stream ? compute : stream) + kTileFixedSec +
                            xbytes / kClusterSplitBytesPerSec) +
           (pd.cg == 2 ? kLaunchFixedSecCtaPair : kLaunchFixedSecOneCta);
}

// GEMM_BF16_CLUSTER_SPLIT=s (2, 4 or 8) forces cluster split-K with s slices wherever the plan
// takes it (tests, tuning); 1 forbids it; unset or 0 leaves the choice to the model.
int forced_csplit() {
    const char* e = std::getenv("GEMM_BF16_CLUSTER_SPLIT");
    if (e) {
        const int v = std::atoi(e);
        if (v == 1 || v == 2 || v == 4 || v == 8) return v;
    }
    return 0;
}

// Modelled time (s) of plan `i` with stream-K geometry `g`: the whole waves and the last wave's
// share of K per cluster, the fixed costs of a launch, and the exposed part of the fixup (the
// last part of a tile reads every part's partial sums; the publishing overlaps the next unit).
double plan_time_sk(int i, const Req& r, int sms, const SkGeom& g) {
    const PlanDesc& pd = kPlans[i];
    const long long tm = 128LL * pd.cg, tn = (long long)pd.bn * pd.nsub;
    const double unit_k = (double)(cdiv(r.K, pd.bk) * pd.bk);
    const long long slots = sms / pd.cg;
    const double compute = 2.0 * (double)(tm * tn) * unit_k / (pd.rate * 1e12 / (double)slots);
    const double stream = (double)(tm + tn) * unit_k * 2.0 / (pd.cg * kCtaOperandBytesPerSec);
    const long long tiles = plan_tiles(pd, r);
    const double waves = (double)((tiles - g.sk_tiles) / g.clusters) + (double)g.sk_tiles / (double)g.clusters;
    const double partial = 128.0 * (double)tn * 4.0;
    // A tile of two MMA sub-tiles holds both accumulator slots, so the next unit's mainloop
    // waits while a part's partial sums are published (measured on B200: 4096^3 and
    // 2048x8192x8192 on plan 4 gained nothing from stream-K).
    const double units = (double)g.sk_tiles * (double)g.max_parts / (double)g.clusters;
    const double publish = pd.nsub == 2 ? units * partial / kSplitWriteBytesPerSec : 0.0;
    return waves * (compute > stream ? compute : stream) + (pd.cg == 2 ? kLaunchFixedSecCtaPair : kLaunchFixedSecOneCta) +
           kTileFixedSec + kSplitFixedSec + (double)g.max_parts * partial / kSplitReadBytesPerSec + publish;
}

// Plan and K split for a request on a device with `sms` SMs that holds `ccap[i]` clusters of
// 2 << i CTAs at once (auto unless overridden); without `allow_split` no global split-K (it
// needs workspace); cluster split-K needs none.
Choice choose(const Req& r, int sms, const int* ccap, bool allow_split) {
    const int fs_env = forced_splits();  // GEMM_BF16_SPLIT_K (0: unset)
    const int fs = allow_split ? fs_env : 1;
    const int fcs = r.index != nullptr ? 1 : forced_csplit();  // dedup units replace K slices
    const int forced = g_plan_override.load();
    int only = -1;  // the one plan to consider, or -1 for every streaming plan
    if (forced >= 0 && plan_serves(forced, r)) {
        if (kPlans[forced].ares) return {forced, 1};
        only = forced;
    } else if (r.index != nullptr && r.b_mn && r.K <= 1024 && r.items >= 32LL * r.n_x && plan_serves(8, r)) {
        // Deduplicated batches with few distinct entries (32 or more items each) are bound by
        // writing the items: the smallest one-CTA tiles spread the writes over the most SMs
        // (B200, 2048 items of 256x128 from 256x512 . 512x128: 16 entries 47.4 -> 43.4 us with
        // plan 8 instead of plan 7, 64 entries 47.4 -> 45.3 us; at 256 entries plan 7 wins).
        return {8, 1};
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
        if (only >= 0 ? i != only : (pd.rate <= 0.0 || !plan_serves(i, r))) continue;
        const int s = fs > 0 && split_valid(pd, r, fs) ? fs : 1;
        const double t = plan_time(i, r, sms, s);
        if (!have || t < best_t * 0.999) best = {i, s}, best_t = t, have = true;
    }
    // Cluster split-K (no workspace): forced, or, when no split is forced either way, where it
    // beats the best so far by 10 %.
    if (fcs > 1 || (fs_env == 0 && fcs == 0)) {
        const double cbar = best_t * 0.90;
        for (int i = 0; i < kNumPlans; ++i) {
            const PlanDesc& pd = kPlans[i];
            if (!plan_csplit_ok(pd)) continue;
            if (only >= 0 ? i != only : (pd.rate <= 0.0 || !plan_serves(i, r))) continue;
            const long long tiles = plan_tiles(pd, r);
            for (int cs = 2; cs <= max_csplit(pd); cs *= 2) {
                if (fcs > 0 && cs != fcs) continue;
                if (!split_valid(pd, r, cs) || cdiv(r.K, pd.bk) < (long long)cs * 2) continue;
                const int cdim = cs * pd.cg;
                const int cap = ccap[cdim == 2 ? 0 : cdim == 4 ? 1 : 2];
                // Automatically only where the unsplit tiles leave at least half the SMs idle and
                // the split tiles' clusters all fit on the device at once: measured on B200, a
                // split that adds a wave (8192x256x4096: 37.8 -> 50 us) or only fills the last
                // SMs loses.
                if (fcs == 0 && (2 * tiles * pd.cg > sms || tiles > cap)) continue;
                const double t = plan_time_csplit(i, r, sms, cs, cap);
                if (fcs > 0 || (t < cbar && t < best_t * 0.999)) {
                    best = {i, 1, cs};
                    best_t = t;
                    if (fcs > 0) return best;
                }
            }
        }
    }
    if (fs > 0 || !allow_split || best.csplit > 1) return best;
    // Stream-K where the last wave is partial: forced, or where it beats the best by 5 %.
    const int fsk = r.index != nullptr ? 2 : forced_stream_k();
    if (fsk != 2) {
        const double sk_bar = best_t * 0.95;
        Choice sk_best{-1, 1};
        double sk_t = 0.0;
        for (int i = 0; i < kNumPlans; ++i) {
            const PlanDesc& pd = kPlans[i];
            if (only >= 0 ? i != only : (pd.rate <= 0.0 || !plan_serves(i, r))) continue;
            const SkGeom g = sk_geometry(pd, r, persistent_clusters(pd, sms, ccap));
            if (g.sk_tiles == 0) continue;
            const double t = plan_time_sk(i, r, sms, g);
            if (sk_best.plan < 0 || t < sk_t) sk_best = Choice{i, 1, 1, 0, 1}, sk_t = t;
        }
        // forced: the plan chosen so far, where stream-K applies to it
        if (fsk == 1 && sk_geometry(kPlans[best.plan], r, persistent_clusters(kPlans[best.plan], sms, ccap)).sk_tiles > 0)
            return Choice{best.plan, 1, 1, 0, 1};
        if (sk_best.plan >= 0 && (fsk == 1 || sk_t < sk_bar)) return sk_best;
    }
    const double split_bar = best_t * 0.90;
    for (int i = 0; i < kNumPlans; ++i) {
        const PlanDesc& pd = kPlans[i];
        if (only >= 0 ? i != only : (pd.rate <= 0.0 || !plan_serves(i, r))) continue;
        // Only few-tile problems (at least half the clusters idle unsplit): with many tiles the
        // partial sums' traffic swamps the gain (4096^3, plan 4, two slices: 102 -> 175 us).
        if (2 * plan_tiles(pd, r) > sms / pd.cg) continue;
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

// ------------------------------------------------------------------ tuning table
// Configurations measured by gemm_autotune, keyed by everything the choice depends on: the
// device's SM count, the shape, the operand form and types, whether C is read, and the
// alignment classes that select the pre-pass and the store path.  Calls whose key is in the
// table take its configuration (unless a plan or split is forced).
struct TuneKey {
    int sms, batch, M, N, K, n_x;
    int b_mn, in_f16, out, c_read, a_ok, b_ok, c_tma;
    bool operator==(const TuneKey& o) const { return std::memcmp(this, &o, sizeof *this) == 0; }
};
static_assert(sizeof(TuneKey) == 13 * sizeof(int), "TuneKey has no padding");

struct TuneKeyHash {
    size_t operator()(const TuneKey& k) const {
        const unsigned char* b = reinterpret_cast<const unsigned char*>(&k);
        uint64_t h = 1469598103934665603ull;  // FNV-1a
        for (size_t i = 0; i < sizeof k; ++i) h = (h ^ b[i]) * 1099511628211ull;
        return (size_t)h;
    }
};

struct TuneVal {
    Choice ch;
    float us;  // measured time of one call (median of the timed runs)
};

std::mutex g_tune_mu;
std::unordered_map<TuneKey, TuneVal, TuneKeyHash> g_tune;

// The configuration the calling thread's most recent GEMM launch used (gemm_last_config).
thread_local Choice t_last{-1, 0, 0, 0};

bool tuned_choice(const TuneKey& k, Choice* out) {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    auto it = g_tune.find(k);
    if (it == g_tune.end()) return false;
    *out = it->second.ch;
    return true;
}

// Strides that a single-entry operand does not use are set to its extent, as the kernels
// address every operand in three dimensions.
void normalize(Req& r) {
    if ((r.index != nullptr ? r.n_x : r.batch) == 1) r.stride_b = r.b_mn ? (long long)r.K * r.ldb : (long long)r.N * r.ldb;
    if (r.batch == 1) r.stride_c = (long long)r.M * r.ldc;
}

// TMA-readability of A and B as given (else the pre-pass copies them) and of C (else the
// row-by-row store path), for a normalized request.
void alignment_classes(const Req& r, bool* a_ok, bool* b_ok, bool* c_tma) {
    const int nb = r.index != nullptr ? r.n_x : r.batch;
    const long long b_rows = r.b_mn ? r.K : r.N;
    const int es = out_bytes(r.out);
    *a_ok = aligned(r.A, 16) && (r.lda % 8) == 0;
    *b_ok = aligned(r.B, 16) && (r.ldb % 8) == 0 && (nb == 1 || ((r.stride_b % 8) == 0 && r.stride_b >= b_rows * r.ldb));
    *c_tma = aligned(r.C, 16) && ((r.ldc * es) % 16) == 0 && (r.batch == 1 || ((r.stride_c * es) % 16) == 0);
}

TuneKey tune_key(const Req& r, int sms) {
    bool a_ok, b_ok, c_tma;
    alignment_classes(r, &a_ok, &b_ok, &c_tma);
    return TuneKey{sms, r.batch, r.M, r.N, r.K, r.index != nullptr ? r.n_x : 0, r.b_mn ? 1 : 0, r.in_f16, r.out,
                   r.beta != 0.0f ? 1 : 0, a_ok ? 1 : 0, b_ok ? 1 : 0, c_tma ? 1 : 0};
}

// Any explicit override (forced plan, forced split of either kind, forced raster group) turns
// the table off for the call.
bool overrides_set() {
    return g_plan_override.load() >= 0 || std::getenv("GEMM_BF16_SPLIT_K") != nullptr ||
           std::getenv("GEMM_BF16_CLUSTER_SPLIT") != nullptr || std::getenv("GEMM_BF16_GROUP_M") != nullptr ||
           std::getenv("GEMM_BF16_STREAM_K") != nullptr;
}

// The cost model's choice per problem (and workspace permission), so that a repeated call skips
// the model.  Not used while an override is set; bounded by clearing it when it grows large.
std::mutex g_memo_mu;
std::unordered_map<TuneKey, Choice, TuneKeyHash> g_memo[2];
constexpr size_t kMemoMax = 4096;

bool memo_choice(const TuneKey& k, bool may_split, Choice* out) {
    std::lock_guard<std::mutex> lk(g_memo_mu);
    auto& m = g_memo[may_split ? 1 : 0];
    auto it = m.find(k);
    if (it == m.end()) return false;
    *out = it->second;
    return true;
}

void memo_store(const TuneKey& k, bool may_split, const Choice& c) {
    std::lock_guard<std::mutex> lk(g_memo_mu);
    auto& m = g_memo[may_split ? 1 : 0];
    if (m.size() >= kMemoMax) m.clear();
    m[k] = c;
}

// ------------------------------------------------------------------ auxiliary launches
gemm_status_t launch_scale(const Req& r) {
    const long long total = (long long)r.batch * r.M * r.N;
    const int threads = 256;
    long long blocks = cdiv(total, threads);
    if (blocks > 148LL * 32) blocks = 148LL * 32;
    (void)cudaGetLastError();  // report only what this launch raises
    switch (r.out) {
        case OUT_F32:
            scale_c_kernel<OUT_F32><<<(unsigned)blocks, threads, 0, r.stream>>>(r.C, r.ldc, r.stride_c, r.batch,
                                                                                r.M, r.N, r.beta);
            break;
        case OUT_BF16:
            scale_c_kernel<OUT_BF16><<<(unsigned)blocks, threads, 0, r.stream>>>(r.C, r.ldc, r.stride_c, r.batch,
                                                                                 r.M, r.N, r.beta);
            break;
        default:
            scale_c_kernel<OUT_F16><<<(unsigned)blocks, threads, 0, r.stream>>>(r.C, r.ldc, r.stride_c, r.batch,
                                                                                r.M, r.N, r.beta);
            break;
    }
    return cudaGetLastError() == cudaSuccess ? GEMM_OK : GEMM_ERR_CUDA;
}

// Enqueue the alignment pre-pass copy of a batch x rows x cols operand; GEMM_ERR_CUDA when the
// launch fails (the GEMM must then not run on the copy's destination).
gemm_status_t launch_pad(const void* src, long long ld_src, long long bs_src, void* dst, long long ld_dst,
                         long long bs_dst, int batch, int rows, int cols, cudaStream_t st) {
    const int threads = 128;
    int gx = (int)cdiv(cdiv(cols, 8), threads);
    if (gx > 8) gx = 8;
    int gy = rows < 4096 ? (rows > 0 ? rows : 1) : 4096;
    int gz = batch < 65535 ? batch : 65535;
    // extent of the source: from its first element to one past its last
    const uintptr_t lo = reinterpret_cast<uintptr_t>(src);
    const uintptr_t hi = lo + 2 * (uintptr_t)((long long)(batch - 1) * bs_src + (long long)(rows - 1) * ld_src + cols);
    (void)cudaGetLastError();  // report only what this launch raises
    pad_copy_kernel<<<dim3(gx, gy, gz), threads, 0, st>>>(
        static_cast<const uint16_t*>(src), ld_src, bs_src, static_cast<uint16_t*>(dst), ld_dst, bs_dst,
        batch, rows, cols, lo, hi);
    return cudaGetLastError() == cudaSuccess ? GEMM_OK : GEMM_ERR_CUDA;
}

// ------------------------------------------------------------------ workspace sources
// gemm_bf16_noalloc's scratch: the padded copies of A and B written by the alignment pre-pass
// and read by the GEMM kernel.  Every device that loads this library holds it until the process
// exits.  In host code this name is only a host-side stand-in, never a device address: kernels
// are given the address that static_scratch() obtains once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GEMM_BF16_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
std::array<void*, kMaxDevices> g_scratch_ptr{};

// Device address of the scratch on device `dev`, which must be the current device.  The first
// call per device asks the runtime for it; later calls reuse the cached value.
gemm_status_t static_scratch(int dev, void** out) {
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

// Where a call's workspace comes from: the library's stream-ordered pool (gemm_bf16 and the
// other allocating entry points), or the fixed static scratch (gemm_bf16_noalloc), which never
// allocates and therefore never splits K (split-K needs partial sums sized by the problem).
enum class Workspace { Pool, Static };

// ------------------------------------------------------------------ the GEMM call
gemm_status_t run(Req r, Workspace wsrc) {
    gemm_status_t v = validate(r);
    if (v != GEMM_OK) return v;
    if (r.batch == 0 || r.M == 0 || r.N == 0) return GEMM_OK;
    normalize(r);
    if (r.K == 0 || r.alpha == 0.0f) return launch_scale(r);

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GEMM_ERR_CUDA;
    DevInfo di;
    if (!device_info(dev, di)) return GEMM_ERR_CUDA;
    if (di.major != 10 || di.minor != 0) return GEMM_ERR_UNSUPPORTED;

    // Deduplicated form: the GEMM runs over the n_x distinct entries of X (rg); its epilogue
    // stores each entry's result to the r.batch output items that use it.
    const bool dedup = r.index != nullptr;
    Req rg = r;
    if (dedup) rg.batch = r.n_x, rg.items = r.batch;

    // Operands TMA cannot read as given go through a padded, 16-byte aligned copy; C that TMA
    // cannot address takes the row-by-row store path.
    bool a_ok, b_ok, c_tma;
    alignment_classes(r, &a_ok, &b_ok, &c_tma);
    const long long b_rows = r.b_mn ? r.K : r.N;  // rows of the stored B matrix per batch
    const long long b_cols = r.b_mn ? r.N : r.K;
    long long lda_p = r.lda, ldb_p = r.ldb, sb_p = r.stride_b;
    size_t ws_a = 0, ws_b = 0;
    if (!a_ok) {
        lda_p = round_up(r.K, 8);
        ws_a = (size_t)round_up((long long)r.M * lda_p * 2, 256);
    }
    if (!b_ok) {
        ldb_p = round_up(b_cols, 8);
        sb_p = b_rows * ldb_p;
        ws_b = (size_t)round_up(sb_p * 2 * rg.batch, 256);
    }
    const int es = out_bytes(r.out);
    // The configuration: the caller's (autotuner candidates), a tuned one, or the model's.
    const bool may_split = wsrc == Workspace::Pool && !dedup;
    const TuneKey key = tune_key(r, di.sms);
    Choice ch{0, 1};
    Choice tuned{0, 1};
    if (r.force != nullptr) {
        ch = *r.force;
        if (ch.plan < 0 || ch.plan >= kNumPlans || !plan_serves(ch.plan, rg)) return GEMM_ERR_INVALID_ARG;
        if (ch.splits > 1 && (!may_split || !split_valid(kPlans[ch.plan], rg, ch.splits))) return GEMM_ERR_INVALID_ARG;
        if (ch.csplit > 1 && (dedup || !plan_csplit_ok(kPlans[ch.plan]) || ch.csplit > max_csplit(kPlans[ch.plan]) ||
                              !split_valid(kPlans[ch.plan], rg, ch.csplit)))
            return GEMM_ERR_INVALID_ARG;
        if (ch.sk && (!may_split || ch.splits > 1 || ch.csplit > 1 ||
                      sk_geometry(kPlans[ch.plan], rg, persistent_clusters(kPlans[ch.plan], di.sms, di.cluster_cap))
                              .sk_tiles == 0))
            return GEMM_ERR_INVALID_ARG;
    } else if (!overrides_set() && tuned_choice(key, &tuned) && ((tuned.splits <= 1 && !tuned.sk) || may_split)) {
        ch = tuned;
    } else if (overrides_set()) {
        ch = choose(rg, di.sms, di.cluster_cap, may_split);
    } else if (!memo_choice(key, may_split, &ch)) {
        ch = choose(rg, di.sms, di.cluster_cap, may_split);
        memo_store(key, may_split, ch);
    }
    // Split-K partial sums (fp32, one 128 x tile_n slab per CTA, tile and slice) and the
    // per-(tile, CTA, epilogue warp) arrival counters, which must start at zero.
    const int plan = ch.plan;
    const PlanDesc pd = kPlans[plan];
    const long long tiles_est = plan_tiles(pd, rg);
    size_t ws_p = 0, ws_n = 0;
    SkGeom skg;
    if (ch.sk) skg = sk_geometry(pd, rg, persistent_clusters(pd, di.sms, di.cluster_cap));
    if (ch.sk && skg.sk_tiles == 0) return GEMM_ERR_INVALID_ARG;  // a tuned entry that no longer applies
    const bool partials = ch.splits > 1 || ch.sk;
    if (partials) {
        // slots for split-K's slices of every tile, or stream-K's parts of the cut tiles
        const long long ptiles = ch.sk ? skg.sk_tiles : tiles_est;
        const int parts = ch.sk ? skg.max_parts : ch.splits;
        ws_p = (size_t)ptiles * pd.cg * parts * 128 * pd.bn * pd.nsub * sizeof(float);
        ws_n = (size_t)round_up(ptiles * pd.cg * kSplitCountersPerCta * (long long)sizeof(unsigned int), 256);
    }
    // Deduplicated form: per-entry item lists (offsets, cursor scratch, items).
    size_t ws_d = 0;
    if (dedup) ws_d = (size_t)round_up((2LL * r.n_x + 1 + r.batch) * (long long)sizeof(int), 256);
    const size_t ws_total = ws_a + ws_b + ws_p + ws_n + ws_d;
    void* ws = nullptr;
    bool pooled = false;
    if (ws_total) {
        if (wsrc == Workspace::Static) {
            if (ws_total > (size_t)GEMM_BF16_NOALLOC_SCRATCH_BYTES) return GEMM_ERR_INVALID_ARG;
            const gemm_status_t s = static_scratch(dev, &ws);
            if (s != GEMM_OK) return s;
        } else {
            cudaMemPool_t pool = nullptr;
            const gemm_status_t ps = workspace_pool(dev, &pool);
            if (ps != GEMM_OK) return ps;
            if (cudaMallocFromPoolAsync(&ws, ws_total, pool, r.stream) != cudaSuccess) return GEMM_ERR_NO_MEMORY;
            pooled = true;
        }
    }
    auto fail = [&](gemm_status_t s) {
        if (pooled) cudaFreeAsync(ws, r.stream);
        return s;
    };
    float* ws_partials = partials ? reinterpret_cast<float*>(static_cast<char*>(ws) + ws_a + ws_b) : nullptr;
    unsigned int* ws_counters =
        partials ? reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + ws_a + ws_b + ws_p) : nullptr;
    if (ws_n && cudaMemsetAsync(ws_counters, 0, ws_n, r.stream) != cudaSuccess) return fail(GEMM_ERR_CUDA);
    int* dd_off = nullptr;
    int* dd_dst = nullptr;
    if (dedup) {
        dd_off = reinterpret_cast<int*>(static_cast<char*>(ws) + ws_a + ws_b + ws_p + ws_n);
        int* cursor = dd_off + r.n_x + 1;
        dd_dst = cursor + r.n_x;
        (void)cudaGetLastError();  // report only what this launch raises
        dedup_groups_kernel<<<1, 1024, 0, r.stream>>>(r.index, r.batch, r.n_x, dd_off, cursor, dd_dst, di.status,
                                                      kStatusBadIndex);
        if (cudaGetLastError() != cudaSuccess) return fail(GEMM_ERR_CUDA);
    }
    const void* A = r.A;
    const void* B = r.B;
    if (!a_ok) {
        if (launch_pad(r.A, r.lda, 0, ws, lda_p, 0, 1, r.M, r.K, r.stream) != GEMM_OK) return fail(GEMM_ERR_CUDA);
        A = ws;
    }
    if (!b_ok) {
        void* dst = static_cast<char*>(ws) + ws_a;
        if (launch_pad(r.B, r.ldb, r.stride_b, dst, ldb_p, sb_p, rg.batch, (int)b_rows, (int)b_cols, r.stream) !=
            GEMM_OK)
            return fail(GEMM_ERR_CUDA);
        B = dst;
    }

    const int b_chunk = pd.bn * pd.nsub / pd.cg;  // B rows per CTA and stage
    const int stg_cols = r.out == OUT_F32 ? 32 : 64;

    CUtensorMap ma, mb, mc;
    std::memset(&mc, 0, sizeof mc);
    const CUtensorMapDataType in_t = r.in_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle ksw = pd.bk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    gemm_status_t st = encode_3d(&ma, A, in_t, (uint64_t)r.K, (uint64_t)r.M, 1, (uint64_t)lda_p * 2,
                                 (uint64_t)lda_p * 2 * (uint64_t)r.M, (uint32_t)pd.bk, 128, ksw);
    if (st == GEMM_OK) {
        if (!r.b_mn)
            st = encode_3d(&mb, B, in_t, (uint64_t)r.K, (uint64_t)r.N, (uint64_t)rg.batch, (uint64_t)ldb_p * 2,
                           (uint64_t)sb_p * 2, (uint32_t)pd.bk, (uint32_t)b_chunk, ksw);
        else
            st = encode_3d(&mb, B, in_t, (uint64_t)r.N, (uint64_t)r.K, (uint64_t)rg.batch, (uint64_t)ldb_p * 2,
                           (uint64_t)sb_p * 2, 64, (uint32_t)pd.bk);
    }
    if (st == GEMM_OK && c_tma)
        st = encode_3d(&mc, r.C, out_dtype(r.out), (uint64_t)r.N, (uint64_t)r.M, (uint64_t)r.batch,
                       (uint64_t)r.ldc * es, (uint64_t)r.stride_c * es, (uint32_t)stg_cols, 32);
    if (st != GEMM_OK) return fail(st);

    LaunchArgs la;
    std::memset(&la, 0, sizeof la);
    la.b_mn = r.b_mn;
    la.out = r.out;
    la.ma = &ma;
    la.mb = &mb;
    la.mc = &mc;
    la.dev = dev;
    la.sms = di.sms;
    la.stream = r.stream;
    KParams& p = la.p;
    p.M = r.M;
    p.N = r.N;
    p.K = r.K;
    p.m_blocks = (int)cdiv(r.M, 128 * pd.cg);
    p.pack = pack_factor(pd, r.b_mn, r.N);
    p.batch_real = rg.batch;
    if (p.pack > 1) {
        p.n_blocks = (int)cdiv(rg.batch, p.pack);
        p.batch = 1;
    } else {
        p.n_blocks = (int)cdiv(r.N, pd.bn * pd.nsub);
        p.batch = rg.batch;
    }
    p.tiles = p.m_blocks * p.n_blocks * p.batch;
    p.k_blocks = (int)cdiv(r.K, pd.bk);
    if (ch.splits > 1) {
        p.splits = ch.splits;
        p.kb_per_split = (int)cdiv(p.k_blocks, ch.splits);
        p.ws = ws_partials;
        p.ws_parts = ch.splits;
        p.counters = ws_counters;
    } else if (ch.sk) {
        p.sk_tiles = skg.sk_tiles;
        p.sk_clusters = skg.clusters;
        p.ws = ws_partials;
        p.ws_parts = skg.max_parts;
        p.counters = ws_counters;
    } else if (ch.csplit > 1) {
        p.csplit = ch.csplit;
        p.kb_per_split = (int)cdiv(p.k_blocks, ch.csplit);
    }
    p.group_m = ch.group_m > 0 ? ch.group_m : group_m();
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
    p.batch_out = r.batch;
    if (dedup) {
        // Few distinct entries (few tiles) leave clusters idle: give each tile up to as many
        // work units as the clusters allow (at most the items per entry on average), each unit
        // storing its share of the entry's items.
        const long long cap = di.sms / pd.cg;
        long long ds = p.tiles > 0 ? cap / p.tiles : 1;
        const long long per_entry = cdiv(r.batch, r.n_x);
        if (ds > per_entry) ds = per_entry;
        p.dd_off = dd_off;
        p.dd_dst = dd_dst;
        p.dsplit = (int)(ds < 1 ? 1 : ds);
    }
    p.status = di.status;
    p.in_f16 = r.in_f16;
    p.timeout_ns = g_timeout_ns.load();
    p.test_stall = test_stall_requested() ? 1 : 0;
    st = launch_by_plan(plan, la);
    if (st == GEMM_OK)
        t_last = Choice{plan, p.splits > 1 ? p.splits : 1, p.csplit > 1 ? p.csplit : 1, p.group_m, p.sk_tiles > 0 ? 1 : 0};
    if (pooled) cudaFreeAsync(ws, r.stream);
    return st;
}

gemm_status_t guarded(const Req& r, Workspace w) {
    try {
        return run(r, w);
    } catch (...) {
        return GEMM_ERR_CUDA;
    }
}

// Candidate configurations for a request: every plan that serves it (resident-A plans as they
// are), unsplit, with stream-K where it applies, with each valid split of K through the workspace
// (2, 4, 8 slices) or across a cluster (2, 4, 8 CTAs or 2, 4 CTA pairs), and raster groups of 8,
// 16 and 32 m-blocks when the tiles fill more than two waves.
std::vector<Choice> candidates(const Req& rg, int sms, const int* ccap, bool dedup) {
    std::vector<Choice> c;
    for (int i = 0; i < kNumPlans; ++i) {
        const PlanDesc& pd = kPlans[i];
        if (!plan_serves(i, rg)) continue;
        const long long tiles = plan_tiles(pd, rg);
        const bool many_waves = tiles > 2LL * (sms / pd.cg);
        const int groups[3] = {16, 8, 32};
        for (int g = 0; g < (many_waves ? 3 : 1); ++g) c.push_back(Choice{i, 1, 1, groups[g]});
        if (!dedup && sk_geometry(pd, rg, persistent_clusters(pd, sms, ccap)).sk_tiles > 0)
            c.push_back(Choice{i, 1, 1, kGroupM, 1});
        if (pd.ares || dedup || many_waves) continue;
        for (int s = 2; s <= kMaxSplits; s *= 2) {
            if (!split_valid(pd, rg, s) || cdiv(rg.K, pd.bk) < (long long)s * 2) continue;
            c.push_back(Choice{i, s, 1, kGroupM});
            if (plan_csplit_ok(pd) && s <= max_csplit(pd)) c.push_back(Choice{i, 1, s, kGroupM});
        }
    }
    return c;
}

// Time every candidate on the caller's operands, writing into a scratch copy of C, and record
// the fastest in the tuning table.  Synchronous: returns after the measurements.
gemm_status_t autotune(Req r, float* best_us) {
    gemm_status_t v = validate(r);
    if (v != GEMM_OK) return v;
    if (r.batch == 0 || r.M == 0 || r.N == 0 || r.K == 0 || r.alpha == 0.0f) return GEMM_OK;  // nothing to tune
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GEMM_ERR_CUDA;
    DevInfo di;
    if (!device_info(dev, di)) return GEMM_ERR_CUDA;
    if (di.major != 10 || di.minor != 0) return GEMM_ERR_UNSUPPORTED;
    const bool dedup = r.index != nullptr;
    normalize(r);
    const TuneKey key = tune_key(r, di.sms);
    Req rg = r;
    if (dedup) rg.batch = r.n_x, rg.items = r.batch;
    const std::vector<Choice> cand = candidates(rg, di.sms, di.cluster_cap, dedup);
    if (cand.empty()) return GEMM_ERR_UNSUPPORTED;

    // Scratch C: the whole extent of the caller's C, at the same offset from a 256-byte
    // boundary (so the store path is the same), holding a copy of C when it is read.
    const int es = out_bytes(r.out);
    const size_t extent = (size_t)((long long)(r.batch - 1) * r.stride_c + (long long)(r.M - 1) * r.ldc + r.N) * es;
    const size_t off = reinterpret_cast<uintptr_t>(r.C) % 256;
    cudaMemPool_t pool = nullptr;
    gemm_status_t st = workspace_pool(dev, &pool);
    if (st != GEMM_OK) return st;
    void* scratch = nullptr;
    if (cudaMallocFromPoolAsync(&scratch, extent + off, pool, r.stream) != cudaSuccess) return GEMM_ERR_NO_MEMORY;
    void* c2 = static_cast<char*>(scratch) + off;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    auto cleanup = [&](gemm_status_t s) {
        cudaFreeAsync(scratch, r.stream);
        cudaStreamSynchronize(r.stream);
        if (e0) cudaEventDestroy(e0);
        if (e1) cudaEventDestroy(e1);
        return s;
    };
    if (r.beta != 0.0f && cudaMemcpyAsync(c2, r.C, extent, cudaMemcpyDeviceToDevice, r.stream) != cudaSuccess)
        return cleanup(GEMM_ERR_CUDA);
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return cleanup(GEMM_ERR_CUDA);
    Req rc = r;
    rc.C = c2;
    Choice best{-1, 1};
    float best_t = 0.0f;
    for (const Choice& ch : cand) {
        rc.force = &ch;
        if (run(rc, Workspace::Pool) != GEMM_OK) continue;  // warm-up (and a configuration check)
        // Three groups of back-to-back calls (enough for about 1 ms of device time each, 1 to
        // 64 calls); a group's mean is one sample, the smallest sample the candidate's time.
        if (cudaEventRecord(e0, r.stream) != cudaSuccess) return cleanup(GEMM_ERR_CUDA);
        if (run(rc, Workspace::Pool) != GEMM_OK) continue;
        if (cudaEventRecord(e1, r.stream) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess)
            return cleanup(GEMM_ERR_CUDA);
        float one = 0.0f;
        cudaEventElapsedTime(&one, e0, e1);
        int reps = one > 0.0f ? (int)(1.0f / one) : 64;
        reps = reps < 1 ? 1 : reps > 64 ? 64 : reps;
        float t = -1.0f;
        for (int g = 0; g < 3; ++g) {
            if (cudaEventRecord(e0, r.stream) != cudaSuccess) return cleanup(GEMM_ERR_CUDA);
            bool ran = true;
            for (int k = 0; k < reps && ran; ++k) ran = run(rc, Workspace::Pool) == GEMM_OK;
            if (cudaEventRecord(e1, r.stream) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess)
                return cleanup(GEMM_ERR_CUDA);
            float ms = 0.0f;
            if (!ran || cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess) {
                t = -1.0f;
                break;
            }
            if (t < 0.0f || ms / reps < t) t = ms / reps;
        }
        if (t < 0.0f) continue;
        if (best.plan < 0 || t < best_t) best = ch, best_t = t;
    }
    if (gemm_bf16_device_status(r.stream) != GEMM_OK) return cleanup(GEMM_ERR_TIMEOUT);
    if (best.plan < 0) return cleanup(GEMM_ERR_UNSUPPORTED);
    {
        std::lock_guard<std::mutex> lk(g_tune_mu);
        g_tune[key] = TuneVal{best, best_t * 1000.0f};
    }
    if (best_us) *best_us = best_t * 1000.0f;
    return cleanup(GEMM_OK);
}

}  // namespace

extern "C" {

gemm_status_t gemm_bf16(int M, int N, int K, const void* A, int lda, const void* B, int ldb, void* C,
                        int ldc, gemm_out_t out_type, float alpha, float beta, cudaStream_t stream) {
    Req r{1, M, N, K, A, lda, B, ldb, 0, false, C, ldc, 0, (int)out_type, 0, alpha, beta, stream};
    return guarded(r, Workspace::Pool);
}

gemm_status_t gemm_bf16_batched_shared_w(int batch, int M, int N, int K, const void* W, int ldw,
                                         const void* X, int ldx, long long stride_x, void* Y, int ldy,
                                         long long stride_y, gemm_out_t out_type, float alpha,
                                         float beta, cudaStream_t stream) {
    Req r{batch, M, N, K, W, ldw, X, ldx, stride_x, true, Y, ldy, stride_y, (int)out_type, 0, alpha, beta, stream};
    return guarded(r, Workspace::Pool);
}

gemm_status_t gemm_f16(int M, int N, int K, const void* A, int lda, const void* B, int ldb, void* C,
                       int ldc, gemm_out_t out_type, float alpha, float beta, cudaStream_t stream) {
    Req r{1, M, N, K, A, lda, B, ldb, 0, false, C, ldc, 0, (int)out_type, 1, alpha, beta, stream};
    return guarded(r, Workspace::Pool);
}

gemm_status_t gemm_f16_batched_shared_w(int batch, int M, int N, int K, const void* W, int ldw,
                                        const void* X, int ldx, long long stride_x, void* Y, int ldy,
                                        long long stride_y, gemm_out_t out_type, float alpha,
                                        float beta, cudaStream_t stream) {
    Req r{batch, M, N, K, W, ldw, X, ldx, stride_x, true, Y, ldy, stride_y, (int)out_type, 1, alpha, beta, stream};
    return guarded(r, Workspace::Pool);
}

gemm_status_t gemm_bf16_batched_shared_w_dedup(int batch, int n_unique, int M, int N, int K, const void* W,
                                               int ldw, const void* X, int ldx, long long stride_x,
                                               const int* index, void* Y, int ldy, long long stride_y,
                                               gemm_out_t out_type, float alpha, float beta,
                                               cudaStream_t stream) {
    if (index == nullptr && batch > 0) return GEMM_ERR_INVALID_ARG;
    Req r{batch, M, N, K, W, ldw, X, ldx, stride_x, true, Y, ldy, stride_y, (int)out_type, 0, alpha, beta, stream};
    r.index = index;
    r.n_x = n_unique;
    return guarded(r, Workspace::Pool);
}

gemm_status_t gemm_bf16_noalloc(int M, int N, int K, const void* A, int lda, const void* B, int ldb,
                                void* C, int ldc, gemm_out_t out_type, float alpha, float beta,
                                cudaStream_t stream) {
    Req r{1, M, N, K, A, lda, B, ldb, 0, false, C, ldc, 0, (int)out_type, 0, alpha, beta, stream};
    return guarded(r, Workspace::Static);
}

gemm_status_t gemm_autotune(int in_type, int form, int batch, int n_unique, int M, int N, int K, const void* A,
                            int lda, const void* B, int ldb, long long stride_b, const int* index, const void* C,
                            int ldc, long long stride_c, gemm_out_t out_type, float alpha, float beta,
                            cudaStream_t stream, float* best_us) {
    if ((in_type != 0 && in_type != 1) || form < 0 || form > 2) return GEMM_ERR_INVALID_ARG;
    if (form == 2 && (in_type != 0 || (index == nullptr && batch > 0))) return GEMM_ERR_INVALID_ARG;
    if (form == 0 && batch != 1) return GEMM_ERR_INVALID_ARG;
    Req r{batch, M, N, K, A, lda, B, ldb, form == 0 ? 0 : stride_b, form != 0, const_cast<void*>(C), ldc,
          form == 0 ? 0 : stride_c, (int)out_type, in_type, alpha, beta, stream};
    if (form == 2) {
        r.index = index;
        r.n_x = n_unique;
    }
    try {
        return autotune(r, best_us);
    } catch (...) {
        return GEMM_ERR_CUDA;
    }
}

gemm_status_t gemm_tuning_clear(void) {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    g_tune.clear();
    return GEMM_OK;
}

int gemm_tuning_size(void) {
    std::lock_guard<std::mutex> lk(g_tune_mu);
    return (int)g_tune.size();
}

// One entry per line: "gemmtune1" and the key (sms batch M N K n_x b_mn in_f16 out c_read a_ok
// b_ok c_tma), then the configuration (plan splits csplit group_m) and the measured time (us).
gemm_status_t gemm_tuning_save(const char* path) {
    if (path == nullptr) return GEMM_ERR_INVALID_ARG;
    std::FILE* f = std::fopen(path, "w");
    if (f == nullptr) return GEMM_ERR_INVALID_ARG;
    {
        std::lock_guard<std::mutex> lk(g_tune_mu);
        for (const auto& kv : g_tune) {
            const TuneKey& k = kv.first;
            const TuneVal& v = kv.second;
            std::fprintf(f, "gemmtune1 %d %d %d %d %d %d %d %d %d %d %d %d %d %d %d %d %d %.3f\n", k.sms, k.batch, k.M,
                         k.N, k.K, k.n_x, k.b_mn, k.in_f16, k.out, k.c_read, k.a_ok, k.b_ok, k.c_tma, v.ch.plan,
                         v.ch.sk ? 0 : v.ch.splits, v.ch.csplit, v.ch.group_m, (double)v.us);
        }
    }
    return std::fclose(f) == 0 ? GEMM_OK : GEMM_ERR_INVALID_ARG;
}

// Adds the file's entries to the table (replacing entries with the same key).  Every line is
// checked first; a malformed line or an impossible configuration rejects the whole file and
// leaves the table as it was.
gemm_status_t gemm_tuning_load(const char* path) {
    if (path == nullptr) return GEMM_ERR_INVALID_ARG;
    std::FILE* f = std::fopen(path, "r");
    if (f == nullptr) return GEMM_ERR_INVALID_ARG;
    std::vector<std::pair<TuneKey, TuneVal>> rows;
    char line[512];
    bool ok = true;
    while (ok && std::fgets(line, sizeof line, f) != nullptr) {
        if (line[0] == '\n' || line[0] == '#') continue;
        TuneKey k;
        std::memset(&k, 0, sizeof k);
        TuneVal v{};
        double us = 0.0;
        int consumed = 0;
        const int n = std::sscanf(line, "gemmtune1 %d %d %d %d %d %d %d %d %d %d %d %d %d %d %d %d %d %lf %n", &k.sms,
                                  &k.batch, &k.M, &k.N, &k.K, &k.n_x, &k.b_mn, &k.in_f16, &k.out, &k.c_read, &k.a_ok,
                                  &k.b_ok, &k.c_tma, &v.ch.plan, &v.ch.splits, &v.ch.csplit, &v.ch.group_m, &us,
                                  &consumed);
        v.us = (float)us;
        if (n == 18 && v.ch.splits == 0) {  // stream-K
            v.ch.splits = 1;
            v.ch.sk = 1;
        }
        const PlanDesc* pd = (v.ch.plan >= 0 && v.ch.plan < kNumPlans) ? &kPlans[v.ch.plan] : nullptr;
        ok = n == 18 && line[consumed] == '\0' && pd != nullptr && k.sms > 0 && k.batch >= 1 && k.M >= 1 &&
             k.N >= 1 && k.K >= 1 && k.n_x >= 0 && (k.b_mn | k.in_f16 | k.c_read | k.a_ok | k.b_ok | k.c_tma) >= 0 &&
             (k.b_mn | k.in_f16 | k.c_read | k.a_ok | k.b_ok | k.c_tma) <= 1 && k.out >= OUT_F32 &&
             k.out <= OUT_F16 && v.ch.splits >= 1 && v.ch.splits <= kMaxSplits &&
             (v.ch.csplit == 1 || v.ch.csplit == 2 || v.ch.csplit == 4 || v.ch.csplit == 8) &&
             !(v.ch.splits > 1 && v.ch.csplit > 1) &&
             (v.ch.csplit == 1 || (plan_csplit_ok(*pd) && v.ch.csplit <= max_csplit(*pd))) &&
             (v.ch.splits == 1 || !pd->ares) && !(v.ch.sk && (pd->ares || v.ch.csplit > 1)) && v.ch.group_m >= 1 &&
             v.ch.group_m <= 64;
        if (ok) rows.emplace_back(k, v);
    }
    std::fclose(f);
    if (!ok) return GEMM_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_tune_mu);
    for (const auto& kv : rows) g_tune[kv.first] = kv.second;
    return GEMM_OK;
}

gemm_status_t gemm_last_config(int* plan, int* splits, int* csplit, int* group_m) {
    if (!plan || !splits || !csplit || !group_m) return GEMM_ERR_INVALID_ARG;
    *plan = t_last.plan;
    *splits = t_last.sk ? 0 : t_last.splits;
    *csplit = t_last.csplit;
    *group_m = t_last.group_m;
    return GEMM_OK;
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
        return (v & ~kStatusBadIndex) != 0 ? GEMM_ERR_TIMEOUT : GEMM_ERR_INVALID_ARG;
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

gemm_status_t gemm_bf16_tensor_map_cache_stats(unsigned long long* hits, unsigned long long* misses) {
    if (hits == nullptr || misses == nullptr) return GEMM_ERR_INVALID_ARG;
    *hits = g_map_hits.load();
    *misses = g_map_misses.load();
    return GEMM_OK;
}

int gemm_bf16_version(void) { return 200; }

}  // extern "C"
