// launch.cuh -- launch of one instantiation of the persistent GEMM kernel: shared-memory
// attribute, cluster occupancy (queried once per device) and the persistent grid size.
// Each plan*.cu translation unit instantiates the launches of one tile plan, so the plans
// compile in parallel; api.cu calls them through the declarations at the end of this file.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <array>
#include <atomic>

#include "gemm_bf16.h"
#include "gemm_kernel.cuh"
#include "plans.h"

namespace pw {

constexpr int kMaxDevices = 64;

// Everything a plan's launch needs besides its template parameters.
struct LaunchArgs {
    bool b_mn;                 // B operand N-major (batched shared-W form)
    int out;                   // OUT_F32 / OUT_BF16 / OUT_F16
    const CUtensorMap* ma;     // A (or W), K-major
    const CUtensorMap* mb;     // B (K-major) or X (N-major)
    const CUtensorMap* mc;     // C, when tensor stores are possible (zeroed otherwise)
    KParams p;
    int dev, sms;
    cudaStream_t stream;
};

template <int CG, int BN, int NSUB, int STAGES, int BK, int B_MN, int OUT, int ARES>
gemm_status_t launch_persistent(const LaunchArgs& a) {
    using T = Tile<CG, BN, NSUB, STAGES, BK, B_MN, OUT, ARES>;
    auto kern = gemm_persistent<CG, BN, NSUB, STAGES, BK, B_MN, OUT, ARES>;
    static std::array<std::atomic<int>, kMaxDevices> attr_done{};
    static std::array<std::atomic<int>, kMaxDevices> max_clusters{};
    const int dev = a.dev;
    if (dev < 0 || dev >= kMaxDevices) return GEMM_ERR_CUDA;
    if (!attr_done[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::SMEM_ALLOC) !=
            cudaSuccess)
            return GEMM_ERR_CUDA;
        int clusters = a.sms / CG;
        if constexpr (CG == 2) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3(a.sms, 1, 1);
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
    // Cluster split-K: one cluster of csplit slices per tile, a slice being a CTA or a CTA pair
    // (not persistent: each CTA computes one K slice of one tile).  Otherwise a persistent grid of
    // CG-CTA clusters, at most as many as fit on the device at once.
    const bool csplit = T::CSPLIT_OK && a.p.csplit > 1;
    if (a.p.csplit > 1 && !csplit) return GEMM_ERR_UNSUPPORTED;
    const int cdim = csplit ? a.p.csplit * CG : CG;
    long long ctas;
    if (csplit) {
        ctas = (long long)a.p.tiles * cdim;
    } else if (a.p.sk_tiles > 0) {
        // stream-K: exactly the clusters its K ranges were cut for (correct even if fewer fit at
        // once: no CTA waits for another)
        if (a.p.sk_clusters <= 0) return GEMM_ERR_INVALID_ARG;
        ctas = (long long)a.p.sk_clusters * CG;
    } else {
        const int upt = a.p.splits > 1 ? a.p.splits : (a.p.dd_off != nullptr && a.p.dsplit > 1) ? a.p.dsplit : 1;
        const long long units = (long long)a.p.tiles * upt;  // work units
        const long long cap = max_clusters[dev].load();
        ctas = (units < cap ? units : cap) * CG;
    }
    if (ctas > 0x7FFFFFFFLL) return GEMM_ERR_UNSUPPORTED;
    if (csplit) {
        // A cluster size the device cannot place is refused here, once per device and size.
        static std::array<std::array<std::atomic<int>, 3>, kMaxDevices> fits{};  // 0 unknown, 1 yes, 2 no
        if (cdim != 2 && cdim != 4 && cdim != 8) return GEMM_ERR_UNSUPPORTED;
        const size_t ci = cdim == 2 ? 0 : cdim == 4 ? 1 : 2;
        if (fits[dev][ci].load() == 0) {
            cudaLaunchConfig_t q = {};
            q.gridDim = dim3((unsigned)cdim, 1, 1);
            q.blockDim = dim3(T::THREADS, 1, 1);
            q.dynamicSmemBytes = T::SMEM_ALLOC;
            cudaLaunchAttribute qa[1];
            qa[0].id = cudaLaunchAttributeClusterDimension;
            qa[0].val.clusterDim.x = (unsigned)cdim;
            qa[0].val.clusterDim.y = 1;
            qa[0].val.clusterDim.z = 1;
            q.attrs = qa;
            q.numAttrs = 1;
            int n = 0;
            fits[dev][ci].store(cudaOccupancyMaxActiveClusters(&n, kern, &q) == cudaSuccess && n > 0 ? 1 : 2);
        }
        if (fits[dev][ci].load() != 1) return GEMM_ERR_UNSUPPORTED;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    cfg.blockDim = dim3(T::THREADS, 1, 1);
    cfg.dynamicSmemBytes = T::SMEM_ALLOC;
    cfg.stream = a.stream;
    cudaLaunchAttribute attrs[1];
    if (cdim > 1) {
        attrs[0].id = cudaLaunchAttributeClusterDimension;
        attrs[0].val.clusterDim.x = (unsigned)cdim;
        attrs[0].val.clusterDim.y = 1;
        attrs[0].val.clusterDim.z = 1;
        cfg.attrs = attrs;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kern, *a.ma, *a.mb, *a.mc, a.p) == cudaSuccess ? GEMM_OK
                                                                                     : GEMM_ERR_CUDA;
}

// One plan, every operand layout and output type it serves.
template <int CG, int BN, int NSUB, int STAGES, int BK, int ARES>
gemm_status_t launch_plan(const LaunchArgs& a) {
    if (a.b_mn) {
        if constexpr ((BN / CG) % 64 == 0) {
            switch (a.out) {
                case OUT_F32: return launch_persistent<CG, BN, NSUB, STAGES, BK, 1, OUT_F32, ARES>(a);
                case OUT_BF16: return launch_persistent<CG, BN, NSUB, STAGES, BK, 1, OUT_BF16, ARES>(a);
                case OUT_F16: return launch_persistent<CG, BN, NSUB, STAGES, BK, 1, OUT_F16, ARES>(a);
                default: return GEMM_ERR_INVALID_ARG;
            }
        } else {
            return GEMM_ERR_UNSUPPORTED;
        }
    }
    switch (a.out) {
        case OUT_F32: return launch_persistent<CG, BN, NSUB, STAGES, BK, 0, OUT_F32, ARES>(a);
        case OUT_BF16: return launch_persistent<CG, BN, NSUB, STAGES, BK, 0, OUT_BF16, ARES>(a);
        case OUT_F16: return launch_persistent<CG, BN, NSUB, STAGES, BK, 0, OUT_F16, ARES>(a);
        default: return GEMM_ERR_INVALID_ARG;
    }
}

// Defined in plan<N>.cu, one per plan.
gemm_status_t launch_plan0(const LaunchArgs& a);
gemm_status_t launch_plan1(const LaunchArgs& a);
gemm_status_t launch_plan2(const LaunchArgs& a);
gemm_status_t launch_plan3(const LaunchArgs& a);
gemm_status_t launch_plan4(const LaunchArgs& a);
gemm_status_t launch_plan5(const LaunchArgs& a);
gemm_status_t launch_plan6(const LaunchArgs& a);
gemm_status_t launch_plan7(const LaunchArgs& a);
gemm_status_t launch_plan8(const LaunchArgs& a);

}  // namespace pw

// Body of plan<N>.cu.
#define PW_DEFINE_PLAN(N) \
    namespace pw { \
    gemm_status_t launch_plan##N(const LaunchArgs& a) { return launch_plan<PW_PLAN##N##_ARGS>(a); } \
    }
