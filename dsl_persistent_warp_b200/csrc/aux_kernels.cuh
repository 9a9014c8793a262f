// aux_kernels.cuh -- the two small kernels around the GEMM: the K == 0 / alpha == 0 update
// of C, and the alignment pre-pass copy that lets TMA read operands whose leading dimension or
// base it cannot address.  Included by api.cu only.
#pragma once
#include <cstdint>

#include "gemm_kernel.cuh"

namespace pw {

// C = beta * C (C = 0 when beta == 0) over batch x M x N: the K == 0 / alpha == 0 case.
// OUT is the element type of C (OUT_F32, OUT_BF16 or OUT_F16).
template <int OUT>
__global__ void scale_c_kernel(void* Cv, long long ldc, long long stride_c, int batch, int M, int N,
                               float beta) {
    const long long per = (long long)M * N;
    const long long total = per * batch;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long b = i / per;
        const long long r = (i - b * per) / N;
        const long long c = i - b * per - r * N;
        const long long off = b * stride_c + r * ldc + c;
        float x = 0.0f;
        if constexpr (OUT != OUT_F32) {
            uint16_t* e = static_cast<uint16_t*>(Cv) + off;
            if (beta != 0.0f) x = beta * dec16_lo<OUT>(*e);
            *e = (uint16_t)(pack16<OUT>(x, 0.0f) & 0xFFFFu);
        } else {
            float* e = static_cast<float*>(Cv) + off;
            if (beta != 0.0f) x = beta * *e;
            *e = x;
        }
    }
}

// Copy a batch x rows x cols array of 16-bit elements (bf16 or fp16) into a buffer whose leading dimension is a multiple
// of 8 elements and whose base is 16-byte aligned, so that TMA can read it.  Each thread writes
// 8 elements with one 16-byte store.  Interior threads read the two aligned 16-byte words that
// cover their (2-byte aligned) source window and realign them with byte permutes; threads whose
// aligned window would reach outside [src_lo, src_hi) -- the source allocation's extent -- and
// row tails use 2-byte loads.
__global__ void pad_copy_kernel(const uint16_t* __restrict__ src, long long ld_src, long long bs_src,
                                uint16_t* __restrict__ dst, long long ld_dst, long long bs_dst,
                                int batch, int rows, int cols, uintptr_t src_lo, uintptr_t src_hi) {
    const int vec_per_row = (cols + 7) >> 3;
    for (int b = blockIdx.z; b < batch; b += gridDim.z) {
        for (int r = blockIdx.y; r < rows; r += gridDim.y) {
            const uint16_t* s = src + b * bs_src + (long long)r * ld_src;
            uint16_t* d = dst + b * bs_dst + (long long)r * ld_dst;
            for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < vec_per_row;
                 v += gridDim.x * blockDim.x) {
                const int c = v << 3;
                if (c + 8 <= cols) {
                    const uintptr_t a = reinterpret_cast<uintptr_t>(s + c);
                    const uintptr_t a0 = a & ~(uintptr_t)15;
                    const uint32_t sh = (uint32_t)(a - a0);  // 0, 2, ..., 14
                    uint32_t e[4];
                    if (a0 >= src_lo && a0 + 32 <= src_hi) {
                        const uint4 lo = *reinterpret_cast<const uint4*>(a0);
                        const uint4 hi = sh ? *reinterpret_cast<const uint4*>(a0 + 16) : lo;
                        // y[j] = word (sh/4 + j) of the 32-byte window, selected without indexing
                        const uint32_t wo = sh >> 2;
                        const uint32_t y0 = wo == 0 ? lo.x : wo == 1 ? lo.y : wo == 2 ? lo.z : lo.w;
                        const uint32_t y1 = wo == 0 ? lo.y : wo == 1 ? lo.z : wo == 2 ? lo.w : hi.x;
                        const uint32_t y2 = wo == 0 ? lo.z : wo == 1 ? lo.w : wo == 2 ? hi.x : hi.y;
                        const uint32_t y3 = wo == 0 ? lo.w : wo == 1 ? hi.x : wo == 2 ? hi.y : hi.z;
                        const uint32_t y4 = wo == 0 ? hi.x : wo == 1 ? hi.y : wo == 2 ? hi.z : hi.w;
                        const uint32_t sel = (sh & 2) ? 0x5432u : 0x3210u;  // half-word shift or none
                        e[0] = __byte_perm(y0, y1, sel);
                        e[1] = __byte_perm(y1, y2, sel);
                        e[2] = __byte_perm(y2, y3, sel);
                        e[3] = __byte_perm(y3, y4, sel);
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            e[j] = (uint32_t)s[c + 2 * j] | ((uint32_t)s[c + 2 * j + 1] << 16);
                    }
                    *reinterpret_cast<uint4*>(d + c) = make_uint4(e[0], e[1], e[2], e[3]);
                } else {
                    for (int j = c; j < cols; ++j) d[j] = s[j];
                }
            }
        }
    }
}

// Group the items of a deduplicated batch by their distinct entry: after it, items
// dst[off[e] .. off[e+1]) are those b with index[b] == e (in no particular order; each item is
// listed once).  One CTA of up to 1024 threads: count per entry, exclusive scan, placement.
// `cursor` is n ints of scratch.  An index outside [0, n) is not listed (that item's output is
// left untouched) and sets `bad_bit` in *status.
__global__ void dedup_groups_kernel(const int* __restrict__ index, int batch, int n, int* __restrict__ off,
                                    int* __restrict__ cursor, int* __restrict__ dst, unsigned int* status,
                                    unsigned int bad_bit) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int lane = tid & 31, wid = tid >> 5, nw = (nt + 31) >> 5;
    for (int e = tid; e < n; e += nt) cursor[e] = 0;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int b = tid; b < batch; b += nt) {
        const int e = index[b];
        if (e >= 0 && e < n) atomicAdd(&cursor[e], 1);
        else atomicOr(status, bad_bit);
    }
    __syncthreads();
    // exclusive scan of the counts, nt entries at a time
    for (int base = 0; base < n; base += nt) {
        const int e = base + tid;
        const int c = e < n ? cursor[e] : 0;
        int x = c;  // inclusive scan within the warp
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, d);
            if (lane >= d) x += y;
        }
        if (lane == 31) warp_tot[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, d);
                if (lane >= d) t += y;
            }
            if (lane < nw) warp_tot[lane] = t;  // inclusive totals of warps 0..lane
        }
        __syncthreads();
        const int before = carry + (wid > 0 ? warp_tot[wid - 1] : 0);
        if (e < n) off[e] = before + x - c;
        __syncthreads();
        if (tid == 0) carry += warp_tot[nw - 1];
        __syncthreads();
    }
    if (tid == 0) off[n] = carry;
    for (int e = tid; e < n; e += nt) cursor[e] = off[e];
    __syncthreads();
    for (int b = tid; b < batch; b += nt) {
        const int e = index[b];
        if (e >= 0 && e < n) dst[atomicAdd(&cursor[e], 1)] = b;
    }
}

}  // namespace pw
