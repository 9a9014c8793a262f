// gemm_kernel.cuh -- the persistent, warp-specialized BF16 GEMM for sm_100a.
//
// Computes C = alpha * A * B + beta * C (bf16 in, fp32 accumulate) over a grid of output
// tiles, following the producer/consumer structure described for TLX on the page
// "Meta presente TLX pour combler le fosse entre la complexite du materiel GPU et la
// productivite des developpeurs", section "Comment cela fonctionne": one warp loads tiles
// asynchronously through TMA while another drives the tensor cores, and lightweight
// barriers (mbarriers) hand each stage over, giving a deep pipeline that overlaps data
// movement and math.  The multi-stage shared-memory ring and the K loop over staged tiles
// correspond to the Hopper sketch on the page "Triton 3.7 permite extender el compilador de
// GPU sin forks", section "NVIDIA H100 (Hopper): GEMM persistente" (NUM_STAGES buffers,
// prefetch ahead, accumulate, store); the grouped tile order is its GROUP_SIZE_M parameter.
//
// Blackwell design (not from the pages):
//   * warp 0, one lane      : TMA producer.  Waits empty[s], arms full[s] with the stage's
//                             byte count, issues the A and B tile loads (no multicast).
//   * warp 1, one lane      : MMA issuer (leader CTA only).  Waits full[s], issues
//                             tcgen05.mma (K=16 per instruction) into a TMEM accumulator,
//                             commits empty[s]; after the last k-block commits tmem_full.
//   * warps 2..5            : epilogue.  Wait tmem_full, tcgen05.ld 32 rows x 32 columns per
//                             warp, release the accumulator (tmem_empty), apply alpha/beta,
//                             convert, stage through swizzled shared memory and TMA-store.
//   * two TMEM accumulators : the epilogue of tile i overlaps the mainloop of tile i+1.
//   * CG = 2                : a 2-CTA cluster computes a 256-row tile with
//                             tcgen05.mma.cta_group::2; each CTA loads its 128 rows of A and
//                             half of the tile's B columns; loads of both CTAs complete on the
//                             leader's full barrier, commits go to both CTAs' barriers.
//   * every barrier wait is bounded (global timer); on expiry the kernel records a status
//     bit, raises an abort flag, lets in-flight copies land, frees TMEM and returns.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx_sm100.cuh"

#ifndef PW_OPERAND_L2_POLICY
#define PW_OPERAND_L2_POLICY 1
#endif
#ifndef PW_B_L2_POLICY
#define PW_B_L2_POLICY PW_OPERAND_L2_POLICY
#endif
// Tiles of two MMA sub-tiles (both TMEM accumulator slots) with 16-bit output use 8 epilogue
// warps, two per TMEM lane quarter, which drain both slots before storing when C is not read
// (1), or 4 warps that store chunk by chunk (0).
#ifndef PW_EPI8_NSUB2
#define PW_EPI8_NSUB2 1
#endif
// Resident-A plans (short mainloops, so the epilogue sets the pace) use 8 epilogue warps, two per
// TMEM lane quarter, each storing half of the columns (1), or 4 (0).  B200, RecSys 2048 x
// (256x512 . 512x128): 94.3 -> 85.6 us; 512 distinct entries x 4 items, dedup: 59.8 -> 54.3 us.
#ifndef PW_EPI8_ARES
#define PW_EPI8_ARES 1
#endif
// The same for the other 2-CTA plans whose CTA holds at least two epilogue chunks per slot (1),
// or 4 warps (0).  B200: 4099^3 (beta = 1, row-by-row epilogue) 174.4 -> 168.3 us, 2048^2 x 8192
// 61.4 -> 60.4 us; on the one-CTA plans it was neutral or slower (1024^2 x 8192 cut over a
// cluster of 4: 31.7 -> 32.8 us).
#ifndef PW_EPI8_PAIR
#define PW_EPI8_PAIR 1
#endif

namespace pw {

enum : int { OUT_F32 = 0, OUT_BF16 = 1, OUT_F16 = 2 };

// 16-bit output element <-> fp32.  Packed words hold element 2j in bits 0..15 and element
// 2j+1 in bits 16..31; both conversions to 16 bits round to nearest even once.
template <int OUT>
__device__ __forceinline__ float dec16_lo(uint32_t w) {
    if constexpr (OUT == OUT_BF16) return __uint_as_float(w << 16);
    else return f16_to_f32((uint16_t)(w & 0xFFFFu));
}
template <int OUT>
__device__ __forceinline__ float dec16_hi(uint32_t w) {
    if constexpr (OUT == OUT_BF16) return __uint_as_float(w & 0xFFFF0000u);
    else return f16_to_f32((uint16_t)(w >> 16));
}
template <int OUT>
__device__ __forceinline__ uint32_t pack16(float lo, float hi) {
    if constexpr (OUT == OUT_BF16) return pack_bf16x2(lo, hi);
    else return pack_f16x2(lo, hi);
}

enum : unsigned int {
    kStatusProducer = 1u,
    kStatusMma = 2u,
    kStatusEpilogue = 4u,
};

struct KParams {
    int M, N, K;
    int m_blocks, n_blocks;  // cluster tiles along M and N
    int batch;
    int tiles;               // batch * m_blocks * n_blocks
    int k_blocks;            // ceil(K / 64)
    int group_m;             // grouped raster: m-blocks per group
    float alpha, beta;
    void* C;                 // output base (also the beta input)
    long long ldc;           // elements
    long long stride_c;      // elements between batches of C
    int c_tma;               // 1: epilogue uses TMA stores (aligned C), 0: direct stores
    int n_store_tma;         // columns [0, n_store_tma) may be TMA-stored; a chunk reaching past
                             // it (a row end that is not 16-byte aligned) is stored directly,
                             // because a tensor store writes whole 16-byte granules
    int c_read;              // 1: beta != 0
    int pack;                // batch entries side by side in one tile (MN-major B; 1 = none):
                             // tile column c belongs to entry nb*pack + c/N, column c%N
    int batch_real;          // number of batch entries (p.batch counts tile batches)
    int splits;              // K slices per tile (split-K; <= 1: none).  Work unit u covers tile
                             // u / splits and k-blocks [s*kb_per_split, (s+1)*kb_per_split), s = u % splits
    int kb_per_split;        // k-blocks per slice (global or cluster split-K)
    int csplit;              // cluster split-K: K slices per tile, computed by the csplit CTAs (CTA
                             // pairs) of one thread-block cluster, one slice each; the partial
                             // sums are added through distributed shared memory (<= 1: none)
    int sk_tiles;            // stream-K: tiles [0, sk_tiles) are computed as K ranges spread evenly
                             // over sk_clusters clusters (0: none), the rest whole
    int sk_clusters;         // stream-K: clusters of the grid (the launch has exactly this many)
    float* ws;               // split-K partials: per (tile, CTA rank, part) the CTA's 128 rows x
                             // TILE_N columns in fp32, as 4 KiB pieces per epilogue warp
    int ws_parts;            // partial slots per (tile, CTA rank): splits, or stream-K's most
                             // K ranges of one tile
    unsigned int* counters;  // split-K arrivals per (tile, CTA rank, epilogue warp); zero on entry,
                             // and the last arrival puts it back to zero
    // Deduplicated batches (shared-W form): the tiles cover the batch_real distinct X entries;
    // the result of entry e goes to the items dd_dst[dd_off[e] .. dd_off[e+1]) of the output
    // (Y has `batch_out` entries).  Each tile is computed by `dsplit` work units, unit part k
    // storing destinations k, k + dsplit, ... of each entry (nullptr: no deduplication).
    const int* dd_off;
    const int* dd_dst;
    int dsplit;
    int batch_out;
    unsigned int* status;    // device status word: bit i set = a bounded wait of role i expired
    int in_f16;              // 1: A and B hold fp16 values, 0: bf16
    int test_stall;          // test hook: the producer issues nothing, so the first bounded
                             // wait of the MMA thread expires (failure-detection tests)
    unsigned long long timeout_ns;
};

// CG: CTAs per cluster tile (1, or 2 computing together with cta_group::2).  BN: N of one MMA,
// i.e. the columns of one TMEM accumulator slot.  NSUB: MMA sub-tiles along N per tile (tile N =
// BN * NSUB).  There are two accumulator slots: with NSUB == 1 they alternate between tiles (the
// epilogue of a tile overlaps the next tile's mainloop); with NSUB == 2 a tile owns both, the
// epilogue drains slot 0 while the last sub-tile 1 MMAs run, and the next tile starts in slot 0
// as soon as it is drained.
// ARES: the A operand is resident -- the whole M x K panel of A (one M tile, K <= KB_RES * BK) is
// loaded into shared memory once per CTA and the ring streams only B.  This is the shared-W
// form: W is read from HBM once per CTA and never per batch entry.
template <int CG, int BN, int NSUB, int STAGES, int BK_, int B_MN, int OUT, int ARES = 0>
struct Tile {
    static constexpr int BK = BK_;                  // K per stage: 64 (128-B rows) or 32 (64-B rows)
    static constexpr int BM = 128 * CG;             // rows of the cluster tile (MMA M)
    static constexpr int TILE_N = BN * NSUB;        // columns of the cluster tile
    static constexpr int BN_CTA = BN / CG;          // B rows (N) of one sub-tile held per CTA
    static constexpr int B_CHUNK = NSUB * BN_CTA;   // contiguous B rows (tile columns) per CTA
    static constexpr int A_BYTES = 128 * BK * 2;
    static constexpr int B_SUB_BYTES = BN_CTA * BK * 2;
    static constexpr int B_BYTES = NSUB * B_SUB_BYTES;
    static constexpr int KB_RES = 8;                // resident k-blocks (K <= 512 at BK = 64)
    static constexpr int STAGE_BYTES = (ARES ? 0 : A_BYTES) + B_BYTES;
    // Epilogue: 4 warps, one per TMEM lane quarter, each with two 4 KiB staging buffers (the TMA
    // store of one chunk overlaps the next chunk's TMEM load and conversion); for two sub-tiles
    // and 16-bit output, 8 warps (two per quarter, each half of the columns, one buffer each),
    // which drain the tile's accumulators into registers before storing so that the next tile's
    // MMAs start sooner (B200, 8192^3: the MMAs' wait between tiles 7.3 -> 4.0 us, 2-3 % faster);
    // for resident A and the other wide 2-CTA tiles, 8 warps storing chunk by chunk (twice the
    // stores in flight).
    static constexpr int EPI_WARPS = ((NSUB == 2 && OUT != OUT_F32 && PW_EPI8_NSUB2) || (ARES && PW_EPI8_ARES) ||
                                      (CG == 2 && PW_EPI8_PAIR && BN / CG >= 2 * (OUT == OUT_F32 ? 32 : 64)))
                                         ? 8 : 4;
    static constexpr int EPI_HALVES = EPI_WARPS / 4;          // warps sharing a lane quarter
    static constexpr int STG_BUFS = 8 / EPI_WARPS;            // staging buffers per warp
    static constexpr int THREADS = 32 * (2 + EPI_WARPS);
    static constexpr int STG_COLS = OUT == OUT_F32 ? 32 : 64;  // 128-byte rows
    static constexpr int STG_BYTES = 32 * 128;
    static constexpr int CHUNKS = BN / STG_COLS;                // per accumulator slot
    static constexpr int TMEM_COLS = 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128
                                   : 2 * BN <= 256 ? 256 : 512;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + (ARES ? KB_RES : STAGES) * A_BYTES;
    static constexpr int OFF_STG = OFF_B + STAGES * B_BYTES;
    static constexpr int STG_REGION = EPI_WARPS * STG_BUFS * STG_BYTES;
    static constexpr int OFF_BAR = OFF_STG + STG_REGION;
    static constexpr int NUM_BARS = 2 * STAGES + 5;  // full/empty ring, tfull/tempty slots, resident A
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // slack to align the base to 1 KiB
    static_assert(BN % (16 * CG) == 0 && BN <= 256, "MMA N");
    static_assert(NSUB == 1 || NSUB == 2, "one or two sub-tiles");
    static_assert(!B_MN || BN_CTA % 64 == 0, "MN-major B is loaded in 64-column boxes");
    static_assert(B_CHUNK <= 256, "one tensor-map box per CTA and stage");
    static_assert(BN_CTA % STG_COLS == 0, "an epilogue chunk maps to contiguous output columns");
    static_assert(BN % (STG_COLS * EPI_HALVES) == 0, "epilogue chunks split evenly between warps");
    // K-major operands: one row of a stage is BK*2 bytes, swizzled at that width.
    static constexpr uint32_t KMAJ_SWIZZLE = BK == 64 ? 2u : 4u;  // descriptor swizzle mode
    static constexpr uint32_t KMAJ_SBO = 8u * BK * 2u;            // bytes between 8-row groups
    // MN-major B: 64-column boxes of BK rows (128-byte rows, 128-byte swizzle).
    static constexpr int MN_BOX_BYTES = 64 * 2 * BK;
    static_assert(BK == 64 || BK == 32, "stage K");
    static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
    // Cluster split-K: after its K slice, a CTA's ring is idle and holds its 128 x BN fp32
    // partial tile (its rows of the tile, every column) for the other slices' CTAs to read.
    static constexpr int XCHG_BYTES = 128 * BN * 4;
    static constexpr bool CSPLIT_OK = NSUB == 1 && ARES == 0 && XCHG_BYTES <= STAGES * STAGE_BYTES;
    static_assert(ARES == 0 || BK == 64, "resident A uses K=64 blocks");
};

// Tile t -> (batch, m-block, n-block); m-blocks are walked in groups of group_m so that
// the CTAs resident at one time share A and B panels in L2.
__device__ __forceinline__ void decode_tile(const KParams& p, int t, int& b, int& mb, int& nb) {
    const int per_batch = p.m_blocks * p.n_blocks;
    b = t / per_batch;
    const int r = t - b * per_batch;
    const int group_size = p.group_m * p.n_blocks;
    const int g = r / group_size;
    const int first_m = g * p.group_m;
    const int gm = min(p.m_blocks - first_m, p.group_m);
    const int w = r - g * group_size;
    mb = first_m + w % gm;
    nb = w / gm;
}

// `ctarank` is the CTA's rank in its cluster; with CG == 2 its pair partner is ctarank ^ 1.
template <int CG>
__device__ __forceinline__ void raise_abort(uint32_t slot_abort, uint32_t ctarank, unsigned int* status,
                                            unsigned int code) {
    atomicOr(status, code);
    st_shared_volatile_u32(slot_abort, 1u);
    if constexpr (CG == 2) st_cluster_u32(map_to_rank(slot_abort, ctarank ^ 1u), 1u);
}

// Slow path of wait_phase: poll with the global-timer bound.
template <int CG, bool CLUSTER_SCOPE>
__device__ __noinline__ bool wait_phase_slow(uint32_t bar, uint32_t parity, uint32_t slot_abort,
                                             uint32_t ctarank, unsigned int* status,
                                             unsigned long long timeout_ns, unsigned int code) {
    const uint64_t t0 = global_timer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (CLUSTER_SCOPE ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity))
                return true;
        if (ld_shared_volatile_u32(slot_abort) != 0u) return false;
        if (global_timer_ns() - t0 > timeout_ns) {
            raise_abort<CG>(slot_abort, ctarank, status, code);
            return false;
        }
    }
}

// Bounded wait on an mbarrier phase.  Returns false when the kernel is aborting (this wait
// expired, or another role raised the abort flag).  The first probe is inline: on the
// critical path (a stage that is already full or free) it costs one instruction.
template <int CG, bool CLUSTER_SCOPE>
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, uint32_t slot_abort,
                                           uint32_t ctarank, unsigned int* status,
                                           unsigned long long timeout_ns, unsigned int code) {
    if (CLUSTER_SCOPE ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    return wait_phase_slow<CG, CLUSTER_SCOPE>(bar, parity, slot_abort, ctarank, status, timeout_ns, code);
}

template <int CG, int BN, int NSUB, int STAGES, int BK, int B_MN, int OUT, int ARES>
__global__ void __launch_bounds__(Tile<CG, BN, NSUB, STAGES, BK, B_MN, OUT, ARES>::THREADS, 1)
    gemm_persistent(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const KParams p) {
    using T = Tile<CG, BN, NSUB, STAGES, BK, B_MN, OUT, ARES>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw);

    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31u;
    // Cluster split-K: the grid holds one cluster of CS K slices per tile, each slice a CTA (CG ==
    // 1) or a CTA pair (CG == 2; pairs are cluster ranks 2j, 2j+1), slice crank computing k-blocks
    // [crank*kb_per_split, ...).  Otherwise a persistent grid of CG-CTA clusters.
    const int CS = (T::CSPLIT_OK && p.csplit > 1) ? p.csplit : 1;
    const uint32_t ctarank = (CG == 2 || CS > 1) ? cluster_ctarank() : 0u;
    const uint32_t rank = CG == 2 ? (ctarank & 1u) : 0u;     // rank in the CTA pair
    const uint32_t pair0 = CG == 2 ? (ctarank & ~1u) : 0u;   // cluster rank of the pair's leader
    const uint32_t crank = CS > 1 ? ctarank / CG : 0u;       // K slice (cluster split-K)
    const int cluster_id = (int)(blockIdx.x / (CG * CS));
    const int num_clusters = (int)(gridDim.x / (CG * CS));
    // K blocks of work unit u (global split-K: unit = (tile, slice); cluster split-K: this CTA's
    // slice of the tile; else all of K).
    const int SG = (ARES == 0 && p.splits > 1) ? p.splits : 1;
    // Work units per tile: global split-K slices, or the deduplicated form's destination parts.
    const int DS = (p.dd_off != nullptr && p.dsplit > 1) ? p.dsplit : 1;
    const int UPT = SG > 1 ? SG : DS;
    // Stream-K: the k-blocks of tiles [0, sk_tiles) form one sequence of sk_tiles * k_blocks
    // iterations, cut into sk_clusters contiguous ranges of equal length (the first `extra` one
    // longer); a tile crossed by several ranges is computed in parts, one per range, and added up
    // by the split-K fixup.  Each cluster runs its range's parts first, then whole tiles
    // sk_tiles + cluster_id, + num_clusters, ...  (This is the persistent tile walk with its last,
    // partial wave spread over every cluster.)
    const int SK = (ARES == 0 && CS == 1 && SG == 1 && DS == 1 && p.sk_tiles > 0) ? 1 : 0;
    const long long sk_total = (long long)p.sk_tiles * p.k_blocks;
    const long long sk_base = SK ? sk_total / p.sk_clusters : 0;
    const long long sk_extra = SK ? sk_total % p.sk_clusters : 0;
    auto sk_start = [&](long long c) { return c * sk_base + (c < sk_extra ? c : sk_extra); };
    auto sk_owner = [&](long long i) {  // the range holding iteration i
        const long long edge = sk_extra * (sk_base + 1);
        return i < edge ? i / (sk_base + 1) : sk_extra + (i - edge) / (sk_base > 0 ? sk_base : 1);
    };
    const long long sk_lo = SK ? sk_start(cluster_id) : 0, sk_hi = SK ? sk_start(cluster_id + 1) : 0;
    const int sk_t0 = (int)(sk_lo / (SK ? p.k_blocks : 1));
    const int sk_units = (SK && sk_hi > sk_lo) ? (int)((sk_hi - 1) / p.k_blocks) - sk_t0 + 1 : 0;
    // Work unit i of this cluster: tile t, k-blocks [kb_lo, kb_hi), part `part` of `parts` whose
    // partial sums the split-K fixup adds (parts == 1: the whole tile; deduplicated batches: part
    // is the destination part and parts 1).  False past the last unit.
    auto get_unit = [&](int i, int& t, int& kb_lo, int& kb_hi, int& part, int& parts) -> bool {
        if (SK) {
            if (i < sk_units) {
                t = sk_t0 + i;
                const long long ts = (long long)t * p.k_blocks, te = ts + p.k_blocks;
                kb_lo = (int)((sk_lo > ts ? sk_lo : ts) - ts);
                kb_hi = (int)((sk_hi < te ? sk_hi : te) - ts);
                const long long first = sk_owner(ts);
                part = (int)(cluster_id - first);
                parts = (int)(sk_owner(te - 1) - first) + 1;
                return true;
            }
            t = p.sk_tiles + cluster_id + (i - sk_units) * num_clusters;
            kb_lo = 0;
            kb_hi = p.k_blocks;
            part = 0;
            parts = 1;
            return t < p.tiles;
        }
        const int u = cluster_id + i * num_clusters;
        t = u / UPT;
        const int sl = u % UPT;
        kb_lo = (SG > 1 || CS > 1) ? (SG > 1 ? sl : (int)crank) * p.kb_per_split : 0;
        kb_hi = (SG > 1 || CS > 1) ? min(p.k_blocks, kb_lo + p.kb_per_split) : p.k_blocks;
        part = sl;
        parts = SG;
        return u < p.tiles * UPT;
    };

    const uint32_t bar0 = sbase + T::OFF_BAR;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto bar_tfull = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto bar_tempty = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
    const uint32_t bar_ares = bar0 + 8u * (2 * STAGES + 4);  // resident A landed
    const uint32_t slot_tmem = sbase + T::OFF_MISC;
    const uint32_t slot_abort = sbase + T::OFF_MISC + 4;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar_tfull(a), 1);
            mbar_init(bar_tempty(a), T::EPI_WARPS * CG);
        }
        mbar_init(bar_ares, 1);
        st_shared_volatile_u32(slot_abort, 0u);
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (p.c_tma) tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc<CG>(slot_tmem, T::TMEM_COLS);
        tmem_relinquish<CG>();
    }
    tc_fence_before();
    if constexpr (CG == 2) cluster_sync(); else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + T::OFF_MISC);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint32_t full_leader0 = CG == 2 ? map_to_rank(bar_full(0), pair0) : bar_full(0);
            // A and B panels are read by several CTAs of a wave: keep them in L2 (build options
            // PW_OPERAND_L2_POLICY for A and PW_B_L2_POLICY for B: 0 evict-normal, 1 evict-last,
            // 2 evict-first).
            auto policy = [](int k) {
                return k == 0 ? l2_policy_evict_normal() : k == 2 ? l2_policy_evict_first() : l2_policy_evict_last();
            };
            const uint64_t pol = policy(PW_OPERAND_L2_POLICY);
            const uint64_t pol_b = policy(PW_B_L2_POLICY);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = p.test_stall == 0;
            if (ARES != 0 && ok) {
                // This CTA's 128 rows of the single M tile, every k-block, once.
                if (rank == 0) mbar_arrive_expect_tx(bar_ares, (uint32_t)(T::A_BYTES * CG * p.k_blocks));
                const uint32_t ares_bar = CG == 2 ? map_to_rank(bar_ares, pair0) : bar_ares;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    const uint32_t sa = sbase + T::OFF_A + kb * T::A_BYTES;
                    if constexpr (CG == 1) tma_load_3d(sa, &tmA, ares_bar, kb * T::BK, (int)rank * 128, 0, pol);
                    else tma_load_3d_pair(sa, &tmA, ares_bar, kb * T::BK, (int)rank * 128, 0, pol);
                }
            }
            int t, kb_lo, kb_hi, part, parts;
            for (int i = 0; ok && get_unit(i, t, kb_lo, kb_hi, part, parts); ++i) {
                int b, mb, nb;
                decode_tile(p, t, b, mb, nb);
                const int a_row = mb * T::BM + (int)rank * 128;
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!wait_phase<CG, false>(bar_empty(stage), phase ^ 1u, slot_abort, ctarank,
                                               p.status, p.timeout_ns, kStatusProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_local = bar_full(stage);
                    if (rank == 0) mbar_arrive_expect_tx(full_local, T::STAGE_BYTES * CG);
                    const uint32_t full_bar = full_leader0 + 8u * stage;
                    const uint32_t sa = sbase + T::OFF_A + stage * T::A_BYTES;
                    const uint32_t sb = sbase + T::OFF_B + stage * T::B_BYTES;
                    const int k0 = kb * T::BK;
                    if constexpr (ARES == 0) {
                        if constexpr (CG == 1) tma_load_3d(sa, &tmA, full_bar, k0, a_row, 0, pol);
                        else tma_load_3d_pair(sa, &tmA, full_bar, k0, a_row, 0, pol);
                    }
                    // This CTA's B chunk: tile columns [rank*B_CHUNK, +B_CHUNK), contiguous.
                    const int b_row = nb * T::TILE_N + (int)rank * T::B_CHUNK;
                    if constexpr (!B_MN) {
                        if constexpr (CG == 1) tma_load_3d(sb, &tmB, full_bar, k0, b_row, b, pol_b);
                        else tma_load_3d_pair(sb, &tmB, full_bar, k0, b_row, b, pol_b);
                    } else {
#pragma unroll
                        for (int j = 0; j < T::B_CHUNK / 64; ++j) {
                            // 64-column box j; with packing it lies inside one batch entry (N % 64 == 0)
                            const int tc = (int)rank * T::B_CHUNK + 64 * j;
                            const int bx = p.pack > 1 ? nb * p.pack + tc / p.N : b;
                            const int cx = p.pack > 1 ? tc % p.N : b_row + 64 * j;
                            if constexpr (CG == 1)
                                tma_load_3d(sb + j * T::MN_BOX_BYTES, &tmB, full_bar, cx, k0, bx, pol_b);
                            else
                                tma_load_3d_pair(sb + j * T::MN_BOX_BYTES, &tmB, full_bar, cx, k0, bx, pol_b);
                        }
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && rank == 0) {
            const uint32_t IDESC = idesc_f16_kind(T::BM, BN, 0, B_MN, p.in_f16);
            // Descriptors of stage 0 (K step 0); other stages and K steps only add to the
            // start-address field, which never carries out of its 14 bits (smem < 256 KiB).
            const uint64_t adesc0 = smem_desc(sbase + T::OFF_A, 16, T::KMAJ_SBO, T::KMAJ_SWIZZLE);
            const uint64_t bdesc0 = B_MN ? smem_desc(sbase + T::OFF_B, T::MN_BOX_BYTES, 1024, 2u)
                                         : smem_desc(sbase + T::OFF_B, 16, T::KMAJ_SBO, T::KMAJ_SWIZZLE);
            const uint32_t empty_r0 = CG == 2 ? map_to_rank(bar_empty(0), pair0) : bar_empty(0);
            const uint32_t empty_r1 = CG == 2 ? map_to_rank(bar_empty(0), pair0 + 1u) : bar_empty(0);
            const uint32_t tfull_r0 = CG == 2 ? map_to_rank(bar_tfull(0), pair0) : bar_tfull(0);
            const uint32_t tfull_r1 = CG == 2 ? map_to_rank(bar_tfull(0), pair0 + 1u) : bar_tfull(0);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t tph = 0u;  // bit i: phase of accumulator slot i's next use
            int acc = 0;                 // slot of the tile when NSUB == 1
            bool ok = true;
            if constexpr (ARES != 0) {
                ok = wait_phase<CG, false>(bar_ares, 0u, slot_abort, ctarank, p.status, p.timeout_ns, kStatusMma);
                tc_fence_after();
            }
            auto commit_tfull = [&](int slot) {
                // accumulator of this slot complete: hand it to the epilogue
                if constexpr (CG == 1) {
                    umma_commit<1>(bar_tfull(slot));
                } else {
                    umma_commit<2>(tfull_r0 + 8u * slot);
                    umma_commit<2>(tfull_r1 + 8u * slot);
                }
            };
            auto commit_empty = [&](int st) {
                if constexpr (CG == 1) {
                    umma_commit<1>(bar_empty(st));
                } else {
                    umma_commit<2>(empty_r0 + 8u * st);
                    umma_commit<2>(empty_r1 + 8u * st);
                }
            };
            int t, kb_lo, kb_hi, part, parts;
            for (int i = 0; ok && get_unit(i, t, kb_lo, kb_hi, part, parts); ++i) {
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
                    if (!wait_phase<CG, false>(bar_full(stage), phase, slot_abort, ctarank, p.status, p.timeout_ns,
                                               kStatusMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // descriptor start-address fields advance in 16-byte units
                    const uint64_t a_st = adesc0 + (uint64_t)(((ARES ? kb : stage) * T::A_BYTES) >> 4);
                    const uint64_t b_st = bdesc0 + (uint64_t)((stage * T::B_BYTES) >> 4);
#pragma unroll
                    for (int sub = 0; sub < NSUB; ++sub) {
                        const int slot = NSUB == 1 ? acc : sub;
                        if (kb == kb_lo) {
                            // the slot must have been drained by the epilogue of its last use
                            if (!wait_phase<CG, CG == 2>(bar_tempty(slot), ((tph >> slot) & 1u) ^ 1u, slot_abort, ctarank,
                                                         p.status, p.timeout_ns, kStatusMma)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        const uint32_t d_tmem = tmem_base + (uint32_t)(slot * BN);
                        const uint64_t b_sub = b_st + (uint64_t)((sub * T::B_SUB_BYTES) >> 4);
#pragma unroll
                        for (int kk = 0; kk < T::BK / 16; ++kk) {
                            // K=16 step: 32 bytes along a K-major row; 16 rows (2 KiB) of an MN-major box
                            const uint64_t adesc = a_st + (uint64_t)((kk * 32) >> 4);
                            const uint64_t bdesc = b_sub + (uint64_t)((B_MN ? kk * 2048 : kk * 32) >> 4);
                            umma_f16<CG>(d_tmem, adesc, bdesc, IDESC, (kb != kb_lo || kk != 0) ? 1u : 0u);
                        }
                        if (kb == kb_hi - 1) commit_tfull(slot);
                    }
                    if (!ok) break;
                    commit_empty(stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (NSUB == 1) {
                    tph ^= 1u << acc;
                    acc ^= 1;
                } else {
                    tph ^= 3u;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = (int)warp - 2;                 // 0..EPI_WARPS-1
        const int q = (int)(warp & 3u);               // TMEM lane quarter this warp may access
        const int half = ew / 4;                      // which part of the slot's columns
        constexpr int CPW = T::CHUNKS / T::EPI_HALVES;  // chunks per warp and slot
        const uint32_t stg = sbase + T::OFF_STG + ew * T::STG_BUFS * T::STG_BYTES;
        const uint32_t tempty_leader0 = CG == 2 ? map_to_rank(bar_tempty(0), pair0) : bar_tempty(0);
        uint32_t tph = 0u;
        int acc = 0;
        int buf = 0;
        bool ok = true;
        // alpha/beta, conversion and store of chunk c (STG_COLS columns) of sub-tile `sub` of the
        // tile (b, nb) for the 32-row slab starting at row0; v holds this lane's row.
        // batch entry of chunk c of sub-tile `sub` of tile (b, nb) (several per tile when packed)
        auto chunk_entry = [&](int b, int nb, int sub, int c) {
            const int jc = c * T::STG_COLS;
            const int tcol = sub * T::BN_CTA + (jc / T::BN_CTA) * T::B_CHUNK + jc % T::BN_CTA;
            return p.pack > 1 ? nb * p.pack + tcol / p.N : b;
        };
        // Does chunk c leave through one tensor store?  Yes when C is TMA-addressable up to the
        // chunk's end (a ragged right edge or unaligned ldc takes the row-by-row path).
        auto chunk_tma = [&](int b, int nb, int sub, int c) {
            const int jc = c * T::STG_COLS;
            const int tcol = sub * T::BN_CTA + (jc / T::BN_CTA) * T::B_CHUNK + jc % T::BN_CTA;
            const int colc = p.pack > 1 ? tcol % p.N : nb * T::TILE_N + tcol;
            return p.c_tma && colc + T::STG_COLS <= p.n_store_tma && chunk_entry(b, nb, sub, c) < p.batch_real;
        };
        // bout >= 0: store to output entry bout instead of the chunk's own batch entry (the
        // deduplicated form's scatter; C_in is read from the same entry).  more != nullptr: the
        // chunk also goes to entries more[0], more[step], ... (n_more of them); when it leaves
        // through a tensor store and C is not read, those are extra tensor stores of the same
        // staged chunk and the call returns true, else it returns false and stores only bout.
        // `packed`: the chunk already scaled and rounded (C not read); v is then not used.
        auto finish_chunk = [&](int b, int nb, int row0, int row, int sub, int c, float (&v)[T::STG_COLS],
                                int bout = -1, const int* more = nullptr, int n_more = 0, int step = 1,
                                const uint32_t* packed = nullptr) -> bool {
            bool fanned = false;
            const int col_tile = sub * T::BN_CTA;  // column within the tile
            const int jc = c * T::STG_COLS;
            const int tcol = col_tile + (jc / T::BN_CTA) * T::B_CHUNK + jc % T::BN_CTA;
            const int bsrc = p.pack > 1 ? nb * p.pack + tcol / p.N : b;
            // a chunk beyond the last entry stores nothing; otherwise bb is the output entry
            const bool entry_in = bsrc < p.batch_real;
            const int bb = !entry_in ? p.batch_real : bout >= 0 ? bout : bsrc;
            const int colc = p.pack > 1 ? tcol % p.N : nb * T::TILE_N + tcol;
            const long long cbase = (long long)bb * p.stride_c + (long long)row * p.ldc;
            const bool row_in = row < p.M && entry_in;
            const bool full_cols = colc + T::STG_COLS <= p.N;
            // A chunk goes out as one tensor store when C is TMA-addressable up to the
            // chunk's end; otherwise (unaligned ldc, a ragged right edge) the warp moves it
            // row by row through the staging buffer so that every access is coalesced.
            const bool tma_chunk = chunk_tma(b, nb, sub, c);
            const bool coop_chunk = !tma_chunk;
            const uint32_t sbuf = stg + buf * T::STG_BYTES;
            // the buffer may still be read by an earlier tensor store
            if (lane == 0) bulk_wait_group_read<T::STG_BUFS - 1>();
            __syncwarp();
            if (packed == nullptr) {
#pragma unroll
                for (int j = 0; j < T::STG_COLS; ++j) v[j] *= p.alpha;
            }
            if (packed == nullptr && p.c_read && coop_chunk) {
                // C_in: lane j reads elements j (and j+32 for bf16) of each of the warp's 32
                // rows; element e of row r sits in 16-byte chunk (e*ES/16) ^ (r & 7).  Rows
                // go RB at a time so that RB (2 RB for bf16) loads per lane are in flight:
                // 16 rows keep the register budget of the other paths (32 spill).
                constexpr int RB = 16;
                constexpr int EPR = OUT != OUT_F32 ? 2 : 1;  // elements per lane and row
                constexpr int ES = OUT != OUT_F32 ? 2 : 4;   // bytes per element
                const int nrows = entry_in ? min(32, p.M - row0) : 0;
                const char* src = static_cast<const char*>(p.C) +
                                  ((long long)bb * p.stride_c + (long long)row0 * p.ldc + colc + (int)lane) * ES;
                const long long sstep = (long long)p.ldc * ES;
                bool ev[EPR];
#pragma unroll
                for (int h = 0; h < EPR; ++h) ev[h] = colc + (int)lane + 32 * h < p.N;
#pragma unroll 1
                for (int r0 = 0; r0 < 32; r0 += RB) {
                    uint32_t x[RB * EPR];
#pragma unroll
                    for (int i = 0; i < RB; ++i) {
                        const bool rv = r0 + i < nrows;
                        const char* rp = src + (long long)(r0 + i) * sstep;
#pragma unroll
                        for (int h = 0; h < EPR; ++h) {
                            x[i * EPR + h] = 0u;
                            if (rv && ev[h]) {
                                if constexpr (OUT != OUT_F32)
                                    x[i * EPR + h] = *reinterpret_cast<const uint16_t*>(rp + 64 * h);
                                else
                                    x[i * EPR + h] = *reinterpret_cast<const uint32_t*>(rp);
                            }
                        }
                    }
#pragma unroll
                    for (int i = 0; i < RB; ++i) {
                        const int r = r0 + i;
                        const uint32_t srow = sbuf + (uint32_t)r * 128u;
#pragma unroll
                        for (int h = 0; h < EPR; ++h) {
                            const int e = (int)lane + 32 * h;
                            if constexpr (OUT != OUT_F32)
                                st_shared_u16(srow + ((uint32_t)((e >> 3) ^ (r & 7)) << 4) + (uint32_t)(e & 7) * 2u,
                                              (uint16_t)x[i * EPR + h]);
                            else
                                st_shared_u32(srow + ((uint32_t)((e >> 2) ^ (r & 7)) << 4) + (uint32_t)(e & 3) * 4u,
                                              x[i * EPR + h]);
                        }
                    }
                }
                __syncwarp();
                if (row_in) {
                    const uint32_t srow = sbuf + lane * 128u;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        uint32_t x0, x1, x2, x3;
                        ld_shared_v4(srow + ((uint32_t)(cc ^ (int)(lane & 7u)) << 4), x0, x1, x2, x3);
                        const uint32_t xs[4] = {x0, x1, x2, x3};
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            if constexpr (OUT != OUT_F32) {
                                const int e = 8 * cc + 2 * h;
                                if (colc + e < p.N) v[e] = fmaf(p.beta, dec16_lo<OUT>(xs[h]), v[e]);
                                if (colc + e + 1 < p.N) v[e + 1] = fmaf(p.beta, dec16_hi<OUT>(xs[h]), v[e + 1]);
                            } else {
                                const int e = 4 * cc + h;
                                if (colc + e < p.N) v[e] = fmaf(p.beta, __uint_as_float(xs[h]), v[e]);
                            }
                        }
                    }
                }
                __syncwarp();  // every lane has its C_in before the buffer is overwritten
            } else if (packed == nullptr && p.c_read && row_in) {
                if (full_cols && p.c_tma) {
                    if constexpr (OUT != OUT_F32) {
                        const uint4* src = reinterpret_cast<const uint4*>(
                            static_cast<const uint16_t*>(p.C) + cbase + colc);
#pragma unroll
                        for (int j = 0; j < T::STG_COLS / 8; ++j) {
                            const uint4 w = src[j];
                            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                v[8 * j + 2 * h] = fmaf(p.beta, dec16_lo<OUT>(ww[h]), v[8 * j + 2 * h]);
                                v[8 * j + 2 * h + 1] = fmaf(p.beta, dec16_hi<OUT>(ww[h]), v[8 * j + 2 * h + 1]);
                            }
                        }
                    } else {
                        const float4* src = reinterpret_cast<const float4*>(
                            static_cast<const float*>(p.C) + cbase + colc);
#pragma unroll
                        for (int j = 0; j < T::STG_COLS / 4; ++j) {
                            const float4 w = src[j];
                            v[4 * j + 0] = fmaf(p.beta, w.x, v[4 * j + 0]);
                            v[4 * j + 1] = fmaf(p.beta, w.y, v[4 * j + 1]);
                            v[4 * j + 2] = fmaf(p.beta, w.z, v[4 * j + 2]);
                            v[4 * j + 3] = fmaf(p.beta, w.w, v[4 * j + 3]);
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < T::STG_COLS; ++j) {
                        if (colc + j < p.N) {
                            float cin;
                            if constexpr (OUT != OUT_F32)
                                cin = dec16_lo<OUT>(static_cast<const uint16_t*>(p.C)[cbase + colc + j]);
                            else
                                cin = static_cast<const float*>(p.C)[cbase + colc + j];
                            v[j] = fmaf(p.beta, cin, v[j]);
                        }
                    }
                }
            }
            // pack the 128-byte row segment into 8 x 16-byte words
            uint32_t w[32];
            if (packed != nullptr) {
#pragma unroll
                for (int j = 0; j < 32; ++j) w[j] = packed[j];
            } else {
                if constexpr (OUT != OUT_F32) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) w[j] = pack16<OUT>(v[2 * j], v[2 * j + 1]);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(v[j]);
                }
            }
            {
                const uint32_t row_addr = sbuf + lane * 128u;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    st_shared_v4(row_addr + ((uint32_t)(j ^ (int)(lane & 7u)) << 4), w[4 * j],
                                 w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                if (tma_chunk) {
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&tmC, sbuf, colc, row0, bb);
                        bulk_commit_group();
                        if (!p.c_read)
                            for (int k = 0; k < n_more; ++k) {
                                tma_store_3d(&tmC, sbuf, colc, row0, __ldg(more + (size_t)k * step));
                                bulk_commit_group();
                            }
                    }
                    fanned = !p.c_read;
                } else {
                    // row by row: lane j writes element j (and j+32) of each row, coalesced.
                    // The column predicates and the swizzle-free part of the shared address are
                    // fixed for the lane and the global pointer advances by ldc, so a row costs
                    // one shared load and one store per element (the loop is issue-bound: one
                    // warp per scheduler, nothing else to hide latency behind).
                    __syncwarp();
                    constexpr int ES = OUT != OUT_F32 ? 2 : 4;  // bytes per element
                    constexpr int EPR = OUT != OUT_F32 ? 2 : 1;  // elements per lane and row
                    const int nrows = entry_in ? min(32, p.M - row0) : 0;
                    char* dst = static_cast<char*>(p.C) +
                                ((long long)bb * p.stride_c + (long long)row0 * p.ldc + colc + (int)lane) * ES;
                    const long long dstep = (long long)p.ldc * ES;
                    bool ev[EPR];
                    uint32_t ch[EPR];
                    const uint32_t inb = OUT != OUT_F32 ? (lane & 7u) * 2u : (lane & 3u) * 4u;
#pragma unroll
                    for (int h = 0; h < EPR; ++h) {
                        const int e = (int)lane + 32 * h;
                        ev[h] = colc + e < p.N;
                        ch[h] = (uint32_t)(e * ES / 16);
                    }
#pragma unroll 8
                    for (int r = 0; r < nrows; ++r, dst += dstep) {
                        const uint32_t srow = sbuf + (uint32_t)r * 128u + inb;
                        const uint32_t sw = (uint32_t)(r & 7);
#pragma unroll
                        for (int h = 0; h < EPR; ++h) {
                            if (!ev[h]) continue;
                            const uint32_t a = srow + ((ch[h] ^ sw) << 4);
                            if constexpr (OUT != OUT_F32)
                                *reinterpret_cast<uint16_t*>(dst + 64 * h) = ld_shared_u16(a);
                            else
                                *reinterpret_cast<uint32_t*>(dst) = ld_shared_u32(a);
                        }
                    }
                    __syncwarp();
                }
                if (T::STG_BUFS == 2) buf ^= 1;
            }
            return fanned;
        };
        // TMEM -> registers: chunk c (STG_COLS columns) of the slot whose lane-quarter row is trow.
        auto load_chunk = [&](uint32_t trow, int c, float (&v)[T::STG_COLS]) {
            uint32_t r0[32];
            tmem_ld_32x32b_x32(trow + c * T::STG_COLS, r0);
            if constexpr (OUT != OUT_F32) {
                uint32_t r1[32];
                tmem_ld_32x32b_x32(trow + c * T::STG_COLS + 32, r1);
                tmem_ld_wait(r0);
                tmem_ld_wait(r1);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[32 + j] = __uint_as_float(r1[j]);
            } else {
                tmem_ld_wait(r0);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r0[j]);
        };
        // Split-K partial sums travel as 4 KiB pieces: 32 rows x 32 fp32 columns, held in global
        // memory as the image of the staging buffer (row r at byte 128 r, 16-byte word w of the
        // row at ((w ^ (r & 7)) << 4)).  Moving a piece through the buffer turns the
        // lane-per-row layout of TMEM into 512-byte coalesced accesses.
        constexpr int PIECES = T::STG_COLS / 32;               // pieces per chunk
        constexpr int WS_TILE = 128 * NSUB * BN;               // floats per (tile, CTA rank, slice)
        constexpr int WS_WARP = WS_TILE / T::EPI_WARPS;        // floats per epilogue warp
        auto put_piece = [&](float* g, const float* x, uint32_t sb) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                st_shared_v4(sb + lane * 128u + ((uint32_t)(j ^ (int)(lane & 7u)) << 4), __float_as_uint(x[4 * j]),
                             __float_as_uint(x[4 * j + 1]), __float_as_uint(x[4 * j + 2]),
                             __float_as_uint(x[4 * j + 3]));
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t x0, x1, x2, x3;
                ld_shared_v4(sb + (uint32_t)i * 512u + lane * 16u, x0, x1, x2, x3);
                reinterpret_cast<uint4*>(g)[i * 32 + (int)lane] = make_uint4(x0, x1, x2, x3);
            }
            __syncwarp();
        };
        // Cluster split-K exchange buffer: the ring, as 4 KiB pieces (32 rows x 32 fp32 columns),
        // piece (32-column block cb, lane quarter qq) at ((cb * 4 + qq) << 12).  Inside a piece,
        // columns 4j..4j+3 of row r sit at j * 512 + r * 16: a warp-wide 16-byte access then
        // covers 512 contiguous bytes, the form distributed shared memory serves fastest
        // (measured on B200: about 3x the rate of the same loads 128 bytes apart).
        const uint32_t xchg = sbase + T::OFF_A;
        // per unit: tile t, part sl of S (split-K slice or stream-K range; or the destination part
        // of a deduplicated batch, S == 1)
        int t, kb_lo_u, kb_hi_u, sl, S;
        for (int i = 0; ok && get_unit(i, t, kb_lo_u, kb_hi_u, sl, S); ++i) {
            int b, mb, nb;
            decode_tile(p, t, b, mb, nb);
            const int row0 = mb * T::BM + (int)rank * 128 + 32 * q;
            const int row = row0 + (int)lane;
            if (p.c_read && p.dd_off == nullptr && (S == 1 || sl == 0) && row < p.M && b < p.batch_real) {
                // C_in of this warp's rows of the tile, fetched into L2 while the mainloop runs:
                // the beta term then reads L2 instead of DRAM (a tile's epilogue is exposed when a
                // CTA has a single tile).  Each lane asks for the first and last line of each of its
                // row's chunk segments, within the matrix only (C rows may start anywhere).
                constexpr int ES = OUT != OUT_F32 ? 2 : 4;
#pragma unroll 1
                for (int sub = 0; sub < NSUB; ++sub)
#pragma unroll 1
                    for (int ci = 0; ci < CPW; ++ci) {
                        const int jc = (half * CPW + ci) * T::STG_COLS;
                        const int tcol = sub * T::BN_CTA + (jc / T::BN_CTA) * T::B_CHUNK + jc % T::BN_CTA;
                        const int bb = p.pack > 1 ? nb * p.pack + tcol / p.N : b;
                        const int colc = p.pack > 1 ? tcol % p.N : nb * T::TILE_N + tcol;
                        if (bb >= p.batch_real || colc >= p.N) continue;
                        const char* seg = static_cast<const char*>(p.C) +
                                          ((long long)bb * p.stride_c + (long long)row * p.ldc + colc) * ES;
                        prefetch_l2(seg);
                        prefetch_l2(seg + (min(T::STG_COLS, p.N - colc) * ES - 1));
                    }
            }
            // this warp's partials of slice s of the tile: pieces in (sub, ci, piece) order
            auto slab = [&](int s) {
                return p.ws + ((size_t)(t * CG + (int)rank) * p.ws_parts + s) * WS_TILE + (size_t)ew * WS_WARP;
            };
            if (S > 1) {
                // the staging buffer must not be read by a tensor store still in flight
                if (lane == 0) bulk_wait_group_read<0>();
                __syncwarp();
            }
            if constexpr (OUT != OUT_F32 && NSUB == 2 && T::EPI_HALVES == 2) {
                if (CS == 1 && S == 1 && p.dd_off == nullptr && !p.c_read) {
                    // Plain two-sub-tile tile, C not read: each warp moves its half of both
                    // accumulator slots into registers (scaled, rounded pairs), handing each slot
                    // back to the MMA warp as soon as it is read; only then are the chunks
                    // staged and stored, while the next tile's mainloop runs.
                    uint32_t pk[NSUB][CPW][32];
#pragma unroll
                    for (int sub = 0; sub < NSUB; ++sub) {
                        int w_ok = 1;
                        if (lane == 0)
                            w_ok = wait_phase<CG, false>(bar_tfull(sub), (tph >> sub) & 1u, slot_abort, ctarank,
                                                         p.status, p.timeout_ns, kStatusEpilogue);
                        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
                        if (!w_ok) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        tph ^= 1u << sub;
                        const uint32_t trow = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(sub * BN);
#pragma unroll
                        for (int ci = 0; ci < CPW; ++ci) {
                            uint32_t ra[32], rb[32];
                            const uint32_t tc = trow + (uint32_t)((half * CPW + ci) * T::STG_COLS);
                            tmem_ld_32x32b_x32(tc, ra);
                            tmem_ld_32x32b_x32(tc + 32, rb);
                            tmem_ld_wait(ra);
                            tmem_ld_wait(rb);
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                pk[sub][ci][j] = pack16<OUT>(__uint_as_float(ra[2 * j]) * p.alpha,
                                                             __uint_as_float(ra[2 * j + 1]) * p.alpha);
                                pk[sub][ci][16 + j] = pack16<OUT>(__uint_as_float(rb[2 * j]) * p.alpha,
                                                                  __uint_as_float(rb[2 * j + 1]) * p.alpha);
                            }
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * sub);
                    }
                    if (!ok) break;
                    float unused[T::STG_COLS];
#pragma unroll
                    for (int sub = 0; sub < NSUB; ++sub)
#pragma unroll
                        for (int ci = 0; ci < CPW; ++ci)
                            finish_chunk(b, nb, row0, row, sub, half * CPW + ci, unused, -1, nullptr, 0, 1, pk[sub][ci]);
                    continue;
                }
            }
            for (int sub = 0; sub < NSUB; ++sub) {
                const int slot = NSUB == 1 ? acc : sub;
                int w_ok = 1;
                if (lane == 0)
                    w_ok = wait_phase<CG, false>(bar_tfull(slot), (tph >> slot) & 1u, slot_abort, ctarank, p.status, p.timeout_ns,
                                                 kStatusEpilogue);
                w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
                if (!w_ok) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tph ^= 1u << slot;
                const uint32_t trow = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(slot * BN);
#pragma unroll 1
                for (int ci = 0; ci < CPW; ++ci) {
                    const int c = half * CPW + ci;
                    float v[T::STG_COLS];
                    load_chunk(trow, c, v);
                    if (CS > 1) {
                        // this CTA's K-slice partial sums, for the cluster's reduction below
                        if (ci == 0) fence_proxy_async_smem();
#pragma unroll
                        for (int h = 0; h < PIECES; ++h) {
                            const uint32_t pc = xchg + ((uint32_t)((c * PIECES + h) * 4 + q) << 12) + lane * 16u;
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                st_shared_v4(pc + (uint32_t)j * 512u, __float_as_uint(v[32 * h + 4 * j]),
                                             __float_as_uint(v[32 * h + 4 * j + 1]), __float_as_uint(v[32 * h + 4 * j + 2]),
                                             __float_as_uint(v[32 * h + 4 * j + 3]));
                        }
                    } else if (S == 1 && p.dd_off == nullptr) {
                        if (ci == CPW - 1) {
                            // Slot drained: hand it back to the MMA warp (leader CTA).
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * slot);
                        }
                        finish_chunk(b, nb, row0, row, sub, c, v);
                    } else if (S == 1) {
                        // Deduplicated batch: the chunk's distinct entry goes to every item that
                        // uses it; this unit stores destinations sl, sl + DS, ... of the entry's
                        // list, reloading the accumulator from TMEM for each one.  The slot is
                        // handed back after the last reload of the warp's last chunk.
                        const int e = chunk_entry(b, nb, sub, c);
                        int k = 0, hi = 0;
                        if (e < p.batch_real) {
                            k = __ldg(p.dd_off + e) + sl;
                            hi = __ldg(p.dd_off + e + 1);
                        }
                        auto release = [&]() {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * slot);
                        };
                        if (k >= hi) {
                            if (ci == CPW - 1) release();
                        } else {
                            // With C not read and the chunk leaving through a tensor store, it is
                            // converted and staged once and every item gets a tensor store of it;
                            // otherwise each item reloads the accumulator and is stored in turn.
                            const bool fan = !p.c_read && chunk_tma(b, nb, sub, c);
                            const int n_more = fan ? (hi - k - 1) / DS : 0;
                            if (ci == CPW - 1 && (fan || k + DS >= hi)) release();
                            finish_chunk(b, nb, row0, row, sub, c, v, __ldg(p.dd_dst + k), p.dd_dst + k + DS, n_more, DS);
                            if (!fan) {
                                for (k += DS; k < hi; k += DS) {
                                    load_chunk(trow, c, v);
                                    if (ci == CPW - 1 && k + DS >= hi) release();
                                    finish_chunk(b, nb, row0, row, sub, c, v, __ldg(p.dd_dst + k));
                                }
                            }
                        }
                    } else {
                        // publish this part's partial sums; the slot is free once its last chunk
                        // is read, so the next unit's mainloop overlaps the publishing and fixup
                        if (ci == CPW - 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * slot);
                        }
                        float* g = slab(sl) + (size_t)((sub * CPW + ci) * PIECES) * 1024;
#pragma unroll
                        for (int h = 0; h < PIECES; ++h) put_piece(g + h * 1024, v + 32 * h, stg + buf * T::STG_BYTES);
                    }
                }
            }
            if (S > 1 && ok) {
                // Split-K fixup, per warp (its 32 rows).  Arrival is counted after the partial
                // sums are visible; the last of the S parts to arrive adds them up in part order
                // 0..S-1, reading every one (its own too) from global memory, so the result is the
                // same whatever the arrival order.  Nothing waits on another CTA.
                __threadfence();
                __syncwarp();
                unsigned int* cnt = p.counters + ((size_t)(t * CG + (int)rank) * T::EPI_WARPS + ew);
                unsigned int old = 0;
                if (lane == 0) {
                    old = atomicAdd(cnt, 1u);
                    if (old == (unsigned int)(S - 1)) *cnt = 0u;  // ready for the next call
                }
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == (unsigned int)(S - 1)) {
                    __threadfence();
                    for (int sub = 0; sub < NSUB; ++sub) {
#pragma unroll 1
                        for (int ci = 0; ci < CPW; ++ci) {
                            const int c = half * CPW + ci;
                            float v[T::STG_COLS];
#pragma unroll
                            for (int j = 0; j < T::STG_COLS; ++j) v[j] = 0.0f;
                            const size_t off = (size_t)((sub * CPW + ci) * PIECES) * 1024;
                            // the buffer finish_chunk will use next; a tensor store may still read it
                            if (lane == 0) bulk_wait_group_read<T::STG_BUFS - 1>();
                            __syncwarp();
                            const uint32_t sb = stg + buf * T::STG_BYTES;
#pragma unroll 1
                            for (int s2 = 0; s2 < S; ++s2) {
                                // every piece of the chunk in flight at once, then through the buffer
                                const uint4* g = reinterpret_cast<const uint4*>(slab(s2) + off);
                                uint4 x[PIECES][8];
#pragma unroll
                                for (int h = 0; h < PIECES; ++h)
#pragma unroll
                                    for (int i = 0; i < 8; ++i) x[h][i] = __ldcg(g + h * 256 + i * 32 + (int)lane);
#pragma unroll
                                for (int h = 0; h < PIECES; ++h) {
#pragma unroll
                                    for (int i = 0; i < 8; ++i)
                                        st_shared_v4(sb + (uint32_t)i * 512u + lane * 16u, x[h][i].x, x[h][i].y,
                                                     x[h][i].z, x[h][i].w);
                                    __syncwarp();
#pragma unroll
                                    for (int j = 0; j < 8; ++j) {
                                        uint32_t y0, y1, y2, y3;
                                        ld_shared_v4(sb + lane * 128u + ((uint32_t)(j ^ (int)(lane & 7u)) << 4), y0, y1,
                                                     y2, y3);
                                        v[32 * h + 4 * j] += __uint_as_float(y0);
                                        v[32 * h + 4 * j + 1] += __uint_as_float(y1);
                                        v[32 * h + 4 * j + 2] += __uint_as_float(y2);
                                        v[32 * h + 4 * j + 3] += __uint_as_float(y3);
                                    }
                                    __syncwarp();
                                }
                            }
                            finish_chunk(b, nb, row0, row, sub, c, v);
                        }
                    }
                }
            }
            if (NSUB == 1) acc ^= 1;
        }
        if constexpr (T::CSPLIT_OK) {
            if (CS > 1) {
                // Cluster split-K reduction.  Once every CTA of the cluster has its partial tile in
                // its shared memory, the EPI_WARPS*CS epilogue warps of the CTAs holding the same 128 rows
                // (one per slice) share those rows' (lane quarter, column chunk) items; each adds
                // the CS partials of its item in slice order 0..CS-1, reading them through
                // distributed shared memory, and runs the normal alpha/beta epilogue on the sum.
                // The result does not depend on timing.
                __syncwarp();
                cluster_sync();
                if (ok && ld_shared_volatile_u32(slot_abort) == 0u) {
                    int b, mb, nb;
                    decode_tile(p, cluster_id, b, mb, nb);
                    constexpr int CH = BN / T::STG_COLS;  // column chunks of the tile
                    for (int it = (int)crank * T::EPI_WARPS + ew; it < 4 * CH; it += T::EPI_WARPS * CS) {
                        const int qq = it & 3, c = it >> 2;
                        const int row0 = mb * T::BM + (int)rank * 128 + 32 * qq;
                        float v[T::STG_COLS];
#pragma unroll 1
                        for (int s2 = 0; s2 < CS; ++s2) {
                            // slice s2's CTA holding the same rows of the tile
                            const uint32_t src = map_to_rank(xchg, (uint32_t)(s2 * CG) + rank) + lane * 16u;
#pragma unroll
                            for (int h = 0; h < PIECES; ++h) {
                                uint32_t x[8][4];
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    ld_cluster_v4(src + ((uint32_t)((c * PIECES + h) * 4 + qq) << 12) + (uint32_t)j * 512u,
                                                  x[j][0], x[j][1], x[j][2], x[j][3]);
#pragma unroll
                                for (int j = 0; j < 8; ++j)
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const float f = __uint_as_float(x[j][e]);
                                        v[32 * h + 4 * j + e] = s2 == 0 ? f : v[32 * h + 4 * j + e] + f;
                                    }
                            }
                        }
                        finish_chunk(b, nb, row0, row0 + (int)lane, 0, c, v);
                    }
                }
            }
        }
        if (p.c_tma && lane == 0) bulk_wait_group_all();
    }
    // Producer and MMA warps meet the epilogue's cluster barrier (all partial tiles written).
    if (CS > 1 && warp < 2) {
        __syncwarp();
        cluster_sync();
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (ld_shared_volatile_u32(slot_abort) != 0u && threadIdx.x == 0) {
        // Aborting: let copies and MMAs already issued by this CTA land (bounded).
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 5000000ull) nanosleep_ns(100000);
    }
    // (cluster split-K: no CTA leaves while another may still read its shared memory)
    if (CG == 2 || CS > 1) cluster_sync(); else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<CG>(tmem_base, T::TMEM_COLS);
    }
}

}  // namespace pw
