/*
 * gemm_bf16.h -- C ABI of the B200 (sm_100a) persistent, warp-specialized BF16 GEMM.
 *
 * The operation is the producer/consumer matrix multiply described on the page
 * "Meta presente TLX pour combler le fosse entre la complexite du materiel GPU et la
 * productivite des developpeurs", section "Comment cela fonctionne" (one warp group loads
 * tiles asynchronously through TMA while another drives the tensor cores, handing over
 * through lightweight barriers), whose accumulator loop is sketched on the page
 * "Triton 3.7 permite extender el compilador de GPU sin forks", section "NVIDIA H100
 * (Hopper): GEMM persistente" (fp32 accumulator, K loop over staged tiles, results stored),
 * with the alpha/beta update of a BLAS GEMM:
 *
 *     C = alpha * A * B + beta * C       bf16 inputs, fp32 accumulation.
 *
 * All matrices are row-major in device memory; leading dimensions and strides are in
 * ELEMENTS.  Calls are asynchronous: they validate the arguments, enqueue the kernels on
 * `stream` and return.  The caller owns every buffer it passes; the library never frees
 * them.  The library owns only a stream-ordered workspace, taken on `stream` from a memory
 * pool of its own (one per device, created on first use) and given back on `stream` at the end
 * of the call.  It holds the padded copies of A or B when the tensor-memory accelerator cannot
 * read them as given (a leading dimension that is not a multiple of 8 elements, a base not
 * 16-byte aligned), and the fp32 partial sums when a call with few output tiles cuts K into
 * slices (split-K).  The pool keeps freed memory for later calls rather than returning it to
 * the driver, so it holds the largest workspace used so far until the process exits.
 *
 * No exceptions cross this boundary.  A call rejected for its arguments enqueues nothing; a
 * CUDA failure during the enqueue (GEMM_ERR_CUDA / GEMM_ERR_NO_MEMORY) may leave the steps
 * already enqueued by that call on `stream` (pre-pass copies, the workspace's allocation and
 * release), which touch only the workspace.
 */
#ifndef GEMM_BF16_H
#define GEMM_BF16_H

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GEMM_API __attribute__((visibility("default")))
#else
#define GEMM_API
#endif

struct CUstream_st; /* cudaStream_t == struct CUstream_st*; NULL is the legacy stream */

typedef enum {
    GEMM_OK = 0,
    GEMM_ERR_INVALID_ARG = 1, /* bad size, leading dimension, pointer or enum */
    GEMM_ERR_UNSUPPORTED = 2, /* valid request this build cannot run (e.g. no sm_100 GPU) */
    GEMM_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (launch, encode, alloc) */
    GEMM_ERR_TIMEOUT = 4,     /* a kernel gave up a bounded wait (see gemm_bf16_device_status) */
    GEMM_ERR_NO_MEMORY = 5    /* the workspace allocation failed */
} gemm_status_t;

typedef enum {
    GEMM_OUT_F32 = 0, /* C is float32 */
    GEMM_OUT_BF16 = 1 /* C is bfloat16 (fp32 result rounded to nearest even once) */
} gemm_out_t;

/*
 * gemm_bf16 -- C[M x N] = alpha * A[M x K] * B + beta * C.
 *
 *   A   bf16, M x K row-major, element (i,k) at A[i*lda + k], lda >= max(1, K).
 *   B   bf16, stored N x K row-major ("K-major"), element (k,j) of the K x N operand at
 *       B[j*ldb + k], ldb >= max(1, K).  So C = alpha * A * B_stored^T + beta * C.
 *   C   out_type, M x N row-major, element (i,j) at C[i*ldc + j], ldc >= max(1, N).
 *       Read only when beta != 0 (so NaN/garbage in C is ignored when beta == 0) and
 *       updated in place.  Elements of the ldc padding columns are never touched.
 *   alpha, beta  fp32 scalars.  D = alpha*acc + beta*C_in is formed in fp32 and, for
 *       bf16 output, rounded once to nearest even.
 *
 * M == 0 or N == 0: returns GEMM_OK with nothing enqueued.  K == 0 or alpha == 0:
 * C = beta * C (C = 0 when beta == 0) without reading A or B.
 * Errors: GEMM_ERR_INVALID_ARG for negative sizes, a leading dimension below its minimum,
 * a NULL pointer where data is needed, a pointer not aligned to its element size, or an
 * unknown out_type.  A or B overlapping C is undefined behaviour (not checked).
 * Results are deterministic: the same inputs give bitwise the same C on every call.
 */
GEMM_API gemm_status_t gemm_bf16(int M, int N, int K, const void* A, int lda, const void* B, int ldb,
                        void* C, int ldc, gemm_out_t out_type, float alpha, float beta,
                        struct CUstream_st* stream);

/*
 * gemm_bf16_batched_shared_w -- Y[b] = alpha * W * X[b] + beta * Y[b] for b < batch.
 *
 * The shared-operand form of the recommendation-model "linear compression" kernel on the
 * page "Meta accelere un noyau GPU d'un facteur 4 avec TLX, une extension du langage
 * Triton", sections "Comment le chargement des donnees gene le calcul" and "Ce que signifie
 * une acceleration d'un facteur quatre": the operand common to every item (W) is read once
 * per tile walk and never replicated per batch entry.
 *
 *   W      bf16, M x K row-major (shared by all b), ldw >= max(1, K).
 *   X      bf16; X[b] = X + b*stride_x is K x N row-major ("N-major"), ldx >= max(1, N),
 *          stride_x >= 0.
 *   Y      out_type; Y[b] = Y + b*stride_y is M x N row-major, ldy >= max(1, N);
 *          when batch > 1, stride_y >= (M-1)*ldy + N (output batches must not overlap).
 * Same conventions and errors as gemm_bf16.  batch == 0: GEMM_OK, nothing enqueued.
 */
GEMM_API gemm_status_t gemm_bf16_batched_shared_w(int batch, int M, int N, int K, const void* W, int ldw,
                                         const void* X, int ldx, long long stride_x, void* Y,
                                         int ldy, long long stride_y, gemm_out_t out_type,
                                         float alpha, float beta, struct CUstream_st* stream);

/* Human-readable name of a status code (static storage, never NULL). */
GEMM_API const char* gemm_bf16_status_string(gemm_status_t s);

/*
 * gemm_bf16_device_status -- synchronizes `stream`, then reports whether any kernel of this
 * library that ran on the current device since the previous call gave up a bounded
 * barrier wait (GEMM_ERR_TIMEOUT; the word is then cleared), or GEMM_ERR_CUDA if the
 * synchronization failed, else GEMM_OK.  A timed-out kernel skips its remaining tiles,
 * releases its tensor memory and exits, so the CUDA context stays usable; its output is
 * incomplete.
 */
GEMM_API gemm_status_t gemm_bf16_device_status(struct CUstream_st* stream);

/*
 * gemm_bf16_set_plan -- force a tile plan for all following calls in this process (for
 * tuning sweeps and tests); -1 restores the automatic choice.
 *   0: 128x128 tile, one CTA       1: 128x256 tile, one CTA
 *   2: 256x256 tile, 2-CTA cluster 3: 256x128 tile, 2-CTA cluster
 *   4: 256x512 tile, 2-CTA cluster (two 256-column MMA sub-tiles sharing the A tile)
 *   5: 256x128 tile, 2-CTA cluster, A resident in shared memory (M <= 256, K <= 512)
 *   6: 128x128 tile, one CTA, A resident in shared memory (M <= 128, K <= 512)
 *   7: 256x256 tile, 2-CTA cluster, A resident in shared memory (M <= 256, K <= 512)
 *   8: 128x64 tile, one CTA (thin problems: twice the tiles of plan 0)
 * In the batched call, a tile wider than N holds several batch entries side by side when N is a
 * multiple of 64 that divides the tile width.
 * Returns GEMM_ERR_INVALID_ARG for an unknown plan.  A plan that cannot serve a given
 * call is replaced by the automatic choice for that call.
 *
 * With few output tiles and a long K, plans 0-4 and 8 may also cut K into slices (split-K): each
 * (tile, slice) unit writes fp32 partial sums to the workspace and the last unit of a tile
 * adds them in slice order, so results stay bitwise reproducible.  The plan and the slice
 * count come from a cost model; environment variables read at every call override it for
 * sweeps and tests:
 *   GEMM_BF16_SPLIT_K=s     (1..8) s slices wherever the plan and K allow it (1: never split)
 *   GEMM_BF16_GROUP_M=g     (1..64) m-blocks per group of the persistent tile order
 */
GEMM_API gemm_status_t gemm_bf16_set_plan(int plan);

/*
 * gemm_bf16_set_wait_timeout_ns -- bound, in nanoseconds of the GPU global timer, of every
 * barrier wait inside the kernels launched afterwards in this process (default 2e9 = 2 s;
 * 0 restores the default).
 */
GEMM_API gemm_status_t gemm_bf16_set_wait_timeout_ns(unsigned long long ns);

/*
 * gemm_bf16_noalloc -- the same operation, arguments, layouts and errors as gemm_bf16, for
 * callers that must not have this library allocate device memory.  (The pages describe no
 * such entry point; it exists for integration only.)
 *
 * Who needs it: a caller whose device memory is already handed out by its own caching
 * allocator or memory budget (a framework that reserves nearly all of the GPU, a service that
 * pins a fixed footprint) cannot let a library draw extra memory from the device's pool, where
 * the request may fail or fragment what the caller manages; a caller on a latency-critical
 * path cannot afford the time an allocation may take.  gemm_bf16 may allocate a stream-ordered
 * workspace when A or B is not laid out for the tensor-memory accelerator; this entry point
 * never calls cudaMalloc, cudaMallocAsync, cudaFree or any allocating routine.
 *
 * Instead it uses one fixed scratch array of GEMM_BF16_NOALLOC_SCRATCH_BYTES (32 MiB) that
 * lives in the library's device image: every GPU on which the library is used holds it until
 * the process exits.  It stores the padded copies of A and/or B that the alignment pre-pass
 * makes (needed when lda or ldb is not a multiple of 8 elements or a base is not 16-byte
 * aligned).  If those copies, each rounded up to 256 bytes, need more than the scratch holds,
 * the call returns GEMM_ERR_INVALID_ARG and enqueues nothing.  Calls whose operands need no
 * copy do not touch the scratch.
 *
 * The scratch is shared by every call on a device and keeps the last call's contents; nothing
 * in it has to start at zero (the copies are fully rewritten by each call that uses them, and
 * their padding columns are never read).  Calls that use the scratch and overlap on the GPU
 * (for instance on two streams without ordering between them) race on it: order them on one
 * stream or with events.
 *
 * The first call on each device looks up the scratch's device address (cudaGetSymbolAddress,
 * with that device current) and caches it; make that first call before any stream capture.
 */
#define GEMM_BF16_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
GEMM_API gemm_status_t gemm_bf16_noalloc(int M, int N, int K, const void* A, int lda, const void* B,
                                         int ldb, void* C, int ldc, gemm_out_t out_type,
                                         float alpha, float beta, struct CUstream_st* stream);

/* Library version as an integer (major*10000 + minor*100 + patch). */
GEMM_API int gemm_bf16_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GEMM_BF16_H */
