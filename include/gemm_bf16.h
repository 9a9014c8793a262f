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
    GEMM_OUT_F32 = 0,  /* C is float32 */
    GEMM_OUT_BF16 = 1, /* C is bfloat16 (fp32 result rounded to nearest even once) */
    GEMM_OUT_F16 = 2   /* C is IEEE binary16 (fp32 result rounded to nearest even once; values
                          beyond +-65504 become +-inf) */
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

/*
 * gemm_f16, gemm_f16_batched_shared_w -- the same operations, arguments, layouts, conventions
 * and errors as gemm_bf16 and gemm_bf16_batched_shared_w, with A and B (W and X) holding IEEE
 * binary16 (fp16) values instead of bfloat16.  Products are exact and accumulate in fp32, as
 * for bf16.  The pages' GEMM measurements (page "Triton 3.7 permite extender el compilador de
 * GPU sin forks", sections "NVIDIA H100 (Hopper): resultados de rendimiento" and "AMD MI350:
 * GEMM segmentado") are FP16 GEMMs; this is that operand type.  The output may be fp32, bf16
 * or fp16 (out_type).
 */
GEMM_API gemm_status_t gemm_f16(int M, int N, int K, const void* A, int lda, const void* B, int ldb,
                                void* C, int ldc, gemm_out_t out_type, float alpha, float beta,
                                struct CUstream_st* stream);

GEMM_API gemm_status_t gemm_f16_batched_shared_w(int batch, int M, int N, int K, const void* W, int ldw,
                                                 const void* X, int ldx, long long stride_x, void* Y,
                                                 int ldy, long long stride_y, gemm_out_t out_type,
                                                 float alpha, float beta, struct CUstream_st* stream);

/*
 * gemm_bf16_batched_shared_w_dedup -- Y[b] = alpha * W * X[index[b]] + beta * Y[b], b < batch:
 * the shared-W form for requests whose items repeat feature entries.
 *
 * The recommendation-model kernel on the page "Meta accelere un noyau GPU d'un facteur 4 avec
 * TLX, une extension du langage Triton" gets part of its speed-up from no longer handling
 * repeated features as copies (sections "Comment le chargement des donnees gene le calcul":
 * a buyer's data are identical across the items scored for that buyer; "Ce que signifie une
 * acceleration d'un facteur quatre").  Here the request carries each distinct entry once: X
 * holds n_unique entries, X[u] = X + u*stride_x (K x N row-major, ldx >= max(1, N)), and
 * item b uses entry index[b].  The GEMM runs once per distinct entry; its epilogue writes
 * the result to every item that uses it (Y[b] = Y + b*stride_y, M x N row-major; when
 * batch > 1, stride_y >= (M-1)*ldy + N).  The items of one entry receive bitwise the same
 * values as gemm_bf16_batched_shared_w gives for the expanded batch X[b] = X[index[b]] when
 * both calls take the same tile plan (no split of K is used here).
 *
 *   index  device memory, `batch` ints in [0, n_unique), 4-byte aligned; read by the device.
 *          An entry outside that range leaves its item's Y untouched and makes the next
 *          gemm_bf16_device_status return GEMM_ERR_INVALID_ARG.
 * Other arguments, conventions and errors as gemm_bf16_batched_shared_w; n_unique < 0, or
 * n_unique == 0 with work to do, or a NULL index with batch > 0 is GEMM_ERR_INVALID_ARG.  The
 * workspace also holds the per-entry item lists (2*n_unique + 1 + batch ints).
 */
GEMM_API gemm_status_t gemm_bf16_batched_shared_w_dedup(int batch, int n_unique, int M, int N, int K,
                                                        const void* W, int ldw, const void* X, int ldx,
                                                        long long stride_x, const int* index, void* Y,
                                                        int ldy, long long stride_y, gemm_out_t out_type,
                                                        float alpha, float beta, struct CUstream_st* stream);

/* Human-readable name of a status code (static storage, never NULL). */
GEMM_API const char* gemm_bf16_status_string(gemm_status_t s);

/*
 * gemm_bf16_device_status -- synchronizes `stream`, then reports whether any kernel of this
 * library that ran on the current device since the previous call gave up a bounded
 * barrier wait (GEMM_ERR_TIMEOUT), or found a deduplicated batch's index out of range
 * (GEMM_ERR_INVALID_ARG); the word is then cleared.  GEMM_ERR_CUDA if the synchronization
 * failed, else GEMM_OK.  A timed-out kernel skips its remaining tiles,
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
 * With few output tiles and a long K, the kernels may also cut K into slices, in one of two ways:
 *   cluster split-K (plans 0-3 and 8): the 2, 4 or 8 slices of a tile run on the CTAs of one
 *     thread-block cluster (plans 2 and 3: 2 or 4 slices, each on a CTA pair), which add their
 *     partial tiles through distributed shared memory (no workspace, so gemm_bf16_noalloc may
 *     use it too);
 *   split-K through the workspace (plans 0-4 and 8): each (tile, slice) unit writes fp32
 *     partial sums to the workspace and the last unit of a tile adds them.
 * With more tiles than the device runs at once and a partial last wave, stream-K (plans 0-4 and
 * 8; workspace) spreads the last wave's tiles over every cluster as equal ranges of k-blocks;
 * a tile cut by several ranges is added up like a workspace split.
 * All of them add the parts in a fixed order, so results stay bitwise reproducible.  The plan and
 * the split come from the tuning table when gemm_autotune measured the problem, else from a cost
 * model whose choice is kept per problem for later calls.  A forced plan or any of these
 * environment variables (read at every call; for sweeps and tests) bypasses both:
 *   GEMM_BF16_SPLIT_K=s        (1..8) s workspace slices wherever the plan and K allow it
 *                              (1: no split of either kind unless the next variable forces one)
 *   GEMM_BF16_CLUSTER_SPLIT=s  (2, 4, 8) cluster split-K with s slices where the plan takes it;
 *                              1: never cluster split-K
 *   GEMM_BF16_STREAM_K=1       stream-K wherever it applies; 0: never
 *   GEMM_BF16_GROUP_M=g        (1..64) m-blocks per group of the persistent tile order
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
 * copy do not touch the scratch.  K is never cut through the workspace here; the cluster form
 * of split-K (partial sums exchanged in shared memory) needs no memory and may be used.
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

/*
 * gemm_bf16_tensor_map_cache_stats -- how many tensor maps (the TMA descriptors of A, B and C)
 * the calls so far took from the library's cache (*hits) and had to encode (*misses).  A map
 * depends only on a buffer's address, extents, strides and tile box, so repeated calls on the
 * same buffers encode nothing.  GEMM_ERR_INVALID_ARG if a pointer is NULL.
 */
GEMM_API gemm_status_t gemm_bf16_tensor_map_cache_stats(unsigned long long* hits,
                                                        unsigned long long* misses);

/*
 * Autotuning.  The pages integrate TLX with Triton's autotuning (page "Meta presente TLX pour
 * combler le fosse...", section "Comment cela fonctionne"); here the tuner searches this
 * library's own configuration space for one problem: the tile plan (0-8 above), K cut into 2, 4
 * or 8 slices through the workspace or across a cluster of 2, 4 or 8 CTAs (few-tile problems),
 * and the raster group of the persistent tile order (8, 16 or 32 m-blocks; many-tile problems).
 *
 * gemm_autotune -- times every candidate configuration on the given operands and records the
 * fastest in a per-process table.  Later calls of the same problem -- same device SM count,
 * form, sizes, operand and output types, beta == 0 or not, and the same alignment of A, B and C
 * (which decides the pre-pass and store paths) -- take the recorded configuration instead of
 * the library's cost model, unless a plan or split is forced (gemm_bf16_set_plan, the
 * GEMM_BF16_* variables).
 *
 *   in_type  0: bf16 operands, 1: fp16 operands.
 *   form     0: gemm_bf16 / gemm_f16 (batch must be 1; stride_b, stride_c, index and n_unique
 *               are ignored); 1: the batched shared-W form (B = X N-major, stride_b = stride_x,
 *               stride_c = stride_y); 2: the deduplicated shared-W form (bf16 only; index and
 *               n_unique as in gemm_bf16_batched_shared_w_dedup).
 *   Other arguments as in the matching entry point.  C is NOT written: candidates write into
 *   a scratch copy of C taken from the library's workspace pool.  *best_us (if best_us != NULL)
 *   receives the winner's time per call in microseconds.
 * Synchronous: returns after the measurements (it synchronizes `stream`); do not call it
 * during stream capture.  Returns GEMM_OK, or an argument/CUDA error; GEMM_OK with nothing
 * recorded when there is nothing to compute (an empty problem, K == 0 or alpha == 0).
 */
GEMM_API gemm_status_t gemm_autotune(int in_type, int form, int batch, int n_unique, int M, int N, int K,
                                     const void* A, int lda, const void* B, int ldb, long long stride_b,
                                     const int* index, const void* C, int ldc, long long stride_c,
                                     gemm_out_t out_type, float alpha, float beta, struct CUstream_st* stream,
                                     float* best_us);

/* Empties the tuning table. */
GEMM_API gemm_status_t gemm_tuning_clear(void);

/* Number of problems in the tuning table. */
GEMM_API int gemm_tuning_size(void);

/*
 * gemm_tuning_save / gemm_tuning_load -- write the tuning table to a text file, or add a file's
 * entries to it (same key: replaced).  One line per problem:
 *   gemmtune1 sms batch M N K n_unique b_mn in_f16 out c_read a_ok b_ok c_tma plan splits csplit group_m us
 * (b_mn: batched forms; c_read: beta != 0; a_ok/b_ok: operand read in place by TMA; c_tma: C
 * stored by TMA; splits: workspace K slices, 0 for stream-K; csplit: cluster K slices; us:
 * measured time).
 * Lines starting with '#' and empty lines are skipped.  A file that cannot be opened, or any
 * malformed line or impossible configuration, returns GEMM_ERR_INVALID_ARG and loads nothing.
 */
GEMM_API gemm_status_t gemm_tuning_save(const char* path);
GEMM_API gemm_status_t gemm_tuning_load(const char* path);

/*
 * gemm_last_config -- the configuration of the calling thread's most recent GEMM kernel launch
 * (plan, workspace K slices -- 0 for stream-K --, cluster K slices, raster group); plan -1 before
 * any launch.
 * GEMM_ERR_INVALID_ARG if a pointer is NULL.
 */
GEMM_API gemm_status_t gemm_last_config(int* plan, int* splits, int* csplit, int* group_m);

/* Library version as an integer (major*10000 + minor*100 + patch). */
GEMM_API int gemm_bf16_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GEMM_BF16_H */
