/*
 * b200gemm -- dense GEMM for NVIDIA B200 (sm_100a), plain C ABI.
 *
 *   C = A . B      A: M x K,  B: K x N,  C: M x N
 *
 * The operation is the matrix product C_{MxN} = A_{MxK} B_{KxN} of
 * "GPU 执行模型" (wineandchord.com/llm/systems/gpu-execution/), section
 * "Tile 的容量约束"; the kernels follow the Blackwell GEMM construction of
 * "Modern GPU Programming For MLSys - 书籍总结" (omica.com.cn), part III
 * (steps 1-9: tiling, K loop, TMA, software pipeline, persistent kernel,
 * warp specialisation, 2-CTA cluster), and the argument contract below
 * follows the checklist of "GPU 执行模型", section "正确性契约" (shape,
 * stride, layout, dtype, alignment, tails, accumulation and rounding,
 * aliasing, stream lifetime, determinism).
 *
 * Layouts (all row-major with explicit leading dimensions, in ELEMENTS):
 *   A  element (i,k) at A[i*lda + k]            (M rows of K)
 *   B  element (k,j) at B[j*ldb + k]            (stored K-major: N rows of K)
 *   C  element (i,j) at C[i*ldc + j]            (M rows of N)
 *   MXFP8 scales: sfa[i*(K/32) + kb], sfb[j*(K/32) + kb], one E8M0 byte per
 *   32 consecutive K elements (kb = k/32), rows packed (leading dim K/32).
 *
 * Ownership: every pointer is a DEVICE pointer owned by the caller, valid
 * until the work queued on `stream` has finished.  The library keeps, per
 * device, a small status block (allocated on the first call on a device of
 * every entry point except gemm_bf16_noalloc, which uses a static array),
 * cached launch attributes and, for the skinny and block-scaled paths, a
 * workspace that grows on demand.  A workspace that a larger one replaces
 * is kept, never freed, while the library is loaded.
 *
 * Execution: calls are asynchronous on `stream` (0 = the legacy default
 * stream) and never synchronise, except gemm_check_device_status().
 * gemm_bf16 and gemm_mxfp8 overwrite C; gemm_bf16_ex and gemm_bf16_fused
 * add alpha/beta, a bias and an activation.  Results are deterministic for
 * a given shape and configuration (fixed per-element accumulation order).
 *
 * CUDA graphs: every call may be captured into a graph, whose replays then
 * reuse the captured addresses ("GPU 执行模型", section "Launch、CUDA Graph
 * 与动态 shape": fixed shapes and reusable input, output and workspace
 * addresses).  One-time set-up cannot run inside a capture: the first call
 * on a device, the first call of each kernel configuration and output
 * type, and any workspace growth return GEMM_ERR_CAPTURE there, with
 * nothing queued.  So make one call of the same shapes and types outside
 * the capture first.  Because replaced workspaces are never freed, a graph
 * captured before a workspace grew still replays on valid memory.
 * gemm_check_device_status() synchronises and may not be captured.
 *
 * Errors: every function returns a status and never aborts or throws.
 * Argument checks run on the host before anything is queued.  A device-side
 * watchdog bounds every wait inside the kernels; if one expires, the kernel
 * records GEMM_ERR_TIMEOUT in the status block and exits cleanly, and the
 * next gemm_check_device_status() reports it.
 */
#ifndef B200GEMM_H
#define B200GEMM_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define B200GEMM_API __attribute__((visibility("default")))
#else
#define B200GEMM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GEMM_OK = 0,
    GEMM_ERR_INVALID_VALUE = 1,     /* negative size, ld too small, bad enum, null pointer */
    GEMM_ERR_MISALIGNED = 2,        /* pointer or ld*elem_size not a multiple of 16 bytes */
    GEMM_ERR_ALIAS = 3,             /* C overlaps an input */
    GEMM_ERR_UNSUPPORTED_DEVICE = 4,/* no device, or not compute capability 10.0 */
    GEMM_ERR_LAUNCH = 5,            /* a CUDA runtime call failed (see gemm_last_cuda_error) */
    GEMM_ERR_TIMEOUT = 6,           /* a kernel's bounded wait expired (device watchdog) */
    GEMM_ERR_TOO_LARGE = 7,         /* a dimension exceeds 2^31-1 (TMA coordinates are int32) */
    GEMM_ERR_CAPTURE = 8            /* one-time set-up requested inside a stream capture (below) */
} gemm_status_t;

typedef enum {
    GEMM_OUT_F32 = 0,               /* C is float32 */
    GEMM_OUT_BF16 = 1               /* C is bfloat16, rounded to nearest even */
} gemm_out_t;

/* How an operand is stored (gemm_bf16_ex).  K-major is the layout of
 * gemm_bf16: A as M rows of K (a(i,k) at A[i*lda + k]), B as N rows of K
 * (b(k,j) at B[j*ldb + k]).  MN-major stores the other way round: A as K rows
 * of M (a(i,k) at A[k*lda + i]), B as K rows of N (b(k,j) at B[k*ldb + j],
 * the row-major K x N matrix of C = A.B as most frameworks hold it). */
typedef enum {
    GEMM_LAYOUT_KMAJOR = 0,
    GEMM_LAYOUT_MNMAJOR = 1
} gemm_layout_t;

/* Pointwise activation of the fused epilogue (gemm_bf16_fused). */
typedef enum {
    GEMM_ACT_NONE = 0,
    GEMM_ACT_RELU = 1,              /* x < 0 ? 0 : x  (NaN stays NaN) */
    GEMM_ACT_GELU = 2,              /* x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)), erff in fp32 */
    GEMM_ACT_GELU_TANH = 3          /* 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), the tanh
                                       form of GELU (within 4.8e-4 of GELU), with the hardware
                                       tanh approximation (PTX tanh.approx.f32) */
} gemm_act_t;

/* Kernel configurations.  GEMM_CFG_AUTO picks by shape (gemm_select_config);
 * the others force a configuration (for tests and benchmarks) through
 * gemm_force_config().
 *
 * Narrow tail: on 1CTA_128x128, 1CTA_128x256, 2CTA_256x256 and their CLC
 * forms, with B stored N x K, a last wave of tiles that would occupy at most
 * half of the co-resident clusters runs as half-width units (BN / 2 columns
 * each), so that the idle clusters take the other halves.  The result is the
 * same element by element; only the schedule changes.  ("GPU 执行模型",
 * section "编译与 autotune": tile shape and persistent strategy.) */
typedef enum {
    GEMM_CFG_AUTO = 0,
    GEMM_CFG_1CTA_128x256 = 1,      /* one CTA per tile, tile 128 x 256, tcgen05 cta_group::1 */
    GEMM_CFG_1CTA_128x128 = 2,      /* one CTA per tile, tile 128 x 128 */
    GEMM_CFG_2CTA_256x256 = 3,      /* CTA pair per tile, tile 256 x 256, cta_group::2 */
    GEMM_CFG_SKINNY = 4,            /* M <= 256: swap A/B (128 rows of B per MMA).  For M <= 64
                                       with enough 128-row tiles of B, K split over a cluster of 2
                                       or 4 CTAs per tile, partials summed through shared memory;
                                       otherwise stream-K over all SMs with a deterministic fix-up
                                       of split tiles in a library-owned workspace (cudaMalloc on
                                       first use) */
    GEMM_CFG_2CTA_256x256_CLC = 5,  /* as 2CTA_256x256, tiles handed out by Cluster Launch Control:
                                       one cluster per tile, running pairs claim pending ones */
    GEMM_CFG_1CTA_128x256_CLC = 6,  /* as 1CTA_128x256 with Cluster Launch Control */
    GEMM_CFG_MXFP8_1CTA_128x256 = 7,/* gemm_mxfp8: one CTA per 128 x 256 tile */
    GEMM_CFG_MXFP8_2CTA_256x256 = 8,/* gemm_mxfp8: CTA pair per 256 x 256 tile, cta_group::2 */
    GEMM_CFG_2CTA_512x256_CLC = 9,  /* CTA pair per 512 x 256 tile, two MMA consumers sharing each
                                       B k-tile, one TMEM accumulator each (TMEM single-buffered);
                                       Cluster Launch Control; chosen by shape only for K >= 8192,
                                       e.g. 8192 x 8192 x 8192 */
    GEMM_CFG_2CTA_256x256_SK = 10,  /* CTA pair per 256 x 256 tile, stream-K: every co-resident pair
                                       takes an equal contiguous share of the (tile, 64-wide K block)
                                       iterations; a tile split between pairs is summed from fp32
                                       partials by its last contributor, in contributor order
                                       (deterministic); uses the library-owned split workspace;
                                       never chosen by shape */
    GEMM_CFG_2CTA_256x224 = 11,     /* CTA pair per 256 x 224 tile (fills the waves of some shapes
                                       better); fp32 C with B stored K-major only (bf16 C or a B
                                       stored K x N runs 2CTA_256x256); never chosen by shape */
    GEMM_CFG_1CTA_128x128_SPLITK = 12, /* cluster split-K: a cluster of S = 2, 4 or 8 CTAs per 128 x 128
                                       tile, each over a contiguous share of K; member j sums
                                       column slice j from every member's fp32 partial in member
                                       order (deterministic), the partials crossing through
                                       distributed shared memory (no workspace).  S: the largest
                                       whose clusters all fit at once and give every member two
                                       64-wide K blocks (else the unsplit 1CTA_128x128); the
                                       environment variable B200GEMM_KSPLIT = 2, 4 or 8, read
                                       once, forces it (tests) */
    GEMM_CFG_1CTA_128x256_SPLITK = 13, /* the same with 128 x 256 tiles (else 1CTA_128x256) */
    GEMM_CFG_SMALL = 14,            /* latency path for tiny products: warp-level mma.sync
                                       (m16n8k16, bf16 in, fp32 accumulate) straight from global
                                       memory, 32 x 32 of C per CTA; no tensor memory, no shared
                                       memory, no barriers.  Chosen by shape below a measured work
                                       bound (gemm_select_config); any size when forced */
    GEMM_CFG_COUNT_ = 15
} gemm_config_t;

/*
 * gemm_bf16: C = A . B with bf16 A and B, fp32 accumulation in tensor memory,
 * C written as fp32 or bf16 (c_type): the matrix product C_{MxN} = A_{MxK}
 * B_{KxN} of "GPU 执行模型", section "Tile 的容量约束", with the argument
 * rules of that page's section "正确性契约" (shape, stride, layout, dtype,
 * alignment, tail predicates, accumulation and rounding, aliasing).
 *
 *   A, B     device pointers to bfloat16; C device pointer to c_type
 *   M, N, K  >= 0.  M == 0 or N == 0: nothing to do (GEMM_OK).
 *            K == 0 with M, N > 0: C is set to zero (the empty sum).
 *   lda, ldb >= K, ldc >= N (elements); lda*2, ldb*2 and ldc*sizeof(c_type)
 *            multiples of 16 bytes; A, B, C 16-byte aligned.
 *   Tails: any M, N, K are accepted; partial tiles are zero-filled on load
 *   and clipped on store, so no element outside the M x N (x K) ranges is
 *   read or written.
 *   C must not overlap A or B.
 */
B200GEMM_API gemm_status_t gemm_bf16(const void *A, const void *B, void *C,
                        int64_t M, int64_t N, int64_t K,
                        int64_t lda, int64_t ldb, int64_t ldc,
                        gemm_out_t c_type, cudaStream_t stream);

/*
 * gemm_bf16_ex: C = alpha * A . B + beta * C, with each operand stored
 * K-major or MN-major (gemm_layout_t).  bf16 A and B, fp32 accumulation,
 * C as c_type; alpha and beta are applied in fp32 to the fp32 accumulator
 * and the (widened) old C before the single rounding to c_type.  C is read
 * only when beta != 0 (beta == 0: C's old contents, NaN included, are
 * ignored).  K == 0 gives C = beta * C.  These are the epilogue and operand
 * variants of a GEMM's correctness contract ("GPU 执行模型", section
 * "正确性契约": layout, stride, which buffers are read and written).
 *   a_layout K-major: lda >= K; MN-major: lda >= M.
 *   b_layout K-major: ldb >= K; MN-major: ldb >= N.
 * Other rules as gemm_bf16, which is gemm_bf16_ex with both operands
 * K-major, alpha = 1, beta = 0.
 */
B200GEMM_API gemm_status_t gemm_bf16_ex(const void *A, const void *B, void *C,
                                        int64_t M, int64_t N, int64_t K,
                                        int64_t lda, int64_t ldb, int64_t ldc,
                                        gemm_out_t c_type, gemm_layout_t a_layout, gemm_layout_t b_layout,
                                        float alpha, float beta, cudaStream_t stream);

/*
 * gemm_bf16_fused: C = act(alpha * A . B + beta * C + bias), the bias one
 * fp32 value per column of C (bias[j] for every row), act a gemm_act_t.
 * The pointwise steps run on the fp32 accumulator in registers inside the
 * GEMM's write-back, in that order, before the single rounding to c_type:
 * the unfused sequence would write the M x N intermediate to memory and
 * read it back, two intermediate-sized transfers that fusion saves ("GPU
 * 执行模型", section "Fusion 的收益与上限").
 *   bias  device pointer to N floats, 16-byte aligned, or NULL (no bias);
 *         it must not overlap C.  Read only, owned by the caller.
 *   act   GEMM_ACT_NONE, GEMM_ACT_RELU, GEMM_ACT_GELU or GEMM_ACT_GELU_TANH;
 *         anything else is GEMM_ERR_INVALID_VALUE.
 * K == 0 gives C = act(beta * C + bias).  Every other argument, rule and
 * layout is gemm_bf16_ex's, which is gemm_bf16_fused with bias == NULL and
 * act == GEMM_ACT_NONE.
 */
B200GEMM_API gemm_status_t gemm_bf16_fused(const void *A, const void *B, void *C,
                                           int64_t M, int64_t N, int64_t K,
                                           int64_t lda, int64_t ldb, int64_t ldc,
                                           gemm_out_t c_type, gemm_layout_t a_layout, gemm_layout_t b_layout,
                                           float alpha, float beta, const float *bias, gemm_act_t act,
                                           cudaStream_t stream);

/*
 * gemm_bf16_allgather: one GPU's part of a row-sharded C = A . B with the
 * all-gather of C fused into the GEMM's write-back.
 *
 * With A's rows split over G GPUs (each holding its slab of A and all of B),
 * every GPU computes its rows of C and every GPU needs all of C: the GEMM is
 * followed by an all-gather.  Here one kernel does both: each finished chunk
 * of this GPU's slab goes from shared memory straight into every destination
 * C by TMA stores, so the transfer to the other GPUs overlaps the next tiles'
 * math instead of following the whole GEMM.  (The row-sharded GEMM is the
 * distributed step the tile ledger of "GPU 执行模型", section "Tile 小账本",
 * leaves to a later chapter; fusing its gather into the epilogue is this
 * library's design.)
 *
 *   A, B      this GPU's slab of A (M rows, row-major, lda >= K) and all of B
 *             (stored N x K, ldb >= K), bf16, on this GPU.
 *   C_dst     HOST array of n_dst (1 .. 8) pointers, each the base of a whole
 *             C (c_type, leading dimension ldc >= N, at least row0 + M rows):
 *             this GPU's own C first, then the other GPUs' C buffers mapped
 *             into this process (CUDA IPC or symmetric memory).  The slab is
 *             written to rows [row0, row0 + M) of every one of them.
 *   M, N, K   the slab's rows, C's columns, the reduction length.
 *   row0      the slab's first row in C.
 *   Other rules (alignment, leading dimensions, tails, K == 0) as gemm_bf16;
 *   no destination's slab may overlap A, B or another destination's slab.
 * It runs the 256 x 256 CTA-pair kernel with Cluster Launch Control.  The
 * call orders nothing across GPUs: a GPU may read its C only after every
 * GPU's call has finished (for example a barrier on each stream after the
 * call).  No TMA load ever reads another GPU's memory; only stores cross.
 */
B200GEMM_API gemm_status_t gemm_bf16_allgather(const void *A, const void *B, void *const *C_dst, int n_dst,
                                               int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                                               int64_t ldc, int64_t row0, gemm_out_t c_type, cudaStream_t stream);

/*
 * gemm_mxfp8: block-scaled C = (sa . A) . (sb . B) with FP8 E4M3 A and B and
 * one E8M0 scale per 32 consecutive K elements of every row of A and of the
 * K-major B -- the block-scaled MMA with its scale factors in tensor memory
 * of "Modern GPU Programming For MLSys - 书籍总结", sections 2.4 and 2.6:
 *
 *   C[i][j] = sum_k (a_ik 2^(sfa[i][k/32]-127)) (b_kj 2^(sfb[j][k/32]-127))
 *
 * fp32 accumulation, C written as bf16 (round to nearest even).
 *   A   M x lda bytes of E4M3 codes (row i, element k at A[i*lda + k])
 *   B   N x ldb bytes of E4M3 codes (stored K-major: b(k,j) at B[j*ldb + k])
 *   sfa M x (K/32) E8M0 bytes, rows packed: sfa[i*(K/32) + k/32]
 *   sfb N x (K/32) E8M0 bytes, rows packed: sfb[j*(K/32) + k/32]
 *   C   M x ldc bf16
 * K must be a multiple of 32; lda and ldb multiples of 16; ldc*2 a multiple
 * of 16; A, B and C 16-byte aligned (the scales need no alignment).  C must
 * not overlap A, B, sfa or sfb.  M == 0 or N == 0: nothing to do; K == 0:
 * C = 0.  An E8M0 byte 0xFF (NaN) makes its block NaN.
 * Each call queues two kernels: a repack of the scales into a per-device
 * workspace of 512 bytes per (128 rows x 128 K) block of A and of B, which
 * the library allocates on first use and grows when a larger problem needs
 * it (cudaMalloc), then the GEMM.  Calls on streams that are not ordered
 * with each other share that workspace and must not overlap.
 */
B200GEMM_API gemm_status_t gemm_mxfp8(const void *A, const uint8_t *sfa, const void *B, const uint8_t *sfb,
                                      void *C, int64_t M, int64_t N, int64_t K,
                                      int64_t lda, int64_t ldb, int64_t ldc, cudaStream_t stream);

/*
 * gemm_bf16_noalloc: gemm_bf16 for callers that cannot allocate device memory.
 * (No counterpart in the pages: it is a packaging choice of this library.)
 *
 * gemm_bf16 allocates a small status block with cudaMalloc on its first call
 * on each device.  Some callers cannot allow that: code that runs while a
 * framework's caching allocator owns the whole device memory, allocator or
 * memory-pool callbacks that must not re-enter the allocator, and latency-
 * critical loops where cudaMalloc's implicit device synchronisation is not
 * allowed.  This entry point computes what gemm_bf16 computes, with the same
 * arguments, checks and kernels, but it allocates nothing: the kernels'
 * scratch (the 16-byte watchdog status block) lives in a static 256-byte
 * device array inside the library, which every GPU that loads the library
 * holds until the process exits.  One difference in kernel choice: where
 * GEMM_CFG_SKINNY would fall back to its stream-K form, whose workspace
 * gemm_bf16 allocates, this runs GEMM_CFG_1CTA_128x128_SPLITK instead (no
 * workspace: its partials meet in shared memory).  A call that would need more scratch than that array is
 * rejected with GEMM_ERR_TOO_LARGE (no shape does today: the scratch does
 * not grow with M, N or K).  Each call queues exactly one kernel.
 *
 * The first call on each device does a one-time set-up with that device
 * current (it looks up the array's device address and zeroes it); make that
 * first call before any stream capture.  The status block then keeps a
 * recorded watchdog timeout until gemm_check_device_status() reads and
 * clears it, exactly as for the other entry points.  All calls share the one
 * array, so calls that overlap on the GPU (different streams, no ordering)
 * race on it.
 */
B200GEMM_API gemm_status_t gemm_bf16_noalloc(const void *A, const void *B, void *C,
                                             int64_t M, int64_t N, int64_t K,
                                             int64_t lda, int64_t ldb, int64_t ldc,
                                             gemm_out_t c_type, cudaStream_t stream);

/* Synchronises `stream`, then reports and clears the device watchdog status
 * of the current device (the status blocks of every entry point, the static
 * one of gemm_bf16_noalloc included): GEMM_OK, or GEMM_ERR_TIMEOUT if a
 * kernel's bounded wait expired since the last check.  GEMM_ERR_LAUNCH if
 * the stream itself reports a CUDA error.  It serves two items of the
 * correctness contract of "GPU 执行模型", section "正确性契约": the
 * lifetime of the stream's asynchronous work (it returns once that work has
 * finished) and the barrier happens-before of the shared-memory stages (the
 * kernels bound every barrier wait, and an expired one is what it reports).
 * The device watchdog itself has no counterpart in the pages. */
B200GEMM_API gemm_status_t gemm_check_device_status(cudaStream_t stream);

/* Detail of the last watchdog event read by gemm_check_device_status():
 * which wait expired (role * 16 + barrier kind) and in which CTA; -1 if none.
 * (No counterpart in the pages.) */
B200GEMM_API void gemm_last_timeout_detail(int32_t *where, int32_t *block);

/* Static description of a status code.  The codes name the argument checks
 * of the correctness contract ("GPU 执行模型", section "正确性契约": shape,
 * stride, alignment, aliasing, stream and capture rules) plus the library's
 * own launch and watchdog failures, which have no counterpart in the pages. */
B200GEMM_API const char *gemm_status_string(gemm_status_t status);

/* The CUDA error behind the last GEMM_ERR_LAUNCH on this host thread. */
B200GEMM_API int gemm_last_cuda_error(void);

/* Force a kernel configuration for subsequent calls in this process
 * (GEMM_CFG_AUTO restores shape-based selection).  A bf16 configuration
 * applies to gemm_bf16, gemm_bf16_ex and gemm_bf16_fused (except that an A
 * stored K x M runs GEMM_CFG_SKINNY as GEMM_CFG_1CTA_128x128_SPLITK) and to
 * gemm_bf16_noalloc (which runs GEMM_CFG_SKINNY's stream-K form as
 * GEMM_CFG_1CTA_128x128_SPLITK); an MXFP8 one applies to gemm_mxfp8, and
 * leaves the bf16 entry points choosing by shape.
 * A forced GEMM_CFG_SKINNY with M > 256 fails with GEMM_ERR_INVALID_VALUE.
 * Returns GEMM_ERR_INVALID_VALUE for an unknown configuration. */
B200GEMM_API gemm_status_t gemm_force_config(gemm_config_t config);

/* The configuration the next gemm_bf16 call with this shape would use.
 * M <= 32 with K >= 4096: GEMM_CFG_SKINNY.  K >= 2048 with at most 74
 * tiles of 128 x 128 (else of 128 x 256): GEMM_CFG_1CTA_128x128_SPLITK
 * (GEMM_CFG_1CTA_128x256_SPLITK).  Every 128 x 128 tile on an SM of its
 * own: GEMM_CFG_1CTA_128x128.
 * Otherwise the configuration with the lowest predicted time among the
 * 1-CTA 128 x 256 (up to two waves), the 256 x 256 pair (static, or with
 * Cluster Launch Control when K > 2048) and, for K >= 8192, the 512 x 256
 * pair tile and the 1-CTA 128 x 256 CLC kernel.  The prediction is a fixed
 * cost plus the waves of tiles times each SM's work per wave, at rates
 * measured on a B200: the autotuning search over tile shape and persistent
 * strategy ("GPU 执行模型", section "编译与 autotune"), done once offline so
 * that no call pays for it.
 * gemm_bf16_ex and gemm_bf16_fused use it too, except that with a non-plain
 * epilogue (beta != 0, alpha != 1, a bias or an activation) they take
 * GEMM_CFG_2CTA_256x256_CLC where this returns GEMM_CFG_2CTA_512x256_CLC
 * (the 256 x 256 tile's second TMEM buffer hides the longer epilogue), and
 * an A stored K x M takes GEMM_CFG_1CTA_128x128_SPLITK where this returns
 * GEMM_CFG_SKINNY. */
B200GEMM_API gemm_config_t gemm_select_config(int64_t M, int64_t N, int64_t K);

/* Number of kernels that one call queues for this shape: gemm_bf16 /
 * gemm_bf16_noalloc (block_scaled = 0) or gemm_mxfp8 (block_scaled = 1);
 * 0 for an empty problem. */
B200GEMM_API int gemm_launches_per_call(int64_t M, int64_t N, int64_t K, int block_scaled);

#ifdef __cplusplus
}
#endif

#endif /* B200GEMM_H */
