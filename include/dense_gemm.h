/*
 * dense_gemm.h -- C ABI of the B200 (sm_100a) tiled GEMM library.
 *
 * The operation is the tiled dense GEMM the pages build in Triton:
 *
 *     C = act(A . B + bias)          act = identity or ReLU
 *
 * with fp16 or bf16 inputs and an fp32 accumulator ("用Triton跨芯片优化GEMM：
 * 实测性能反超原生算子库", section 2.1 for the tiled product with an fp32
 * accumulator and section 3.4 for the bias + ReLU epilogue fused into the
 * same kernel; "Triton 学习笔记", section 2.1: always accumulate in fp32).
 * The grouped entry point runs the many GEMMs of an MoE layer in a single
 * launch (first page, section 2.3).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.   All matrices are addressed through a leading dimension, in
 *           elements, the way the pages pass a stride per dimension
 *           ("Triton 学习笔记" section 1, strides and transposes):
 *             A[i,k] = A[i*lda + k]                        (row-major, M x K)
 *             B[k,j] = B[k*ldb + j]                        (row-major, K x N)
 *             B[k,j] = B[j*ldb + k]  with GEMM_B_COL_MAJOR (stored N x K)
 *             C[i,j] = C[i*ldc + j]                        (row-major, M x N)
 *           bias is a length-N vector of the input type, broadcast over rows.
 * Memory.   Every pointer except the grouped call's host scalars is a DEVICE
 *           pointer owned by the caller.  The library never frees or keeps
 *           a reference to a caller buffer after the call.  Its own device
 *           memory is a status word per device and, only for calls that need
 *           it, per-stream scratch: split-K / stream-K partial tiles, tile
 *           counters and the im2col matrix of conv2d_im2col, each allocated
 *           with cudaMalloc on the first such call on a stream and grown on
 *           demand (gemm_splitk_noalloc never allocates).  The scratch is
 *           keyed by the stream handle and kept until gemm_free_scratch().
 *           Destroy a stream only after gemm_free_scratch(stream), or a new
 *           stream that is given the same handle would share its scratch.
 * Alignment. A, B and C must be 16-byte aligned; lda*sizeof(input),
 *           ldb*sizeof(input) and ldc*sizeof(output) must be multiples of 16
 *           bytes (the tensor-memory-access unit copies 16-byte granules):
 *           multiples of 8 elements for 16-bit data, 4 for fp32.
 *           bias needs only its element alignment.  Anything else returns
 *           GEMM_ERR_MISALIGNED; there is no slower fallback.
 * Sizes.    M, N, K >= 0.  M == 0 or N == 0 is a no-op that returns GEMM_OK.
 *           K == 0 writes C = act(bias) (or 0) -- the plain definition.
 * Streams.  `stream` is a cudaStream_t (NULL = the legacy default stream).
 *           Calls are asynchronous: GEMM_OK means the work was enqueued;
 *           a device-side fault shows up at the caller's next synchronisation,
 *           and a watchdog time-out is reported by gemm_device_status().
 * Graphs.   Calls may be captured into a CUDA graph (stream capture).  A
 *           capture cannot allocate, so make one uncaptured call of the same
 *           shape and config on the capture stream first: it sizes that
 *           stream's scratch.  Kernels leave their split-K / stream-K tile
 *           counters at zero, so a graph replays any number of times.
 * Errors.   Every function returns a gemm_status; nothing throws, aborts or
 *           exits.  Argument errors are detected before anything is launched.
 * Threads.  All entry points are thread-safe.  The only mutable global state
 *           is a per-device cache (SM count, status-word address, kernel
 *           attributes) filled once per device, and the config override.
 */
#ifndef DENSE_GEMM_H
#define DENSE_GEMM_H

#include <stdint.h>

#if defined(__GNUC__)
#define GEMM_API __attribute__((visibility("default")))
#else
#define GEMM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GEMM_OK = 0,
  GEMM_ERR_INVALID_ARG = -1,    /* null pointer, negative size, ld too small */
  GEMM_ERR_UNSUPPORTED = -2,    /* unknown dtype, epilogue bit or config id */
  GEMM_ERR_MISALIGNED = -3,     /* pointer or leading dimension breaks the 16-byte rule */
  GEMM_ERR_CUDA = -4,           /* a CUDA runtime / driver call failed (incl. no device) */
  GEMM_ERR_DEVICE_TIMEOUT = -5  /* a kernel's bounded wait ran out (see gemm_device_status) */
} gemm_status;

typedef enum {
  GEMM_F16 = 0,          /* fp16 in, fp32 accumulate, fp16 out (round to nearest even) */
  GEMM_BF16 = 1,         /* bf16 in, fp32 accumulate, bf16 out (round to nearest even) */
  GEMM_F16_OUT_F32 = 2,  /* fp16 in, fp32 accumulate, fp32 out */
  GEMM_BF16_OUT_F32 = 3, /* bf16 in, fp32 accumulate, fp32 out */
  GEMM_F32_TF32 = 4      /* fp32 in, multiplied as tf32 (low 13 mantissa bits ignored),
                            fp32 accumulate, fp32 out; bias fp32; gemm() and
                            gemm_strided_batched() only, 128 x 128/256 tiles */
} gemm_dtype;

/* `epilogue` bits. */
#define GEMM_EPI_BIAS 0x1u     /* add bias[j] (input dtype) to every row, in fp32 */
#define GEMM_EPI_RELU 0x2u     /* then max(x, 0), before the output cast */
#define GEMM_B_COL_MAJOR 0x100u /* B is stored N x K: B[k,j] = B[j*ldb + k] */

/*
 * gemm -- C = act(A . B + bias) on one GPU, one launch.
 *
 * Defined by "用Triton跨芯片优化GEMM" section 2.1 (tiled GEMM, fp32
 * accumulator) and section 3.4 (bias and ReLU applied to the accumulator
 * inside the kernel before the single store).  The result of each element is
 * the exact sum of its K products rounded only by the fp32 accumulation (in
 * an unspecified order) and by the final cast.
 *
 *   M, N, K   problem size (elements), each >= 0
 *   A         device, M x K, leading dimension lda (>= K when K > 0)
 *   B         device, K x N row-major with ldb >= N, or N x K (ldb >= K)
 *             with GEMM_B_COL_MAJOR
 *   C         device, M x N, ldc >= N, output dtype per `dtype`; C must not
 *             overlap A, B or bias
 *   bias      device, N elements of the input dtype; required iff
 *             GEMM_EPI_BIAS, ignored otherwise
 *   epilogue  OR of GEMM_EPI_BIAS, GEMM_EPI_RELU, GEMM_B_COL_MAJOR
 *   dtype     a gemm_dtype
 *   stream    cudaStream_t
 * Returns GEMM_OK or an error status; on error nothing was launched.
 */
GEMM_API int gemm(int M, int N, int K, const void* A, int64_t lda, const void* B, int64_t ldb, void* C,
         int64_t ldc, const void* bias, unsigned epilogue, int dtype, void* stream);

/*
 * gemm_strided_batched -- `batch` independent GEMMs in one launch
 * ("用Triton跨芯片优化GEMM" section 4.3 benchmarks single and multi-batch
 * GEMMs).  For b in [0, batch):
 *     C_b = act(A_b . B_b + bias_b),  X_b = X + b*stride_x  (elements)
 * with every other argument as in gemm() (one lda/ldb/ldc, one layout flag,
 * one dtype for all batches).  gemm() is this call with batch = 1.
 *
 *   batch      >= 0; 0 is a no-op
 *   stride_a   0 (every batch reads the same A) or >= lda*M
 *   stride_b   0 (shared B) or >= ldb*K (row-major) / ldb*N (column-major)
 *   stride_c   >= ldc*M: outputs never overlap
 *   stride_bias 0 (one bias vector for all batches) or the distance between
 *              the batches' length-N bias vectors
 * stride_a*2, stride_b*2 and stride_c*sizeof(output) must be multiples of 16
 * bytes when batch > 1 (else GEMM_ERR_MISALIGNED); a stride that breaks the
 * rules above returns GEMM_ERR_INVALID_ARG.  With batch == 1 the strides are
 * ignored.
 */
GEMM_API int gemm_strided_batched(int batch, int M, int N, int K, const void* A, int64_t lda,
                                  int64_t stride_a, const void* B, int64_t ldb, int64_t stride_b,
                                  void* C, int64_t ldc, int64_t stride_c, const void* bias,
                                  int64_t stride_bias, unsigned epilogue, int dtype, void* stream);

/*
 * conv2d_im2col -- 2-D convolution as a GEMM ("FlagOS众智跨芯算子优化实践"
 * section 5.3: convolution reuses the GEMM through im2col):
 *
 *   y[n][oh][ow][co] = act( sum_{kh,kw,ci} x[n][ih][iw][ci] * w[kh][kw][ci][co] + bias[co] )
 *   ih = oh*stride_h - pad_h + kh*dil_h,  iw = ow*stride_w - pad_w + kw*dil_w,
 *
 * x taken as 0 outside the image.  The sliding windows are gathered into an
 * (batch*OH*OW) x (KH*KW*cin) matrix, then multiplied by the filter on the
 * tensor cores with bias and ReLU fused into the GEMM epilogue.
 *
 *   x      device, NHWC [batch][H][W][cin], 16-bit (dtype GEMM_F16/BF16[_OUT_F32])
 *   w      device, [KH][KW][cin][cout] (a K x N row-major matrix, K = KH*KW*cin)
 *   y      device, NHWC [batch][OH][OW][cout], OH = (H + 2 pad_h - dil_h (KH-1) - 1)
 *          / stride_h + 1, OW likewise
 *   bias   device, cout elements iff GEMM_EPI_BIAS
 *   epilogue  GEMM_EPI_BIAS | GEMM_EPI_RELU (no layout bits)
 * cout must be a multiple of 8; x, w, y 16-byte aligned.  The gathered matrix
 * lives in a per-stream scratch buffer the library allocates (cudaMalloc) on
 * the first call on a stream and grows when a larger one is needed.
 */
GEMM_API int conv2d_im2col(int batch, int H, int W, int cin, int cout, int KH, int KW,
                           int stride_h, int stride_w, int pad_h, int pad_w, int dil_h, int dil_w,
                           const void* x, const void* w, void* y, const void* bias,
                           unsigned epilogue, int dtype, void* stream);

/*
 * grouped_gemm -- the per-expert GEMMs of an MoE layer in one launch
 * ("用Triton跨芯片优化GEMM" section 2.3: a MoE layer runs dozens of GEMMs).
 *
 * Rows of A (and C) are sorted by group: group g owns rows
 * [r_g, r_g + group_rows[g]) with r_g = sum_{h<g} group_rows[h], and
 *     C[r, :] = act(A[r, :] . B_g + bias_g)   for every row r of group g,
 * B_g = B + g*stride_b (same layout rules as gemm(), ldb shared by all
 * groups), bias_g = bias + g*N.
 *
 *   num_groups  1..1024
 *   group_rows  DEVICE int32[num_groups]; read by the kernel, so a routing
 *               step earlier on the same stream may produce it (no host sync)
 *   total_rows  host int, the rows of A and C (= sum of group_rows); rows the
 *               device counts place beyond total_rows are neither read nor
 *               written, and a negative count is treated as 0 -- both set
 *               the device status (gemm_device_status) to GEMM_ERR_INVALID_ARG
 *   N, K        per-group GEMM size (shared by all groups)
 *   A, lda      device, total_rows x K
 *   B, ldb      device, num_groups matrices, each K x N (or N x K with
 *               GEMM_B_COL_MAJOR); stride_b elements apart (stride_b*2 a
 *               multiple of 16 bytes)
 *   C, ldc      device, total_rows x N
 *   bias        device, num_groups x N (input dtype) iff GEMM_EPI_BIAS
 * Empty groups cost nothing; rows of a group's last tile that belong to the
 * next group are computed but never stored.
 */
GEMM_API int grouped_gemm(int num_groups, const int32_t* group_rows, int total_rows, int N, int K,
                 const void* A, int64_t lda, const void* B, int64_t ldb, int64_t stride_b,
                 void* C, int64_t ldc, const void* bias, unsigned epilogue, int dtype,
                 void* stream);

/* Human-readable name of a gemm_status value (static storage). */
GEMM_API const char* gemm_status_string(int status);

/* Library version string (static storage). */
GEMM_API const char* gemm_version(void);

/*
 * gemm_device_status -- synchronise `stream`, then read the current device's
 * status word that the kernels' watchdogs and argument checks write.  Returns
 * GEMM_OK, GEMM_ERR_DEVICE_TIMEOUT (a bounded wait inside a kernel ran out
 * and the kernel returned early; its output is undefined) or
 * GEMM_ERR_INVALID_ARG (grouped row counts were inconsistent).  With clear
 * != 0 the word is reset to 0 afterwards.
 * After a time-out, the pieces of a split tile that gave up may have left
 * that tile's counter set in the stream's scratch: call
 * gemm_free_scratch(stream, 0) before the next split-K / stream-K call on
 * that stream (the next call then allocates zeroed counters).
 * gemm_splitk_noalloc clears its counters on every call and needs nothing.
 */
GEMM_API int gemm_device_status(void* stream, int clear);

/*
 * gemm_set_timeout_ns -- bound, in nanoseconds, of every wait inside the
 * kernels (default 2e9).  A wait that runs out sets the device status word,
 * and every warp of that block leaves its loop, waits (again bounded) for
 * its own copies and MMAs in flight, frees its tensor memory and returns.
 * 0 restores the default.  Returns the previous value.
 */
GEMM_API uint64_t gemm_set_timeout_ns(uint64_t ns);

/*
 * gemm_watchdog_selftest -- launch one block whose wait is on a barrier that
 * nothing ever completes, with the given bound; the kernel must give up,
 * record GEMM_ERR_DEVICE_TIMEOUT and return.  Synchronises `stream` and
 * returns what gemm_device_status(stream, 1) then reports (expected:
 * GEMM_ERR_DEVICE_TIMEOUT).  No fault, trap or hang is involved.
 */
GEMM_API int gemm_watchdog_selftest(uint64_t timeout_ns, void* stream);

/*
 * gemm_free_scratch -- synchronise `stream` and free the scratch the library
 * holds for it on the current device (NULL is the default stream).  With
 * all_streams != 0, `stream` is ignored and every stream's scratch on the
 * current device is freed, each after synchronising its stream.  Later calls
 * allocate anew.  Returns GEMM_OK (also when there was nothing to free) or
 * GEMM_ERR_CUDA.
 */
GEMM_API int gemm_free_scratch(void* stream, int all_streams);

/* ---- tracing ----------------------------------------------------------- */

/* Events a traced launch records per block (indices into its row). */
enum {
  GEMM_TRACE_ENTRY = 0,      /* the block started */
  GEMM_TRACE_SETUP = 1,      /* barriers, tensor memory and tables ready */
  GEMM_TRACE_FIRST_LOAD = 2, /* the producer issued its first copy */
  GEMM_TRACE_FIRST_DATA = 3, /* the MMA issuer saw its first full stage */
  GEMM_TRACE_LAST_MMA = 4,   /* the MMA issuer committed its last accumulator */
  GEMM_TRACE_FIRST_EPI = 5,  /* the first epilogue warp got its first accumulator */
  GEMM_TRACE_EPI_DONE = 6,   /* that warp finished its last tile (stores issued) */
  GEMM_TRACE_EXIT = 7,       /* the block is about to return */
  GEMM_TRACE_EVENTS = 8
};

/*
 * gemm_set_trace -- record where launches spend their time.  `buffer` is
 * caller-owned device memory of `bytes` bytes; NULL (or bytes too small for
 * one block) turns tracing off, which is the default.  While it is set,
 * every GEMM kernel launched by this library writes, for each block b below
 * bytes / (8 * GEMM_TRACE_EVENTS), the device's global timer (nanoseconds,
 * uint64) at event e into buffer[b * GEMM_TRACE_EVENTS + e].  Events a block
 * never reaches (a block with no tile has no FIRST_DATA) keep their old
 * value, so zero the buffer before the launch of interest.  Every launch
 * overwrites the rows of its blocks, so trace one launch at a time.  The
 * setting is process-wide and not synchronised with launches in flight.
 * Returns GEMM_OK, or GEMM_ERR_MISALIGNED for a buffer that is not 8-byte
 * aligned.
 */
GEMM_API int gemm_set_trace(void* buffer, int64_t bytes);

/* ---- tile configurations (the offline sweep's table) ------------------- */

/* Number of tile configurations compiled into the library. */
GEMM_API int gemm_num_configs(void);

/* Name of configuration `id` into buf (NUL-terminated, truncated to
 * buflen); returns GEMM_OK or GEMM_ERR_UNSUPPORTED for a bad id. */
GEMM_API int gemm_config_name(int id, char* buf, int buflen);

/* Id of the configuration gemm() would use for this problem (the table's
 * choice, or the forced id), or a negative gemm_status if none applies. */
GEMM_API int gemm_select_config(int M, int N, int K, int dtype, unsigned epilogue);

/* Force every later gemm() / grouped_gemm() call in this process onto
 * configuration `id` (-1 restores the table).  For the offline sweep and for
 * tests; a forced config that cannot run a problem makes that call return
 * GEMM_ERR_UNSUPPORTED.  Returns GEMM_OK or GEMM_ERR_UNSUPPORTED. */
GEMM_API int gemm_force_config(int id);

/* ---- split-K without any device allocation ------------------------------ */

/* Size of the library's fixed split-K scratch array (bytes per device). */
#define GEMM_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * gemm_splitk_noalloc -- the split-K GEMM (C = act(A . B + bias), arguments
 * exactly as for gemm()) with its scratch memory taken from a fixed array that
 * is part of the library itself, so the call never allocates device memory.
 * The pages have no counterpart to this entry point.
 *
 * Who needs it: gemm() gets its split-K scratch from cudaMalloc, once per
 * stream.  Some callers cannot allow that -- a service whose device memory
 * is carved up by its own allocator up front (cudaMalloc behind its back
 * breaks its accounting or fails once the pool owns the GPU), or a
 * latency-critical loop that cannot take cudaMalloc's implicit device-wide
 * synchronisation.  This entry point calls no cudaMalloc, cudaFree or any
 * other allocating routine.
 *
 *   splits   split-K factor, 1..64: each output tile's K range is cut into
 *            `splits` pieces (fewer if K is short; empty pieces are dropped)
 *   others   as gemm().  Tiles are 128 x 128, or 128 rows of B by 16 rows
 *            of A when M <= 32 and B is column-major.
 * Limits: the scratch holds GEMM_NOALLOC_SCRATCH_BYTES per device: 16 KiB of
 * tile counters (at most 4096 output tiles) and the fp32 partial tiles
 * (tiles x pieces x 128 x tile-width x 4 bytes).  A problem that needs more
 * returns GEMM_ERR_UNSUPPORTED before anything is launched.
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents; each call first clears the counters it uses on `stream`.
 * Calls whose kernels overlap on the GPU (different streams, or graph
 * branches) race on the array and produce wrong results: serialise them.
 * Set-up: the first call on each device (with that device current) looks up
 * the array's device address (cudaGetSymbolAddress); make that first call
 * before any stream capture.  Every GPU that loads the library holds the
 * array until the process exits.
 */
GEMM_API int gemm_splitk_noalloc(int M, int N, int K, const void* A, int64_t lda, const void* B,
                                 int64_t ldb, void* C, int64_t ldc, const void* bias,
                                 unsigned epilogue, int dtype, int splits, void* stream);

/* ---- host-side helpers (no GPU needed) --------------------------------- */

/* Bytes of the shared-memory operand ring for a BM x BN output tile with a
 * BK-deep K step and `stages` buffers: (BM*BK + BK*BN) * elem_bytes * stages,
 * the formula of the crowd-sourced tuning page ("FlagOS众智跨芯算子优化实践",
 * section 2.1; its worked example 128/128/32, fp16, 3 stages = 49152 bytes).
 * Returns -1 on a negative argument. */
GEMM_API int64_t gemm_smem_ring_bytes(int bm, int bn, int bk, int stages, int elem_bytes);

/* K-loop trip count ceil(K / bk) (same page, section 2.2: K = 512 with
 * BLOCK_K = 64 runs 8 iterations).  Returns -1 on a bad argument. */
GEMM_API int gemm_k_iterations(int K, int bk);

/* Grouped-M rasterisation of a linear tile index onto a grid_m x grid_n tile
 * grid, groups of group_m tile rows walked column by column ("Triton 学习笔记"
 * section 2.3.7 on L2 reuse; the grouped pid mapping of the Gluon/Triton
 * page's matmul example).  Writes the tile's row and column block.  Returns
 * GEMM_OK or GEMM_ERR_INVALID_ARG. */
GEMM_API int gemm_tile_coord(int64_t tile, int grid_m, int grid_n, int group_m, int* m_block,
                    int* n_block);

#ifdef __cplusplus
}
#endif

#endif /* DENSE_GEMM_H */
