/*
 * bq.h -- C ABI of the block-quantised weight GEMV library for B200 (sm_100a).
 *
 * The operation is the decode step of an LLM inference runtime: block-quantised
 * weight matrices are streamed from HBM once per token and multiplied against
 * a small batch of activation vectors, with the dequantisation done inside the
 * dot-product loop so dequantised weights never exist in memory (BaseRT:
 * Best-in-Class LLM Inference on Apple Silicon via Native Metal, gist.science
 * technical summary, "Methodologie" -> "Kernel Fusie en Specialisatie"; the
 * same page's "De 'Big Model' Realiteit" paragraph states that decode is
 * bound by memory bandwidth).
 *
 *   y[b][n] = sum_k deq(W)[n][k] * x[b][k],   0 <= b < B <= 8,  0 <= n < N
 *
 * Block formats (32 consecutive weights along K share one fp16 scale d):
 *   Q8: int8 code q, weight = d * q,        d = fp16(absmax / 127)
 *   Q4: 4-bit code q, weight = d * (q - 8), d = fp16(absmax / 7); byte i
 *       (0..15) of a block holds element i in its low nibble and element
 *       i + 16 in its high nibble.
 *
 * Physical layout of a quantised matrix (bq_qmat), "planes":
 *   codes  : Q4 uint8 [N][K/2], Q8 int8 [N][K]; row n at codes + n*(K/2) (Q4)
 *            or codes + n*K (Q8); block j of a row at byte offset 16*j (Q4) or
 *            32*j (Q8).
 *   scales : fp16 bit patterns, [N][ldS] with ldS = bq_scales_ld(K) =
 *            roundup(K/32, 8); entry (n, j) is the scale of block j of row n;
 *            entries j >= K/32 are padding (ignored by the GEMV, written as 0
 *            by the quantisers).  Every scale row therefore starts on a
 *            16-byte boundary.
 *   Both planes must start on a 16-byte boundary; K must be a multiple of 32.
 *   bq_planes_to_blocks_* converts planes to the interleaved per-block form
 *   (fp16 scale followed by the 16 or 32 code bytes) and back, bit-exactly.
 *
 * Activations x are fp16 bit patterns, [B][K] row-major (row b at x + b*K),
 * 16-byte aligned.  Outputs y are fp32 [B][N] row-major, 16-byte aligned, and
 * are overwritten (never accumulated).
 *
 * Conventions for every call:
 *   - Ownership: the caller owns every buffer.  The library never allocates
 *     device or pinned memory (the zero-allocation decode loop: gist.science
 *     technical summary, "Methodologie" -> "Zero-Allocation Decode Loop").
 *   - Pointers marked "device" are CUDA device pointers of the current
 *     device; "host" pointers are ordinary CPU memory.
 *   - GPU calls are asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and return after the launch.
 *   - Workspace: calls that take `ws` need ws_bytes >= the matching
 *     bq_*_workspace_bytes() value.  The workspace must be zero-filled once
 *     (e.g. cudaMemsetAsync) before its first use; every call that completes
 *     leaves all of it zero again (counters and scratch), so one zero-fill
 *     suffices and calls of any shapes may use one workspace one after
 *     another on a stream.  Two calls that may run at the same time must not
 *     share a workspace.  After a call that reported a timeout the workspace
 *     must be zero-filled again.
 *   - Errors: the return code covers everything the host can check before
 *     launching (null pointers, shapes, alignment, batch range, workspace
 *     size) and launch failures; nothing is launched when it is not BQ_OK.
 *     Errors the device detects (an expert index outside [0, E), a bounded
 *     wait that ran out) are OR-ed as (1 << code) into *dev_status when
 *     dev_status is not NULL; the caller reads it after synchronising.  The
 *     device never traps.
 *   - Results are deterministic for a given device, shape and batch: every
 *     split sum is combined in a fixed order.
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BQ_API __attribute__((visibility("default")))
#else
#define BQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BQ_OK = 0,
    BQ_ERR_NULL = 1,         /* a required pointer is NULL */
    BQ_ERR_SHAPE = 2,        /* N < 1, K < 32, K % 32 != 0, topk/E out of range */
    BQ_ERR_ALIGN = 3,        /* a pointer or stride is not 16-byte aligned */
    BQ_ERR_BATCH = 4,        /* B outside [1, 8] (or B*topk > 64 for MoE) */
    BQ_ERR_EXPERT_INDEX = 5, /* device: an expert index outside [0, E) */
    BQ_ERR_CUDA = 6,         /* a CUDA runtime call or launch failed */
    BQ_ERR_TIMEOUT = 7,      /* device: a bounded wait ran out */
    BQ_ERR_WORKSPACE = 8,    /* ws NULL or smaller than required */
    BQ_ERR_RANGE = 9         /* quantiser input not finite or scale overflows fp16 */
} bq_status;

/* A quantised matrix: N output rows, K inputs, in the plane layout above.
 * codes and scales are device pointers for the GEMV calls and host pointers
 * for the host-side pack/unpack calls. */
typedef struct bq_qmat {
    const void *codes;
    const uint16_t *scales;
    int32_t N;
    int32_t K;
} bq_qmat;

/* Human-readable name of a status code (static string, never NULL). */
BQ_API const char *bq_status_string(int32_t status);

/* Entries per scale-plane row for a K-column matrix: roundup(K/32, 8).
 * Returns 0 when K is not a positive multiple of 32. */
BQ_API int32_t bq_scales_ld(int32_t K);

/* ---------------------------------------------------------------- GEMV --- */

/* Bytes of workspace bq_gemv_q4 / bq_gemv_q8 need for an N x K matrix
 * (independent of B and of the format).  0 on a bad shape. */
BQ_API size_t bq_gemv_workspace_bytes(int32_t N, int32_t K);

/* Q4 decode GEMV: y[b][n] = sum_k d(n,k/32) * (q(n,k) - 8) * x[b][k].
 * The operation is the per-format decode GEMV with dequantisation in the
 * inner loop (gist.science technical summary, "Kernel Fusie en
 * Specialisatie").
 *   W          host pointer to a bq_qmat whose planes are device pointers
 *   x          device, fp16 bits [B][K]
 *   B          batch, 1..8
 *   y          device, fp32 [B][N], overwritten
 *   ws         device workspace, ws_bytes >= bq_gemv_workspace_bytes(N, K)
 *   dev_status device int32 or NULL (see conventions)
 *   stream     cudaStream_t
 * The launch carries the programmatic-dependent-launch attribute: its CTAs
 * may become resident while the previous kernel on the stream drains, and
 * they read or write no memory before that kernel has completed.  The work
 * unit height and whether bands summed across CTAs run as thread-block
 * clusters are chosen per call from N, K, B and the device
 * (bq_gemv_geometry_of reports the choice); y is deterministic for a given
 * device and shape. */
BQ_API int32_t bq_gemv_q4(const bq_qmat *W, const uint16_t *x, int32_t B, float *y,
                   void *ws, size_t ws_bytes, int32_t *dev_status, void *stream);

/* Q8 decode GEMV: y[b][n] = sum_k d(n,k/32) * q(n,k) * x[b][k].
 * Arguments as bq_gemv_q4. */
BQ_API int32_t bq_gemv_q8(const bq_qmat *W, const uint16_t *x, int32_t B, float *y,
                   void *ws, size_t ws_bytes, int32_t *dev_status, void *stream);

/* Q4 decode GEMV for callers that cannot allocate device memory: code inside
 * a framework that owns every device allocation, or a decode loop that must
 * never call cudaMalloc (it can synchronise the device).  The pages have no
 * counterpart of this entry point; it exists for such callers only.
 * Same operation, arguments and results as bq_gemv_q4, without ws/ws_bytes:
 * the scratch the kernel needs lives in one fixed array inside the library
 * (917,504 bytes, about 0.9 MB: 65,536 band counters plus cross-CTA partial
 * sums for up to 320 CTAs; reserved on every GPU that loads the library until
 * the process exits).
 *   - Always 32-row work units (bq_gemv_q4 chooses 16 or 32 rows per call);
 *     at most 320 CTAs.  Results are within the same tolerance as
 *     bq_gemv_q4's, but not necessarily bit-identical to them.
 *   - N must be <= 1048576 rows; larger N returns BQ_ERR_WORKSPACE and
 *     launches nothing.  Nothing is allocated: no cudaMalloc / cudaFree.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - Every call shares the one array and clears the part that must start at
 *     zero (an async memset on `stream`) before its kernel.  Calls that can
 *     overlap on the GPU (other streams, other host threads) race on it and
 *     must be serialised by the caller. */
BQ_API int32_t bq_gemv_q4_noalloc(const bq_qmat *W, const uint16_t *x, int32_t B, float *y,
                                  int32_t *dev_status, void *stream);

/* Where bq_gemv_q4_noalloc's fixed scratch array lives on the current device:
 * *dev_ptr its device address, *bytes its size (917,504).  Allocates and
 * launches nothing.  For tests and tools that inspect the array, or clear or
 * poison it to check that a call does not depend on what an earlier one left
 * there.  Same once-per-device address lookup as the first
 * bq_gemv_q4_noalloc call.  BQ_ERR_NULL if an argument is NULL, BQ_ERR_CUDA
 * if the lookup fails. */
BQ_API int32_t bq_gemv_q4_noalloc_scratch(void **dev_ptr, size_t *bytes);

/* ------------------------------------------------------------ epilogues --- */

/* What a GEMV writes.
 *
 * BQ_EPI_NONE: y is fp32 [B][N], the GEMV result.
 *
 * BQ_EPI_SWIGLU: the feed-forward activation fused into the gate|up
 * projection, so the down projection reads its input straight from this
 * output.  The pages' runtime fuses operator sequences inside feed-forward
 * blocks to save global-memory round trips and launches (gist.science
 * technical summary, "Methodologie" -> "Kernel Fusie en Specialisatie"); the
 * activation of the families they evaluate (Qwen3, Llama 3.2) is SwiGLU.
 *   W   the gate and up projections of one block (each F x K) in "SwiGLU pair
 *       order": N = 2F with F a multiple of 8; rows 16j .. 16j+7 are gate rows
 *       8j .. 8j+7 and rows 16j+8 .. 16j+15 are up rows 8j .. 8j+7 (each row
 *       quantised on its own, so the planes of the two projections are just
 *       interleaved 8 rows at a time).
 *   y   fp16 bits [B][F]: h[b][i] = silu(g) * u, g and u the GEMV results for
 *       gate row i and up row i, silu(z) = z / (1 + e^-z), evaluated in fp32
 *       and rounded to the nearest fp16 -- the input format of the next GEMV. */
enum { BQ_EPI_NONE = 0, BQ_EPI_SWIGLU = 1 };

/* Flags of bq_gemv_ex.
 *
 * BQ_GEMV_STATIC_WEIGHTS: the caller guarantees that no kernel still running
 * on (or before) the stream writes W's planes.  The launch then starts
 * streaming the weights as soon as its CTAs are resident -- while the
 * previous kernel on the stream drains (programmatic dependent launch) --
 * and waits for that kernel only before it reads x or writes y and the
 * workspace.  In a chain of per-projection launches (a decode step) this
 * hides each launch's weight latency behind the previous one's tail.
 *
 * BQ_GEMV_ROWS16 / BQ_GEMV_ROWS32: the work unit's height for Q4 (the rows
 * of one chunk of 256 weights along K).  Without either flag the library
 * picks it per call from N, K and the device's SM count: 32-row chunks take
 * fewer instructions per weight (two 16-row tiles share each x fragment),
 * 16-row chunks give twice the work units, which pays when a launch is too
 * small to give every warp a 32-row chunk.  The result is the same up to
 * fp32 summation order.  Chunks of the other formats are always 16 rows: ROWS16 is accepted,
 * ROWS32 returns BQ_ERR_SHAPE, and so does setting both. */
enum { BQ_GEMV_STATIC_WEIGHTS = 1, BQ_GEMV_ROWS16 = 2, BQ_GEMV_ROWS32 = 4 };

/* The launch geometry bq_gemv_ex chooses for one matrix (nothing is
 * launched).  Work is cut into chunks of `rows` rows x 256 weights along K;
 * a band (the rows of one chunk height) has chunks_per_band of them, and
 * workers (warps, 8 per CTA) take chunks_per_worker consecutive chunks each.
 *   sm_count   > 0: computed for a device with that many SMs, assuming it
 *              holds every cluster grid at once (no device is touched);
 *              0: the current device, as bq_gemv_ex would launch on it
 *   out        host pointer, filled on BQ_OK
 * Arguments fmt, N, K, B, flags as bq_gemv_ex; errors as its validation
 * (BQ_ERR_SHAPE, BQ_ERR_BATCH, BQ_ERR_NULL), BQ_ERR_CUDA if sm_count is 0
 * and no device can be queried. */
typedef struct bq_gemv_geometry {
    int32_t rows;               /* rows per chunk: 16 or 32 (Q4), 16 (other formats) */
    int32_t chunks;             /* bands x chunks_per_band */
    int32_t chunks_per_band;    /* ceil(K / 256) */
    int32_t chunks_per_worker;
    int32_t grid;               /* CTAs launched */
    int32_t cluster;            /* CTAs per thread-block cluster; 1: no clusters */
    int32_t cross_cta_bands;    /* 1: some band's chunks span CTAs (summed across CTAs:
                                   inside its cluster when cluster > 1, else through the
                                   workspace) */
    int32_t reserved;
} bq_gemv_geometry;
BQ_API int32_t bq_gemv_geometry_of(int32_t fmt, int32_t N, int32_t K, int32_t B, int32_t flags,
                                   int32_t sm_count, bq_gemv_geometry *out);

/* Q2, Q3, Q4, Q5, Q6 or Q8 decode GEMV with an output epilogue.
 *   fmt        2, 3, 4, 5, 6 or 8 (Q6: K a multiple of 64, codes as
 *              bq_quantize_q6 lays them out, rows of 3K/4 bytes; Q5: K a
 *              multiple of 128, as bq_quantize_q5, rows of 5K/8 bytes; Q3: K a
 *              multiple of 128, as bq_quantize_q3, rows of 3K/8 bytes; Q2: K a
 *              multiple of 64, as bq_quantize_q2, rows of K/4 bytes; all four
 *              in 16-row work units)
 *   y          device: fp32 [B][N] (BQ_EPI_NONE) or fp16 bits [B][N/2]
 *              (BQ_EPI_SWIGLU, N a multiple of 16), 16-byte aligned
 *   epilogue   BQ_EPI_*; anything else returns BQ_ERR_SHAPE
 *   flags      0 or an OR of BQ_GEMV_*; other bits return BQ_ERR_SHAPE
 * Other arguments, errors and launch behaviour as bq_gemv_q4. */
BQ_API int32_t bq_gemv_ex(int32_t fmt, const bq_qmat *W, const uint16_t *x, int32_t B, void *y,
                          int32_t epilogue, int32_t flags, void *ws, size_t ws_bytes,
                          int32_t *dev_status, void *stream);

/* --------------------------------------------------------- decode step --- */

/* One matrix of a decode step.  All planes and buffers are device memory. */
typedef struct bq_step_mat {
    bq_qmat W;            /* the quantised matrix (plane layout above) */
    const uint16_t *x;    /* fp16 bits [B][K], 16-byte aligned */
    void *y;              /* output per `epilogue` (fp32 [B][N] by default), 16-byte
                             aligned, overwritten */
    int32_t B;            /* 1..8 */
    int32_t stage;        /* >= 0; stages run in increasing order */
    int32_t epilogue;     /* BQ_EPI_* */
    int32_t reserved;     /* 0 */
} bq_step_mat;

/* Host-side description of a built plan (filled by bq_step_plan). */
typedef struct bq_step_info {
    int32_t fmt, n_mats, n_stages, grid, max_stage_bands, reserved;
    uint64_t stages_off, mats_off;   /* byte offsets inside the device plan */
    uint64_t ws_bytes;               /* workspace bq_step_run needs */
} bq_step_info;

/* Device bytes a plan of n_mats matrices needs (0 if n_mats < 1). */
BQ_API size_t bq_step_plan_bytes(int32_t n_mats);

/* Build, once (e.g. at model load), the plan of a whole decode step: every
 * matrix of one token's forward pass, grouped in stages.  Matrices of one
 * stage are independent; a later stage may read what an earlier one wrote,
 * so stages are separated by a grid-wide barrier inside the single launch
 * bq_step_run makes.  The launch-per-projection overhead that dominates
 * small models at decode (gist.science technical summary, "Resultaten":
 * the fixed per-token overhead; "Kernel Fusie": launch overhead matters
 * because decode kernels are short) becomes one launch per token.
 *   fmt        4 or 8 (every matrix of the plan has this format)
 *   mats       host array of n_mats matrices (any order; stable by stage),
 *              1 <= n_mats <= 256
 *   plan       device buffer, 64-byte aligned, >= bq_step_plan_bytes(n_mats);
 *              written synchronously (cudaMemcpy) -- do not call during
 *              stream capture
 *   info       host struct filled on success
 * The plan holds the planes' addresses and x / y pointers; those buffers
 * must stay allocated while the plan is used. */
BQ_API int32_t bq_step_plan(int32_t fmt, const bq_step_mat *mats, int32_t n_mats, void *plan,
                            size_t plan_bytes, bq_step_info *info);

/* Run one decode step of a plan: one cooperative launch (its grid is sized
 * for co-residency on the device the plan was built on).
 *   ws      device workspace, >= info->ws_bytes, zero-filled before first use
 *           (left zero-filled on completion) */
BQ_API int32_t bq_step_run(const bq_step_info *info, const void *plan, void *ws, size_t ws_bytes,
                           int32_t *dev_status, void *stream);

/* Bounded waits of a plan run.  Every wait in the library's kernels gives up
 * after a bounded number of SM clock cycles and reports the bit
 * 1 << BQ_ERR_TIMEOUT in *dev_status instead of hanging; the device never
 * traps.
 *   wait_cycles     cycles a grid-barrier wait may last (0 or above 4e9:
 *                   the default, 4e9, about 2 s at 1.9 GHz)
 *   extra_arrivals  arrivals each grid barrier waits for beyond the grid's
 *                   own (0 in normal use; at most 1024).  A value > 0 asks
 *                   for arrivals that no CTA makes: every CTA's first barrier
 *                   then runs out after wait_cycles, reports the timeout and
 *                   stops (it drains its own copies in flight and exits).  It
 *                   exists so that the timeout path can be exercised without
 *                   a fault or a missing CTA.
 * After a run that reported BQ_ERR_TIMEOUT the workspace must be zero-filled
 * again before the next run; the outputs of the stages after the failed
 * barrier are not written. */
typedef struct bq_step_wait {
    int64_t wait_cycles;
    int32_t extra_arrivals, reserved;
} bq_step_wait;

/* bq_step_run with explicit bounded-wait options (wait may be NULL: the
 * defaults, as bq_step_run).  BQ_ERR_SHAPE on a negative option. */
BQ_API int32_t bq_step_run_ex(const bq_step_info *info, const void *plan, void *ws,
                              size_t ws_bytes, const bq_step_wait *wait, int32_t *dev_status,
                              void *stream);

/* ---------------------------------------- batched verification GEMM --- */

/* Bytes of workspace bq_verify_gemm needs (tile arrival counters + per-CTA
 * partial sums).  0 on a bad shape. */
BQ_API size_t bq_verify_workspace_bytes(int32_t N, int32_t K, int32_t B);

/* Batched verification GEMM: y[b][n] = sum_k d(n,k/32) * (q(n,k) - z) * x[b][k]
 * for a batch of B = 1..32 activation rows -- the step that checks a batch
 * of drafted tokens in speculative decoding, which the pages name as the way
 * past decode's bandwidth ceiling: its matrix products are compute-shaped
 * and suit the tensor cores (romaanj.github.io review of the M5 follow-up
 * paper, "Future work").  Same operation as the decode GEMV at a wider
 * batch, on the 5th-generation tensor cores (tcgen05.mma, fp32 accumulators
 * in tensor memory), one CTA per SM.
 *   fmt      4 or 8 (the Q4 / Q8 planes of bq_gemv_q4 / bq_gemv_q8)
 *   W        device planes, N x K, K a multiple of 32
 *   x        device fp16 bits [B][K], 16-byte aligned
 *   B        1..32 (else BQ_ERR_BATCH); the MMA's N is 16 for B <= 16 and
 *            32 above (absent rows read as zero and are never stored)
 *   y        device fp32 [B][N], overwritten
 *   ws       device workspace >= bq_verify_workspace_bytes, zero-filled
 *            before first use and left zero-filled by every call that
 *            completes (calls of any shape may share one); not shared with
 *            calls that may run at the same time
 *   dev_status, stream as bq_gemv_q4 (a bounded wait that runs out sets the
 *            bit 1 << BQ_ERR_TIMEOUT; the workspace must then be zero-filled
 *            again)
 * Rounding: each weight d (q - z) enters the tensor core rounded once to
 * fp16 (times a per-row power of two that keeps every value in fp16's normal
 * range, undone exactly afterwards): |y - y_exact| <= 2^-11 sum_k |w x| plus
 * fp32 accumulation -- inside the decode tolerance 1e-3 sum_k |w x| + 1e-5,
 * but not bit-identical to bq_gemv_q4 / _q8 (whose codes enter exactly).
 * Deterministic for a given device and shape (split tiles are summed in a
 * fixed order). */
BQ_API int32_t bq_verify_gemm(int32_t fmt, const bq_qmat *W, const uint16_t *x, int32_t B,
                              float *y, void *ws, size_t ws_bytes, int32_t *dev_status,
                              void *stream);

/* ----------------------------------- decode attention over a Q8 KV cache --- */

/* A preallocated KV cache of Tmax positions per (sequence, KV head), keys and
 * values block-quantised in the Q8 format of the weights (32-element blocks
 * along the head dimension, fp16 scale = absmax/127, int8 codes).  Device
 * pointers, 16-byte aligned; caller-owned.
 *   k_codes   int8 [B][Hkv][Tmax][D]    one row of D codes per position
 *   k_scales  fp16 [B][Hkv][Tmax][D/32]
 *   vt_codes  int8 [B][Hkv][D][Tmax]    values transposed: row d holds
 *                                       component d of every position (a new
 *                                       token writes one byte in each of the D
 *                                       rows)
 *   v_scales  fp16 [B][Hkv][Tmax][D/32] scale of position t's block j */
typedef struct bq_kv_cache {
    const int8_t *k_codes;
    const uint16_t *k_scales;
    const int8_t *vt_codes;
    const uint16_t *v_scales;
    int32_t D, Tmax;
} bq_kv_cache;

/* Bytes of workspace bq_attn_decode_q8 needs (arrival counters per sequence
 * and head + per-CTA partial results).  0 on a bad shape. */
BQ_API size_t bq_attn_workspace_bytes(int32_t B, int32_t Hkv);

/* Decode attention: for each sequence b and query head i (KV head h = i / G),
 *   s_t = scale * sum_d q[b][i][d] K[t][d],  p = softmax over t < lens[b],
 *   o[b][i][d] = sum_t p_t V[t][d],
 * with K and V dequantised from the cache (d * code).  The KV cache is kept
 * preallocated for the whole decode loop (gist.science technical summary,
 * "Methodologie" -> "Zero-Allocation Decode Loop"), and decode attention is
 * the other memory-bound kernel of the decode step beside the GEMV
 * (romaanj.github.io review of the M5 follow-up paper, "Method").
 *   kv      the cache; D must be 128, Tmax a multiple of 128
 *   q       device fp16 bits [B][Hkv*G][D]
 *   lens    device int32 [B]: positions 0 .. lens[b]-1 are attended to
 *           (clamped to [0, Tmax]; a sequence with none gets o = 0); nothing
 *           past lens[b] is read into the result
 *   B, Hkv  sequences, KV heads; G query heads per KV head, 1..8
 *   scale   softmax scale (typically 1/sqrt(D))
 *   o       device fp32 [B][Hkv*G][D], overwritten
 *   ws      device workspace >= bq_attn_workspace_bytes(B, Hkv), zero-filled
 *           before first use, left zero-filled by every call that completes
 *   dev_status, stream as bq_gemv_q4
 * Both products run on tensor cores with the cache codes as exact fp16
 * operands; the softmax weights times the value scales enter rounded once to
 * fp16 (relative 2^-11), so |o - o_exact| <= ~2^-11 sum_t p_t |V[t][d]| plus
 * fp32 accumulation and exp2 approximation error.  Deterministic for a given
 * device and shape.  BQ_ERR_SHAPE for D != 128, Tmax not a multiple of 128,
 * or G outside 1..8. */
BQ_API int32_t bq_attn_decode_q8(const bq_kv_cache *kv, const uint16_t *q, const int32_t *lens,
                                 int32_t B, int32_t Hkv, int32_t G, float scale, float *o,
                                 void *ws, size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------------------ routed experts --- */

/* Bytes of workspace bq_moe_gemv_q4 needs.  0 on a bad shape. */
BQ_API size_t bq_moe_workspace_bytes(int32_t N, int32_t K, int32_t B, int32_t topk, int32_t E);

/* Grouped Q4 GEMV over routed experts (decode step of a mixture-of-experts
 * layer; the pages discuss expert GEMMs in the technical summary's
 * "Prefill Throughput" results for Qwen3-30B-A3B and in the follow-up
 * paper's method paragraph).  Each routed expert's weights are streamed
 * once and applied to every token routed to it.
 *   Wstack        host pointer to a bq_qmat describing expert 0 (device
 *                 planes); expert e's planes start at codes + e*codes_stride
 *                 bytes and scales + e*scales_stride fp16 entries.
 *                 codes_stride must be >= N*K/2 and a multiple of 16;
 *                 scales_stride >= N*ldS and a multiple of 8.
 *   E             number of experts (1..65535)
 *   x             device fp16 bits: [B][K] (x_per_slot == 0, a token's input
 *                 is shared by its experts) or [B][topk][K] (x_per_slot == 1)
 *   expert_idx    device int32 [B][topk]
 *   route_w       device fp32 [B][topk] or NULL
 *   y             device fp32: route_w == NULL -> [B][topk][N] per-slot
 *                 outputs y[b][s] = W_{idx[b][s]} x_{b,s};
 *                 otherwise [B][N], y[b] = sum_s route_w[b][s] * W_{idx[b][s]} x_{b,s}
 *                 summed in fp32 in slot order.
 *   B, topk       1 <= B <= 8, 1 <= topk, B*topk <= 64
 * A slot whose index lies outside [0, E) contributes zero (its per-slot
 * output is zero) and sets bit BQ_ERR_EXPERT_INDEX in *dev_status. */
BQ_API int32_t bq_moe_gemv_q4(const bq_qmat *Wstack, int32_t E, int64_t codes_stride,
                       int64_t scales_stride, const uint16_t *x, int32_t x_per_slot,
                       const int32_t *expert_idx, const float *route_w, int32_t B,
                       int32_t topk, float *y, void *ws, size_t ws_bytes,
                       int32_t *dev_status, void *stream);

/* bq_moe_gemv_q4 with an output epilogue (see BQ_EPI_*).  With
 * BQ_EPI_SWIGLU each expert's planes hold its gate and up projections in
 * SwiGLU pair order (N = 2F, N a multiple of 16), route_w must be NULL, and y
 * is fp16 bits [B][topk][F]: per slot h = silu(gate) * up of the slot's
 * expert, the per-slot input (x_per_slot = 1) of the down projection -- the
 * routed-expert feed-forward block with its activation fused.  An invalid
 * slot's h is zero.  Anything else as bq_moe_gemv_q4; a bad epilogue, or
 * SwiGLU with route_w or with N not a multiple of 16, returns BQ_ERR_SHAPE. */
BQ_API int32_t bq_moe_gemv_ex(const bq_qmat *Wstack, int32_t E, int64_t codes_stride,
                              int64_t scales_stride, const uint16_t *x, int32_t x_per_slot,
                              const int32_t *expert_idx, const float *route_w, int32_t B,
                              int32_t topk, void *y, int32_t epilogue, void *ws, size_t ws_bytes,
                              int32_t *dev_status, void *stream);

/* ---------------------------------------------- host-side pack / unpack --- */
/* All host pointers; no CUDA call is made.  Bit-exact by construction. */

/* Quantise fp32 weights [N][K] (row-major) into planes.  Per 32-block:
 * a = max|w| (fp32), d = fp16_rne(a / 127) (Q8) or fp16_rne(a / 7) (Q4),
 * q = round-half-away(w / d) clamped to [-127, 127] (Q8), or
 * clamp(round-half-away(w / d) + 8, 0, 15) (Q4); a block whose fp16 scale is
 * zero gets code 0 (Q8) or 8 (Q4).  codes: Q8 int8 [N][K], Q4 uint8 [N][K/2];
 * scales: uint16 [N][bq_scales_ld(K)], padding written as 0.
 * BQ_ERR_RANGE if an input is not finite or a scale overflows fp16. */
BQ_API int32_t bq_quantize_q8(const float *w, int32_t N, int32_t K, int8_t *codes, uint16_t *scales);
BQ_API int32_t bq_quantize_q4(const float *w, int32_t N, int32_t K, uint8_t *codes, uint16_t *scales);

/* Q6, a third format of the family (the pages list formats from Q2 to FP16
 * without defining them; BaseRT abstract): d = fp16_rne(a / 31),
 * q = clamp(round-half-away(w / d) + 32, 0, 63), zero-point code 32.  codes:
 * uint8 [N][3K/4], each row the low-nibble plane (K/2 bytes, Q4's layout:
 * block j at byte 16j, byte i = low 4 bits of element i | those of element
 * i+16 << 4) followed by the top-bit plane (K/4 bytes: block j at byte
 * K/2 + 8j, byte i = top 2 bits of elements i, i+8, i+16, i+24 in bits 0-1,
 * 2-3, 4-5, 6-7).  Errors as bq_quantize_q4. */
BQ_API int32_t bq_quantize_q6(const float *w, int32_t N, int32_t K, uint8_t *codes, uint16_t *scales);

/* Q5, the same construction with one top bit: d = fp16_rne(a / 15),
 * q = clamp(round-half-away(w / d) + 16, 0, 31), zero-point code 16.  codes:
 * uint8 [N][5K/8], each row the low-nibble plane (K/2 bytes, as Q4) followed
 * by the top-bit plane (K/8 bytes: block j at byte K/2 + 4j, byte i = 0..3
 * holds the top bit of element i + 4p in bit p, p = 0..7). */
BQ_API int32_t bq_quantize_q5(const float *w, int32_t N, int32_t K, uint8_t *codes, uint16_t *scales);

/* Q3, the 3-bit member: d = fp16_rne(a / 3), q = clamp(round-half-away(w / d)
 * + 4, 0, 7), zero-point code 4.  codes: uint8 [N][3K/8], each row a 2-bit
 * plane of the low 2 bits (K/4 bytes: block j at byte 8j, byte i = those of
 * elements i, i+8, i+16, i+24 in bits 0-1, 2-3, 4-5, 6-7) followed by a
 * 1-bit plane of bit 2 (K/8 bytes: block j at byte K/4 + 4j, byte i = 0..3
 * holds that of element i + 4p in bit p). */
BQ_API int32_t bq_quantize_q3(const float *w, int32_t N, int32_t K, uint8_t *codes, uint16_t *scales);

/* Q2, the 2-bit member: d = fp16_rne(a / 1), q = clamp(round-half-away(w / d)
 * + 2, 0, 3), zero-point code 2 (the quantiser emits codes 1..3; code 0 is
 * -2d).  codes: uint8 [N][K/4], the 2-bit plane alone (laid out as Q3's). */
BQ_API int32_t bq_quantize_q2(const float *w, int32_t N, int32_t K, uint8_t *codes, uint16_t *scales);

/* Dequantise planes into fp32 weights [N][K] (exact: d * q fits fp32). */
BQ_API int32_t bq_dequantize_q8(const int8_t *codes, const uint16_t *scales, int32_t N, int32_t K,
                         float *w);
BQ_API int32_t bq_dequantize_q4(const uint8_t *codes, const uint16_t *scales, int32_t N, int32_t K,
                         float *w);
BQ_API int32_t bq_dequantize_q6(const uint8_t *codes, const uint16_t *scales, int32_t N, int32_t K,
                         float *w);
BQ_API int32_t bq_dequantize_q5(const uint8_t *codes, const uint16_t *scales, int32_t N, int32_t K,
                         float *w);
BQ_API int32_t bq_dequantize_q3(const uint8_t *codes, const uint16_t *scales, int32_t N, int32_t K,
                         float *w);
BQ_API int32_t bq_dequantize_q2(const uint8_t *codes, const uint16_t *scales, int32_t N, int32_t K,
                         float *w);

/* Planes <-> interleaved blocks.  blocks: N*(K/32) records, row-major over
 * (n, j); each record is the fp16 scale (2 bytes, little-endian) followed by
 * 16 code bytes (Q4, 18-byte records) or 32 code bytes (Q8, 34-byte records). */
BQ_API int32_t bq_planes_to_blocks_q4(const uint8_t *codes, const uint16_t *scales, int32_t N,
                               int32_t K, uint8_t *blocks);
BQ_API int32_t bq_planes_to_blocks_q8(const int8_t *codes, const uint16_t *scales, int32_t N,
                               int32_t K, uint8_t *blocks);
BQ_API int32_t bq_blocks_to_planes_q4(const uint8_t *blocks, int32_t N, int32_t K, uint8_t *codes,
                               uint16_t *scales);
BQ_API int32_t bq_blocks_to_planes_q8(const uint8_t *blocks, int32_t N, int32_t K, int8_t *codes,
                               uint16_t *scales);

/* ------------------------------------------------ device-side quantiser --- */

/* Same arithmetic as bq_quantize_q4 / _q8, on the GPU (for building large
 * resident weight sets without a host round trip).  w: device fp32 [N][K];
 * codes / scales: device planes.  Non-finite inputs or fp16-overflowing
 * scales set bit BQ_ERR_RANGE in *dev_status (if not NULL) and produce the
 * zero-point codes for that block. */
BQ_API int32_t bq_quantize_q4_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                           uint16_t *scales, int32_t *dev_status, void *stream);
BQ_API int32_t bq_quantize_q8_dev(const float *w, int32_t N, int32_t K, int8_t *codes,
                           uint16_t *scales, int32_t *dev_status, void *stream);
/* Q6 on the GPU: K must be a multiple of 64 (rows of 3K/4 bytes stay
 * 16-byte aligned), else BQ_ERR_SHAPE. */
BQ_API int32_t bq_quantize_q6_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                           uint16_t *scales, int32_t *dev_status, void *stream);
/* Q5 on the GPU: K must be a multiple of 128 (rows of 5K/8 bytes stay
 * 16-byte aligned), else BQ_ERR_SHAPE. */
BQ_API int32_t bq_quantize_q5_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                           uint16_t *scales, int32_t *dev_status, void *stream);
/* Q3 on the GPU: K must be a multiple of 128 (rows of 3K/8 bytes keep both
 * planes aligned for the block stores), else BQ_ERR_SHAPE. */
BQ_API int32_t bq_quantize_q3_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                           uint16_t *scales, int32_t *dev_status, void *stream);
/* Q2 on the GPU: any K that is a multiple of 32. */
BQ_API int32_t bq_quantize_q2_dev(const float *w, int32_t N, int32_t K, uint8_t *codes,
                           uint16_t *scales, int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H */
