/*
 * qgemm.h — C ABI of the mixed-bitwidth (EXL2-style) quantised matrix multiply
 * for NVIDIA B200 (sm_100a).
 *
 * The operation.  y = x[:, perm] . dequant(Wq):
 *   - W is K x N (K input rows in act-order, N output columns).  Its rows are cut
 *     into 32-row blocks; block j is quantised at b_j bits, b_j in {2,3,4,5,6,8},
 *     widths mixed inside one matrix to hit a target average bits-per-weight,
 *     more important (act-order-first) rows holding more bits
 *     (nightvoyager.top exllamav2 report, "核心价值提炼" / "关键设计决策";
 *     promptquorum "EXL2量化是什么").
 *   - Each (128-row group, column) pair has one fp16 scale (GPTQ "group 128"
 *     lineage, ainews.cool ExLlamaV3 article, benchmark table).
 *   - w[k][n] = (q[k][n] - 2^(b_j - 1)) * s[k/128][n]           (symmetric codes)
 *   - y[m][n] = sum_k x[m][perm[k]] * w[k][n], fp32 accumulation, fp16 result.
 * The pages give no bit layout; this library uses (and documents as) the
 * following one.  For column n and block j the 32 codes form a little-endian
 * bit stream of 32*b_j bits, code r in stream bits [r*b_j, r*b_j + b_j); stream
 * bit t is bit (t mod 32) of word row off_j + t/32, off_j = sum_{i<j} b_i.
 * Words are stored row-major, qw[row][n], so one word row is N contiguous
 * uint32 values.
 *
 * Conventions for every device call:
 *   - d_* pointers are device memory owned by the caller; h_* pointers are host
 *     memory.  The library never allocates, frees or synchronises; each call is
 *     asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - fp16 values are passed as uint16_t bit patterns (IEEE binary16).
 *   - Shapes: K % 32 == 0, N % 8 == 0, M >= 1, K <= 65536, N <= 2^24.
 *     Every device pointer must be 16-byte aligned.
 *   - Schedule: d_bits[K/32] holds b_j, d_offs[K/32 + 1] its prefix sums
 *     (d_offs[0] = 0, d_offs[K/32] = qw_rows).  qgemm_offsets() computes them on
 *     the host.  Kernels read the table before touching the weights and refuse
 *     an inconsistent one (see qgemm_device_error()).
 *   - Return value: QGEMM_OK, or a negative qgemm_status for an argument error
 *     found on the host (nothing is launched) or a launch failure
 *     (QGEMM_ERR_CUDA).  Errors found on the device (an inconsistent schedule,
 *     perm out of range, a pipeline wait that timed out) make the kernel write
 *     nothing it should not, record a code in a per-device error word and
 *     return; read it with qgemm_device_error().  Nothing traps or aborts and
 *     no C++ exception crosses this boundary.
 */
#ifndef QGEMM_H
#define QGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QGEMM_OK = 0,
    QGEMM_ERR_NULL = -1,        /* a required pointer is NULL                        */
    QGEMM_ERR_SHAPE = -2,       /* M, K, N or qw_rows outside the supported range    */
    QGEMM_ERR_BITS = -3,        /* a block width not in {2,3,4,5,6,8} / bad offsets   */
    QGEMM_ERR_ALIGN = -4,       /* a device pointer is not 16-byte aligned           */
    QGEMM_ERR_WORKSPACE = -5,   /* workspace missing or smaller than required        */
    QGEMM_ERR_DTYPE = -6,       /* x_dtype is not a qgemm_dtype                      */
    QGEMM_ERR_CUDA = -7,        /* a CUDA runtime call or launch failed              */
    QGEMM_ERR_UNSUPPORTED = -8  /* valid request this build does not handle          */
} qgemm_status;

typedef enum { QGEMM_F16 = 0, QGEMM_BF16 = 1 } qgemm_dtype;

/* Device error word codes (qgemm_device_error). */
#define QGEMM_DEV_OK 0
#define QGEMM_DEV_BAD_SCHEDULE 1   /* d_bits/d_offs inconsistent or not matching qw_rows */
#define QGEMM_DEV_BAD_PERM 2       /* a perm entry outside [0, K)                        */
#define QGEMM_DEV_TIMEOUT 4        /* a pipeline wait gave up after ~1 s                 */

/* ---------------------------------------------------------------- host only */

/* Library version (major*10000 + minor*100 + patch). */
int qgemm_version(void);

/* Human-readable name of a qgemm_status value (static string). */
const char* qgemm_status_string(int status);

/* sum_j h_bits[j] over the K/32 blocks = number of packed word rows, or a
 * negative qgemm_status (QGEMM_ERR_SHAPE for K % 32 != 0, QGEMM_ERR_BITS for a
 * width outside {2,3,4,5,6,8}). */
int64_t qgemm_packed_word_rows(const uint8_t* h_bits, int K);

/* Writes h_offs[0..K/32] = prefix sums of h_bits (h_offs[0] = 0).  Returns
 * QGEMM_OK or a negative status as qgemm_packed_word_rows. */
int qgemm_offsets(const uint8_t* h_bits, int K, int32_t* h_offs);

/* Checks a host copy of the schedule: widths allowed, offsets equal to their
 * prefix sums and h_offs[K/32] == qw_rows. */
int qgemm_validate_schedule(const uint8_t* h_bits, const int32_t* h_offs, int K, int64_t qw_rows);

/* Bytes of workspace qgemm() needs for this shape (0 is possible).  The first
 * call with a given workspace needs it zero-filled; every completed call leaves
 * it reusable (its counters return to zero).  Two calls that overlap in time
 * must not share a workspace. */
size_t qgemm_workspace_bytes(int M, int K, int N);

/* Number of bytes the packed weights of one K x N matrix occupy:
 * 4 * N * qw_rows (words) and 2 * N * ceil(K/128) (scales). */
size_t qgemm_packed_bytes(int64_t qw_rows, int N);
size_t qgemm_scale_bytes(int K, int N);

/* Reads (and with clear != 0 resets) the device error word of the current CUDA
 * device.  Synchronises the device. Returns QGEMM_OK or QGEMM_ERR_CUDA. */
int qgemm_device_error(int* h_code, int clear);

/* Which kernel family qgemm() uses for this shape: the autotuner's recorded
 * choice, else the built-in one (crossovers measured on B200):
 *   0 = split-K integer GEMV (M <= 4): activations rounded per (128-row group,
 *       token) to int16 with a power-of-two scale (plus a second, 2^15-finer
 *       part for the blocks next to an outlier activation), exact int32 dot
 *       products;
 *   1 = split-K tensor-core GEMV (5 <= M <= 16): the exact fp16 (q - z) 2^P
 *       codes in TMEM, tcgen05.mma against the activations;
 *   2 = tcgen05 tensor-core GEMM with dequantisation into shared memory
 *       (M > 16, and 12 <= M <= 16 when its output tiles are too few to fill
 *       the GPU and it splits k across the SMs). */
int qgemm_path_for(int M, int K, int N);

/* Launch plan qgemm() would use for this shape on the current device (or on a
 * 148-SM device when no GPU is visible).  out[0] = kernel family (as
 * qgemm_path_for), out[1] = grid size, out[2] = shared-memory ring rows (GEMV)
 * or number of k splits (GEMM),
 * out[3] = CTAs resident per SM, out[4] = dynamic shared
 * memory bytes, out[5] = SM count used.  Host only; returns a qgemm_status. */
int qgemm_plan_info(int M, int K, int N, int64_t qw_rows, int64_t* out);

/* ------------------------------------------------------------ autotuning
 * Per-shape choice of the kernel variant, after the runtime autotuning of the
 * EXL2 kernels (nightvoyager.top exllamav2 report, "创新之处" and "关键设计决策":
 * each (M, K, N) is timed once, 20 warm-up and 200 timed runs ranked by an
 * interquartile mean, and the choice cached with the built-in heuristic as
 * the fallback).  A variant is a kernel family (as qgemm_path_for) and one
 * knob: the integer GEMV's CTAs per SM (1 or 2), none for the tensor-core
 * GEMV (0), the GEMM's largest k split (1, 2 or 4).  Candidates for M rows:
 * the integer GEMV (M <= 4), the tensor-core GEMV (M <= 16), the GEMM (any M).
 * Choices are kept per (current device, M, K, N) for the life of the process;
 * qgemm(), qgemm_path_for, qgemm_plan_info and qgemm_workspace_bytes consult
 * them (the workspace size covers every candidate of M, so any choice fits).
 * Host state is guarded by a mutex; the choice of a shape can change results
 * in the last bits (another kernel or split), never beyond the tolerance. */

/* Times every candidate on these operands on `stream` (warmup untimed calls,
 * then iters calls with an event between consecutive calls; the result in
 * d_y is the last call's, a correct product), ranks them by the mean of the
 * per-call times between the 5/16 and 11/16 quantiles and records the
 * fastest.  Candidates whose workspace exceeds ws_bytes are skipped.
 * Synchronises `stream`.  Refuses (QGEMM_ERR_UNSUPPORTED) a stream that is
 * being captured: timing needs a live stream.
 *   h_results  optional host array of 3 * max_results int64: per candidate
 *              {path, knob, IQM time in ns, or -1 if skipped};
 * Returns the number of rows written (>= 0) or a negative qgemm_status
 * (QGEMM_ERR_WORKSPACE when no candidate fits the workspace). */
int qgemm_autotune(const void* d_x, int x_dtype, const int32_t* d_perm, const uint32_t* d_qw, int64_t qw_rows,
                   const uint16_t* d_scales, const uint8_t* d_bits, const int32_t* d_offs, int M, int K, int N,
                   uint16_t* d_y, void* d_ws, size_t ws_bytes, int warmup, int iters, void* stream,
                   int64_t* h_results, int max_results);

/* mode 1: qgemm() runs qgemm_autotune (20 warm-up, 200 timed calls) on the
 * first call of a shape without a recorded choice, unless its stream is being
 * captured (the built-in choice is used then, and tuning waits for an eager
 * call); mode 0 (default): never.  Host only. */
int qgemm_set_autotune(int mode);

/* The recorded choice for (M, K, N) on the current device: returns 1 and
 * writes *h_path, *h_knob; 0 when there is none.  Host only. */
int qgemm_tune_lookup(int M, int K, int N, int* h_path, int* h_knob);

/* Records a choice without timing (a caller's saved table, or tests);
 * QGEMM_ERR_UNSUPPORTED for a variant that cannot serve M rows.  Host only. */
int qgemm_tune_record(int M, int K, int N, int path, int knob);

/* Forgets every recorded choice.  Host only. */
int qgemm_tune_clear(void);

/* The ranking statistic: mean of h_values[0..n) sorted, from index
 * floor(5n/16) to ceil(11n/16) (at least one value); -1 for n <= 0. */
double qgemm_iqm(const float* h_values, int n);

/* ----------------------------------------------------------- device calls */

/* Quantise fp16 weights into codes and fp16 scales, the step before
 * qgemm_pack (nightvoyager.top exllamav2 report, "关键设计决策": the adaptive
 * scale with a 4-bit second-level quantisation of the group scale and a scan
 * of 96 candidate factors per layer keeping the lowest squared error).
 * This library's reading of the method, per column n:
 *   base[g] = max over the blocks j of group g of max |W[k][n]| / 2^(b_j-1);
 *   qmax = max_g base[g];  qs[g] = clamp(rint(sqrt(base[g] / qmax) * 16), 1, 16);
 *   candidate i = 0..95: p = (32 + i) / 96, s[g] = fp16(p * (qmax * qs[g]^2 / 256)),
 *   q = clamp(rint(W * (1 / s)) + 2^(b-1), 0, 2^b - 1) (zero point where s = 0);
 *   E(i) = sum over columns (in order) of the sum over rows (in order) of
 *   (W - (q - 2^(b-1)) s)^2 in double; the smallest E wins, the lowest i on ties.
 * Single precision with each operation rounded to nearest even decides the
 * codes; the result is bit-exact against any implementation of the same steps.
 *   d_w      [K][N] fp16 weights, act-order rows (as qgemm_pack's codes);
 *   d_bits   [K/32] widths;
 *   d_codes  [K][N] uint8 out, feed to qgemm_pack;  d_scales [ceil(K/128)][N] fp16 out;
 *   d_err    optional double [96] out: E(i);  d_best optional int32 [1] out: the i kept;
 *   d_ws     qgemm_quantize_workspace_bytes(K, N) bytes (need not be zeroed).
 * Widths outside {2,3,4,5,6,8} set QGEMM_DEV_BAD_SCHEDULE.  Finite weights only. */
/* KV-cache quantisation with a Hadamard rotation (nightvoyager.top exllamav2
 * report, "创新之处": rotated K/V in a 4-bit cache; navi2ai ExLlamaV3 page,
 * "核心能力": 2-8 bit caches).  Each of the nvec (token, head) vectors of
 * length D (32, 64, 128 or 256) is rotated by the Sylvester Hadamard matrix
 * (u = H_D v, fast Walsh-Hadamard transform in single precision, strides 1 ..
 * D/2, each operation rounded to nearest even), cut into groups of 32 with
 * one fp16 scale s = fp16(max|u| / (2^(b-1) - 1)) each, and rounded to codes
 * q = clamp(rint(u * (1 / s)) + 2^(b-1), 0, 2^b - 1) (the zero point where
 * s = 0), packed as the weights' blocks: b uint32 words per group, code r at
 * bits [r b, r b + b) of the LSB-first stream.  Dequantisation rotates back:
 * v' = fp16(H_D ((q - 2^(b-1)) s) / D).
 *   d_v      [nvec][D] fp16 (in for quantise, out for dequantise);
 *   d_codes  [nvec][D/32][bits] uint32;  d_scales [nvec][D/32] fp16;
 *   bits     2, 3, 4, 5, 6 or 8 (QGEMM_ERR_BITS otherwise).
 * Pointers: d_v 8-byte aligned (each lane moves D/32 consecutive elements in
 * one access), d_codes 4-byte, d_scales 2-byte (QGEMM_ERR_ALIGN otherwise).
 * Finite inputs only.  Asynchronous on `stream`; nvec = 0 launches nothing. */
int qgemm_kv_quantize(const uint16_t* d_v, int64_t nvec, int D, int bits, uint32_t* d_codes,
                      uint16_t* d_scales, void* stream);
int qgemm_kv_dequantize(const uint32_t* d_codes, const uint16_t* d_scales, int64_t nvec, int D, int bits,
                        uint16_t* d_v, void* stream);

size_t qgemm_quantize_workspace_bytes(int K, int N);
int qgemm_quantize(const uint16_t* d_w, const uint8_t* d_bits, int K, int N, uint8_t* d_codes,
                   uint16_t* d_scales, double* d_err, int32_t* d_best, void* d_ws, size_t ws_bytes,
                   void* stream);

/* Pack codes into the layout above.
 *   d_codes [K][N] uint8, row k = act-order row, value < 2^b_j (higher bits of a
 *           wider value are ignored);
 *   d_qw    [qw_rows][N] uint32 output, fully written.
 * Source: the EXL2 mixed-width format (nightvoyager.top exllamav2 report,
 * "核心价值提炼"); the bit layout is this library's reading. */
int qgemm_pack(const uint8_t* d_codes, const uint8_t* d_bits, const int32_t* d_offs,
               int K, int N, int64_t qw_rows, uint32_t* d_qw, void* stream);

/* Dequantise to fp16: d_w[k][n] = RNE_fp16((q - 2^(b-1)) * s[k/128][n]),
 * computed exactly before the one rounding (bit-exact with any correct
 * implementation).  d_scales [ceil(K/128)][N] fp16, d_w [K][N] fp16 (act-order
 * rows).  Source: per-group scale of the format (nightvoyager.top exllamav2
 * report, "关键设计决策", AdaptiveQuantizer paragraph). */
int qgemm_dequant(const uint32_t* d_qw, int64_t qw_rows, const uint16_t* d_scales,
                  const uint8_t* d_bits, const int32_t* d_offs, int K, int N,
                  uint16_t* d_w, void* stream);

/* y = x[:, perm] . dequant(qw)   (the Q-GEMM the pages credit to exllamav2_ext,
 * nightvoyager.top report "解法哲学"; bandwidth-bound decode per the navi2ai
 * ExLlamaV3 page, "核心能力").
 *   d_x      [M][K] fp16 or bf16 (x_dtype), row-major;
 *   d_perm   [K] int32, perm[k] = column of x that multiplies W row k;
 *   d_qw     [qw_rows][N] uint32; d_scales [ceil(K/128)][N] fp16;
 *   d_y      [M][N] fp16 output (RNE of the fp32 sum);
 *   d_ws     workspace of at least qgemm_workspace_bytes(M, K, N) bytes
 *            (may be NULL when that is 0).
 * M <= 16 runs a split-K GEMV, larger M the tcgen05 GEMM (qgemm_path_for).
 * The integer GEMV (M <= 4) rounds each activation to the nearest multiple of
 * 2^-e, 2^e being the power of two that brings the largest magnitude of its
 * (128-row group, token) into [2^13, 2^14): an error of at most 2^-14 of that
 * largest magnitude. */
int qgemm(const void* d_x, int x_dtype, const int32_t* d_perm,
          const uint32_t* d_qw, int64_t qw_rows, const uint16_t* d_scales,
          const uint8_t* d_bits, const int32_t* d_offs,
          int M, int K, int N, uint16_t* d_y,
          void* d_ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------- allocation-free decode
 * The paper has no counterpart to this entry point; it serves callers that
 * cannot allocate device memory.  qgemm() needs a caller-provided workspace,
 * and some callers have no way to get one: a runtime that plans every byte of
 * device memory up front and owns the only allocator, a plugin that is not
 * allowed to allocate behind its host's back, or a latency-bound decode loop
 * that cannot afford cudaMalloc/cudaFree (cudaFree synchronises the device).
 *
 * qgemm_decode_noalloc computes exactly what qgemm() computes for M <= 4 with
 * the built-in choice or a tuned integer-GEMV variant (the integer decode
 * GEMV, same kernels and same split, so the same result) but
 * takes its scratch from a buffer of QGEMM_NOALLOC_SCRATCH_BYTES built into
 * the library.  Every GPU that loads the library holds that buffer until the
 * process exits.  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *
 *   Arguments, layouts and ownership as qgemm(), without d_ws / ws_bytes.
 *   Limits: 1 <= M <= 4 (QGEMM_ERR_SHAPE otherwise); a shape whose scratch
 *     (qgemm_noalloc_scratch_bytes(M, K, N)) exceeds
 *     QGEMM_NOALLOC_SCRATCH_BYTES is refused with QGEMM_ERR_WORKSPACE before
 *     anything is launched.
 *   First call on a device: looks up the buffer's device address
 *     (cudaGetSymbolAddress, with that device current) and sets the kernels'
 *     shared-memory attributes; make this first call before any stream
 *     capture.
 *   Shared state: every call on a device uses the same buffer.  Its first
 *     256 KiB hold the per-tile tickets of every shape served; they are zero
 *     when the library loads and every completed call leaves them at zero, so
 *     calls need no memset; the rest is overwritten before it is read.  A call
 *     that gave up on a wait (QGEMM_DEV_TIMEOUT in the device error word) can
 *     leave tickets behind: qgemm_noalloc_reset() zeroes them again.  Calls
 *     that overlap on the GPU (other streams, other threads) race on the
 *     buffer and give wrong results: order them, e.g. on one stream.
 *   Returns a qgemm_status as qgemm(). */
#define QGEMM_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/* Scratch bytes qgemm_decode_noalloc needs for this shape (the integer GEMV's
 * workspace), 0 when M is outside 1..4 or the shape is invalid.  Host only. */
size_t qgemm_noalloc_scratch_bytes(int M, int K, int N);

/* Zeroes the tickets of the built-in buffer on `stream` (after a call that
 * reported QGEMM_DEV_TIMEOUT).  Allocates nothing. */
int qgemm_noalloc_reset(void* stream);

int qgemm_decode_noalloc(const void* d_x, int x_dtype, const int32_t* d_perm,
                         const uint32_t* d_qw, int64_t qw_rows, const uint16_t* d_scales,
                         const uint8_t* d_bits, const int32_t* d_offs,
                         int M, int K, int N, uint16_t* d_y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QGEMM_H */
