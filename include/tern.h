/*
 * tern.h -- ternary-g128 weight-only matrix multiply for NVIDIA B200 (sm_100a).
 *
 * The number format.  Each weight is a ternary value t in {-1, 0, +1}; every
 * 128 consecutive weights along K share one FP16 scale s_g, and the weight is
 * w = s_g * t.  ("Bonsai 27B ternary / 1-bit quantization", ThakiCloud blog,
 * section "How compression works": w_i = s_g * t_i with one FP16 scale per
 * 128-weight group; "Ternary-Bonsai-27B" model summary, aitrends.kr, section
 * "Technical features": the group scale is applied inside the matrix multiply
 * and the kernels consume the packed 2-bit slots directly, without an FP16
 * copy of the weights.)
 *
 * The storage ("2-bit slots": "Ternary quantization: 27B in 7 GB", devnsb
 * blog, section "Limits") is this library's own contract; the pages do not
 * fix a byte layout.  For a weight matrix W with N rows and K columns
 * (K contiguous), G = K / 128:
 *
 *   slots   uint8 [N][K/4]   weight (n,k) is the 2-bit code c = t + 1
 *                            (0 -> -1, 1 -> 0, 2 -> +1; 3 is invalid) in byte
 *                            n*K/4 + k/4, bits 2*(k%4) .. 2*(k%4)+1
 *                            (least significant pair first);
 *   scales  fp16  [N][G]     weight (n,k) uses scales[n][k/128].
 *
 * Bytes: K*N/4 + 2*K*N/128, i.e. 2.125 bits per weight (the ideal for this
 * format, log2(3) + 16/128 ~= 1.71, needs a non-power-of-two packing).
 *
 * The products.  y[M][N] = x[M][K] * W^T: fp16 activations, fp32
 * accumulation, fp16 output (round to nearest even).  y is overwritten.
 *
 * Conventions for every entry point:
 *   - All buffers are DEVICE memory owned by the caller; the library keeps no
 *     pointer after a call returns and allocates no device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it.
 *   - Argument errors are detected on the host before anything is launched
 *     and returned synchronously; nothing is written in that case.
 *   - A launch failure returns TERN_ERR_CUDA; tern_last_error() has the text.
 *     Errors raised while kernels run surface on the caller's next
 *     synchronisation, as for any CUDA work.
 *   - K must be a positive multiple of 128; M and N must be >= 1.
 *   - x, slots, codes and y must be 16-byte aligned.  scales must be 16-byte
 *     aligned for the products (tern_gemv, tern_gemm, tern_gemv_grouped, the
 *     step calls and tern_gemv_noalloc) and 2-byte aligned for pack, unpack
 *     and the embedding gather.  The products bring the scale rows on chip
 *     with the tensor memory accelerator, whose global addresses must be
 *     16-byte aligned; a misaligned scales pointer returns TERN_ERR_ALIGN
 *     before any launch.  (Allocations from cudaMalloc / PyTorch are 256-byte
 *     aligned, and a scale row is K/64 bytes.)
 *   - An invalid slot value (3) in tern_gemv / tern_gemm contributes an
 *     unspecified finite value for that weight; it never faults.  Validation
 *     is the job of tern_pack_g128.
 *   - Thread safety: calls on different streams may run concurrently.
 *     tern_set_option changes process-wide state and is meant for tests and
 *     benchmarks only.
 */
#ifndef TERN_H
#define TERN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tern_status {
    TERN_OK = 0,
    TERN_ERR_INVALID_ARG = 1, /* null pointer, negative or zero count, bad option */
    TERN_ERR_ALIGN = 2,       /* a pointer is not aligned as documented */
    TERN_ERR_SHAPE = 3,       /* K not a positive multiple of 128, M or N < 1, too large */
    TERN_ERR_WORKSPACE = 4,   /* workspace smaller than tern_workspace_bytes() */
    TERN_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
    TERN_ERR_TIMEOUT = 6,     /* a bounded on-device wait gave up (see tern_gemm) */
    TERN_ERR_DEVICE = 7,      /* current device is not compute capability 10.0 */
    TERN_ERR_GUARD = 8        /* an in-kernel index check failed (debug build only; see tern_sync_status) */
} tern_status;

/* Library version, e.g. 100 for 0.1.0. */
int tern_version(void);

/* Static text for a status code ("ok", "invalid argument", ...). */
const char *tern_status_string(int status);

/* Text of the most recent error raised on the calling host thread ("" if
 * none).  Valid until the next library call on that thread. */
const char *tern_last_error(void);

/* Size in bytes of the slot buffer / scale buffer of an N x K matrix;
 * 0 if N < 1 or K is not a positive multiple of 128. */
size_t tern_slots_bytes(int64_t N, int64_t K);
size_t tern_scales_bytes(int64_t N, int64_t K);

/*
 * Workspace.  With TERN_OPT_GEMV_VARIANT = 3 and M <= 4 the bandwidth kernel
 * splits long rows along K over several warpgroups when the caller passes a
 * workspace of at least
 * tern_workspace_bytes(M, N, K) bytes (tern_gemv_grouped_workspace_bytes() for
 * a grouped call): partial sums go there and the last part of each 16x128-row
 * tile to finish adds them up in a fixed order, so results do not depend on
 * scheduling.  Without it (NULL or too small) tiles are not split: the result
 * is the same, the balance across SMs may be worse.
 *   - The workspace is device memory owned by the caller, 256-byte aligned,
 *     and its first 128 KiB (per-tile arrival counters) must be ZERO before
 *     its first use; every call that completes leaves them zero again, so one
 *     workspace can serve calls of any shape in turn.  The rest holds partial
 *     sums and needs no initialisation.  After a call that reported
 *     TERN_ERR_TIMEOUT, zero the first 128 KiB again.
 *   - Calls that may run concurrently must not share a workspace.
 *   - The size depends on the current device's SM count (148 is assumed when
 *     no device is visible) and is 0 when no split is planned.
 */
size_t tern_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * tern_pack_g128 -- build the slot layout from ternary values.
 *   codes      int8 [N][K], each value in {-1, 0, +1}          (device, read)
 *   scales_in  fp16 [N][K/128] as raw 16-bit patterns           (device, read)
 *   slots_out  uint8 [N][K/4]                                  (device, written)
 *   scales_out fp16 [N][K/128], a bit-exact copy of scales_in   (device, written;
 *              may equal scales_in, then nothing is copied)
 *   invalid_count  optional device int32: atomically incremented by the
 *              number of codes outside {-1,0,+1}; such a code is stored as
 *              slot value 3.  NULL to skip counting.
 * Alignment: codes and slots_out 16 bytes; scales 2 bytes.  Any N >= 1.
 * Result is bit-exact and independent of launch configuration.
 * Format: ternary weights with one FP16 scale per 128-weight group ("Bonsai
 * 27B ternary / 1-bit quantization", ThakiCloud blog, section "How
 * compression works"), stored in 2-bit slots ("Ternary quantization: 27B in
 * 7 GB", devnsb blog, section "Limits"); the code and bit order are this
 * library's (see the top of this file).
 */
tern_status tern_pack_g128(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K,
                           uint8_t *slots_out, uint16_t *scales_out, int32_t *invalid_count,
                           void *stream);

/*
 * tern_unpack_g128 -- inverse of the slot layout.
 *   slots      uint8 [N][K/4]  (device, read)
 *   codes_out  int8  [N][K]    (device, written): t = c - 1; slot value 3 is
 *              written as the sentinel 2.
 * Alignment: 16 bytes for both.
 */
tern_status tern_unpack_g128(const uint8_t *slots, int64_t N, int64_t K, int8_t *codes_out,
                             void *stream);

/*
 * tern_gemv -- decode matrix-vector product, M = 1:  y[n] = sum_k x[k] * w[n][k].
 *   x       fp16 [K]        (device, read)
 *   slots   uint8 [N][K/4]  (device, read)
 *   scales  fp16 [N][K/128] (device, read)
 *   y       fp16 [N]        (device, written)
 *   workspace / ws_bytes: optional, see tern_workspace_bytes.
 * Bandwidth-bound: the weights are streamed from HBM once, unpacked on chip
 * and never written back in any other precision.  Generation is bound by the
 * weight bytes read per token ("Bonsai 27B ternary / 1-bit quantization",
 * ThakiCloud blog, section "Throughput and speculative decoding"); the kernels
 * read the packed slots directly and apply the group scale inside the
 * product ("Ternary-Bonsai-27B" model summary, aitrends.kr, section
 * "Technical features").  With K a multiple of 1024 it runs the decode-step
 * kernel of tern_gemv_step (one product).
 */
tern_status tern_gemv(const uint16_t *x, const uint8_t *slots, const uint16_t *scales, uint16_t *y,
                      int64_t N, int64_t K, void *workspace, size_t ws_bytes, void *stream);

/*
 * tern_gemm -- y[M][N] = x[M][K] * W^T for any M >= 1.
 *   x  fp16 [M][K] row-major (device, read);  y  fp16 [M][N] row-major (device, written).
 * M <= 8 (speculative-verify batches) runs the same bandwidth-bound kernels as
 * tern_gemv (M = 2 with K a multiple of 1024: the step kernel's two-row
 * form), reading the weights once for all rows wherever the M rows of x fit
 * on chip (M = 5..8 with K above ~7000: two passes of up to four rows).
 * M >= 32 runs the
 * tensor-core prefill kernel (tcgen05), which unpacks weight tiles on chip to
 * s*t (exact in fp16) straight into tensor memory and accumulates in fp32;
 * 8 < M < 32 runs the bandwidth kernel once per eight rows.  Small M is the
 * verification pass of speculative decoding (several drafted tokens checked
 * in one pass of the target) and large M the compute-bound prompt
 * processing ("Bonsai 27B ternary / 1-bit quantization", ThakiCloud blog,
 * section "Throughput and speculative decoding").
 */
tern_status tern_gemm(const uint16_t *x, const uint8_t *slots, const uint16_t *scales, uint16_t *y,
                      int64_t M, int64_t N, int64_t K, void *workspace, size_t ws_bytes,
                      void *stream);

/*
 * tern_gemv_noalloc -- the same product as tern_gemv (M = 1), for callers that
 * may not allocate device memory themselves: code running while a CUDA graph
 * is captured into a memory pool it does not own, runtimes that forbid
 * allocation after start-up, plug-ins whose host framework owns all device
 * memory.  It runs the tensor-core (tcgen05) bandwidth kernel and takes the
 * kernel's split-K scratch from a 4 MiB area compiled into the library
 * instead of a workspace, and allocates nothing (no cudaMalloc, no cudaFree).
 * The method described by the pages has no counterpart to this entry point;
 * it exists only for such callers.
 *   x, slots, scales, y, N, K, stream: as for tern_gemv.
 *   - Every GPU that loads the library holds the 4 MiB area until exit.
 *   - The first call on a device looks the area up (once per device, with
 *     that device current); make that first call before any stream capture.
 *   - Shapes whose scratch would exceed 4 MiB return TERN_ERR_WORKSPACE and
 *     launch nothing.  (The 5120 x 151936 output head at M = 1 fits.)
 *   - All calls on a device share the area: calls that may overlap on the GPU
 *     race on it and must be serialised by the caller.  Each call clears the
 *     area's arrival counters on `stream` before its kernel.
 */
tern_status tern_gemv_noalloc(const uint16_t *x, const uint8_t *slots, const uint16_t *scales, uint16_t *y,
                              int64_t N, int64_t K, void *stream);

/* One matrix of a grouped product (all fields describe device buffers as in
 * tern_gemm; every descriptor of one call has the same M). */
typedef struct tern_gemv_desc {
    const uint16_t *x;      /* fp16 [M][K] */
    const uint8_t *slots;   /* uint8 [N][K/4] */
    const uint16_t *scales; /* fp16 [N][K/128] */
    uint16_t *y;            /* fp16 [M][N] */
    int64_t N;
    int64_t K;
} tern_gemv_desc;

/* Largest number of descriptors accepted by tern_gemv_grouped. */
#define TERN_MAX_GROUP 16

/*
 * tern_gemv_grouped -- up to TERN_MAX_GROUP independent products with the same
 * M (1..8) in ONE kernel launch (two at M = 5..8 when some x does not fit on
 * chip), e.g. the q/k/v projections of a layer, or all seven projections of
 * one synthetic decode layer.  Descriptors are read
 * on the host during the call (the array need not outlive it).  Outputs must
 * not overlap inputs or each other.
 */
tern_status tern_gemv_grouped(const tern_gemv_desc *descs, int32_t count, int64_t M, void *workspace,
                              size_t ws_bytes, void *stream);

/* Workspace for one tern_gemv_grouped call with these descriptors (only N and
 * K are read); 0 if none is needed or the arguments are invalid. */
size_t tern_gemv_grouped_workspace_bytes(const tern_gemv_desc *descs, int32_t count, int64_t M);

/* Largest number of descriptors accepted by tern_gemv_step. */
#define TERN_MAX_STEP 512

/*
 * tern_gemv_step -- products of up to TERN_MAX_STEP independent matrices with
 * the same M (1..8 token rows: a decode step, M = 1, or a speculative-verify
 * step) in ONE persistent launch, e.g. every projection of every layer plus
 * the output head of one step whose inputs do not depend on each other.
 * Generation speed is set by the bytes of weights read per token ("Bonsai
 * 27B ternary / 1-bit quantization", ThakiCloud blog, section "Throughput
 * and speculative decoding"); one launch streams all of them without the
 * start-up and drain every separate launch pays.
 *   descs   count descriptors as for tern_gemv_grouped: x fp16 [M][K], slots
 *           uint8 [N][K/4], scales fp16 [N][K/128], y fp16 [M][N]; device
 *           buffers owned by the caller, 16-byte aligned; read on the host
 *           during the call (the array need not outlive it)
 *   count   1..TERN_MAX_STEP
 *   M       1..8 (TERN_ERR_SHAPE otherwise)
 * Every K must be a multiple of 1024.  The M rows of a product's x are
 * staged in shared memory beside the weight rings; a product whose x does
 * not fit (at M = 8 above K ~ 8900, at M = 4 above K ~ 17900) runs as up to
 * four K segments of whole 1024-k units, in launches of their own after the
 * others: the first writes y, each later one adds its partial sum to the
 * fp16 y (one more fp16 rounding each, at most 2^-11 of sum_k |x_k w_k|; four
 * stay within the tolerance below); beyond four segments TERN_ERR_SHAPE
 * (at M = 8, K above ~36000).  Each weight is read once either way.  Results are
 * within |y - y_ref| <= 2e-3 sum_k |x_k w_k| + 1e-5 of the exact product, as
 * for tern_gemv / tern_gemm (fixed summation order per tile);
 * outputs must not overlap inputs or each other.  Argument errors return
 * before any launch; a device wait that gives up is reported by
 * tern_sync_status.  Internally a list longer than 96 matrices becomes a few
 * launches of equal size (the tensor maps travel in the kernel parameters).
 */
tern_status tern_gemv_step(const tern_gemv_desc *descs, int32_t count, int64_t M, void *stream);

/*
 * tern_step_plan -- the split of one step-kernel launch over CTAs, for
 * inspection and tests; host only (no device is touched).  The pages have no
 * counterpart: it states how the bytes a step streams are shared out.
 *   N, K        count row counts and depths (host arrays), in launch order;
 *               every K a multiple of 1024
 *   count       1..96 (the products of one launch; tern_gemv_step cuts longer
 *               lists into launches of at most 96)
 *   M           1..8 token rows
 *   grid        1..160 CTAs (one per SM on B200: 148)
 *   first_tile  int32 [grid + 1] (host, written): CTA c streams the 16-row
 *               tiles first_tile[c] .. first_tile[c + 1] - 1 of the flat list
 *               (tiles of product 0 first); first_tile[0] = 0 and
 *               first_tile[grid] = all tiles; trailing CTAs may get empty
 *               ranges (always when there are fewer tiles than CTAs).
 * Ranges are cut so that each CTA's streaming (1024-k units) plus the
 * staging of every product it starts is about equal.  Returns TERN_OK, or
 * TERN_ERR_SHAPE / TERN_ERR_INVALID_ARG for arguments out of range.
 */
tern_status tern_step_plan(const int64_t *N, const int64_t *K, int32_t count, int64_t M, int32_t grid,
                           int32_t *first_tile);

/*
 * tern_embed_gather -- ternary embedding lookup: rows of a ternary-g128
 * matrix gathered by token id, written as fp16.  The pages count the
 * embeddings among the ternary matrices ("Ternary-Bonsai-27B" model summary,
 * aitrends.kr, section "Differentiators"; "Bonsai 27B ternary / 1-bit
 * quantization", ThakiCloud blog, section "What it is"); with tied weights
 * the output head's slots and scales are the table.
 *   ids        int32 [M] token ids (device)
 *   M          rows to gather, >= 1 (0 returns TERN_OK without a launch)
 *   slots      uint8 [V][K/4], scales fp16 [V][K/128]: the table, as packed
 *              by tern_pack_g128
 *   V, K       table rows and row length (K a multiple of 128)
 *   out        fp16 [M][K]: out[m][k] = s[id][k/128] * t[id][k], exact
 *              (t is -1, 0 or +1; a zero keeps the sign of the scale, as
 *              IEEE multiplication gives it); an invalid slot value 3 gives
 *              an unspecified value
 *   bad_count  nullable device int32: incremented once per id outside
 *              [0, V); such rows are written as zeros
 * All buffers are device memory owned by the caller; ids, bad_count 4-byte
 * aligned, slots and out 16-byte aligned, scales 2-byte aligned.  Argument
 * errors return before any launch.
 */
tern_status tern_embed_gather(const int32_t *ids, int64_t M, const uint8_t *slots, const uint16_t *scales,
                              int64_t V, int64_t K, uint16_t *out, int32_t *bad_count, void *stream);

/*
 * The 1-bit variant.  Weights in {-1, +1} with the same fp16 scale per 128
 * weights along K, w = s_g * t: 1 + 16/128 = 1.125 bits per weight, about
 * 14.2x smaller than fp16 ("Bonsai 27B ternary / 1-bit quantization",
 * ThakiCloud blog, sections "What it is" and "How compression works").  The
 * pages fix no bit layout; this library's, for W with N rows and K columns:
 *
 *   bits    uint8 [N][K/8]   bit b = (t + 1) / 2 (0 -> -1, 1 -> +1) of weight
 *                            (n,k) at bit k%8 of byte n*K/8 + k/8
 *                            (least significant bit first);
 *   scales  fp16  [N][K/128] as for the ternary slots.
 *
 * tern_b1_pack -- build the bit layout.
 *   codes      int8 [N][K], each value -1 or +1                 (device, read)
 *   scales_in  fp16 [N][K/128] raw 16-bit patterns              (device, read)
 *   bits_out   uint8 [N][K/8]                                   (device, written)
 *   scales_out fp16 [N][K/128], a bit-exact copy (may equal scales_in)
 *   invalid_count  nullable device int32, incremented by the number of codes
 *              other than -1 and +1; such a code is stored as bit 0 (-1).
 * Alignment: codes and bits_out 16 bytes; scales 2 bytes; invalid_count 4.
 */
tern_status tern_b1_pack(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *bits_out,
                         uint16_t *scales_out, int32_t *invalid_count, void *stream);

/*
 * tern_b1_unpack -- inverse of the bit layout: codes_out int8 [N][K] gets -1
 * or +1 (device, written).  bits and codes_out 16-byte aligned.
 */
tern_status tern_b1_unpack(const uint8_t *bits, int64_t N, int64_t K, int8_t *codes_out, void *stream);

/*
 * tern_b1_gemv_step -- tern_gemv_step for 1-bit matrices: y = x * W^T with
 * w = s_g * t, t in {-1, +1}, for up to TERN_MAX_STEP matrices with the same
 * M (1..4) in one persistent launch.  Each descriptor's `slots` field points
 * to the bits (uint8 [N][K/8], as built by tern_b1_pack); everything else,
 * including the shape rules (K a multiple of 1024, x in shared memory), the
 * arithmetic (fp32 accumulation, fp16 output rounded to nearest even),
 * argument checking and error reporting, is as for tern_gemv_step.
 */
tern_status tern_b1_gemv_step(const tern_gemv_desc *descs, int32_t count, int64_t M, void *stream);

/*
 * Five trits per byte: a denser ternary storage, the "native ternary" packing
 * the pages expect closer to the log2(3) + 16/128 ~= 1.71 bits/weight ideal
 * than 2-bit slots ("Ternary-Bonsai-27B" model summary, aitrends.kr, sections
 * "TL;DR" and "Technical features"; "Ternary quantization: 27B in 7 GB",
 * devnsb blog, section "Limits").  The pages fix no layout; this library's,
 * for W with N rows and K columns (K a multiple of 128):
 *
 *   bytes   uint8 [N][R], R = 26 K / 128 rounded up to a multiple of 16: in
 *           each 128-weight group g of a row, weight j (0..127) is base-3
 *           digit j % 5 (least significant first) of byte 26 g + j / 5, the
 *           digit being the code c = t + 1 (0 -> -1, 1 -> 0, 2 -> +1); byte
 *           25 of a group holds weights 125..127 (digits 3, 4 are 0); the
 *           row padding is zero.  Byte values 243..255 are invalid.
 *   scales  fp16 [N][K/128] as for the 2-bit slots.
 *
 * 26 * 8 / 128 + 16 / 128 = 1.75 bits per weight (2-bit slots: 2.125).
 *
 * tern_t5_bytes -- N * R, or 0 for invalid arguments.
 */
size_t tern_t5_bytes(int64_t N, int64_t K);

/*
 * tern_t5_pack -- build the five-per-byte layout.
 *   codes      int8 [N][K] in {-1, 0, +1}                        (device, read)
 *   scales_in  fp16 [N][K/128] raw 16-bit patterns               (device, read)
 *   bytes_out  uint8 [N][R], R as above (tern_t5_bytes / N)      (device, written)
 *   scales_out fp16 [N][K/128], a bit-exact copy (may equal scales_in)
 *   invalid_count  nullable device int32, incremented by the number of codes
 *              outside {-1, 0, +1}; such a code is stored as t = 0.
 * Alignment: codes and bytes_out 16 bytes; scales 2 bytes; invalid_count 4.
 */
tern_status tern_t5_pack(const int8_t *codes, const uint16_t *scales_in, int64_t N, int64_t K, uint8_t *bytes_out,
                         uint16_t *scales_out, int32_t *invalid_count, void *stream);

/*
 * tern_t5_unpack -- inverse: codes_out int8 [N][K] gets t = c - 1, or the
 * sentinel 2 for the five weights of an invalid byte.  16-byte alignment.
 */
tern_status tern_t5_unpack(const uint8_t *bytes, int64_t N, int64_t K, int8_t *codes_out, void *stream);

/*
 * tern_t5_gemv_step -- tern_gemv_step for five-per-byte matrices: each
 * descriptor's `slots` field points to the bytes (uint8 [N][R]); shapes
 * (K a multiple of 1024, M in 1..8), arithmetic, argument checks and error
 * reporting as for tern_gemv_step.  The kernel keeps a 32 KiB decode table
 * in shared memory, so products are cut into K segments at a smaller K than
 * for tern_gemv_step (M = 4 at K = 17408 runs as two).
 * An invalid byte contributes an unspecified finite value for its weights.
 */
tern_status tern_t5_gemv_step(const tern_gemv_desc *descs, int32_t count, int64_t M, void *stream);

/*
 * tern_sync_status -- wait for `stream`, then report whether any kernel of
 * this library on the current device gave up a bounded on-device wait since
 * the previous call (TERN_ERR_TIMEOUT), clearing that record.  No kernel of
 * this library spins without a limit: a wait that exceeds it (1 s by default)
 * makes the kernel stop, release its resources and return, leaving its output
 * undefined and the CUDA context usable.  A library built with in-kernel
 * index checks (build.py: debug) also reports TERN_ERR_GUARD when a check in
 * the decode-step kernels failed since the previous call (the access was
 * skipped, nothing trapped); the normal build has no such checks.
 */
tern_status tern_sync_status(void *stream);

/*
 * Process-wide tuning knobs, for tests and benchmarks.  Value 0 restores the
 * built-in default.  Not thread-safe.
 *   TERN_OPT_GEMV_KSPLIT   warps sharing one 16-row tile along K (1,2,4,8;
 *                          the TMA kernel may lower it for short K)
 *   TERN_OPT_GEMV_CLUSTER  CTAs sharing one tile along K through a thread
 *                          block cluster and distributed shared memory (1,2,4,8)
 *   TERN_OPT_GEMV_CTAS     cap on resident CTAs per SM used for the grid; for
 *                          the TMA-staged kernel 3 also selects the build with
 *                          the smaller register budget (default: 2 per SM)
 *   TERN_OPT_GEMM_PATH     1 = force the bandwidth kernel (M<=8 chunks),
 *                          2 = force the tensor-core kernel
 *   TERN_OPT_GEMM_MIN_M    smallest M (> 8) sent to the tensor-core kernel
 *                          (default 32)
 *   TERN_OPT_GEMV_VARIANT  bandwidth kernel: 0 = default (M = 1: the
 *                          decode-step kernel of tern_gemv_step where its
 *                          shape rules hold; M = 2..8: variant 4 where its
 *                          shape rules hold; else variant 2),
 *                          2 = TMA-staged mma.sync,
 *                          3 = tcgen05 kernel for M <= 4 (splits K through the
 *                          workspace), 4 = producer/consumer mma.sync kernel
 *                          for K a multiple of 1024 (one CTA per SM, one
 *                          logic operation per weight pair; other shapes take
 *                          the default kernel), 6 = variant 4 with token rows
 *                          in the mma columns also at M = 1 (variant 4 puts
 *                          the eight scale groups of a 1024-k slice there
 *                          when M = 1); 1 and 5 are not accepted (kernels
 *                          removed)
 *   TERN_OPT_GEMV_GRID     cap on the CTAs of the producer/consumer and
 *                          tensor-memory kernels
 *                          (0 = one per SM); smaller grids give every CTA
 *                          more tiles to split among its warps
 *   TERN_OPT_GEMV_PREFETCH L2 prefetch distance of the producer/consumer
 *                          kernel, in 16-row x 1024-k units per consumer warp;
 *                          0 or n <= ring depth = none (the default: measured
 *                          slower)
 *   TERN_OPT_STEP_FORM     arithmetic of the decode-step kernels (all three
 *                          weight storages): 0 = default (M = 1, 2: the digit
 *                          form -- 8-bit integer mma on weights unpacked four
 *                          per instruction against activations split into
 *                          four exact signed 8-bit digits; M = 3..8: the fp16
 *                          group-per-column form), 1 = the fp16 form at every
 *                          M, 2 = the digit form also at M = 3, 4 (measured
 *                          slower there: its staged activations leave one ring
 *                          stage per warp)
 *   TERN_OPT_TEST_STALL_US TESTS ONLY: the TMA loaders of the tensor-core and
 *                          the TMA-staged bandwidth kernels issue no loads, so
 *                          their waits can never complete, and every bounded
 *                          wait gives up after this many microseconds.
 *                          Exercises the timeout path; 0 = normal operation.
 */
enum {
    TERN_OPT_GEMV_KSPLIT = 1,
    TERN_OPT_GEMV_CLUSTER = 2,
    TERN_OPT_GEMV_CTAS = 3,
    TERN_OPT_GEMM_PATH = 4,
    TERN_OPT_GEMM_MIN_M = 5,
    TERN_OPT_TEST_STALL_US = 6,
    TERN_OPT_GEMV_VARIANT = 7,
    TERN_OPT_GEMV_GRID = 8,
    TERN_OPT_GEMV_PREFETCH = 9,
    TERN_OPT_STEP_FORM = 10
};
tern_status tern_set_option(int option, int64_t value);

#ifdef __cplusplus
}
#endif

#endif /* TERN_H */
