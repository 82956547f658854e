/*
 * ternary_b200.h -- C ABI of libternary_b200.so: the ternary-g128 linear layer
 * with a signed block-Hadamard rotation, on NVIDIA B200 (sm_100a).
 *
 * What the layer is (the pages' sections):
 *   - Ternary g128 weights: each weight t is -1, 0 or +1 and each run of 128
 *     consecutive weights along K shares one FP16 scale s, so w = s * t
 *     (news.ditty.ir, "Bonsai 2 27B", second paragraph; ai4coding.ru,
 *     "What is a ternary model").
 *   - A signed Hadamard rotation on blocks of 1024 inputs is folded into every
 *     weight matrix; its inverse must be applied to the activations at run
 *     time, and forgetting it gives silently wrong output (news.ditty.ir,
 *     second and third paragraphs; openbonsai.org, "How it works", "Rotate").
 *   - Multiplying by a ternary weight is an add, a subtract or nothing
 *     (ai4coding.ru, "What is a ternary model", last paragraph).
 *   - Two packings are named (a dense trit packing and a 2-bit slot packing,
 *     news.ditty.ir, paragraph on the CUDA GGUF files); the byte layouts below
 *     are this library's own.
 *
 * Conventions for every entry point:
 *   - Shapes: W is [N, K] (N outputs, K inputs), x is [M, K], y is [M, N],
 *     all row-major and densely packed (row stride = row length).
 *   - Every data pointer is a DEVICE pointer owned by the caller.  The library
 *     never allocates device memory and keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All device
 *     work is enqueued asynchronously on it; results are ready when the stream
 *     says so.
 *   - Arguments are validated synchronously, before anything is enqueued; a
 *     non-zero status means nothing was launched (TB_ERR_CUDA excepted, which
 *     reports a failed launch).
 *   - Bad data (codes outside {-1,0,1}, invalid packed bytes) is never trapped:
 *     pack/unpack count it into an optional device uint32 counter (added to,
 *     never reset, by the call).
 *   - Calls are thread-safe.  The only library state is a per-device cache of
 *     device attributes and one per-device fault word (see
 *     tb_get_device_fault).
 *   - Kernels are launched with programmatic dependent launch: a call may
 *     start reading its packed weights, scales and signs while the previous
 *     kernel on the stream is still running (activations and outputs wait for
 *     it).  Weights, scales and signs are layer constants; they must not be
 *     written by a kernel that lets its dependents launch early (the library's
 *     own pack kernel, like any plain kernel or copy, does not).
 *
 * Packed formats (codes only; the FP16 scales always live in a separate
 * [N, K/128] array, row-major, scale g of row n covering k = 128g..128g+127):
 *   TB_FMT_2BIT  : c = t + 1 in {0,1,2}.  Byte i of a row holds k = 4i..4i+3,
 *                  weight k = 4i+j in bits 2j..2j+1.  Row stride K/4 bytes.
 *                  c = 3 is invalid.  2 + 16/128 = 2.125 bits per weight.
 *   TB_FMT_BASE3 : each 128-group is its own run of 26 bytes.  Bytes 0..24 hold
 *                  k = 5i..5i+4 as sum_j c_{5i+j} * 3^j; byte 25 holds
 *                  k = 125..127 as c125 + 3 c126 + 9 c127 + 108 (digits 3 and 4
 *                  are the padding value 1).  Row stride 26*K/128 bytes.  A byte
 *                  >= 243, or a last byte whose digits 3, 4 are not both 1, is
 *                  invalid.  1.625 + 16/128 = 1.75 bits per weight.
 *   TB_FMT_1BIT  : 1-bit g128, the pages' other shipped format (each weight
 *                  -1 or +1 with one FP16 scale per 128; dev.to, "How Prism ML
 *                  Squeezed a 27B Model Into 3.9 GB", "Two formats ship
 *                  today").  Byte i of a row holds k = 8i..8i+7, weight 8i+j in
 *                  bit j, bit 1 = +1 and bit 0 = -1.  Row stride K/8 bytes.
 *                  Every byte is valid; the packer counts any code other than
 *                  -1, +1 (0 included) and packs it as -1.  1 + 16/128 =
 *                  1.125 bits per weight.
 *
 * Rotation (this library's reading of "signed block Hadamard"): for block b of
 * 1024 inputs with signs d_b in {-1,+1}, R_b = diag(d_b) H / 32 where H is the
 * Sylvester Hadamard matrix of order 1024 in natural order.  The weights are
 * stored as W' = W R; the run time applies x' = R^T x, i.e. per block
 * x'_b = H (d_b * x_b) / 32, so that W' x' = W x.
 */
#ifndef TERNARY_B200_H
#define TERNARY_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int tb_status;
#define TB_OK 0
#define TB_ERR_NULL 1      /* a required pointer is NULL                      */
#define TB_ERR_SHAPE 2     /* a size is <= 0 or breaks a divisibility rule    */
#define TB_ERR_DTYPE 3     /* unsupported dtype or dtype combination          */
#define TB_ERR_FORMAT 4    /* unknown packed format                            */
#define TB_ERR_ALIGN 5     /* a pointer breaks its alignment rule              */
#define TB_ERR_CUDA 6      /* a CUDA call or launch failed                     */
#define TB_ERR_WORKSPACE 7 /* workspace NULL or smaller than required          */
#define TB_ERR_DEVICE 8    /* current device is not a B200-class sm_100 GPU    */

typedef int tb_format;
#define TB_FMT_2BIT 0
#define TB_FMT_BASE3 1
#define TB_FMT_1BIT 2

typedef int tb_dtype;
#define TB_BF16 0
#define TB_FP16 1
#define TB_FP32 2
#define TB_INT8 3
#define TB_INT32 4

typedef int tb_path;
#define TB_PATH_AUTO 0   /* choose by shape (what tb_ternary_linear does)       */
#define TB_PATH_GEMV 1   /* CUDA-core streaming kernels on 16-bit fixed-point
                            activations, for M <= 4 (base-3: M <= 7, in chunks
                            of 4 tokens; 1-bit: M = 1).  One token (2-bit,
                            1-bit): one launch that rotates x itself for
                            K <= 8192                                          */
#define TB_PATH_GEMM 2   /* tcgen05 tensor-core kernel on CTA pairs (weights
                            unpacked into TMEM as the A operand: exact fp16
                            s*t against fp16 x', fp32 accumulators; integer
                            mode: kind::i8, the ternary codes as signed bytes
                            against int8 x, exact int32 accumulators, from 16
                            tokens, any K % 128, base-3 only with a workspace
                            to re-encode into);
                            base-3 from 8 tokens, re-encoded to 2-bit slots in
                            the workspace first; 1-bit from 2 tokens.  Chosen
                            by TB_PATH_AUTO past 16 tokens, or from 8 base-3
                            tokens when N is above the tensor-core decode's
                            148 * 128 rows                                    */
#define TB_PATH_SIMPLE 3 /* plain per-row kernel: any K % 128, any alignment    */
#define TB_PATH_GEMV_TC 4 /* tcgen05 decode kernel (codes unpacked into TMEM as
                            the u8 A operand, int8 activation planes as B in
                            shared memory, per-group int32 sums read back and
                            scaled), for M <= 16, any N; K is split over CTAs
                            when rows are few (partial sums in the workspace,
                            added in a fixed order).  base-3 with 8-16 tokens is
                            first re-encoded to 2-bit slots in the workspace.
                            Chosen by TB_PATH_AUTO from 4 tokens (2-bit) or 8
                            tokens (base-3)                                    */

/* Human-readable name of a status code (static string, never NULL). */
const char* tb_status_string(tb_status st);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int tb_version(void);

/* Bytes of packed codes for an [N, K] matrix in format f (scales excluded;
 * they take N * K/128 * 2 bytes).  Returns 0 for an unknown format, N <= 0,
 * K <= 0 or K % 128 != 0. */
size_t tb_packed_bytes(tb_format f, int64_t N, int64_t K);

/* Pack int8 codes [N, K] (values -1, 0, +1) into format f.
 *   codes  : device, N*K int8.
 *   packed : device, tb_packed_bytes(f, N, K) bytes, written in full.
 *   d_invalid_count : device uint32 or NULL.  Every code outside {-1,0,1} is
 *            packed as 0 (1-bit: every code outside {-1,+1} is packed as -1)
 *            and, when non-NULL, adds 1 to *d_invalid_count.
 * Requires K % 128 == 0; codes and packed 16-byte aligned (else TB_ERR_ALIGN).
 * Defined by the format description above; no counterpart kernel on the pages. */
tb_status tb_pack_ternary(tb_format f, const int8_t* codes, int64_t N, int64_t K,
                          uint8_t* packed, uint32_t* d_invalid_count, void* stream);

/* Unpack format-f bytes into int8 codes [N, K].  Invalid slots/bytes decode to
 * 0 and, when d_invalid_count is non-NULL, add 1 each (2-bit: per slot holding
 * 3; base-3: per invalid byte; 1-bit has none).  Same size/alignment rules as
 * tb_pack_ternary. */
tb_status tb_unpack_ternary(tb_format f, const uint8_t* packed, int64_t N, int64_t K,
                            int8_t* codes, uint32_t* d_invalid_count, void* stream);

/* Apply the block rotation to each row of x [M, K] (K % 1024 == 0).
 *   inverse = 0 : y_b = H (d_b * x_b) / 32   (x' = R^T x, the run-time step
 *                 before a rotated linear layer, news.ditty.ir third paragraph)
 *   inverse = 1 : y_b = d_b * (H x_b) / 32   (x = R x')
 *   xt in {BF16, FP16, FP32}, yt in {BF16, FP16, FP32}; computed in fp32.
 *   signs : device, K int8, each -1 or +1 (other values are used as given).
 *   y may equal x when xt == yt (in place); any other overlap is undefined.
 * Alignment: x, y 16-byte aligned. */
tb_status tb_hadamard_rotate(const void* x, tb_dtype xt, void* y, tb_dtype yt,
                             const int8_t* signs, int64_t M, int64_t K, int inverse,
                             void* stream);

/* Producer side: fold the block rotation into a dense weight matrix and round
 * it to ternary g128 (openbonsai.org, "How it works", steps 1 "Rotate" and
 * 2 "Round"; the pages round with sequential GPTQ on calibration data, which
 * needs a model and data; this is the plain stand-in).
 *   w      : device [N, K] row-major, wt in {BF16, FP16, FP32}, 4-byte aligned.
 *   signs  : device K int8 (+-1) of the layer's rotation, 8-byte aligned; NULL
 *            = w is already folded (only rounded).
 *   Fold   : w'_b = H (d_b * w_b) / 32 per row and 1024-block (W' = W R).
 *   Round  : per 128-group s = fp16(mean |w'|) (nearest, ties to even),
 *            t = clip(rint(w' / s), -1, 1) (rint: halves to even), t = 0 where
 *            s = 0.
 *   packed : device, tb_packed_bytes(f, N, K) bytes, 16-byte aligned (2-bit
 *            slots or base-3); scales: device [N, K/128] fp16 bits.  Both
 *            written in full, nothing else touched.
 * Computed in fp64 with one rounding to fp16 for the scale: wherever the fp64
 * sums of the fold and of the group's |w'| are exact (all bf16 and fp16 input;
 * fp32 input spanning fewer than about 40 binary orders inside a block) the
 * codes and scales equal those of exact arithmetic.  K % 1024 == 0 (else
 * TB_ERR_SHAPE); TB_FMT_2BIT or TB_FMT_BASE3 (else TB_ERR_FORMAT). */
tb_status tb_prepare_weights(const void* w, tb_dtype wt, const int8_t* signs, int64_t N, int64_t K,
                             tb_format f, uint8_t* packed, uint16_t* scales, void* stream);

/* Device workspace bytes tb_ternary_linear needs for these sizes (any path,
 * any dtype).  0 means none.  Returns 0 also for invalid sizes. */
size_t tb_ternary_linear_workspace(tb_format f, int64_t M, int64_t N, int64_t K);

/* y = x' W^T with W the ternary g128 matrix given by (packed, scales, f).
 *   x       : device [M, K].  xt in {BF16, FP16, FP32}: float mode; xt = INT8:
 *             integer mode.
 *   signs   : device [K] int8, each -1 or +1, or NULL.  Non-NULL: x is
 *             unrotated and the rotation x' = R^T x is applied first (needs
 *             K % 1024 == 0).
 *             NULL: x is taken as already rotated.  Must be NULL in integer mode.
 *   scales  : device [N, K/128] fp16 bit patterns.  Ignored in integer mode.
 *   y       : device [M, N]; yt in {FP32, BF16} in float mode, INT32 in integer
 *             mode (y[m,n] = sum_k t[n,k] x[m,k], exact).
 *   Integer mode needs no workspace (pass NULL, 0), except that base-3 weights
 *   reach the tensor-core path (16 tokens and more) only when a workspace of
 *   tb_ternary_linear_workspace bytes is passed to re-encode them into;
 *   without one they take the plain kernel (same exact result).
 *   workspace : device, at least tb_ternary_linear_workspace(f, M, N, K) bytes,
 *             16-byte aligned; its contents on entry do not matter and are
 *             overwritten.  Must not be shared by calls in flight at once.
 * Requires M >= 1, N >= 1, K % 128 == 0; packed, scales, x, y 16-byte aligned
 * (else the plain kernel is used; pointers only need natural alignment then).
 * Float results agree with the exact product to relative L2 error <= 2e-3 and
 * per element <= 1e-2 * max|s| * ||x_m||_2.  Invalid packed bytes give
 * unspecified values in the affected outputs (no fault). */
tb_status tb_ternary_linear(const void* x, tb_dtype xt, const uint8_t* packed,
                            const uint16_t* scales, tb_format f, int64_t M, int64_t N,
                            int64_t K, const int8_t* signs, void* y, tb_dtype yt,
                            void* workspace, size_t ws_bytes, void* stream);

/* tb_ternary_linear with the kernel path chosen by the caller (tests, tuning).
 * A path that cannot take the arguments returns TB_ERR_SHAPE without launching
 * anything: GEMV needs float mode, M <= 4 (base-3: M <= 7), K % 1024 == 0 and
 * 16-byte aligned packed/scales; GEMV_TC needs float mode, M <= 16 (base-3:
 * 8 <= M <= 16), K % 1024 == 0, aligned pointers and a plan that fits the
 * SMs; GEMM needs float mode, K % 1024 == 0 and aligned pointers (base-3:
 * M >= 8, re-encoded to 2-bit slots in the workspace first); SIMPLE takes
 * everything tb_ternary_linear takes. */
tb_status tb_ternary_linear_ex(const void* x, tb_dtype xt, const uint8_t* packed,
                               const uint16_t* scales, tb_format f, int64_t M, int64_t N,
                               int64_t K, const int8_t* signs, void* y, tb_dtype yt,
                               void* workspace, size_t ws_bytes, tb_path path,
                               void* stream);

/* Which path tb_ternary_linear would take for these arguments (a tb_path
 * value), or -1 if it would reject them. */
int tb_ternary_linear_path(tb_dtype xt, tb_format f, int64_t M, int64_t N, int64_t K,
                           int has_signs, int aligned16);

/* Bytes of the library's fixed device scratch used by tb_ternary_linear_noalloc
 * (576 KiB). */
#define TB_NOALLOC_SCRATCH_BYTES 589824

/* tb_ternary_linear without a workspace argument: the decode (GEMV) path with
 * its activation scratch in a fixed array inside the library instead of in
 * caller memory.  The pages have no counterpart; it exists for callers that
 * cannot allocate device memory: a plugin inside a host runtime that owns every
 * device allocation and hands plugins none, or a latency-critical decode loop
 * that must not call cudaMalloc / cudaFree, which can synchronise the device.
 * It allocates nothing itself (no cudaMalloc, no cudaFree, no library routine
 * that allocates).
 *   Takes the arguments of tb_ternary_linear minus the workspace, with the
 *   GEMV path's rules: float mode, TB_FMT_2BIT, M <= 4, K % 1024 == 0, all
 *   pointers 16-byte aligned (else TB_ERR_SHAPE / TB_ERR_ALIGN / TB_ERR_DTYPE).
 *   The decode path needs M * (2K + K/16 + 8448) bytes of scratch, and for
 *   one token at least K/128 * 280 bytes (the one-token kernel's activation
 *   words when K is too long for it to rotate x itself); the larger figure
 *   must fit TB_NOALLOC_SCRATCH_BYTES (576 KiB), which allows K up to 269312
 *   at M = 1, 138240 at M = 2, 91136 at M = 3 and 66560 at M = 4.  Larger
 *   sizes return TB_ERR_WORKSPACE ("too big for the library's fixed
 *   scratch") and nothing is launched.
 *   Every GPU that loads the library holds the scratch until the process exits.
 *   The first call on a device looks up the scratch's device address (a host
 *   call that does not allocate); make that first call before any stream
 *   capture.  All calls on a device share the one scratch and every call
 *   overwrites the part it reads, so nothing needs clearing between calls, but
 *   calls that can overlap on the GPU (different streams without ordering)
 *   race on it: order them on one stream. */
tb_status tb_ternary_linear_noalloc(const void* x, tb_dtype xt, const uint8_t* packed,
                                    const uint16_t* scales, int64_t M, int64_t N, int64_t K,
                                    const int8_t* signs, void* y, tb_dtype yt, void* stream);

/* Read, and with clear != 0 reset, the fault word of the current device.  Every
 * wait inside the library's kernels is bounded; a wait that gives up (a
 * producer that never delivered) records a non-zero code here and the kernel
 * returns early instead of hanging, leaving its outputs incomplete.  0 = no
 * fault recorded.  Synchronous (waits for the device's work to finish). */
tb_status tb_get_device_fault(uint32_t* code, int clear);

/* Failure-detection test hook (no counterpart on the pages).  With stall != 0
 * the weight-copy producers of the one-token decode kernel and of the fp16
 * GEMM issue nothing, so every wait for those copies runs out: the kernel
 * records FAULT code 1 (a consumer gave up waiting for a stage) in the fault
 * word, returns without hanging and leaves its output incomplete.
 * wait_limit_ns sets how long a bounded wait lasts (0 = the default 2 s), for
 * every kernel of the library on the current device.  Synchronous; call it
 * between kernels, with nothing of the library in flight, and call it again
 * with (0, 0) to restore normal operation. */
tb_status tb_test_stall_copies(uint32_t stall, uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* TERNARY_B200_H */
