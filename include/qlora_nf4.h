/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) frozen-base NF4 LoRA linear layer.
 *
 * The layer is the QLoRA base linear: the frozen weight W0 [n_out, n_in] is
 * stored as 4-bit NormalFloat codes in blocks of 64 with one absmax scale per
 * block, and those scales are quantized again to 8 bits in groups of 256 with
 * one fp32 constant per group ("QLoRA double quantization and block-wise
 * quantization memory" page, sections 1.2, 2.2 and 2.3; "5.8 QLoRA: 4-bit
 * base + 16-bit sticky notes" page, "three parts that make it work").  The
 * forward pass is y = W0 x + (alpha / r) B (A x) ("Training LoRA directly on
 * GGUF quantized weights" page, section 2.1 formula and section 3.2 module);
 * the backward pass treats W0 as a read-only operator and returns dX, dA and
 * dB (same page, section 2.1).
 *
 * Conventions shared by every call
 * --------------------------------
 * Layouts are row-major.  W0 is [N, K] = [n_out, n_in]; X [M, K];
 * A [r, K]; B [N, r]; Y [M, N]; dY [M, N]; dX [M, K]; U = X A^T [M, r];
 * G = dY B [M, r].  bf16 tensors are passed as pointers to 16-bit words
 * (qlora_bf16) holding IEEE bfloat16 bit patterns.
 *
 * Memory: every pointer is DEVICE memory owned by the caller, except where a
 * parameter says "host".  The library allocates no device memory in any
 * call; scratch space is the caller's `ws` buffer of at least
 * qlora_workspace_bytes(...) bytes, except in
 * qlora_lora_linear_fwd_static_ws, which uses a fixed scratch array held by
 * the library.  Device pointers must be 16-byte aligned.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream).  Calls only enqueue work; they do not synchronise.
 *
 * Errors: every call validates its arguments on the host before launching
 * anything and returns a qlora_status; on failure nothing is launched and
 * qlora_last_error() returns a message (thread-local).  Kernels never trap:
 * a pipeline wait that exceeds its time limit (about two seconds) sets a
 * device error word and the kernel returns; qlora_sync_status() reports it
 * as QLORA_ERR_TIMEOUT.  Non-finite weights give unspecified codes.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t qlora_bf16;

typedef enum {
    QLORA_OK = 0,
    QLORA_ERR_ARG = 1,        /* null pointer, bad flag, bad scaling             */
    QLORA_ERR_SHAPE = 2,      /* sizes out of range or not multiples of 64 / 8   */
    QLORA_ERR_ALIGN = 3,      /* a device pointer is not 16-byte aligned         */
    QLORA_ERR_WORKSPACE = 4,  /* ws missing or smaller than qlora_workspace_bytes */
    QLORA_ERR_CUDA = 5,       /* a CUDA runtime call or launch failed            */
    QLORA_ERR_TIMEOUT = 6,    /* a kernel gave up waiting (reported by sync)     */
    QLORA_ERR_UNSUPPORTED = 7 /* no sm_100 device / wrong architecture           */
} qlora_status;

/* 4-bit level sets ("QLoRA double quantization ..." page, section 3.3: the
 * quant type is nf4 or fp4).  NF4: the normal-quantile levels of
 * qlora_nf4_codebook.  FP4 (a reading; the pages print no values): the E2M1
 * 4-bit float magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 divided by 6, both signs,
 * ascending, with -0 at index 7 and +0 at index 8; a zero or tiny negative
 * normalised value takes index 7, a tiny positive one index 8. */
enum { QLORA_QT_NF4 = 0, QLORA_QT_FP4 = 1 };

/* Storage format of the first-level scales, as bit flags ("QLoRA double
 * quantization ..." page, section 3.1: block size 64 or 128; section 3.2: the
 * double-quantization switch; sections 1.3 and 2.3 give what each costs).
 * 0 is the QLoRA default: blocks of 64, double quantization on. */
enum {
    QLORA_FMT_BLOCK128 = 1,      /* first-level blocks of 128 weights (n_in % 128 == 0) */
    QLORA_FMT_NO_DQ = 2,         /* scales are the fp32 block absmaxes; scales2 unused   */
    QLORA_FMT_CODES_AFTER_DQ = 4 /* encode only: codes are taken against the dequantized
                                    scale fp32(q_b * d_g) instead of a_b (needs DQ);
                                    a normalised value beyond +-1 takes the end level    */
};

/* Packed 4-bit weight.  All buffers are device memory owned by the caller.
 * With B = 64 (or 128 under QLORA_FMT_BLOCK128): numel = n_out * n_in must be a
 * multiple of B and n_in a multiple of B (blocks never straddle rows).
 * quant_type selects the 16 levels (QLORA_QT_NF4 or QLORA_QT_FP4); format the
 * scale storage (QLORA_FMT_* flags, 0 = default).  Every call encodes,
 * dequantizes and multiplies with the weight's levels and format.  The
 * descriptor is 48 bytes.
 *   codes   : numel / 2 bytes; weight element 2j (row-major flattening) is
 *             in bits 0-3 of byte j, element 2j+1 in bits 4-7; each code
 *             indexes the 16 levels of the weight's quant type (see
 *             qlora_codebook).
 *   scales  : double quant: numel / B bytes; block b (elements [Bb, Bb+B)) has
 *             first-level scale q_b in 0..255.  No double quant: numel / B
 *             floats, the block absmax a_b itself.
 *   scales2 : double quant: ceil(numel / (256 B)) floats; group g (blocks
 *             [256g, 256g+256)) has second-level step d_g.  Unused (may be
 *             NULL) without double quant.
 * The dequantized block scale is s_b = fp32(q_b * d_g) (or a_b) and the weight
 * is fp32(c[code] * s_b). */
typedef struct {
    int64_t n_out;
    int64_t n_in;
    uint8_t *codes;
    uint8_t *scales;
    float *scales2;
    int32_t quant_type;
    int32_t format;
} qlora_nf4_weight;

/* Bytes of the three packed buffers together: numel/2 + numel/64 +
 * 4*ceil(numel/16384) (the closed form of the "QLoRA double quantization"
 * page, section 2.3).  Returns 0 if numel is not a positive multiple of 64. */
size_t qlora_packed_bytes(int64_t numel);

/* The same for a storage format (QLORA_FMT_* flags): numel/2 + numel/B +
 * 4*ceil(numel/(256 B)) with double quantization, numel/2 + 4*numel/B without
 * (B = 64 or 128).  Returns 0 for a numel that is not a positive multiple of B
 * or an invalid format. */
size_t qlora_packed_bytes_fmt(int64_t numel, int32_t format);

/* Writes the 16 NF4 levels (ascending float32, out[0] = -1, out[7] = 0,
 * out[15] = +1) to the HOST array out.  The levels are the normal quantiles
 * of the "5.8 QLoRA" page's NF4 paragraph: 8 positive and 7 negative
 * quantiles at equal probability steps below the offset
 * delta = ((1 - 1/30) + (1 - 1/32)) / 2, each divided by Phi^-1(delta),
 * plus an exact zero.  Returns QLORA_ERR_ARG if out is NULL. */
qlora_status qlora_nf4_codebook(float out[16]);

/* The 16 levels of quant type `quant_type` (QLORA_QT_NF4 or QLORA_QT_FP4) as
 * float32, ascending, into the HOST array out.  QLORA_ERR_ARG for another
 * type or a NULL out. */
qlora_status qlora_codebook(int quant_type, float *out);

/* Encode: W [n_out, n_in] fp32 (device) -> w->codes, w->scales, w->scales2.
 * Per block of B (64, or 128 under QLORA_FMT_BLOCK128): a_b = max |w|;
 * code = index of the level nearest to fp32(w / a_b), exact ties to the lower
 * index (a_b = 0 gives the code of 0).  Per group of 256 blocks:
 * d_g = fp32(max a_b / 255) and q_b = clamp(round_half_even(fp32(a_b / d_g)),
 * 0, 255) (d_g = 0 gives 0).  QLORA_FMT_NO_DQ stores a_b instead of q_b and
 * d_g; QLORA_FMT_CODES_AFTER_DQ normalises by s_b = fp32(q_b * d_g) instead of
 * a_b (s_b = 0 gives the code of 0).  Sections 1.2-3.2 of the "QLoRA double
 * quantization" page.  Bit-exact. */
qlora_status qlora_quantize_nf4_dq(const float *W, const qlora_nf4_weight *w, void *stream);

/* Dequant the whole weight (the "one-shot dequant" route of the GGUF page,
 * section 2.2): out [n_out, n_in] receives fp32(c[code] * fp32(q_b * d_g)),
 * as float32 (out_is_bf16 = 0) or rounded to bfloat16 ties-to-even
 * (out_is_bf16 = 1).  Bit-exact. */
qlora_status qlora_dequant(const qlora_nf4_weight *w, void *out, int out_is_bf16, void *stream);

/* Merge the adapter into the base and quantize again (the deployment step of
 * the "Course notes: LLM basics and quantized fine-tuning" page, section 3.3,
 * and of the GGUF page, sections 3.3 and 4.3: dequantize the base to bf16,
 * merge at high precision, rerun the quantization):
 *   m[n, k] = bf16(fp32(bf16(w'[n, k]) + scaling * sum_j B[n, j] A[j, k])),
 * the sum and the add in float64 with j ascending, then w_out = the NF4 +
 * double-quant encode of m (as qlora_quantize_nf4_dq).  A [r, K] and B [N, r]
 * are bf16 with the rank rules of qlora_lora_linear_fwd; r = 0 requantizes
 * bf16(w').  W_scratch: caller-owned device float32 [n_out, n_in] (4 * numel
 * bytes); it holds m when the call completes.  w_out has the shape of w_in and
 * may be w_in itself (the merge reads all of w_in before the encode writes).
 * Bit-exact. */
qlora_status qlora_lora_merge_requant(const qlora_nf4_weight *w_in, const qlora_bf16 *A, const qlora_bf16 *B, int r,
                                      float scaling, float *W_scratch, const qlora_nf4_weight *w_out, void *stream);

/* Scratch bytes needed by qlora_lora_linear_fwd / qlora_lora_linear_bwd_dx for
 * these sizes (N = n_out, K = n_in).  0 is never returned for valid sizes. */
size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/* Forward: Y = X W'^T + scaling * (X A^T) B^T, W' the dequantized base.
 *   X [M, K] bf16, A [r, K] bf16, B [N, r] bf16, Y [M, N] bf16 (output).
 *   r = 0 disables the adapter (A, B may then be NULL); otherwise
 *   8 <= r <= 128 and r % 8 == 0.  scaling = alpha / r, computed by the
 *   caller (the GGUF page's section 3.2 module).
 *   U_save [M, r] bf16 receives U = X A^T (needed by qlora_lora_grad_AB), or
 *   NULL.  ws / ws_bytes: caller scratch of qlora_workspace_bytes(M, N, K, r).
 * The base term is computed on tensor cores from bf16 operands with fp32
 * accumulation; the weight operand is bf16(bf16(c[code]) * bf16(s_b)). */
qlora_status qlora_lora_linear_fwd(const qlora_nf4_weight *w, const qlora_bf16 *X, int64_t M,
                                   const qlora_bf16 *A, const qlora_bf16 *B, int r, float scaling,
                                   qlora_bf16 *Y, qlora_bf16 *U_save,
                                   void *ws, size_t ws_bytes, void *stream);

/* Size of the library's static device scratch used by
 * qlora_lora_linear_fwd_static_ws: 8 MiB on each device. */
#define QLORA_STATIC_SCRATCH_BYTES ((size_t)8 << 20)

/* The forward of qlora_lora_linear_fwd (same arguments, same kernels, same
 * results) with no ws / ws_bytes: its scratch is a file-scope
 * `__device__` array of QLORA_STATIC_SCRATCH_BYTES that the library's module
 * holds on every device where it is loaded.  The QLoRA paper has no
 * counterpart to this call; it exists for callers that cannot allocate
 * device memory for a workspace: a plain-C host that is handed only the
 * layer's tensors and has no allocator of its own; a process whose free
 * device memory is already reserved by a caching allocator (torch's, for
 * one), where a cudaMalloc of its own fails with out-of-memory; and a loop
 * in which cudaFree's implicit device synchronisation would stall the
 * other streams.  This call makes no cudaMalloc, cudaFree or other
 * allocating call.
 *   Set-up: the first call on each device, with that device current, looks
 *   up the array's device address (cudaGetSymbolAddress) and keeps it for
 *   later calls; a failure of that lookup returns QLORA_ERR_CUDA.  Make
 *   this first call on a device before any stream capture.
 *   Limit: when the forward's scratch need for these sizes (the rank-r
 *   buffers, about 6 * M * r bytes, plus a 4 * M * N byte split-K
 *   accumulator when M < 64 and K is split) exceeds
 *   QLORA_STATIC_SCRATCH_BYTES, the call
 *   returns QLORA_ERR_WORKSPACE before touching the device; use
 *   qlora_lora_linear_fwd with a caller workspace instead.
 *   Zeroing: the fp32 accumulators in the scratch are cleared on `stream`
 *   by every call before its kernels add into them.
 *   Concurrency: every call on a device uses the same scratch, so two calls
 *   whose work overlaps in time (different streams, or host threads with no
 *   ordering between their streams) race and give wrong results; order them
 *   on one stream or with events. */
qlora_status qlora_lora_linear_fwd_static_ws(const qlora_nf4_weight *w, const qlora_bf16 *X, int64_t M,
                                             const qlora_bf16 *A, const qlora_bf16 *B, int r, float scaling,
                                             qlora_bf16 *Y, qlora_bf16 *U_save, void *stream);

/* Backward to the input: dX = dY W' + scaling * (dY B) A  (the frozen base
 * is a read-only operator; no gradient is formed for W0).
 *   dY [M, N] bf16, dX [M, K] bf16 (output), G_save [M, r] bf16 receives
 *   G = dY B, or NULL.  Other arguments as in qlora_lora_linear_fwd. */
qlora_status qlora_lora_linear_bwd_dx(const qlora_nf4_weight *w, const qlora_bf16 *dY, int64_t M,
                                      const qlora_bf16 *A, const qlora_bf16 *B, int r, float scaling,
                                      qlora_bf16 *dX, qlora_bf16 *G_save,
                                      void *ws, size_t ws_bytes, void *stream);

/* Adapter gradients ("only A and B are updated", course-notes page LoRA
 * section): dA = scaling * G^T X  [r, K] fp32 and dB = scaling * dY^T U
 * [N, r] fp32, with U and G as saved by the two calls above.  accumulate = 1
 * adds into dA and dB, 0 overwrites them.  8 <= r <= 128, r % 8 == 0,
 * K % 64 == 0, N % 8 == 0. */
qlora_status qlora_lora_grad_AB(const qlora_bf16 *X, const qlora_bf16 *dY, const qlora_bf16 *U,
                                const qlora_bf16 *G, int64_t M, int64_t N, int64_t K, int r,
                                float scaling, float *dA, float *dB, int accumulate, void *stream);

/* ------------------------------------------------------------------ Q8_0 route
 * The Q8_0 block format ("Training LoRA directly on GGUF quantized weights"
 * page, section 1.1: 32 weights share one fp16 scale, a little over one byte
 * per weight; section 2.2: the blocks are dequantized inside the GEMM, or the
 * whole matrix at once).  Reading (the page gives no formula): symmetric int8
 * per block as in the "Quantized vs. non-quantized weights" page, section
 * 2.1: d = fp16(max |w| / 127), q = clamp(round_half_even(w / d), -127, 127),
 * w' = q * d (exact in fp32); d = 0 gives q = 0.  The page fixes no byte layout:
 * the codes and the scales are two row-major arrays.  n_in % 64 == 0.
 *   q : numel int8 codes, [n_out, n_in] row-major (device)
 *   d : numel / 32 fp16 scales as IEEE binary16 bit patterns; block b covers
 *       elements [32b, 32b + 32) of the row-major flattening (device) */
typedef struct {
    int64_t n_out;
    int64_t n_in;
    int8_t *q;
    uint16_t *d;
} qlora_q8_0_weight;

/* numel + 2 * numel / 32 bytes (34 bytes per 32 weights); 0 unless numel is a
 * positive multiple of 32. */
size_t qlora_q8_0_packed_bytes(int64_t numel);

/* Encode W [n_out, n_in] fp32 (device) into w->q and w->d, as above.  Bit-exact. */
qlora_status qlora_quantize_q8_0(const float *W, const qlora_q8_0_weight *w, void *stream);

/* One-shot dequant: out [n_out, n_in] receives q * d as float32 (out_is_bf16 =
 * 0) or rounded to bfloat16 ties-to-even (1).  Bit-exact. */
qlora_status qlora_dequant_q8_0(const qlora_q8_0_weight *w, void *out, int out_is_bf16, void *stream);

/* qlora_lora_linear_fwd with a Q8_0 base: the int8 codes and fp16 scales are
 * expanded in the GEMM main loop to the bf16 operand bf16(q * d).  Same
 * arguments, rules and workspace (qlora_workspace_bytes covers it). */
qlora_status qlora_q8_0_lora_linear_fwd(const qlora_q8_0_weight *w, const qlora_bf16 *X, int64_t M,
                                        const qlora_bf16 *A, const qlora_bf16 *B, int r, float scaling,
                                        qlora_bf16 *Y, qlora_bf16 *U_save, void *ws, size_t ws_bytes, void *stream);

/* qlora_lora_linear_bwd_dx with a Q8_0 base (the transposed dequant in the main
 * loop); dA and dB come from qlora_lora_grad_AB as for the 4-bit base. */
qlora_status qlora_q8_0_lora_linear_bwd_dx(const qlora_q8_0_weight *w, const qlora_bf16 *dY, int64_t M,
                                           const qlora_bf16 *A, const qlora_bf16 *B, int r, float scaling,
                                           qlora_bf16 *dX, qlora_bf16 *G_save, void *ws, size_t ws_bytes,
                                           void *stream);

/* Waits for `stream`, then reports and clears a device-side error recorded by
 * any earlier kernel of this library on the current device: a pipeline wait
 * that timed out (QLORA_ERR_TIMEOUT) or a tensor-memory store whose read-back
 * check failed (QLORA_ERR_CUDA). */
qlora_status qlora_sync_status(void *stream);

/* Message describing the last failure on the calling thread ("" if none). */
const char *qlora_last_error(void);

/* Sets, on the current device, the time after which any pipeline wait of this
 * library's kernels gives up (the pages have no counterpart: this is the
 * failure-detection path of the kernels).  ns must lie in [1e6, 6e10]; the
 * default is 2e9 (two seconds).  The copy is synchronous: call it with no
 * kernel of this library in flight and outside stream capture.  QLORA_ERR_ARG
 * for an out-of-range ns. */
qlora_status qlora_set_wait_limit_ns(uint64_t ns);

/* Self-test of that path: enqueues on `stream` one tiny kernel whose single
 * pipeline wait has nothing to wait for.  It gives up after the current limit,
 * records a timeout in the device error word and returns, so the next
 * qlora_sync_status reports QLORA_ERR_TIMEOUT and clears it; the CUDA context
 * stays usable.  Nothing else is touched. */
qlora_status qlora_probe_wait_timeout(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
