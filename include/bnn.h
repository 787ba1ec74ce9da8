/*
 * bnn.h -- C ABI of libbnn.so: the binary (+1/-1 weights, +1/-1 activations)
 * matrix product on bit-packed operands, on NVIDIA B200 (sm_100a).
 *
 * What is computed (page title, section / equation):
 *  - "Extreme Quantization: Binary, Ternary & 1-bit LLMs", XNOR-Net section,
 *    eq. (4) and eq. (6): w_b = sign(w), x_b = sign(x),
 *    w_b^T x_b = K - 2 * popcount(w~ XOR x~).
 *  - same page, Notation: sign(x) = +1 for x >= 0, -1 for x < 0.
 *  - same page, Binary Neural Networks section, eq. (1):
 *    y = alpha * (w_b^T x), alpha = (1/n) * sum_i |w_i| (one alpha per filter,
 *    i.e. per output channel, as in the "Binary Neural Network (BNN)" glossary
 *    paragraph on BatchNorm and scaling factors).
 *  - "First Principles: Why Binary Ops Can Be Exponentially Faster",
 *    section "1. Arithmetic: MAC -> XNOR + popcount": encoding bit 0 -> +1,
 *    bit 1 -> -1; bits packed into machine words; pad bits encode +1.
 *
 * PACKED LAYOUT (used by every call).  A packed row of K elements is an array
 * of uint32 words; bit j of word w is element 32*w + j (least significant bit
 * first), 1 meaning -1 and 0 meaning +1.  The row holds
 * bnn_packed_ld_words(K) = ceil(K/32) rounded up to a multiple of 4 words, so
 * each row is a whole number of 16-byte units; the bits past element K-1 and
 * the words past ceil(K/32) are 0 (they encode +1 in both operands, so they
 * never add to the popcount).  The uint64 view of the same bytes (little
 * endian) is the 64-bit packing.  Row r of a packed matrix starts at word
 * r * ld, where ld (the row stride, in words) is >= bnn_packed_ld_words(K)
 * and a multiple of 4.  Words between bnn_packed_ld_words(K) and ld are never
 * read or written.
 *
 * CONVENTIONS.
 *  - Device pointers are CUDA device (or managed) memory on the current
 *    device, owned by the caller; the library keeps no pointer after a call
 *    returns and allocates no device memory: a call that needs scratch space
 *    takes a caller-owned workspace.  The one exception is
 *    bnn_ternary_pack_noalloc, whose scratch is a fixed library-owned device
 *    array (about 2 MiB per GPU that loads the library; see there).  Host
 *    pointers are named so.
 *  - Every device call is asynchronous on `stream` (NULL = legacy default
 *    stream).  It returns after the launch; results are visible to later
 *    work on the same stream.
 *  - Arguments are checked on the host before anything is launched; a failed
 *    check returns an error status and writes nothing.  Launch failures
 *    return BNN_ERR_CUDA.  No exception crosses the ABI, nothing traps on the
 *    device, and there is no CPU fallback.
 *  - Packed operands and all vector loads need 16-byte aligned pointers.
 *  - A kernel that waits on an asynchronous copy gives up after about one
 *    second, records BNN_ERR_DEVICE_TIMEOUT in a device-side flag and returns;
 *    bnn_device_error() reads and clears that flag.
 */
#ifndef BNN_H_
#define BNN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
struct CUstream_st;
typedef struct CUstream_st* bnn_stream_t;

typedef enum bnn_status {
    BNN_OK = 0,
    BNN_ERR_INVALID_ARG = 1,     /* null pointer, negative or too-large size, bad mode */
    BNN_ERR_ALIGNMENT = 2,       /* pointer or leading dimension not 16-byte aligned */
    BNN_ERR_UNSUPPORTED = 3,     /* valid but not implemented (e.g. dtype/mode combination) */
    BNN_ERR_CUDA = 4,            /* a CUDA runtime call or kernel launch failed */
    BNN_ERR_DEVICE_TIMEOUT = 5   /* a kernel gave up waiting (reported by bnn_device_error) */
} bnn_status;

typedef enum bnn_dtype {
    BNN_F32 = 0,                 /* IEEE binary32 */
    BNN_BF16 = 1                 /* bfloat16, taken as stored */
} bnn_dtype;

/* Output of a binary product (the epilogue).  s = K - 2 d is the +1/-1 dot
 * product, d the popcount of the XOR (eq. (6)). */
typedef enum bnn_out_mode {
    BNN_OUT_INT32 = 1,           /* int32 s */
    BNN_OUT_SCALED_F32 = 2,      /* fp32 alpha_n * s                    (eq. (1)) */
    BNN_OUT_AFFINE_F32 = 4,      /* fp32 gamma_n * (alpha_n * s) + beta_n */
    BNN_OUT_THRESHOLD_PACK = 8   /* packed sign of a folded BatchNorm, see bnn_fold_bn_threshold */
} bnn_out_mode;

/* Per-output-channel epilogue parameters (device pointers, length = number of
 * output channels).  Unused fields may be NULL.
 *   INT32:           none.
 *   SCALED_F32:      alpha.
 *   AFFINE_F32:      alpha, gamma, beta.
 *   THRESHOLD_PACK:  popc_thresh, thresh_mode (from bnn_fold_bn_threshold):
 *                    thresh_mode 0 -> output bit = (d > popc_thresh),
 *                    thresh_mode 1 -> output bit = (d < popc_thresh);
 *                    bit 1 means -1. */
typedef struct bnn_epilogue {
    int32_t mode;                /* one bnn_out_mode value */
    const float* alpha;
    const float* gamma;
    const float* beta;
    const int32_t* popc_thresh;
    const int8_t* thresh_mode;
} bnn_epilogue;

/* Words in one packed row of K elements: ceil(K/32) rounded up to a multiple
 * of 4 ("First Principles ...", section 1: pack bits into words).  Returns -1
 * for K < 1. */
int64_t bnn_packed_ld_words(int64_t K);

/* Words in one packed 3x3 filter row for `cin` input channels: the 9 taps in
 * (kh, kw) order, each ceil(cin/32) words, rounded up to a multiple of 4.
 * Returns -1 for cin < 1. */
int64_t bnn_conv3x3_ld_words(int64_t cin);

/* Static text for a status code. */
const char* bnn_status_string(int status);

/* Reads and clears the device-side error flag set by a kernel that gave up
 * waiting (BNN_OK if none).  Synchronises the current device first.  Writes
 * the flag value to *code_out (host pointer). */
bnn_status bnn_device_error(int32_t* code_out);

/* bnn_probe_int_pipes -- measures the integer-pipe rates that bound the
 * popcount engine ("First Principles: Why Binary Ops Can Be Exponentially
 * Faster", section "1. Arithmetic: MAC -> XNOR + popcount": one 32-bit XOR +
 * popcount stands for 32 binary multiply-accumulates, so a word rate times 32
 * is a binary MAC rate).  Runs, on the current device, one 1024-thread CTA
 * per SM of register-only chains, timed with the SM clock, and writes (host
 * pointers) the median over SMs of:
 *   *popc_per_clk_sm       32-bit population counts per SM clock;
 *   *lop3_per_clk_sm       three-input logic ops per SM clock;
 *   *csa_words_per_clk_sm  XOR words per SM clock through the popcount GEMM's
 *                          own inner step (XOR, 7:3 carry-save counter, 4
 *                          POPC per 8 words).
 * `iters` (1 .. 2^24) loop iterations per thread; each does 32 operations
 * (words in the third mode).  Synchronous: launches on the legacy default
 * stream and synchronises the device; a diagnostic for roofline
 * denominators, not part of the product path.  Uses a small library-owned
 * device array for the per-SM clock counts (no allocation).
 * Errors: INVALID_ARG, UNSUPPORTED (more than 1024 SMs), CUDA. */
bnn_status bnn_probe_int_pipes(int64_t iters, double* popc_per_clk_sm, double* lop3_per_clk_sm,
                               double* csa_words_per_clk_sm);

/* bnn_selftest_wait_timeout -- diagnostic for the bounded waits.  Runs one
 * kernel that waits on an mbarrier nothing arrives on, with a limit of
 * timeout_ns (1 .. 1e10); the wait must give up, record
 * BNN_ERR_DEVICE_TIMEOUT in the device-side flag (read it with
 * bnn_device_error) and return, leaving the context usable.  Synchronous
 * (it synchronises the current device); allocates nothing.
 * *waited_out (host) is 1 when the wait ran out, 0 if it completed.
 * The pages have no counterpart: it exists to test the library's failure
 * detection without faulting or hanging the GPU.
 *   Errors: INVALID_ARG, CUDA. */
bnn_status bnn_selftest_wait_timeout(int64_t timeout_ns, int32_t* waited_out);

/* bnn_pack_sign -- sign-binarise and bit-pack a real matrix along K, and
 * optionally compute alpha per row.
 *   Passage: "Extreme Quantization ...", Notation (sign) and eq. (4);
 *   "First Principles ...", section 1 (encoding, packing, pad = +1);
 *   eq. (1) (alpha = mean |w| over the row).
 *   x        device, [rows, K] row-major, dtype `dt`, row stride ld_x elements
 *            (ld_x >= K).
 *   packed   device, uint32 [rows, ld_words]; ld_words >= bnn_packed_ld_words(K),
 *            a multiple of 4.  Words [0, bnn_packed_ld_words(K)) of every row
 *            are written, pad bits and pad words as 0.
 *   alpha_out device fp32 [rows] or NULL: (sum_k |x_rk|) / K accumulated in
 *            fp64 over the true K, rounded once to fp32.
 *   Bit k of a row is 1 exactly when x_rk < 0 (so -0.0 and NaN give +1).
 *   rows may be 0 (nothing launched).  K >= 1.
 *   Errors: INVALID_ARG (null, K < 1, ld_x < K, ld_words too small or not a
 *   multiple of 4), ALIGNMENT (packed not 16-byte aligned). */
bnn_status bnn_pack_sign(const void* x, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                         uint32_t* packed, int64_t ld_words, float* alpha_out,
                         bnn_stream_t stream);

/* bnn_pack_sign_nchw -- sign-binarise and pack an NCHW activation tensor into
 * per-pixel channel words, the operand layout of bnn_binary_conv3x3_fused.
 *   Passage: as bnn_pack_sign (eq. (4): activations are binarised too).
 *   x          device, [n, c, h, w] contiguous, dtype `dt`.
 *   packed_nhwc device, uint32 [n, h, w, cw] contiguous with cw = ceil(c/32):
 *              bit q of word j of pixel (n, y, x) is channel 32*j + q; bits for
 *              channels >= c are 0.
 *   Errors: INVALID_ARG, ALIGNMENT (packed_nhwc not 4-byte aligned). */
bnn_status bnn_pack_sign_nchw(const void* x, bnn_dtype dt, int64_t n, int64_t c, int64_t h,
                              int64_t w, uint32_t* packed_nhwc, bnn_stream_t stream);

/* bnn_pack_sign_rsign, bnn_pack_sign_nchw_rsign -- bnn_pack_sign (without
 * alpha) and bnn_pack_sign_nchw with a learned threshold per channel:
 * bit = 1 (-1) exactly where x < beta_c, i.e. sign(x - beta_c) with the
 * Notation tie rule (x = beta_c gives +1; NaN in x or beta gives +1).
 *   Passage: "State of the Art Survey (2016 -> 2026)", classic CNN BNN table,
 *   ReActNet row (RSign: a per-channel reshape of the activation
 *   distribution before binarisation); the pages give no formula, this
 *   reading is sign(x - beta_c).
 *   beta     device fp32, required: [K] per column for bnn_pack_sign_rsign
 *            (the channels of a [rows, K] activation matrix), [c] per channel
 *            for bnn_pack_sign_nchw_rsign.  4-byte aligned.
 *   Other arguments, layouts and errors as bnn_pack_sign / bnn_pack_sign_nchw;
 *   INVALID_ARG for a NULL beta.  Pad bits and padded channels stay 0 (+1). */
bnn_status bnn_pack_sign_rsign(const void* x, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                               const float* beta, uint32_t* packed, int64_t ld_words, bnn_stream_t stream);
bnn_status bnn_pack_sign_nchw_rsign(const void* x, bnn_dtype dt, int64_t n, int64_t c, int64_t h, int64_t w,
                                    const float* beta, uint32_t* packed_nhwc, bnn_stream_t stream);

/* bnn_pack_conv3x3_weights -- pack OIHW 3x3 filters into rows of K = 9 * cin
 * elements in (kh, kw, c) order, and compute alpha per output channel.
 *   Passage: eq. (1) and the glossary's "scaling factors for each weight
 *   filter"; encoding and padding as bnn_pack_sign.
 *   w_oihw   device, [cout, cin, 3, 3] contiguous, dtype `dt`.
 *   packed   device, uint32 [cout, ld_words], ld_words >= bnn_conv3x3_ld_words(cin),
 *            multiple of 4.  Word t*cw + j (t = kh*3 + kw, cw = ceil(cin/32))
 *            holds channels 32*j .. 32*j+31 of tap t; unused channel bits and
 *            words [9*cw, bnn_conv3x3_ld_words(cin)) are 0.
 *   alpha_out device fp32 [cout] or NULL: mean |w| over the 9*cin true weights.
 *   Errors: INVALID_ARG, ALIGNMENT. */
bnn_status bnn_pack_conv3x3_weights(const void* w_oihw, bnn_dtype dt, int64_t cout, int64_t cin,
                                    uint32_t* packed, int64_t ld_words, float* alpha_out,
                                    bnn_stream_t stream);

/* Engine used by bnn_xnor_gemm, bnn_binary_linear_fused and
 * bnn_binary_conv3x3_fused.  All engines return identical results (the
 * product is exact integer arithmetic):
 *   POPCOUNT: XOR + population count on the integer pipes, with carry-save
 *             compression (any shape).
 *   TENSOR:   the sign bits expanded to +1/-1 values in shared memory and
 *             multiplied on the tensor cores: as 4-bit e2m1 values
 *             (tcgen05.mma kind::mxf4 with unit block scales, fp32
 *             accumulators holding exact integers) while K rounded up to a
 *             multiple of 256 is at most 2^20, as int8 bytes (kind::i8,
 *             int32 accumulators) beyond that; for large products.
 *   TENSOR_I8: the int8 tensor-core kernels at every K (GEMM, 3x3
 *             convolution and the multi-bit products below).
 *   AUTO:     TENSOR when M >= 128, N >= 128 and K >= 512, else POPCOUNT
 *             (the default).  Convolutions: the stride-1 tensor-core kernel
 *             when cout >= 64, c <= 64 and n*oh*ow >= 16384, else POPCOUNT.
 * Under TENSOR the convolution uses the tensor cores where its shared memory
 * fits: stride 1 with cout <= 256 (the filters stay resident next to two
 * input buffers of at least one 128-pixel window; e2m1 operands when the
 * channels fill an even number of 32-bit words and cout <= 240, int8
 * otherwise); other strides with c <= 64 and cout <= 256 when the filters and
 * two gathered tiles fit (int8).  Other shapes use the popcount kernel. */
typedef enum bnn_gemm_engine {
    BNN_GEMM_ENGINE_AUTO = 0,
    BNN_GEMM_ENGINE_POPCOUNT = 1,
    BNN_GEMM_ENGINE_TENSOR = 2,
    BNN_GEMM_ENGINE_TENSOR_I8 = 3
} bnn_gemm_engine;

/* Selects the GEMM engine for later calls from every thread of the process
 * (one process-wide setting).  Errors: INVALID_ARG for an unknown engine. */
bnn_status bnn_set_gemm_engine(int engine);

/* The current process-wide GEMM engine setting. */
int bnn_get_gemm_engine(void);

/* bnn_xnor_gemm -- C[m, n] = K - 2 * popcount(A[m, :] XOR W[n, :]) for packed
 * A [M, K] and W [N, K]; optionally also the alpha-scaled fp32 product.
 *   Passage: eq. (6) of "Extreme Quantization ..." (XNOR-Net), eq. (1) for
 *   the scale; "First Principles ...", section 1.
 *   A, W     device, packed rows (layout above), strides lda, ldw words.
 *   alpha    device fp32 [N]; required when C_f32 is given.
 *   C_i32    device int32 [M, ldc] or NULL: s.
 *   C_f32    device fp32 [M, ldf] or NULL: alpha[n] * s in fp32.
 *   At least one of C_i32, C_f32.  M, N >= 0, K >= 1.
 *   Errors: INVALID_ARG, ALIGNMENT (A, W not 16-byte aligned, lda/ldw not a
 *   multiple of 4). */
bnn_status bnn_xnor_gemm(const uint32_t* A, int64_t lda, const uint32_t* W, int64_t ldw,
                         int64_t M, int64_t N, int64_t K, const float* alpha,
                         int32_t* C_i32, int64_t ldc, float* C_f32, int64_t ldf,
                         bnn_stream_t stream);

/* bnn_xnor_gemv -- batch-1 product y[n] = K - 2 * popcount(W[n, :] XOR
 * pack(sign(x))), the real activation vector binarised and packed inside the
 * kernel.  Memory-bound: the packed W is streamed once.
 *   Passage: eq. (4) and eq. (6); "First Principles ...", "Bandwidth math"
 *   (batch-1 y = Wx moves MN/8 bytes when packed).
 *   W        device, packed [N, ldw] (layout above).
 *   x        device, [K] of dtype x_dt.
 *   alpha    device fp32 [N]; required when y_f32 is given.
 *   y_i32    device int32 [N] or NULL; y_f32 device fp32 [N] or NULL (alpha * s);
 *            at least one.
 *   Errors: INVALID_ARG, ALIGNMENT. */
bnn_status bnn_xnor_gemv(const uint32_t* W, int64_t ldw, const void* x, bnn_dtype x_dt,
                         int64_t N, int64_t K, const float* alpha,
                         int32_t* y_i32, float* y_f32, bnn_stream_t stream);

/* Flags of bnn_xnor_gemv_ex. */
typedef enum bnn_gemv_flags {
    BNN_GEMV_WEIGHTS_STATIC = 1,  /* W and its scale (alpha, w_scale) are not written by any work still in flight */
    BNN_GEMV_INPUTS_STATIC = 2,   /* x (and x_scale) are not written by any work still in flight */
    BNN_GEMV_OUTPUT_FREE = 4      /* y is neither read nor written by any work still in flight */
} bnn_gemv_flags;

/* bnn_xnor_gemv_ex -- bnn_xnor_gemv with flags.  Both calls launch the kernel
 * with programmatic dependent launch: it may be scheduled while the previous
 * kernel on the stream is still running, and it waits for that kernel to
 * complete before it reads x, alpha or W or writes y.  With
 * BNN_GEMV_WEIGHTS_STATIC the loads of W and of alpha (the weights' per-row
 * scale, eq. (1)) are issued before that wait, so consecutive GEMVs over
 * resident weights (one decode step through many layers) stream their
 * weights back to back and only x waits.  The caller guarantees that no
 * earlier work on the stream that may still be running writes W or alpha;
 * otherwise pass 0 (then equivalent to bnn_xnor_gemv).  With
 * BNN_GEMV_INPUTS_STATIC (the caller guarantees the same for x) x is packed
 * before the wait as well; with both flags the whole product is computed before it and
 * only the store of y waits, so GEMVs over independent, resident inputs
 * overlap their prologues with the previous kernel.  With all three flags
 * the call depends on nothing still in flight: it computes and stores y
 * while the previous kernel may still run; one block of the launch waits for
 * that kernel before it exits, so the launch completes only after it (stream
 * order stays transitive for later work), and the other blocks leave as soon
 * as their rows are stored.  GEMVs over independent inputs and outputs then
 * run concurrently.  A flag is a
 * permission: shapes served by the general kernel (rows of more than 128
 * words, or x not 16-byte aligned) ignore BNN_GEMV_INPUTS_STATIC and
 * BNN_GEMV_OUTPUT_FREE.
 *   Errors: as bnn_xnor_gemv; INVALID_ARG for unknown flag bits. */
bnn_status bnn_xnor_gemv_ex(const uint32_t* W, int64_t ldw, const void* x, bnn_dtype x_dt,
                            int64_t N, int64_t K, const float* alpha,
                            int32_t* y_i32, float* y_f32, uint32_t flags, bnn_stream_t stream);

/* bnn_xnor_gemv_host -- bnn_xnor_gemv_ex for a caller whose x and y live in
 * host memory: on `stream`, copies x (K elements) from host to device, runs
 * the GEMV, and copies y (N fp32 values) back.  When both host buffers are
 * pinned memory that the device can address (cudaHostAlloc / cudaMallocHost
 * or cudaHostRegister, mapped into the unified address space), both buffers
 * and y_dev are 16-byte aligned and both byte counts are multiples of 16, the
 * copies are two small kernels whose loads and stores cross PCIe, chained to
 * the GEMV by programmatic dependent launch.  Otherwise each copy is one
 * cudaMemcpyAsync.
 *   Passage: as bnn_xnor_gemv ("First Principles ...", "Bandwidth math";
 *   eq. (4), (6) and (1) of "Extreme Quantization ...").
 *   W, ldw, alpha  device, as in bnn_xnor_gemv (W and alpha are the model's
 *                  resident weights).
 *   x_host   host memory, K elements of x_dt; pinned (page-locked) memory
 *            makes the copy asynchronous, pageable memory is copied too but
 *            the call may then block the host until the copy is done.
 *   x_dev    device scratch for x, >= K elements of x_dt, 16-byte aligned,
 *            owned by the caller (the library allocates nothing).
 *   y_dev    device scratch for y, >= N fp32, 4-byte aligned (16 for the
 *            kernel copies).
 *   y_host   host memory for the N fp32 outputs alpha[n] * s (pinned for an
 *            asynchronous copy); valid once `stream` reaches the end of the
 *            call's work (e.g. after cudaStreamSynchronize).
 *   flags    0, BNN_GEMV_WEIGHTS_STATIC (as in bnn_xnor_gemv_ex) and/or
 *            BNN_GEMV_INPUTS_STATIC, which here says that no earlier work on
 *            the stream that may still be running writes x_host: the copy
 *            kernel then reads x_host before waiting for that work (its PCIe
 *            latency overlaps it) and writes x_dev after.  Without it the
 *            read follows the wait, as a copy in stream order would.
 *            BNN_GEMV_OUTPUT_FREE does not apply (y is read by the copy
 *            after the kernel).
 *   Errors: INVALID_ARG (null pointer, bad size or flag), ALIGNMENT, and the
 *   errors of bnn_xnor_gemv; BNN_ERR_CUDA when a copy cannot be enqueued. */
bnn_status bnn_xnor_gemv_host(const uint32_t* W, int64_t ldw, const void* x_host, bnn_dtype x_dt, int64_t N,
                              int64_t K, const float* alpha, void* x_dev, float* y_dev, float* y_host, uint32_t flags,
                              bnn_stream_t stream);

/* bnn_binary_weight_gemv -- binary weights times a REAL activation vector:
 *   y[n] = alpha[n] * sum_k sign(W[n,k]) * x[k]
 * ("Extreme Quantization: Binary, Ternary & 1-bit LLMs", Binary Neural
 * Networks, eq. (1)-(2): every term is +x_k or -x_k, no multiplication).
 * Unlike bnn_xnor_gemv, x is not binarised.
 *   W        device, packed [N, ldw] as produced by bnn_pack_sign (16-B aligned,
 *            ldw % 4 == 0, pad bits zero).  kw = bnn_packed_ld_words(K) <= 384
 *            (K <= 12288; the per-block add table lives in shared memory).
 *   x        device fp32 or bf16 [K] (x_dt).
 *   alpha    device fp32 [N], required; y device fp32 [N].
 *   flags    as for bnn_xnor_gemv_ex (BNN_GEMV_WEIGHTS_STATIC,
 *            BNN_GEMV_INPUTS_STATIC, BNN_GEMV_OUTPUT_FREE).
 *   N        <= 2^30.
 * Accumulation is fp32: a 16-entry table of +-x0 +-x1 +-x2 +-x3 per group
 * of 4 elements, then one lookup and one add per 4 weights on 4 accumulators
 * per lane (each lane holds 128 consecutive weights of a row per pass), and
 * the lanes of a row added by a butterfly of shuffles.
 *   Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (K too large), CUDA.  A
 *   launch whose shared-memory window is laid out where the 32 KiB-aligned
 *   table does not fit (not expected on sm_100) records
 *   BNN_ERR_UNSUPPORTED in the device flag (bnn_device_error) and writes
 *   nothing. */
bnn_status bnn_binary_weight_gemv(const uint32_t* W, int64_t ldw, const void* x, bnn_dtype x_dt,
                                  int64_t N, int64_t K, const float* alpha, float* y,
                                  uint32_t flags, bnn_stream_t stream);

/* TERNARY LAYOUT (bnn_ternary_pack, bnn_ternary_gemv_i8).  A ternary weight
 * t in {-1, 0, +1} is stored as the 2-bit code t + 1 (0 = -1, 1 = 0, 2 = +1;
 * code 3 is not a weight and must not occur).  Weight k of a row sits at bits
 * 2(k mod 16), 2(k mod 16)+1 of uint32 word k / 16 (least significant first).
 * A row holds bnn_ternary_ld_words(K) = ceil(K/16) rounded up to a multiple of
 * 4 words; positions past K hold code 1.  Row r starts at word r * ldq, ldq a
 * multiple of 4 and >= bnn_ternary_ld_words(K).  2 bits per weight: the pages
 * give ~1.58 bits (log2 3) as the information content and ~0.2 bytes per
 * weight for packed ternary; the 2-bit code is the densest layout whose
 * weights can be addressed with shifts and masks. */

/* bnn_binary_weight_gemv_i8 -- binary weights times an INT8 activation vector:
 *   acc[n]   = sum_k sign(W[n,k]) * x[k]              (exact, int32)
 *   y_f32[n] = fp32( fp32(a_n * x_scale) * fp32(acc[n]) ),
 *   a_n = alpha[n] (alpha_per_row = 1, eq. (1): one scale per output row) or
 *   alpha[0] (alpha_per_row = 0, eq. (8): one scale for the whole matrix).
 * ("Extreme Quantization: Binary, Ternary & 1-bit LLMs", Binary Neural
 * Networks, eq. (1)-(2): each term is +x_k or -x_k; BitNet: activations
 * quantised to INT8, weights binarised with the matrix scale of eq. (8).)
 * The pages give no activation quantiser: x arrives as int8 with its scale.
 *   W        device, packed [N, ldw] as produced by bnn_pack_sign (16-B
 *            aligned, ldw % 4 == 0, pad bits zero); kw = bnn_packed_ld_words(K)
 *            <= 1536 (K <= 49152).
 *   x        device int8 [K]; x_scale device fp32 [1] or NULL (1.0).
 *   alpha    device fp32 [N] or [1] (see alpha_per_row); required with y_f32.
 *   y_i32, y_f32  device [N]; either may be NULL, not both.  N <= 2^30.
 *   flags    as for bnn_xnor_gemv_ex.
 * Per 4 weights the kernel does one shift, one byte permute and one dp4a
 * against x staged in that byte order; the int32 result is exact.
 *   Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (K too large), CUDA. */
bnn_status bnn_binary_weight_gemv_i8(const uint32_t* W, int64_t ldw, const int8_t* x, int64_t N, int64_t K,
                                     const float* alpha, int alpha_per_row, const float* x_scale, int32_t* y_i32,
                                     float* y_f32, uint32_t flags, bnn_stream_t stream);

/* Words in one ternary row of K weights; -1 for K < 1. */
int64_t bnn_ternary_ld_words(int64_t K);

/* Bytes of device workspace bnn_ternary_pack needs for `rows` rows when it
 * computes gamma: 8 * (rows + 1).  -1 for rows < 0. */
int64_t bnn_ternary_workspace_bytes(int64_t rows);

/* bnn_ternary_pack -- quantise a real matrix to ternary weights and pack them.
 *   Passage: "Extreme Quantization: Binary, Ternary & 1-bit LLMs",
 *   Ternary Quantization, eq. (7), and BitNet b1.58, eq. (9).
 *   delta < 0  -- eq. (9): W_t = RoundClip(W / gamma, -1, 1),
 *                 gamma = sum |w| / (rows * K) over the whole matrix.
 *                 Halves round to even, so the weight is +-1 exactly where
 *                 |w| > gamma / 2 and 0 elsewhere; that comparison is made in
 *                 fp64 with gamma summed in fp64 (per row, then the rows in a
 *                 fixed order: the same codes on every run).  All-zero W gives
 *                 gamma = 0 and all weights 0.
 *   delta >= 0 -- eq. (7) with Delta = delta: +1 where w > delta, -1 where
 *                 w < -delta, 0 otherwise (compared in fp64).
 *   NaN weights quantise to 0.
 *   w         device, [rows, K] row-major, dtype dt, row stride ld_w >= K.
 *   codes     device, uint32 [rows, ldq] (TERNARY LAYOUT, 16-byte aligned);
 *             words [0, bnn_ternary_ld_words(K)) of each row are written.
 *   gamma_out device fp32 [1] or NULL: gamma rounded once to fp32 (the scale
 *             of eq. (9): W is approximated by gamma * W_t).
 *   workspace device, >= bnn_ternary_workspace_bytes(rows) bytes, 8-byte
 *             aligned, owned by the caller; required when delta < 0 or
 *             gamma_out is given, else may be NULL.  Its contents on entry do
 *             not matter; it must not be used by other work until the call's
 *             kernels are done (stream order).
 *   Launches up to three kernels (row sums of |w|, gamma, pack).
 *   Errors: INVALID_ARG (null, sizes, NaN delta, workspace missing or too
 *   small), ALIGNMENT. */
bnn_status bnn_ternary_pack(const void* w, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_w,
                            double delta, uint32_t* codes, int64_t ldq, float* gamma_out,
                            void* workspace, int64_t workspace_bytes, bnn_stream_t stream);

/* Largest `rows` bnn_ternary_pack_noalloc accepts. */
#define BNN_TERNARY_PACK_NOALLOC_MAX_ROWS 262144

/* bnn_ternary_pack_noalloc -- bnn_ternary_pack without a caller workspace.
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory themselves -- code that only receives the
 * input and output pointers from a host framework (a plugin or custom
 * operator of another runtime, whose allocator it cannot reach), or a
 * latency-critical path where cudaMalloc, which may synchronise the device,
 * is not allowed.  It computes exactly what bnn_ternary_pack computes, with
 * the same arguments minus the workspace, and allocates nothing: the row sums
 * and gamma go to one array of BNN_TERNARY_PACK_NOALLOC_MAX_ROWS + 1 doubles
 * (about 2 MiB) that the library holds in device memory on every GPU that
 * loads it, for the life of the process.
 *   rows > BNN_TERNARY_PACK_NOALLOC_MAX_ROWS: BNN_ERR_UNSUPPORTED (use
 *   bnn_ternary_pack with a workspace).
 *   The first call on a device looks up that array's device address (one
 *   cudaGetSymbolAddress, with the device current) and keeps it for the life
 *   of the process; make that first call before any stream capture.  After
 *   cudaDeviceReset() the array may sit at another address while the kept
 *   one stays: do not call this entry point on a device that was reset
 *   after its first call (use bnn_ternary_pack there).
 *   Every call on a device shares the one array.  Calls whose kernels may
 *   overlap on the GPU (on different streams without ordering between them)
 *   race on it and must not be issued; calls in stream order are safe.
 *   Nothing in the array needs to start at zero: each call writes every entry
 *   it reads.
 *   Errors: as bnn_ternary_pack (INVALID_ARG, ALIGNMENT), UNSUPPORTED (too
 *   many rows), CUDA (the address look-up failed). */
bnn_status bnn_ternary_pack_noalloc(const void* w, bnn_dtype dt, int64_t rows, int64_t K, int64_t ld_w,
                                    double delta, uint32_t* codes, int64_t ldq, float* gamma_out,
                                    bnn_stream_t stream);

/* bnn_ternary_gemv_i8 -- ternary weights times an int8 activation vector:
 *   acc[n]   = sum_k t_nk * x_k                    (exact, int32)
 *   y_f32[n] = fp32( fp32(w_scale * x_scale) * fp32(acc[n]) )
 * ("Extreme Quantization ...", BitNet: INT8 activations; BitNet b1.58:
 * ternary weights; "First Principles ...", op-per-element table: add / skip /
 * sub).  The pages do not define the activation quantiser: x arrives
 * quantised, with its scale.
 *   codes    device, [N, ldq] words (TERNARY LAYOUT), 16-byte aligned.
 *   x        device int8 [K] (any alignment; 16-byte aligned is faster).
 *   w_scale, x_scale  device fp32 [1] each, or NULL for 1.0 (read only when
 *            y_f32 is given).  w_scale is typically gamma from
 *            bnn_ternary_pack.
 *   y_i32    device int32 [N] or NULL; y_f32 device fp32 [N] or NULL; at
 *            least one.  fp32(acc) is exact for K <= 65536.
 *   flags    as for bnn_xnor_gemv_ex (the x vector and both scales are the
 *            inputs of BNN_GEMV_INPUTS_STATIC).
 *   K <= 98304 (x is staged in shared memory).
 *   Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (K too large), CUDA. */
bnn_status bnn_ternary_gemv_i8(const uint32_t* codes, int64_t ldq, const int8_t* x, int64_t N, int64_t K,
                               const float* w_scale, const float* x_scale, int32_t* y_i32, float* y_f32,
                               uint32_t flags, bnn_stream_t stream);

/* bnn_binary_linear_fused -- packed binary GEMM with one fused epilogue.
 *   Passage: eq. (6) (product), eq. (1) (alpha), the glossary's BatchNorm
 *   paragraph (normalise, then binarise for the next layer).
 *   A, W, lda, ldw, M, N, K as bnn_xnor_gemm.
 *   ep       host pointer to the epilogue (mode + device parameter arrays of
 *            length N).
 *   out      device: int32 or fp32 [M, ld_out] (ld_out in elements) for the
 *            INT32 / SCALED_F32 / AFFINE_F32 modes; for THRESHOLD_PACK a
 *            packed uint32 [M, ld_out] matrix of N elements per row (ld_out in
 *            words, >= bnn_packed_ld_words(N), multiple of 4; pad bits and
 *            pad words written as 0), i.e. directly the A operand of the next
 *            layer with K_next = N.
 *   Errors: INVALID_ARG (incl. missing parameter for the mode), ALIGNMENT. */
bnn_status bnn_binary_linear_fused(const uint32_t* A, int64_t lda, const uint32_t* W, int64_t ldw,
                                   int64_t M, int64_t N, int64_t K, const bnn_epilogue* ep,
                                   void* out, int64_t ld_out, bnn_stream_t stream);

/* bnn_binary_conv3x3_fused -- binary 3x3 convolution as an implicit GEMM over
 * packed per-pixel channel words, with a fused epilogue.  Output pixel
 * (n, y, x) gathers the 9 taps (kh, kw); a tap outside the image reads all-0
 * words (+1: zero-padded real input, then sign).  K = 9 * c.
 *   Passage: eq. (4), eq. (6), eq. (1) per filter; glossary BatchNorm paragraph.
 *   X_nhwc_bits device, from bnn_pack_sign_nchw: [n, h, w, ceil(c/32)] words.
 *   W_packed device, from bnn_pack_conv3x3_weights: [cout, ldw] words.
 *   stride >= 1, pad >= 0; output spatial size (h + 2 pad - 3)/stride + 1 by
 *   (w + 2 pad - 3)/stride + 1, both >= 1.
 *   ep       host pointer; modes INT32, SCALED_F32, AFFINE_F32.
 *   out_nchw device int32/fp32 [n, cout, oh, ow] contiguous.
 *   Supports c <= 128.  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED. */
bnn_status bnn_binary_conv3x3_fused(const uint32_t* X_nhwc_bits, int64_t n, int64_t c, int64_t h,
                                    int64_t w, const uint32_t* W_packed, int64_t ldw, int64_t cout,
                                    int64_t stride, int64_t pad, const bnn_epilogue* ep,
                                    void* out_nchw, bnn_stream_t stream);

/* bnn_binary_conv1x1_fused -- binary 1x1 convolution with stride (the
 * downsampling projection of a ResNet-class block), fused epilogue.  Output
 * pixel (n, y, x) reads input pixel (n, s*y, s*x); no padding.  K = c.
 *   Passage: eq. (4), eq. (6), eq. (1) per filter of "Extreme Quantization
 *   ..."; the glossary's BatchNorm paragraph for the affine epilogue.
 *   X_nhwc_bits device, from bnn_pack_sign_nchw (or its RSign variant):
 *            [n, h, w, ceil(c/32)] words.
 *   W_packed device, [cout, ldw] words, ldw >= ceil(c/32): the filters
 *            [cout, c, 1, 1] packed as rows of c elements, e.g. by
 *            bnn_pack_sign on the [cout, c] view (which also gives alpha).
 *   stride >= 1; output spatial size (h - 1)/stride + 1 by (w - 1)/stride + 1.
 *   ep       host pointer; modes INT32, SCALED_F32, AFFINE_F32.
 *   out_nchw device int32/fp32 [n, cout, oh, ow] contiguous.
 *   Supports c <= 512, n*oh*ow < 2^31 - 4096 and cout*oh*ow < 2^31 (32-bit
 *   pixel indices).  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED. */
bnn_status bnn_binary_conv1x1_fused(const uint32_t* X_nhwc_bits, int64_t n, int64_t c, int64_t h, int64_t w,
                                    const uint32_t* W_packed, int64_t ldw, int64_t cout, int64_t stride,
                                    const bnn_epilogue* ep, void* out_nchw, bnn_stream_t stream);

/* bnn_fold_bn_threshold -- HOST function: fold inference BatchNorm of
 * alpha * s followed by sign() into an integer popcount threshold per channel.
 *   Passage: glossary "Binary Neural Network (BNN)", BatchNorm paragraph (BN
 *   before binarisation, alpha per filter); the pages give no BN formula.
 *   The decision folded is, in IEEE double with each fp32 input widened:
 *     v(s) = ((alpha*s - mean) / sqrt(var + eps)) * gamma + beta,
 *     output +1 (bit 0) iff v(s) >= 0,
 *   for every reachable s = K - 2d, d = 0..K.  The result reproduces that
 *   decision exactly for every d: thresh_mode 0 -> bit = (d > popc_thresh),
 *   thresh_mode 1 -> bit = (d < popc_thresh).  A constant decision is
 *   encoded as mode 0 with popc_thresh = K (always +1) or -1 (always -1).
 *   alpha, gamma, beta, mean, var: host fp32 [N]; popc_thresh: host int32 [N];
 *   thresh_mode: host int8 [N].
 *   Errors: INVALID_ARG (null, N < 0, K < 1, a non-finite parameter,
 *   var + eps <= 0, alpha < 0). */
bnn_status bnn_fold_bn_threshold(const float* alpha, const float* gamma, const float* beta,
                                 const float* mean, const float* var, double eps, int64_t N,
                                 int64_t K, int32_t* popc_thresh, int8_t* thresh_mode);

/* ------------------------------------------------------------------------
 * Multi-bit products on bit planes ("State of the Art Survey (2016 -> 2026)",
 * classic CNN BNN table: DoReFa-Net -- low-bit weights and activations,
 * bit-convolution; ABC-Net -- several binary bases approximating full
 * precision).
 *
 * PLANE-INTERLEAVED LAYOUT.  An operand of R rows with P planes per row is a
 * packed matrix (PACKED LAYOUT above) of R * P rows: plane p of row r is
 * packed row r * P + p, at word (r * P + p) * ld.  Every plane holds K
 * elements.  A plane of bits (DoReFa) or a +1/-1 base (ABC-Net) uses the
 * same packed encoding as every other call.
 * ------------------------------------------------------------------------ */

/* bnn_pack_bit_planes -- unsigned k-bit codes to bit planes.
 *   codes: device uint8 [rows, ld_codes] (ld_codes >= K); only the low `bits`
 *   bits of each byte are used.  planes: device, plane-interleaved, `bits`
 *   planes per row, row stride ld_words (>= bnn_packed_ld_words(K), multiple of
 *   4, 16-byte aligned): bit j of word w of plane p of row r is bit p of
 *   codes[r, 32 w + j]; code = sum_p 2^p * bit_p.  Elements past K are 0.
 *   bits: 1 .. 8.
 *   Errors: INVALID_ARG, ALIGNMENT, CUDA. */
bnn_status bnn_pack_bit_planes(const uint8_t* codes, int64_t rows, int64_t K, int64_t ld_codes, int bits,
                               uint32_t* planes, int64_t ld_words, bnn_stream_t stream);

/* bnn_bitserial_gemm -- the product of unsigned low-bit integer codes:
 *   C_i32[m, n] = sum_k a[m, k] * w[n, k]      (exact, int32)
 *   C_f32[m, n] = fp32(alpha[n] * fp32(C_i32[m, n]))
 * for codes 0 <= a < 2^a_bits and 0 <= w < 2^w_bits given as bit planes
 * (DoReFa-Net's bit-convolution, which a bit-serial kernel computes as
 * sum over plane pairs of 2^(b + b') * popcount(a_b AND w_b')).  The
 * tensor-core kernels fold each row's planes back into one code per element
 * in shared memory, so all plane pairs cost one pass: codes of up to two bits
 * as exact e2m1 values (code c as c / 2, kind::mxf4, CTA pairs, when
 * M > 128 and 9 * K rounded up to 256 is below 2^22), wider codes -- and every code
 * under BNN_GEMM_ENGINE_TENSOR_I8 -- as unsigned bytes (u8 x u8).
 *   A: plane-interleaved [M rows x a_bits planes], row stride lda words.
 *   W: plane-interleaved [N rows x w_bits planes], row stride ldw words.
 *   a_bits, w_bits: 1 .. 4.  K * (2^a_bits - 1) * (2^w_bits - 1) must fit in
 *   int32.  C_i32 (ldc >= N) and/or C_f32 (ldf >= N, needs alpha [N]); either
 *   may be NULL, not both.
 *   Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA. */
bnn_status bnn_bitserial_gemm(const uint32_t* A, int64_t lda, int a_bits, const uint32_t* W, int64_t ldw, int w_bits,
                              int64_t M, int64_t N, int64_t K, const float* alpha, int32_t* C_i32, int64_t ldc,
                              float* C_f32, int64_t ldf, bnn_stream_t stream);

/* bnn_binary_bases_gemm -- activations approximated by J binary bases,
 * A ~ sum_j beta_j H_j, weights by I bases per output channel,
 * W[n] ~ sum_i alpha_i[n] B_i[n] (ABC-Net):
 *   Y[m, n] = sum_j sum_i beta_j * alpha_i[n] * s_ji[m, n],
 *   s_ji[m, n] = <H_j[m, :], B_i[n, :]>  (a +1/-1 product, eq. (6)),
 * with every s_ji exact and the weighted sum in fp32.  Within a row, v_j =
 * sum_i alpha_i[n] * s_ji is formed by fused multiply-adds in i order, then
 * beta_j * v_j, then the J terms are added pairwise (j, j^1), (j, j^2), ...;
 * |Y - Y_exact| <= (I + J + 2) * 2^-24 * sum_j sum_i |beta_j alpha_i[n] s_ji|.
 * The products run on the e2m1 tensor-core kernel in CTA pairs (when M
 * exceeds 128 / J' rows, J' = J rounded up to a power of two) and on the int8
 * one otherwise or under BNN_GEMM_ENGINE_TENSOR_I8; both give the same s_ji.
 *   H: plane-interleaved +1/-1 bases [M rows x J planes], stride ldh words
 *   (base j of row m, packed as by bnn_pack_sign, at packed row m * J + j).
 *   B: plane-interleaved [N rows x I planes], stride ldb words.
 *   J, I: 1 .. 8.  beta: device fp32 [J]; alpha: device fp32 [I, lda_alpha]
 *   (alpha_i[n] at i * lda_alpha + n, lda_alpha >= N); Y: device fp32 [M, ldy].
 *   Errors: INVALID_ARG, ALIGNMENT, CUDA. */
bnn_status bnn_binary_bases_gemm(const uint32_t* H, int64_t ldh, int J, const uint32_t* B, int64_t ldb, int I,
                                 int64_t M, int64_t N, int64_t K, const float* beta, const float* alpha,
                                 int64_t lda_alpha, float* Y, int64_t ldy, bnn_stream_t stream);

/* One layer of bnn_xnor_gemv_chain.  The layer's K is the previous layer's N
 * (the first layer's is the call's K). */
typedef struct bnn_chain_layer {
    const uint32_t* W;            /* device, packed [N, ldw] as by bnn_pack_sign (16-B aligned, ldw % 4 == 0) */
    int64_t ldw;                  /* >= bnn_packed_ld_words(K) */
    int64_t N;                    /* outputs, 1 .. 2^24; a hidden layer's N is <= 16384 */
    const int32_t* popc_thresh;   /* hidden layers: device int32 [N] (bnn_fold_bn_threshold) */
    const int8_t* thresh_mode;    /* hidden layers: device int8 [N] */
    const float* alpha;           /* last layer: device fp32 [N], needed for y_f32 */
} bnn_chain_layer;

/* Size, in uint32 words, of the workspace of bnn_xnor_gemv_chain. */
int64_t bnn_gemv_chain_workspace_words(void);

/* bnn_xnor_gemv_chain -- a batch-1 fully binary layer chain, the decode step
 * of a binary network, in ONE launch:
 *   a_0 = sign(x)                                  (bit 1 = x < 0)
 *   d_l = popcount(W_l[n, :] XOR a_l)              (eq. (6): s = K_l - 2 d_l)
 *   a_{l+1}[n] = THRESHOLD_PACK bit of d_l[n]      (hidden layers: BatchNorm of
 *                alpha * s followed by sign, folded by bnn_fold_bn_threshold)
 *   last layer: y_i32[n] = s, y_f32[n] = alpha[n] * s (eq. (1)).
 * Each layer is the XNOR GEMV of bnn_xnor_gemv ("Extreme Quantization:
 * Binary, Ternary & 1-bit LLMs", eq. (4) and (6); "First Principles: Why
 * Binary Ops Can Be Exponentially Faster", "Bandwidth math": a batch-1 layer
 * streams its packed weights once).  The layers run in one cooperative launch
 * (every block resident): no launch or grid barrier between layers, the
 * weights of later layers are fetched into L2 while earlier layers run, and
 * a layer's blocks start as soon as the previous layer's output words are
 * complete.  Results are those of the same chain of bnn_binary_linear_fused
 * calls at M = 1 (THRESHOLD_PACK for hidden layers).
 *   layers    HOST array [L] of bnn_chain_layer; 1 <= L <= 16.
 *   x         device [K] fp32 or bf16 (x_dt), element-aligned; 1 <= K <= 16384,
 *             and every layer's K <= 16384 (packed rows of at most 512 words).
 *   y_i32     device int32 [N_{L-1}] or NULL; y_f32 device fp32 [N_{L-1}] or
 *             NULL; at least one.
 *   acts      device uint32 [L-1, ld_acts] or NULL: the packed input of every
 *             layer after the first (row l-1 = a_l, bnn_pack_sign layout);
 *             ld_acts >= bnn_packed_ld_words of every hidden N.
 *   workspace device uint32 [bnn_gemv_chain_workspace_words()], 16-byte
 *             aligned, ZERO before its first use; every call leaves it zero
 *             again (also after a timeout).  Calls that may run concurrently
 *             need separate workspaces.
 *   A block that waits more than about a second for the previous layer's
 *   output gives up and sets the device error flag (bnn_device_error then
 *   reports BNN_ERR_DEVICE_TIMEOUT); outputs are then undefined.
 *   Errors: INVALID_ARG (null or out-of-range argument, missing thresholds
 *   or alpha, small ld_acts), ALIGNMENT, UNSUPPORTED (a layer K > 16384),
 *   CUDA (launch failed, e.g. the grid cannot be co-resident). */
bnn_status bnn_xnor_gemv_chain(const bnn_chain_layer* layers, int32_t L, const void* x, bnn_dtype x_dt, int64_t K,
                               int32_t* y_i32, float* y_f32, uint32_t* acts, int64_t ld_acts, uint32_t* workspace,
                               bnn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BNN_H_ */
