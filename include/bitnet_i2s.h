/*
 * bitnet_i2s.h -- C ABI of the B200 (sm_100a) I2_S ternary x int8 matmul.
 *
 * The library computes, for ternary weights w[n,k] in {-1,0,+1} packed two
 * bits each with one fp32 per-tensor scale s, and per-token int8 activations
 * xq[m,k] with fp32 scales xs[m]:
 *
 *     acc[m,n] = sum_k w[n,k] * xq[m,k]            (exact int32)
 *     y[m,n]   = ((float)acc[m,n] * xs[m]) * s     (two fp32 multiplies)
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "How BitNet's 1-Bit (I2_S) Quantization Works Compared to Standard
 *        LLM Quantization": sections "Ternary Representation and Packing",
 *        "Per-Tensor Scaling Strategy", "How I2_S Kernels Process the Format".
 *   [P2] "BitNet Inference Preprocessing: Converting Hugging Face Checkpoints
 *        to I2S GGUF": "The Two-Stage BitNet Inference Preprocessing
 *        Pipeline" (the packing is lossless; the seven ternary projections).
 *   [P3] "ik_llama.cpp 运行 BitNet b1.58 2B 模型实战：从 bitnet-b1.58 架构兼容到
 *        I2_S 量化转换": section 5.1 (I2_S tensors are dequantized to f32 in
 *        full before requantizing).
 *   [P5] "LLM Quantization Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026":
 *        section 5, figure "BitNet b1.58 Ternary Matrix Multiplication" and
 *        "The Mathematics of BitNet b1.58".
 *
 * I2_S byte layout (the packed tensor of an N x K weight matrix, K % 128 == 0):
 *   bytes [0, N*K/4): 2-bit codes, code = w + 1 (so -1,0,+1 -> 0,1,2; code 3
 *     never occurs).  Weights are taken in row-major order in blocks of 128;
 *     weight j of a block sits in byte j % 32 of the block's 32 bytes, in
 *     bits [7-2g : 6-2g] with g = j / 32 (the shift 6 - 2*group of [P1]).
 *   bytes [N*K/4, N*K/4 + 4): the scale s = max|W| as little-endian fp32 [P1].
 *
 * Conventions for every call below:
 *   - Pointers are DEVICE pointers, allocated and owned by the caller; the
 *     library never allocates, frees or keeps them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream; arguments are
 *     checked on the host before anything is launched.
 *   - The current CUDA device must be a B200-class GPU (sm_100a); the
 *     pointers must belong to it.
 *   - Return value: BITNET_OK, or an error code with a message readable from
 *     bitnet_last_error() (thread-local; valid until the next call on the
 *     same thread).  On an argument error nothing is launched.
 *   - Device-side waits are bounded.  A wait that runs out (about two
 *     seconds) makes the kernel stop early and raise a device error flag;
 *     bitnet_device_status() reports and clears it.
 *   - Shape limits: 1 <= N, M; K a multiple of 128 with K <= 131072, which
 *     keeps |acc| <= 127*K < 2^24 so (float)acc is exact.
 */
#ifndef BITNET_I2S_H
#define BITNET_I2S_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BITNET_API __attribute__((visibility("default")))
#else
#define BITNET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bitnet_status {
  BITNET_OK = 0,
  BITNET_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad buffer size */
  BITNET_ERR_SHAPE = 2,         /* N, M < 1; K not a multiple of 128; over a limit */
  BITNET_ERR_ALIGN = 3,         /* a pointer misses its required alignment */
  BITNET_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  BITNET_ERR_DEVICE_TIMEOUT = 5,/* a bounded device-side wait ran out */
  BITNET_ERR_UNSUPPORTED = 6    /* the current device is not sm_100 */
} bitnet_status;

/* Size in bytes of the I2_S tensor of an N x K weight matrix: N*K/4 code
 * bytes plus the 4-byte scale [P1 "Ternary Representation and Packing",
 * "Per-Tensor Scaling Strategy"].  Returns 0 for an invalid shape. */
BITNET_API size_t bitnet_i2s_packed_bytes(int64_t N, int64_t K);

/* Pack fp32 weights W[N,K] (row-major) into I2_S [P1 "Ternary Representation
 * and Packing", "Per-Tensor Scaling Strategy"; P2: lossless for weights that
 * are already ternary times one scale].
 *   s = max|W|; each weight becomes q = clip(round_half_away(W/s), -1, 1)
 *   (fp32 IEEE divide; s == 0 gives q = 0 everywhere) and code q + 1.
 * W: N*K fp32, 16-byte aligned.  packed: bitnet_i2s_packed_bytes(N,K)
 * bytes, 16-byte aligned; fully overwritten (codes and scale). */
BITNET_API bitnet_status bitnet_i2s_pack(const float* W, int64_t N, int64_t K, uint8_t* packed,
                              void* stream);

/* Per-token absmax int8 quantization [P5 section 5, "The Mathematics of
 * BitNet b1.58"]: for each row m of X[M,K] (row-major fp32),
 *   amax = max_k |x|; xq = clamp(round_half_even(x * (127/amax)), -127, 127);
 *   xs[m] = amax / 127 (fp32 IEEE divides); a zero row gives xq = 0, xs = 0.
 * X: 16-byte aligned; K % 16 == 0.  Xq: M*K int8, 16-byte aligned.
 * xs: M fp32. */
BITNET_API bitnet_status bitnet_act_quant_i8(const float* X, int64_t M, int64_t K, int8_t* Xq, float* xs,
                                  void* stream);

/* Decode-shaped ternary matmul, M = 1..64 tokens [P5 section 5 figure, "BitNet
 * b1.58 Ternary Matrix Multiplication" (add, subtract or skip per ternary
 * weight, integer accumulation); P1 "How I2_S Kernels Process the Format"
 * (unpack the 2-bit codes, multiply by the shared per-tensor scale)].
 *   packed: I2_S tensor of W[N,K] (as written by bitnet_i2s_pack), 16-byte
 *           aligned; the scale is read from its tail.
 *   Xq:     M*K int8 row-major, 16-byte aligned.   xs: M fp32.
 *   Y:      M*N fp32 row-major (token-major), written.
 *   acc_or_null: if not NULL, M*N int32 row-major receives the exact
 *           accumulators.
 * Memory-bound: streams N*K/4 packed bytes once. */
BITNET_API bitnet_status bitnet_i2s_gemv(const uint8_t* packed, int64_t N, int64_t K, const int8_t* Xq,
                              const float* xs, int64_t M, float* Y, int32_t* acc_or_null,
                              void* stream);

/* The same contraction for any M >= 1 (prefill), with the same arguments and
 * results; for M > 64 it uses a tile shaped for tensor-core throughput. */
BITNET_API bitnet_status bitnet_i2s_gemm(const uint8_t* packed, int64_t N, int64_t K, const int8_t* Xq,
                              const float* xs, int64_t M, float* Y, int32_t* acc_or_null,
                              void* stream);

/* Full-tensor dequantization I2_S -> fp32: W_out[n,k] = w[n,k] * s, exact
 * ["ik_llama.cpp 运行 BitNet b1.58 2B 模型实战", section 5.1: an I2_S tensor is
 * dequantized to f32 in full before being requantized; P1 "Ternary
 * Representation and Packing" for the code layout].
 * packed: I2_S tensor, 16-byte aligned.  W_out: N*K fp32, 16-byte aligned. */
BITNET_API bitnet_status bitnet_i2s_dequant_f32(const uint8_t* packed, int64_t N, int64_t K,
                                                float* W_out, void* stream);

/* Device scratch bytes bitnet_ternarize_absmean needs (fixed, 8 KB). */
BITNET_API size_t bitnet_ternarize_absmean_workspace_bytes(void);

/* AbsMean ternarization, the preprocessing step before packing [P5 section
 * 5, "The Mathematics of BitNet b1.58": W~ = RoundClip(W / (gamma + eps),
 * -1, 1) with gamma = mean |W|; P2 Stage 1 applies it to the seven
 * projections].
 *   gamma is summed in fp64 in a fixed order (deterministic run to run) and
 *   written to *gamma_out (device).  The division and the rounding (ties away
 *   from zero) are fp64.  W_out[i] = W~[i] * (float)gamma, so
 *   bitnet_i2s_pack(W_out) is lossless with scale (float)gamma.
 *   W, W_out: `count` fp32 (may be the same buffer).  eps >= 0 (the pages
 *   leave it open; 1e-5 is the usual choice).  workspace: at least
 *   bitnet_ternarize_absmean_workspace_bytes(), 8-byte aligned. */
BITNET_API bitnet_status bitnet_ternarize_absmean(const float* W, int64_t count, double eps,
                                                  float* W_out, double* gamma_out, void* workspace,
                                                  size_t workspace_bytes, void* stream);

/* Bytes of device scratch that bitnet_i2s_quant_gemv needs for M tokens of
 * length K: the int8 activations and their scales and, for one or two
 * tokens, room for split-K partial sums (256 KB per token) and their
 * counters.  0 for a bad shape. */
BITNET_API size_t bitnet_i2s_quant_gemv_workspace_bytes(int64_t M, int64_t K);

/* Activation quantization followed by the ternary matmul: exactly
 * bitnet_act_quant_i8(X) then bitnet_i2s_gemm [P5 section 5: activations
 * quantized per token with AbsMax, then the ternary contraction].
 *   X: M*K fp32 row-major, 16-byte aligned.
 *   workspace: caller-owned device scratch of at least
 *     bitnet_i2s_quant_gemv_workspace_bytes(M,K) bytes, 256-byte aligned;
 *     it must not be used by other work that may run at the same time.
 *     Its contents need not be initialised: the call zeroes what it counts.
 *   With one or two tokens and fewer 128-row tiles than the GPU runs CTAs of
 *   the decode kernel at once, the call cuts K into slices that run on
 *   separate SMs and adds their int32 partial sums in the workspace; integer
 *   sums are exact, so the results are those of the unsplit contraction.
 *   Other arguments as bitnet_i2s_gemv; M >= 1.  The same as
 *   bitnet_i2s_quant_gemv_batched with one problem. */
BITNET_API bitnet_status bitnet_i2s_quant_gemv(const uint8_t* packed, int64_t N, int64_t K, const float* X,
                                    int64_t M, float* Y, int32_t* acc_or_null, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* One independent problem of a batched call (device pointers; layouts as for
 * bitnet_i2s_quant_gemv): Y[M,N] = matmul(I2_S W[N,K], quant(X[M,K])). */
typedef struct bitnet_i2s_problem {
  const uint8_t* packed;  /* I2_S tensor, 16-byte aligned */
  int64_t N;
  int64_t K;              /* multiple of 128 */
  const float* X;         /* M*K fp32, 16-byte aligned */
  float* Y;               /* M*N fp32 */
  int32_t* acc_or_null;   /* M*N int32 or NULL */
} bitnet_i2s_problem;

/* Workspace bytes bitnet_i2s_quant_gemv_batched needs (0 for bad arguments). */
BITNET_API size_t bitnet_i2s_quant_gemv_batched_workspace_bytes(const bitnet_i2s_problem* problems,
                                                                int count, int64_t M);

/* bitnet_i2s_quant_gemv for `count` independent problems that share the token
 * count M, as few launches as possible: one launch quantizes every problem's
 * activations; for M = 1 with K <= 30720 and M = 2 with K <= 8192,
 * persistent launches of up to 160
 * problems stream the packed weights, handing 128-row tiles out through a
 * work counter in the workspace (longest tiles first), so the whole batch
 * (for example the 210 projections of a 30-layer BitNet b1.58 stack) keeps
 * HBM busy end to end; other shapes go to tensor-core launches of up to 96
 * problems.
 * Results are identical to calling bitnet_i2s_quant_gemv on each problem
 * [P5 section 5: per-token AbsMax quantization, then the ternary contraction].
 *   problems: HOST array of `count` descriptors, read during the call only.
 *   workspace: device scratch of at least
 *     bitnet_i2s_quant_gemv_batched_workspace_bytes(problems, count, M) bytes,
 *     256-byte aligned, not shared with work that may run at the same time;
 *     its contents need not be initialised.
 * When a decode launch has fewer 128-row tiles than it runs CTAs (a few
 * small projections, or one of them), each problem's K is cut into slices of
 * whole 512-weight boxes that run on separate SMs; the slices' int32 partial
 * sums meet in the workspace and the last slice of each tile adds them.
 * The problems' outputs must not overlap each other or any input. */
BITNET_API bitnet_status bitnet_i2s_quant_gemv_batched(const bitnet_i2s_problem* problems, int count,
                                                       int64_t M, void* workspace,
                                                       size_t workspace_bytes, void* stream);

/* Workspace bytes bitnet_i2s_quant_gemv_chain needs (0 for bad arguments;
 * the reason is then readable from bitnet_last_error()). */
BITNET_API size_t bitnet_i2s_quant_gemv_chain_workspace_bytes(const bitnet_i2s_problem* problems,
                                                              const int32_t* stage, int count,
                                                              int64_t M);

/* A chain of fused problems in dependency order, in one persistent
 * cooperative launch per 128 problems (plus one that zeroes the workspace's
 * counters; the cooperative launch needs every CTA of the grid resident, so
 * the call fails with BITNET_ERR_CUDA where that cannot be had): the
 * same results as calling bitnet_i2s_quant_gemv_batched once per stage, in
 * stage order, on the problems of that stage.  This is the shape of a
 * decode step through a BitNet b1.58 layer, whose seven projections each
 * quantize the output of one before them [P2, The Two-Stage BitNet Inference
 * Preprocessing Pipeline: q, k, v, o, gate, up, down; P5 section 5: per-token
 * AbsMax quantization before each ternary matmul].
 *   problems: HOST array of `count` descriptors (read during the call only);
 *     M = 1 or 2 tokens.
 *   stage: HOST array of `count` stage numbers: stage[0] = 0, and each next
 *     one equal to the one before it or one more.
 *   A problem's X is either exactly the Y of a problem of an earlier stage
 *     (the same pointer, K equal to that problem's N) -- it then reads that
 *     output as the earlier call would have left it -- or memory that no
 *     problem of the chain writes.  Outputs must not overlap one another;
 *     anything else is BITNET_ERR_INVALID_ARG, checked before any launch.
 *   The kernel never materialises a chained input in fp32: it quantizes
 *     the earlier problem's exact int32 accumulators with that problem's
 *     scales, in the order and rounding of the fp32 output, so the int8
 *     activations, and with them every acc and Y, are bit-identical to
 *     those of the stage-by-stage calls.
 *   workspace: device scratch of at least
 *     bitnet_i2s_quant_gemv_chain_workspace_bytes(problems, stage, count, M)
 *     bytes, 256-byte aligned, not shared with work that may run at the same
 *     time; its contents need not be initialised.
 *   Dependencies are waited for on the device with bounded waits: a wait
 *     that runs out (2 s) raises BITNET_ERR_DEVICE_TIMEOUT in
 *     bitnet_device_status() and the launch ends early. */
BITNET_API bitnet_status bitnet_i2s_quant_gemv_chain(const bitnet_i2s_problem* problems,
                                                     const int32_t* stage, int count, int64_t M,
                                                     void* workspace, size_t workspace_bytes,
                                                     void* stream);

/* One problem of bitnet_i2s_gemv_batched: activations already quantized. */
typedef struct bitnet_i2s_qproblem {
  const uint8_t* packed;  /* I2_S tensor, 16-byte aligned */
  int64_t N;
  int64_t K;              /* multiple of 128 */
  const int8_t* Xq;       /* M*K int8, 16-byte aligned */
  const float* xs;        /* M fp32 */
  float* Y;               /* M*N fp32 */
  int32_t* acc_or_null;   /* M*N int32 or NULL */
} bitnet_i2s_qproblem;

/* Workspace bytes bitnet_i2s_gemv_batched can use (0 for count < 1). */
BITNET_API size_t bitnet_i2s_gemv_batched_workspace_bytes(int count);

/* bitnet_i2s_gemm on `count` independent problems sharing the token count M
 * (for example q, k and v on one quantized input), in persistent launches
 * of up to 160 problems when M = 1 with K <= 30720 or M = 2 with K <= 8192
 * (the integer-ALU kernel),
 * and of up to 96 problems on the tensor-core kernel otherwise.  Same results
 * as the single-problem call [P5 section 5 figure; P1 "How I2_S Kernels
 * Process the Format"].  `problems` is a HOST array read during the call only.
 *   workspace: NULL, or device scratch of at least
 *     bitnet_i2s_gemv_batched_workspace_bytes(count) bytes, 256-byte aligned,
 *     not shared with work that may run at the same time.  With it, the
 *     integer-ALU launches hand out their tiles through work counters there
 *     (zeroed on `stream` first), which evens out the SMs' finishing times,
 *     and split K as bitnet_i2s_quant_gemv_batched does when a launch has
 *     few row tiles; without it each CTA takes a fixed range of whole tiles.
 *     Results are the same either way. */
BITNET_API bitnet_status bitnet_i2s_gemv_batched(const bitnet_i2s_qproblem* problems, int count,
                                                 int64_t M, void* workspace,
                                                 size_t workspace_bytes, void* stream);

/* bitnet_i2s_quant_gemv without a caller-supplied workspace, for callers
 * that cannot allocate device memory: for example a plug-in that receives only
 * raw input/output pointers from a host framework owning all allocations, or
 * a latency-critical loop that must never enter the CUDA allocator.  (This
 * entry point is a deployment convenience; the pages have no counterpart.)
 *   - Scratch: a fixed 1 MiB array inside the library's device image, held by
 *     every GPU that loads the library until the process exits.  The call
 *     needs bitnet_i2s_quant_gemv_workspace_bytes(M,K) <= 1 MiB, i.e.
 *     M*K rounded up to 256 plus 4*M rounded up to 256; larger shapes return
 *     BITNET_ERR_SHAPE before anything is launched.
 *   - It allocates nothing (no cudaMalloc, cudaFree or allocating library
 *     routine).  The first call on a device looks the array's address up
 *     for that device and its current context (with the device current) and
 *     keeps it; a call that finds a different current context on the device
 *     (after a device reset, say) looks it up again.  Make the first call on
 *     each device before any stream capture.
 *   - That first lookup can load the library's device image onto the device
 *     (CUDA loads modules lazily by default), and loading a module may
 *     allocate device memory and synchronize.  Callers whose later calls must
 *     never do either make one warm-up call per device first (or run with
 *     CUDA_MODULE_LOADING=EAGER, which loads the image when the context is
 *     created).
 *   - Every call on a device shares the one array: two calls whose work may
 *     overlap on the GPU (different streams, no ordering) race on it.  Calls
 *     on one stream are ordered and safe.  Nothing in the array needs to
 *     start at zero; each call overwrites what it reads.
 *   Arguments and results as bitnet_i2s_quant_gemv. */
BITNET_API bitnet_status bitnet_i2s_quant_gemv_noalloc(const uint8_t* packed, int64_t N, int64_t K,
                                                       const float* X, int64_t M, float* Y,
                                                       int32_t* acc_or_null, void* stream);

/* ------------------------------------------------------------------------
 * Block-64 formats ["ik_llama.cpp 运行 BitNet b1.58 2B 模型实战", section 5.2:
 * iq2_bn about 2 bits and iq1_bn 1.625 bits per weight, iq2_bn_r4 = iq2_bn
 * packed in groups of 4 rows; section 5.3: K a multiple of the block of 64;
 * section 6: one row quantized at a time, IQ1_BN decoded with multiplies,
 * adds and shifts; section 5.1: the conversion from I2_S goes through f32,
 * i.e. bitnet_i2s_dequant_f32 then one of the packs below].  The page leaves
 * the bits inside a block open; this library's layouts:
 *   IQ2_BN: a block of 64 weights is 16 bytes, weight j in byte j % 16,
 *     bits [7-2g : 6-2g] with g = j / 16, code = w + 1.  Row n is K/64 blocks;
 *     N*K/4 code bytes are followed by N little-endian fp32 row scales
 *     d_n = max_k |W[n,k]|, with w = clip(round_half_away(W/d_n), -1, 1).
 *   IQ2_BN_R4 (r4 != 0; N a multiple of 4): block b of row 4G + r at byte
 *     ((G*(K/64) + b)*4 + r)*16; row scales as IQ2_BN.
 *   IQ1_BN: a block of 64 weights is 13 bytes; byte i < 12 holds weights
 *     5i .. 5i+4, byte 12 weights 60 .. 63, as ceil(256 v / 243) with
 *     v = sum_j (w_j + 1) 3^(4-j); row scales after the N*(K/64)*13 code
 *     bytes, which must be a multiple of 4.
 * Conventions as for I2_S (device pointers, asynchronous on `stream`,
 * host-side argument checks); all buffers 16-byte aligned; K <= 131072.
 */

/* Size in bytes of an IQ2_BN or IQ2_BN_R4 tensor (0 for a bad shape). */
BITNET_API size_t bitnet_iq2bn_bytes(int64_t N, int64_t K);

/* Size in bytes of an IQ1_BN tensor (0 for a bad shape). */
BITNET_API size_t bitnet_iq1bn_bytes(int64_t N, int64_t K);

/* Pack fp32 W[N,K] into IQ2_BN (r4 == 0) or IQ2_BN_R4 (r4 != 0), one scale
 * per row.  out: bitnet_iq2bn_bytes(N,K) bytes, fully written. */
BITNET_API bitnet_status bitnet_iq2bn_pack(const float* W, int64_t N, int64_t K, int r4,
                                           uint8_t* out, void* stream);

/* IQ2_BN / IQ2_BN_R4 -> fp32 W_out[N,K] = w * d_n, exact. */
BITNET_API bitnet_status bitnet_iq2bn_dequant_f32(const uint8_t* packed, int64_t N, int64_t K,
                                                  int r4, float* W_out, void* stream);

/* Pack fp32 W[N,K] into IQ1_BN, one scale per row.  out:
 * bitnet_iq1bn_bytes(N,K) bytes, fully written.  N*(K/64) % 4 == 0. */
BITNET_API bitnet_status bitnet_iq1bn_pack(const float* W, int64_t N, int64_t K, uint8_t* out,
                                           void* stream);

/* IQ1_BN -> fp32 W_out[N,K] = w * d_n, exact. */
BITNET_API bitnet_status bitnet_iq1bn_dequant_f32(const uint8_t* packed, int64_t N, int64_t K,
                                                  float* W_out, void* stream);

/* Decode matmul on IQ2_BN_R4 weights, M = 1 or 2 tokens, K <= 8192
 * [P5 section 5 figure: add, subtract or skip per ternary weight; the row's
 * scale in place of the tensor's]:
 *   acc[m,n] = sum_k w[n,k] * Xq[m,k] (exact int32),
 *   Y[m,n] = ((float)acc[m,n] * xs[m]) * d_n.
 * Layouts of Xq, xs, Y and acc_or_null as bitnet_i2s_gemv. */
BITNET_API bitnet_status bitnet_iq2bn_r4_gemv(const uint8_t* packed, int64_t N, int64_t K,
                                              const int8_t* Xq, const float* xs, int64_t M,
                                              float* Y, int32_t* acc_or_null, void* stream);

/* Waits for all work on the current device, then returns
 * BITNET_ERR_DEVICE_TIMEOUT if any kernel of this library gave up on a
 * bounded wait since the last call (and clears the flag), BITNET_ERR_CUDA if
 * the device reports an error, else BITNET_OK. */
BITNET_API bitnet_status bitnet_device_status(void);

/* Failure-detection check: launches one bounded device wait on a barrier
 * that nothing completes, so it runs out after `timeout_ns` (1e3..1e8 ns)
 * and raises the same device error flag a stuck pipeline would; the next
 * bitnet_device_status() then returns BITNET_ERR_DEVICE_TIMEOUT and clears
 * it.  Nothing faults or hangs: the kernel returns after the timeout.
 * (A deployment check; the pages have no counterpart.) */
BITNET_API bitnet_status bitnet_debug_wait_timeout(int64_t timeout_ns, void* stream);

/* Message of the last error on this thread ("" if none). */
BITNET_API const char* bitnet_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_I2S_H */
