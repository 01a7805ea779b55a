/*
 * w4a16.h — C ABI of the B200 (sm_100a) INT4 group-wise weight-only GEMM library.
 *
 * The operation (Int4GroupwiseGemmPluginV2 page, class description and
 * constructor parameters): activations A [M, K] fp16 times int4 weights W
 * [K, N] with one fp16 scale per group of G consecutive rows of K and per
 * column n, giving C [M, N] fp16:
 *
 *     C[m, n] = fp16( sum_k A[m, k] * q[k, n] * s[floor(k / G), n] )
 *
 * q are signed 4-bit codes in [-8, 7]; s has shape [ceil(K/G), N]; there is
 * no zero point and no bias. The grouped-expert form (Int4MoePlugin page,
 * constructor parameters numExperts, hiddenSize, moeInterSize,
 * quantizationGroupSize) applies one such product per expert to that
 * expert's contiguous block of gathered activation rows.
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev are device pointers (cudaMalloc or torch); the
 *     caller owns every buffer. The library never allocates device memory
 *     on these paths and never frees anything.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). All work is enqueued asynchronously on it; nothing blocks the
 *     host, except w4a16_device_status().
 *   - fp16 tensors are IEEE 754 binary16, passed as w4a16_half (raw bits).
 *   - All matrices are row-major and dense (no row padding).
 *   - Return value: W4A16_OK or one W4A16_ERR_* code. Arguments are fully
 *     validated on the host before anything is enqueued; an argument error
 *     enqueues nothing. No entry point calls exit(), abort() or traps on the
 *     device.
 *   - Errors found on the device (a bounded wait that ran out, malformed
 *     expert offsets) are latched in a per-device status word and read with
 *     w4a16_device_status().
 *
 * Weight layouts:
 *   canonical packed  Wp [ceil(K/2), N] uint8: byte (j, n) holds q[2j, n] in
 *       its low nibble and q[2j+1, n] in its high nibble, each as the
 *       two's-complement nibble (q & 0xF); a missing odd row is 0. This is
 *       the interchange layout (K rows, N columns as on the plugin page).
 *   tiled  Wt, w4a16_tiled_bytes(K, N) bytes: ceil(N/128) x ceil(K/64) tiles
 *       of 4096 bytes (the 128-column x 64-row tile the plugin page's
 *       "fragment weights" use), tile (nt, kt) at byte (nt*ceil(K/64)+kt)*4096.
 *       Inside a tile, half h (k_local 32h..32h+31) of column j (0..127) is 16
 *       bytes at h*2048 + j*16: four little-endian 32-bit words, word w holding
 *       k_local 32h+8w+{0,2,4,6,1,3,5,7} in nibbles 0..7. Rows k >= K and
 *       columns n >= N hold code 0. The GEMM entry points read this layout;
 *       w4a16_repack produces it from the canonical one.
 */
#ifndef W4A16_H
#define W4A16_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t w4a16_half; /* IEEE 754 binary16 bit pattern */

enum {
    W4A16_OK = 0,
    W4A16_ERR_INVALID_ARG = 1,  /* null pointer, negative or zero size, G <= 0, E out of range */
    W4A16_ERR_MISALIGNED = 2,   /* a pointer is not 16-byte aligned */
    W4A16_ERR_UNSUPPORTED = 3,  /* shape outside the GPU contract, or no sm_100 device */
    W4A16_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    W4A16_ERR_TIMEOUT = 5,      /* device status: a bounded wait inside a kernel ran out */
    W4A16_ERR_BAD_OFFSETS = 6,  /* device status: expert offsets not 0 = o[0] <= ... <= o[E] = rows */
    W4A16_ERR_BAD_ROUTING = 7,  /* device status: an expert id out of range or repeated within a token,
                                   or a gathered-row index out of range */
    W4A16_ERR_SCRATCH_TOO_SMALL = 8  /* w4a16_moe_layer_static: the shape needs more intermediates than
                                        the library's static scratch holds */
};

/* Elementwise activations of the expert layer (Int4 Moe Plugin page,
 * constructor parameter activationType), applied to the fp16 result x of the
 * up projection and rounded to fp16 again:
 *   IDENTITY   x
 *   RELU       max(x, 0)
 *   GELU_ERF   x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2))
 *   GELU_TANH  0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
 * evaluated in fp32 on the device. */
enum {
    W4A16_ACT_IDENTITY = 0,
    W4A16_ACT_RELU = 1,
    W4A16_ACT_GELU_ERF = 2,
    W4A16_ACT_GELU_TANH = 3
};

/* Largest topK the expert layer accepts. */
#define W4A16_MAX_TOPK 8

/* Largest number of experts one w4a16_grouped_gemm call accepts. */
#define W4A16_MAX_EXPERTS 64

/* Human-readable name of a status code (static string, never NULL). */
const char* w4a16_status_string(int status);

/* Pack int8 codes q_dev [K, N] (values in [-8, 7]; other values are masked
 * to their low 4 bits) into the canonical layout wp_dev [ceil(K/2), N].
 * Plugin page: weights as K rows by N columns, two int4 codes per byte.
 * Errors: INVALID_ARG (null pointer, K <= 0, N <= 0), CUDA. */
int w4a16_pack(const int8_t* q_dev, uint8_t* wp_dev, int64_t K, int64_t N, void* stream);

/* Group-wise symmetric int4 quantisation of fp16 weights W_dev [K, N]
 * row-major, the export step that produces the GEMM's codes and scales. Rule
 * of the KV Cache INT8 quantization page's symmetric quantisation kernel
 * (scale = max|x| / 127, x_q = round(x / scale)), taken with the int4 code
 * range over each group of G rows of one column, the scale kept in fp16 as
 * the Int4 Groupwise GEMM Plugin V2 page's scales [ceil(K/G), N]:
 *     s[g, n] = fp16_rne(float(max |W[k, n]| over group g) / 7)
 *     q[k, n] = clamp(round(float(W[k, n]) / float(s[g, n])), -8, 7)
 * with IEEE float division and halves rounded away from zero; q = 0 where
 * s = 0. Codes go to wp_dev in the canonical layout [ceil(K/2), N] (as
 * w4a16_pack writes them), scales to S_dev [ceil(K/G), N]. W must be finite.
 * GPU contract: N and G even, K, N < 2^31; W_dev and S_dev 4-byte aligned,
 * wp_dev 2-byte aligned. Errors: INVALID_ARG (null pointer, K, N or G <= 0),
 * MISALIGNED, UNSUPPORTED, CUDA. */
int w4a16_quantize(const w4a16_half* W_dev, uint8_t* wp_dev, w4a16_half* S_dev, int64_t K, int64_t N,
                   int64_t G, void* stream);

/* Inverse of w4a16_pack: canonical wp_dev -> int8 codes q_dev [K, N], sign
 * extended. Same errors as w4a16_pack. */
int w4a16_unpack(const uint8_t* wp_dev, int8_t* q_dev, int64_t K, int64_t N, void* stream);

/* Size in bytes of the tiled layout for K x N codes (0 if K or N <= 0). */
int64_t w4a16_tiled_bytes(int64_t K, int64_t N);

/* One-off repack of canonical weights wp_dev [ceil(K/2), N] into the tiled
 * layout wt_dev (w4a16_tiled_bytes(K, N) bytes, 16-byte aligned), the
 * counterpart of the plugin page's export-time repack into its fragment
 * layout. Errors: INVALID_ARG, MISALIGNED (wt_dev), CUDA. */
int w4a16_repack(const uint8_t* wp_dev, uint8_t* wt_dev, int64_t K, int64_t N, void* stream);

/* C_dev [M, N] = A_dev [M, K] x dequant(Wt) with scales S_dev [ceil(K/G), N].
 * Wt_dev is the tiled layout. Plugin page: inputs [0] activations, [1]
 * weights, [2] scales; output [0]; enqueue on a stream, 0 on success.
 * GPU contract: N % 8 == 0, K % 8 == 0, G % 16 == 0 (G > K is allowed and
 * means one group); A_dev, Wt_dev, S_dev 16-byte aligned; C_dev 2-byte
 * aligned; N, K < 2^31, M < 2^31. M == 0 is a no-op.
 * Accumulation is fp32; each dequantised weight q*s is rounded to fp16
 * before the product; the result is rounded to fp16 once.
 * Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED, CUDA. */
int w4a16_gemm(const w4a16_half* A_dev, const uint8_t* Wt_dev, const w4a16_half* S_dev,
               w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G, void* stream);

/* Flags of w4a16_gemm_ex. */
#define W4A16_FLAG_STATIC_WEIGHTS 1u /* this call's Wt and S are not written by any kernel that may still be
                                        running on the stream (weights prepared at load time): the GEMM may
                                        stream them before the previous kernel on the stream finishes */

/* w4a16_gemm with per-call flags (0 or W4A16_FLAG_STATIC_WEIGHTS): the
 * static-weights promise of w4a16_set_static_weights scoped to this one call,
 * so that one stream's GEMMs can stream their fixed weights early while
 * another stream repacks or requantises others. Same contract and errors as
 * w4a16_gemm; INVALID_ARG also for unknown flag bits. */
int w4a16_gemm_ex(const w4a16_half* A_dev, const uint8_t* Wt_dev, const w4a16_half* S_dev, w4a16_half* C_dev,
                  int64_t M, int64_t N, int64_t K, int64_t G, uint32_t flags, void* stream);

/* Grouped-expert form. A_dev [total_rows, K] holds the activation rows
 * already gathered per expert; rows [off[e], off[e+1]) of A_dev and of
 * C_dev [total_rows, N] belong to expert e, which uses tiled weights
 * Wt[e] and scales S[e] [ceil(K/G), N]. Wt and S are HOST arrays of E device
 * pointers. offsets_dev is a DEVICE array of E+1 int32 with off[0] = 0,
 * non-decreasing, off[E] = total_rows; empty experts are allowed. A kernel
 * that finds the offsets malformed writes nothing and latches
 * W4A16_ERR_BAD_OFFSETS in the device status. 1 <= E <= W4A16_MAX_EXPERTS;
 * total_rows == 0 is a no-op. Same GPU contract and errors as w4a16_gemm. */
int w4a16_grouped_gemm(const w4a16_half* A_dev, const uint8_t* const* Wt, const w4a16_half* const* S,
                       const int32_t* offsets_dev, w4a16_half* C_dev, int64_t E, int64_t total_rows,
                       int64_t N, int64_t K, int64_t G, void* stream);

/* w4a16_grouped_gemm with the activation `act` (W4A16_ACT_*) applied to each
 * fp16 result element in the epilogue: C = fp16(act(fp16(A x dequant(W)))).
 * The expert layer's up projection (Int4 Moe Plugin page: hiddenSize ->
 * moeInterSize, then activationType). Same contract and errors as
 * w4a16_grouped_gemm; INVALID_ARG also for an unknown act. */
int w4a16_grouped_gemm_act(const w4a16_half* A_dev, const uint8_t* const* Wt, const w4a16_half* const* S,
                           const int32_t* offsets_dev, w4a16_half* C_dev, int64_t E, int64_t total_rows,
                           int64_t N, int64_t K, int64_t G, int act, void* stream);

/* ---------------------------------------------------------------------------
 * The INT4 mixture-of-experts layer (Int4 Moe Plugin page: constructor
 * parameters numExperts E, topK k, hiddenSize H, moeInterSize I,
 * activationType, quantizationGroupSize G; getWorkspaceSize; enqueue with a
 * workspace and a stream; one output). The page names the parameters, not the
 * steps; the steps are the plain reading of them, for T tokens:
 *
 *   1. route     ids[t, 0..k-1]: the k experts with the largest router logits
 *                (ties: the lower expert index first), in descending order;
 *                weights[t, j] = softmax over the k selected logits (fp32).
 *   2. dispatch  the T*k (token, slot) pairs grouped by expert, stable in the
 *                flat order t*k + j: offsets[E+1] (expert e owns gathered rows
 *                offsets[e] .. offsets[e+1]-1), pos[t, j] (the gathered row of
 *                the pair), src_row[r] (the token of gathered row r).
 *   3. gather    Xg[r] = X[src_row[r]].
 *   4. up        A = fp16(act(fp16(Xg x dequant(W_up[e])))), per expert [H -> I].
 *   5. down      Y = fp16(A x dequant(W_down[e])), per expert [I -> H].
 *   6. combine   out[t] = fp16(sum over j of weights[t, j] * Y[pos[t, j]]),
 *                fp32 arithmetic in slot order.
 *
 * Each step is an entry point of its own; w4a16_moe_layer enqueues all six on
 * one stream with intermediates in a caller-owned workspace. Sizes: 1 <= E <=
 * W4A16_MAX_EXPERTS, 1 <= k <= min(E, W4A16_MAX_TOPK), T*k < 2^31. Router
 * logits must be finite (a NaN logit is never preferred over a finite one, so
 * the ids stay valid, but its weight is NaN).
 * ------------------------------------------------------------------------- */

/* Step 1. logits_dev [T, E] fp16 -> ids_dev [T, k] int32, weights_dev [T, k]
 * fp32. T == 0 is a no-op. Errors: INVALID_ARG, UNSUPPORTED (no sm_100
 * device), CUDA. */
int w4a16_moe_route(const w4a16_half* logits_dev, int32_t* ids_dev, float* weights_dev, int64_t T, int64_t E,
                    int64_t top_k, void* stream);

/* Step 2. ids_dev [T, k] int32 -> offsets_dev [E+1], pos_dev [T, k],
 * src_row_dev [T*k] (all int32). If any id is outside [0, E) or repeated
 * within a token, the kernel writes offsets all 0, pos and src_row all -1, and
 * latches W4A16_ERR_BAD_ROUTING. T == 0 writes offsets all 0. Errors:
 * INVALID_ARG, UNSUPPORTED, CUDA. */
int w4a16_moe_dispatch(const int32_t* ids_dev, int32_t* offsets_dev, int32_t* pos_dev, int32_t* src_row_dev,
                       int64_t T, int64_t E, int64_t top_k, void* stream);

/* Step 3. X_dev [T, H] -> Xg_dev [rows, H] with Xg[r] = X[src_row[r]]. H % 8
 * == 0; X_dev and Xg_dev 16-byte aligned. A row index outside [0, T) writes
 * zeros and latches W4A16_ERR_BAD_ROUTING. Errors: INVALID_ARG, MISALIGNED,
 * UNSUPPORTED, CUDA. */
int w4a16_moe_gather(const w4a16_half* X_dev, const int32_t* src_row_dev, w4a16_half* Xg_dev, int64_t T,
                     int64_t rows, int64_t H, void* stream);

/* Step 6. Y_dev [T*k, H], weights_dev [T, k] fp32, pos_dev [T, k] -> out_dev
 * [T, H]. H % 8 == 0; Y_dev and out_dev 16-byte aligned. A term whose pos is
 * outside [0, T*k) is left out and W4A16_ERR_BAD_ROUTING latched. Errors:
 * INVALID_ARG, MISALIGNED, UNSUPPORTED, CUDA. */
int w4a16_moe_combine(const w4a16_half* Y_dev, const float* weights_dev, const int32_t* pos_dev,
                      w4a16_half* out_dev, int64_t T, int64_t top_k, int64_t H, void* stream);

/* Bytes of workspace w4a16_moe_layer needs (the page's getWorkspaceSize):
 * ids, weights, pos, src_row, offsets, the gathered rows [T*k, H], the
 * activated up projection [T*k, I] and the down projection [T*k, H], each
 * starting on a 256-byte boundary. Returns -1 for invalid sizes. */
int64_t w4a16_moe_workspace_size(int64_t T, int64_t E, int64_t top_k, int64_t H, int64_t I);

/* The whole layer: out_dev [T, H] from hidden states X_dev [T, H] and router
 * logits logits_dev [T, E]. Wt_up / S_up / Wt_down / S_down are HOST arrays of
 * E device pointers: tiled weights [H -> I] and [I -> H] with scales
 * [ceil(H/G), I] and [ceil(I/G), H]. workspace_dev (16-byte aligned, at least
 * w4a16_moe_workspace_size bytes) is caller-owned; nothing in it needs to be
 * initialised, and two calls that overlap on the GPU must not share it.
 * Contract of the GEMMs (H, I multiples of 8, G % 16 == 0). T == 0 is a no-op.
 * Errors: INVALID_ARG (also workspace too small or unknown act), MISALIGNED,
 * UNSUPPORTED, CUDA. */
int w4a16_moe_layer(const w4a16_half* X_dev, const w4a16_half* logits_dev, const uint8_t* const* Wt_up,
                    const w4a16_half* const* S_up, const uint8_t* const* Wt_down, const w4a16_half* const* S_down,
                    w4a16_half* out_dev, int64_t T, int64_t E, int64_t top_k, int64_t H, int64_t I, int64_t G,
                    int act, void* workspace_dev, int64_t workspace_bytes, void* stream);

/* The whole layer without a caller workspace: the same six steps as
 * w4a16_moe_layer (same kernels, bit-identical results), with the
 * intermediates in a fixed region of device memory that the library itself
 * owns, w4a16_moe_static_scratch_bytes() = 8 MiB per device, created with the
 * library's device code when the CUDA runtime loads it. The plugin pages have
 * no counterpart of this entry point.
 *
 * For callers that cannot provide or obtain device memory at call time: an
 * engine whose execute step was promised a zero-byte workspace when it was
 * built, or C code that owns no device allocator. Allocating inside the call
 * is no option for them (cudaMalloc synchronizes the device and may fail under
 * memory pressure in the middle of a step); nothing here calls cudaMalloc,
 * cudaFree or any other allocating routine.
 *
 * - The first call on a device looks up the region's device address
 *   (cudaGetSymbolAddress, with that device current) and keeps it; make that
 *   first call on each device before any stream capture begins.
 * - Shapes whose intermediates (w4a16_moe_workspace_size) exceed the region
 *   are refused with W4A16_ERR_SCRATCH_TOO_SMALL before anything is enqueued;
 *   at H = 4096 and I = 14336 the region holds about 180 gathered rows
 *   (T * topK), a decode batch.
 * - Nothing in the region needs to start at zero or survive between calls:
 *   every intermediate is written before it is read within a call.
 * - All calls on a device share the one region: two calls whose kernels may
 *   overlap on the GPU (different streams, or different host threads, without
 *   ordering between them) race on it and may return wrong results. Calls
 *   ordered on one stream are safe.
 * Arguments, other errors and T == 0 as for w4a16_moe_layer. */
int w4a16_moe_layer_static(const w4a16_half* X_dev, const w4a16_half* logits_dev, const uint8_t* const* Wt_up,
                           const w4a16_half* const* S_up, const uint8_t* const* Wt_down,
                           const w4a16_half* const* S_down, w4a16_half* out_dev, int64_t T, int64_t E,
                           int64_t top_k, int64_t H, int64_t I, int64_t G, int act, void* stream);

/* Size in bytes of the static scratch region of w4a16_moe_layer_static. */
int64_t w4a16_moe_static_scratch_bytes(void);

/* Declares (enable != 0) or withdraws (enable == 0) the promise that no
 * kernel on the calling streams writes the tiled weights or the scales passed
 * to w4a16_gemm right before that call, i.e. the weights are static (prepared
 * once, as at model load time). Every GEMM kernel is launched with
 * programmatic dependent launch, so it may start while the previous kernel on
 * its stream is still running; it always waits for that kernel before reading
 * activations or writing the output. With static weights declared, the dense
 * kernels also start streaming Wt and S before that wait, which hides the
 * launch and memory-latency ramp between back-to-back GEMMs. Process-wide;
 * off by default. Returns the previous setting. Has no counterpart on the
 * plugin pages. */
int w4a16_set_static_weights(int enable);

/* How w4a16_gemm / w4a16_grouped_gemm will launch for a shape (no work is
 * enqueued): the token tile (MMA N extent), the K split, the grid and the
 * CTAs per SM. Errors as for the GEMM's host validation. */
typedef struct {
    int32_t token_tile;   /* activation rows per CTA tile (16..256) */
    int32_t k_splits;     /* CTAs along K that reduce through a thread-block cluster */
    int32_t grid_x, grid_y, grid_z;
    int32_t threads_per_cta;
    int32_t smem_bytes;
    int32_t ctas_per_sm;
} w4a16_launch_info;

int w4a16_gemm_launch_info(int64_t M, int64_t N, int64_t K, int64_t G, w4a16_launch_info* info);
int w4a16_grouped_launch_info(int64_t E, int64_t total_rows, int64_t N, int64_t K, int64_t G,
                              w4a16_launch_info* info);

/* ---------------------------------------------------------------------------
 * W8A16: the INT8 weight-only variant (the FP8-vs-INT8 TensorRT-LLM comparison
 * page lists INT8 weight-only with an FP16 KV cache among its INT8
 * configurations). The same group-wise product with signed 8-bit codes:
 *     C[m, n] = fp16( sum_k A[m, k] * q8[k, n] * s[floor(k / G), n] ),
 * q8 in [-128, 127], s [ceil(K/G), N] fp16. Canonical codes are int8 [K, N]
 * row-major, one per byte (no packing). Tiled layout (the GEMM's operand),
 * w8a16_tiled_bytes(K, N) bytes: ceil(N/128) x ceil(K/64) tiles of 8192 bytes,
 * tile (nt, kt) at byte (nt*ceil(K/64)+kt)*8192; inside a tile, quarter h
 * (k_local 16h..16h+15) of column j is 16 bytes at h*2048 + j*16, byte b
 * holding k_local 16h + b as a two's-complement byte; rows k >= K and columns
 * n >= N hold 0. The product runs on the tensor-core kernel for every M.
 * ------------------------------------------------------------------------- */

/* Group-wise symmetric 8-bit quantisation of fp16 weights W_dev [K, N], the
 * export step of W8A16: the KV Cache INT8 quantization page's symmetric rule
 * (scale = max|x| / 127, x_q = round(x / scale)) over each group of G rows of
 * one column, the scale kept in fp16:
 *     s[g, n] = fp16_rne(float(max |W[k, n]| over group g) / 127)
 *     q8[k, n] = clamp(round(float(W[k, n]) / float(s[g, n])), -128, 127)
 * with IEEE float division and halves rounded away from zero; q8 = 0 where
 * s = 0. Codes to q8_dev [K, N] int8 row-major, scales to S_dev [ceil(K/G), N].
 * Same contract, alignment and errors as w4a16_quantize (q8_dev 2-byte
 * aligned). */
int w8a16_quantize(const w4a16_half* W_dev, int8_t* q8_dev, w4a16_half* S_dev, int64_t K, int64_t N, int64_t G,
                   void* stream);

/* Size in bytes of the 8-bit tiled layout for K x N codes (0 if K or N <= 0). */
int64_t w8a16_tiled_bytes(int64_t K, int64_t N);

/* One-off repack of int8 codes q_dev [K, N] into the 8-bit tiled layout wt_dev
 * (16-byte aligned). Errors: INVALID_ARG, MISALIGNED, UNSUPPORTED (no sm_100
 * device), CUDA. */
int w8a16_repack(const int8_t* q_dev, uint8_t* wt_dev, int64_t K, int64_t N, void* stream);

/* C_dev [M, N] = A_dev [M, K] x (q8 * s) from the 8-bit tiled layout Wt8_dev and
 * scales S_dev [ceil(K/G), N]. Same GPU contract, rounding and errors as
 * w4a16_gemm (each dequantised weight q*s rounded to fp16 before the product,
 * fp32 accumulation, one rounding of the result). */
int w8a16_gemm(const w4a16_half* A_dev, const uint8_t* Wt8_dev, const w4a16_half* S_dev, w4a16_half* C_dev,
               int64_t M, int64_t N, int64_t K, int64_t G, void* stream);

/* How w8a16_gemm will launch for a shape (no work is enqueued). */
int w8a16_gemm_launch_info(int64_t M, int64_t N, int64_t K, int64_t G, w4a16_launch_info* info);

/* ---------------------------------------------------------------------------
 * Tactics (Int4GroupwiseGemmPluginV2 page: getNbTactics / getValidTactics list
 * the valid variants as ids >= 1, setTactic selects one, 0 is the default
 * variant; configurePlugin captures the optimum M the tuning is done for; the
 * timing cache tunes identical shapes once). A tactic of w4a16_gemm for a
 * shape (M, N, K, G) is one launch form: the skinny kernel (M <= 16 only) with
 * a K split over 1..8 cluster CTAs, one or two K halves per CTA and a ring
 * depth, or the tensor-core kernel with a token tile of 16..256 rows and a K
 * split of 1, 2, 4 or 8. Every tactic computes the same product (the K split
 * changes the fp32 summation order only). The process-wide table maps a shape
 * on a device to its tactic; w4a16_gemm and w4a16_gemm_launch_info use the
 * table's tactic when it holds one for the exact shape, else the built-in
 * heuristic. The table is guarded by a mutex; its lookup is skipped while it
 * is empty.
 * ------------------------------------------------------------------------- */

/* The ids (1..count) of the valid tactics for a shape, skinny forms first.
 * Writes min(count, capacity) ids to `tactics` and the total to *count.
 * Errors: INVALID_ARG, UNSUPPORTED (shape outside the GPU contract). */
int w4a16_get_valid_tactics(int64_t M, int64_t N, int64_t K, int64_t G, int32_t* tactics, int32_t capacity,
                            int32_t* count);

/* The launch form of one tactic id for a shape. Errors: INVALID_ARG (also an
 * id outside 1..count), UNSUPPORTED. */
int w4a16_tactic_launch_info(int64_t M, int64_t N, int64_t K, int64_t G, int32_t tactic,
                             w4a16_launch_info* info);

/* Pins tactic `tactic` for the shape on the current device (0 removes the
 * entry: the heuristic applies again). Errors: INVALID_ARG, UNSUPPORTED. */
int w4a16_set_tactic(int64_t M, int64_t N, int64_t K, int64_t G, int32_t tactic);

/* The table's tactic for the shape on the current device (0 if none). */
int w4a16_get_tactic(int64_t M, int64_t N, int64_t K, int64_t G, int32_t* tactic);

/* Empties the tactic table. Always W4A16_OK. */
int w4a16_clear_tactics(void);

/* Times every valid tactic for the shape and stores the fastest in the table
 * (the page's timing cache). A [M, K] is read and C [M, N] overwritten; Wt and
 * S are HOST arrays of `copies` device pointers to copies of the tiled weights
 * and scales (1 <= copies <= 1024). For each tactic, `reps` launches rotating
 * over the copies are recorded into a CUDA graph (on a stream of its own) and
 * replayed on `stream`: launches back to back, as a model's layers run them,
 * with their programmatic-dependent-launch overlap; when the copies together
 * exceed the L2 cache the weights come from HBM, as they do when many layers'
 * weights stream by. The time of a tactic is the fastest of three replays per
 * launch. Blocks the host until the timing is done: call it at setup, not
 * while `stream` is being captured. Writes the winning id to *best_tactic, its
 * time per launch in microseconds to *best_us (if not NULL), and the time of
 * tactic id t to times_us[t - 1] for the first times_capacity ids (times_us
 * may be NULL when times_capacity is 0). Same contract and errors as
 * w4a16_gemm; INVALID_ARG also for reps outside 1..10000. */
int w4a16_autotune(const w4a16_half* A_dev, const uint8_t* const* Wt, const w4a16_half* const* S, int32_t copies,
                   w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G, int32_t reps,
                   int32_t* best_tactic, float* best_us, float* times_us, int32_t times_capacity, void* stream);

/* Test aid for the failure path of the bounded device waits (no counterpart
 * on the plugin pages). For every later launch of the tensor-core GEMM kernel
 * (w4a16_gemm with M > 16, and w4a16_grouped_gemm) until it is called again:
 * every bounded wait in the kernel runs out after wait_limit_cycles SM clock
 * cycles (<= 0 restores the default of about 2 s), and, if stall_stage >= 0,
 * the dequantising warps withhold the ready signal of that 64-deep K stage
 * (counted from the start of each CTA's K range), so the MMA thread's wait for
 * it runs out. The kernel then latches W4A16_ERR_TIMEOUT, lets every copy and
 * MMA in flight complete, frees its tensor memory and writes no output tile
 * that the stalled stage (or, with K split over a cluster, any CTA of the
 * cluster) contributes to; nothing faults or hangs. Process-wide; always
 * returns W4A16_OK. */
int w4a16_set_fault_injection(int64_t stall_stage, int64_t wait_limit_cycles);

/* Reads (and, if clear != 0, resets) the current device's status word. This
 * synchronizes the current device. Returns W4A16_OK, W4A16_ERR_TIMEOUT,
 * W4A16_ERR_BAD_OFFSETS, or W4A16_ERR_CUDA if the read itself failed. */
int w4a16_device_status(int clear);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
