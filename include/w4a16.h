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
    W4A16_ERR_BAD_OFFSETS = 6   /* device status: expert offsets not 0 = o[0] <= ... <= o[E] = rows */
};

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
