// Group-wise symmetric int4 quantisation of fp16 weights: the export step that
// produces the codes and scales the GEMM consumes.
//
// Rule (KV Cache INT8 quantization page, symmetric quantisation kernel: scale =
// max|x| / 127, x_q = round(x / scale), in float), taken with the int4 code range
// (largest positive code 7) over each group of G rows of one column, the scale
// stored in fp16 as the Int4 Groupwise GEMM Plugin V2 page lays scales out
// ([ceil(K/G), N]):
//     s[g, n] = fp16_rne(float(max |W[k, n]| over the group) / 7)
//     q[k, n] = clamp(round(float(W[k, n]) / float(s[g, n])), -8, 7), 0 if s == 0
// with IEEE float division and round() taking halves away from zero. Codes are
// written straight into the canonical packed layout (include/w4a16.h).
//
// A setup kernel (once per weight matrix, outside any timed GEMM). Each CTA
// takes one group of G rows of a 256-column tile: one TMA copy brings the
// G x 256 fp16 tile into shared memory (read from HBM once). Four slices of
// 128 threads split the group's rows; each thread owns two adjacent columns of
// its slice: the slice maximum, combined with the other slices' through shared
// memory into the group's fp16 scale, then one packed byte per column and row
// pair of the slice, stored 64 columns per warp (coalesced).
// Weights that the copy engine cannot address (W not 16-byte aligned, N % 8,
// G > 256) take a fallback kernel that reads each group twice from global
// memory instead.
//
// The quotient w / s decides an integer, so it must be the IEEE one: the
// kernels take w * (1/s) (within 2 ulp of it) and fall back to the IEEE
// division only when that product lies within 1e-5 (8-bit codes: 1e-4) of a
// rounding boundary (a half-integer); elsewhere both round to the same integer.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/w4a16.h"
#include "ptx.cuh"
#include "w4a16_internal.h"

namespace w4a16 {

__device__ int g_quant_status;  // latched W4A16_ERR_TIMEOUT (0 = none)

namespace {

constexpr int kQuantThreads = 128;          // column pairs of a 256-column tile
constexpr int kTileCols = 2 * kQuantThreads;
constexpr int kSlices = 4;                  // row slices of a group in the staged kernel (one warp group each)
constexpr int kMaxTmaGroup = 256;           // rows of one copy (the copy engine's box limit)
constexpr long long kQuantTimeoutCycles = 4000000000ll;  // about 2 s at the boost clock

// BITS = 4: int4 codes in [-8, 7], scale max/7, two codes per byte (row pairs).
// BITS = 8: 8-bit codes in [-128, 127], scale max/127, one code per byte (the
// W8A16 export step). The boundary window around a half-integer covers the
// product's error (2 ulp of a quotient below 8, or below 128).
template <int BITS>
struct QuantRange {
    static constexpr int kMin = BITS == 4 ? -8 : -128;
    static constexpr int kMax = BITS == 4 ? 7 : 127;
    static constexpr float kWindow = BITS == 4 ? 1e-5f : 1e-4f;
};

// Code of weight w with scale s (inverse rs = 1/s rounded, 0 when s = 0):
// round(w / s), halves away from zero, clamped to the code range; 0 when s = 0
// (then x = w * 0 = 0 for finite w, whose nearest integer is 0 with no
// boundary to check).
// Away from a half-integer the quotient's nearest integer (that of w * (1/s))
// is the rounded code under any tie rule: the true quotient is within 2 ulp of
// the product, far inside the window. Near a half-integer the IEEE quotient
// decides, with halves away from zero.
// The nearest integer of x comes from the magic-number method: for |x| < 2^22
// the float sum x + 1.5 * 2^23 lies in [2^23, 2^24), where the spacing is 1, so
// the sum is rounded to an integer (ties to even) and its bit pattern is
// 0x4B400000 + that integer; subtracting 1.5 * 2^23 again gives it as a float.
// (|x| stays far below 2^22: at most about 2 * 127 for 8-bit codes.)
// Returns a word whose low BITS bits are the code (two's complement).
// CLAMP = false leaves out the clamp, for groups whose scale is 0 or a normal
// fp16 number: then s >= (max / kMax) (1 - 2^-11) (one fp16 and one float
// rounding), so |w| <= max gives |w * (1/s)| <= kMax (1 + 2^-10) < kMax + 0.5,
// and the rounded code is already in range. Below 2^-14 (subnormal scales) the
// fp16 rounding error is relatively larger and the clamp is needed. Without
// the clamp the code is read straight from the low bits of the magic sum
// (0x4B400000 is a multiple of 256, so those bits are the integer's own).
template <int BITS, bool CLAMP>
__device__ __forceinline__ uint32_t quantize_code(float w, float s, float rs) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23, bit pattern 0x4B400000
    const float x = w * rs;
    const float m = x + kMagic;
    int q = __float_as_int(m);
    const bool boundary = fabsf(x - (m - kMagic)) > 0.5f - QuantRange<BITS>::kWindow;
    if constexpr (CLAMP) {
        q -= 0x4B400000;
        if (boundary) q = static_cast<int>(roundf(__fdiv_rn(w, s)));
        q = q < QuantRange<BITS>::kMin ? QuantRange<BITS>::kMin
                                       : (q > QuantRange<BITS>::kMax ? QuantRange<BITS>::kMax : q);
        return static_cast<uint32_t>(q) & (BITS == 4 ? 0xFu : 0xFFu);
    } else {
        if (boundary) q = static_cast<int>(roundf(__fdiv_rn(w, s)));
        return static_cast<uint32_t>(q);
    }
}

template <int BITS>
__device__ __forceinline__ __half2 group_scales(float a0, float a1) {
    constexpr float kDiv = static_cast<float>(QuantRange<BITS>::kMax);
    return __halves2half2(__float2half_rn(__fdiv_rn(a0, kDiv)), __float2half_rn(__fdiv_rn(a1, kDiv)));
}

// Rows 0..nrows-1 of one column pair, read through row(r), whose maxima are
// (a0, a1): the pair's fp16 scales (stored at s_out), then the codes, written
// from out_row0 on with a stride of N2 16-bit words per output row: for int4 one
// packed byte per column and row pair (rows of the canonical packed layout), for
// 8-bit codes one byte per column and row.
// The codes of rows 0..n-1 of one column pair with scales s and inverses
// (r0, r1), written from out on with a stride of N2 16-bit words per row.
template <int BITS, bool CLAMP, typename RowFn>
__device__ __forceinline__ void quantize_rows(RowFn row, int n, uint16_t* __restrict__ out, int64_t N2, float2 s,
                                              float r0, float r1) {
    if constexpr (BITS == 4) {
        // Row pairs (k, k + 1): groups start on even rows (G is even), so a packed
        // byte never spans two groups; a missing last odd row packs 0.
        const int full = n & ~1;
#pragma unroll 4
        for (int r = 0; r < full; r += 2, out += N2) {
            const float2 lo = __half22float2(row(r));
            const float2 hi = __half22float2(row(r + 1));
            const uint32_t b0 = (quantize_code<4, CLAMP>(lo.x, s.x, r0) & 0xFu) |
                                ((quantize_code<4, CLAMP>(hi.x, s.x, r0) & 0xFu) << 4);
            const uint32_t b1 = (quantize_code<4, CLAMP>(lo.y, s.y, r1) & 0xFu) |
                                ((quantize_code<4, CLAMP>(hi.y, s.y, r1) & 0xFu) << 4);
            *out = static_cast<uint16_t>(b0 | (b1 << 8));  // bytes of the pair's two columns
        }
        if (n & 1) {
            const float2 lo = __half22float2(row(full));
            *out = static_cast<uint16_t>((quantize_code<4, CLAMP>(lo.x, s.x, r0) & 0xFu) |
                                         ((quantize_code<4, CLAMP>(lo.y, s.y, r1) & 0xFu) << 8));
        }
    } else {
#pragma unroll 4
        for (int r = 0; r < n; ++r, out += N2) {
            const float2 v = __half22float2(row(r));
            *out = static_cast<uint16_t>((quantize_code<8, CLAMP>(v.x, s.x, r0) & 0xFFu) |
                                         ((quantize_code<8, CLAMP>(v.y, s.y, r1) & 0xFFu) << 8));
        }
    }
}

template <int BITS, typename RowFn>
__device__ __forceinline__ void quantize_pair(RowFn row, int64_t nrows, uint16_t* __restrict__ out_row0,
                                              int64_t N2, __half2* __restrict__ s_out, float a0, float a1) {
    const __half2 sh = group_scales<BITS>(a0, a1);
    *s_out = sh;
    const float2 s = __half22float2(sh);
    const float r0 = s.x != 0.0f ? __frcp_rn(s.x) : 0.0f;
    const float r1 = s.y != 0.0f ? __frcp_rn(s.y) : 0.0f;
    // (nrows is at most G rows of one group, below 2^31)
    const int n = static_cast<int>(nrows);
    constexpr float kMinNormal = 6.103515625e-05f;  // 2^-14, the smallest normal fp16 number
    const bool in_range = (s.x == 0.0f || s.x >= kMinNormal) && (s.y == 0.0f || s.y >= kMinNormal);
    if (in_range)
        quantize_rows<BITS, false>(row, n, out_row0, N2, s, r0, r1);
    else
        quantize_rows<BITS, true>(row, n, out_row0, N2, s, r0, r1);
}

// Group g of a 256-column tile through shared memory (see the file header).
template <int BITS>
__global__ void __launch_bounds__(kQuantThreads * kSlices) quantize_tma_kernel(const __grid_constant__ CUtensorMap tmW,
                                                                      uint16_t* __restrict__ wp,
                                                                      __half2* __restrict__ S, int64_t K,
                                                                      int64_t N, int64_t G, int64_t groups) {
    extern __shared__ __align__(128) uint8_t qsm[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(qsm);
    volatile int* stop = reinterpret_cast<volatile int*>(qsm + 8);
    float2* part = reinterpret_cast<float2*>(qsm + 128);                              // [kSlices][kQuantThreads]
    const __half2* tile = reinterpret_cast<const __half2*>(qsm + 128 + kSlices * kQuantThreads * 8);  // [G][128]
    const int64_t N2 = N / 2;
    const int t = threadIdx.x & (kQuantThreads - 1);
    const int slice = threadIdx.x / kQuantThreads;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * kQuantThreads + t;  // column pair
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    uint32_t phase = 0;
    for (int64_t g = blockIdx.y; g < groups; g += gridDim.y, phase ^= 1u) {
        const int64_t k0 = g * G;
        const int64_t nrows = (k0 + G < K ? k0 + G : K) - k0;
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(G * kTileCols * 2));
            tma_load_2d(const_cast<__half2*>(tile), &tmW, static_cast<int32_t>(blockIdx.x) * kTileCols, static_cast<int32_t>(k0), bar);
            // Bounded wait for the copy. Past the first bound the status is latched
            // and the copy gets a second bound to land. If it has still not landed
            // then, the whole CTA stops with the copy possibly still in flight into
            // its shared memory: the latched status is then the only signal, and
            // the CTA's output tile is not written.
            long long start = 0;
            int bounds = 0;
            for (uint32_t it = 0; !mbar_try_wait(bar, phase); ++it) {
                if ((it & 15u) == 15u) {
                    const long long now = clock64();
                    if (start == 0) {
                        start = now;
                    } else if (now - start > kQuantTimeoutCycles) {
                        if (bounds++ == 0) atomicCAS(&g_quant_status, 0, W4A16_ERR_TIMEOUT);
                        if (bounds == 2) break;
                        start = now;
                    }
                }
            }
            *stop = bounds;
        }
        __syncthreads();
        if (*stop) return;  // the same decision in every thread
        mbar_try_wait(bar, phase);  // (completed: each thread observes the phase the copy completed)
        // This slice's rows [r0, r1): an even count per slice keeps row pairs whole.
        const int64_t per = ((nrows + kSlices - 1) / kSlices + 1) & ~int64_t(1);
        const int64_t r0 = slice * per < nrows ? slice * per : nrows;
        const int64_t r1 = r0 + per < nrows ? r0 + per : nrows;
        // The slice's maxima of |w| in fp16 (exact: no rounding in abs or max).
        __half2 amax = __float2half2_rn(0.0f);
        for (int r = static_cast<int>(r0); r < static_cast<int>(r1); ++r)
            amax = __hmax2(amax, __habs2(tile[r * kQuantThreads + t]));
        float a0 = __low2float(amax), a1 = __high2float(amax);
        part[slice * kQuantThreads + t] = make_float2(a0, a1);
        __syncthreads();
#pragma unroll
        for (int q = 0; q < kSlices; ++q) {  // the group's maximum (the same in every slice)
            const float2 m = part[q * kQuantThreads + t];
            a0 = fmaxf(a0, m.x);
            a1 = fmaxf(a1, m.y);
        }
        if (c < N2) {
            __half2 scratch;
            uint16_t* out = wp + (BITS == 4 ? ((k0 + r0) >> 1) : (k0 + r0)) * N2 + c;
            quantize_pair<BITS>([&](int64_t r) { return tile[(r0 + r) * kQuantThreads + t]; }, r1 - r0, out, N2,
                                slice == 0 ? S + g * N2 + c : &scratch, a0, a1);
        }
        __syncthreads();  // every thread is done with the tile and the partial maxima before they are reused
    }
}

// Fallback: the group's rows read twice from global memory (maximum, then codes).
template <int BITS>
__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(const __half2* __restrict__ W,
                                                                  uint16_t* __restrict__ wp,
                                                                  __half2* __restrict__ S, int64_t K,
                                                                  int64_t N, int64_t G, int64_t groups) {
    const int64_t N2 = N / 2;  // column pairs
    const int64_t c = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x;
    if (c >= N2) return;
    for (int64_t g = blockIdx.y; g < groups; g += gridDim.y) {
        const int64_t k0 = g * G;
        const int64_t nrows = (k0 + G < K ? k0 + G : K) - k0;
        float a0 = 0.0f, a1 = 0.0f;
        for (int64_t r = 0; r < nrows; ++r) {
            const float2 v = __half22float2(W[(k0 + r) * N2 + c]);
            a0 = fmaxf(a0, fabsf(v.x));
            a1 = fmaxf(a1, fabsf(v.y));
        }
        quantize_pair<BITS>([&](int64_t r) { return W[(k0 + r) * N2 + c]; }, nrows,
                            wp + (BITS == 4 ? (k0 >> 1) : k0) * N2 + c, N2, S + g * N2 + c, a0, a1);
    }
}

}  // namespace

}  // namespace w4a16

using namespace w4a16;

namespace {

// Codes to out_dev (int4: canonical packed [ceil(K/2), N]; 8-bit: [K, N] int8),
// scales to S_dev [ceil(K/G), N].
template <int BITS>
int quantize_launch(const w4a16_half* W_dev, void* out_dev, w4a16_half* S_dev, int64_t K, int64_t N, int64_t G,
                    void* stream) {
    if (!W_dev || !out_dev || !S_dev || K <= 0 || N <= 0 || G <= 0) return W4A16_ERR_INVALID_ARG;
    if ((N & 1) || (G & 1) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(W_dev) & 3u) || (reinterpret_cast<uintptr_t>(S_dev) & 3u) ||
        (reinterpret_cast<uintptr_t>(out_dev) & 1u))
        return W4A16_ERR_MISALIGNED;
    int rc = check_device();
    if (rc) return rc;
    const int64_t groups = (K + G - 1) / G;
    const int64_t pairs = N / 2;
    const int64_t bx = (pairs + kQuantThreads - 1) / kQuantThreads;
    if (bx > 0x7FFFFFFF) return W4A16_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(groups < 65535 ? groups : 65535), 1);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool tma = G <= kMaxTmaGroup && (N % 8) == 0 && (reinterpret_cast<uintptr_t>(W_dev) & 15u) == 0;
    CUtensorMap map;
    if (tma && make_half_map_2d(&map, W_dev, static_cast<uint64_t>(N), static_cast<uint64_t>(K),
                                static_cast<uint64_t>(N) * 2, kTileCols, static_cast<uint32_t>(G)) == W4A16_OK) {
        static bool attr_done[64] = {};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return W4A16_ERR_CUDA;
        const size_t smem = 128 + kSlices * kQuantThreads * 8 + static_cast<size_t>(kMaxTmaGroup) * kTileCols * 2;
        if (!attr_done[dev]) {
            if (cudaFuncSetAttribute(reinterpret_cast<const void*>(quantize_tma_kernel<BITS>),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
                cudaSuccess)
                return W4A16_ERR_CUDA;
            attr_done[dev] = true;
        }
        quantize_tma_kernel<BITS><<<grid, kQuantThreads * kSlices,
                                    128 + kSlices * kQuantThreads * 8 + static_cast<size_t>(G) * kTileCols * 2, st>>>(
            map, reinterpret_cast<uint16_t*>(out_dev), reinterpret_cast<__half2*>(S_dev), K, N, G, groups);
    } else {
        quantize_kernel<BITS><<<grid, kQuantThreads, 0, st>>>(reinterpret_cast<const __half2*>(W_dev),
                                                              reinterpret_cast<uint16_t*>(out_dev),
                                                              reinterpret_cast<__half2*>(S_dev), K, N, G, groups);
    }
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

}  // namespace

extern "C" int w4a16_quantize(const w4a16_half* W_dev, uint8_t* wp_dev, w4a16_half* S_dev, int64_t K, int64_t N,
                              int64_t G, void* stream) {
    return quantize_launch<4>(W_dev, wp_dev, S_dev, K, N, G, stream);
}

extern "C" int w8a16_quantize(const w4a16_half* W_dev, int8_t* q8_dev, w4a16_half* S_dev, int64_t K, int64_t N,
                              int64_t G, void* stream) {
    return quantize_launch<8>(W_dev, q8_dev, S_dev, K, N, G, stream);
}

namespace w4a16 {

int quant_device_status(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_quant_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_quant_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

}  // namespace w4a16
