// Weight packing kernels: int8 codes -> canonical packed int4, its inverse, and
// the one-off repack from the canonical layout into the tiled layout the GEMM
// kernels stream. Layout definitions are in include/w4a16.h.
//
// These are setup kernels (run once per weight matrix, outside the timed GEMM),
// so they favour simple, fully coalesced writes over peak bandwidth.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/w4a16.h"
#include "w4a16_internal.h"

namespace w4a16 {

// One thread per packed byte (j, n): q[2j, n] in the low nibble, q[2j+1, n]
// in the high nibble (Int4GroupwiseGemmPluginV2 page: K rows x N columns,
// two int4 codes per byte; low nibble = even row).
__global__ void pack_kernel(const int8_t* __restrict__ q, uint8_t* __restrict__ wp, int64_t K, int64_t N) {
    const int64_t rows = (K + 1) / 2;
    const int64_t total = rows * N;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = i / N, n = i - j * N;
        const uint32_t lo = static_cast<uint8_t>(q[(2 * j) * N + n]) & 0xFu;
        const uint32_t hi = (2 * j + 1 < K) ? (static_cast<uint8_t>(q[(2 * j + 1) * N + n]) & 0xFu) : 0u;
        wp[i] = static_cast<uint8_t>(lo | (hi << 4));
    }
}

__global__ void unpack_kernel(const uint8_t* __restrict__ wp, int8_t* __restrict__ q, int64_t K, int64_t N) {
    const int64_t total = K * N;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t k = i / N, n = i - k * N;
        const uint32_t b = wp[(k >> 1) * N + n];
        const int32_t v = static_cast<int32_t>((k & 1) ? (b >> 4) : (b & 0xFu));
        q[i] = static_cast<int8_t>(v >= 8 ? v - 16 : v);
    }
}

// One thread per 32-bit word of the tiled layout. Word (tile, h, j, w) gathers
// the eight codes k_local = 32h + 8w + {0,2,4,6,1,3,5,7} of column j, so that
// the GEMM's nibble decoder yields (k, k+1) pairs in natural order.
__global__ void repack_kernel(const uint8_t* __restrict__ wp, uint32_t* __restrict__ wt, int64_t K, int64_t N,
                              int64_t KT, int64_t total_words) {
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total_words;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tile = idx >> 10;       // 1024 words per 4096-byte tile
        const int32_t r = static_cast<int32_t>(idx & 1023);
        const int32_t h = r >> 9;             // 512 words per 32-row half
        const int32_t j = (r >> 2) & 127;     // column inside the tile
        const int32_t w = r & 3;              // word inside the column's 16 bytes
        const int64_t nt = tile / KT, kt = tile - nt * KT;
        const int64_t n = nt * 128 + j;
        const int64_t kbase = kt * 64 + 32 * h + 8 * w;
        uint32_t word = 0;
        if (n < N) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t k = kbase + ((i < 4) ? 2 * i : 2 * (i - 4) + 1);
                if (k < K) {
                    const uint32_t b = wp[(k >> 1) * N + n];
                    const uint32_t code = (k & 1) ? (b >> 4) : (b & 0xFu);
                    word |= code << (4 * i);
                }
            }
        }
        wt[idx] = word;
    }
}

// One thread per 16-byte chunk of the 8-bit tiled layout: chunk (tile, h, j)
// holds the codes k_local = 16h .. 16h+15 of column j, byte b = k_local 16h + b.
__global__ void repack8_kernel(const int8_t* __restrict__ q, uint4* __restrict__ wt, int64_t K, int64_t N,
                               int64_t KT, int64_t total_chunks) {
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total_chunks;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tile = idx >> 9;        // 512 chunks per 8192-byte tile
        const int32_t r = static_cast<int32_t>(idx & 511);
        const int32_t h = r >> 7;             // 128 chunks per 16-row quarter
        const int32_t j = r & 127;            // column inside the tile
        const int64_t nt = tile / KT, kt = tile - nt * KT;
        const int64_t n = nt * 128 + j;
        const int64_t kbase = kt * 64 + 16 * h;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if (n < N) {
#pragma unroll
            for (int b = 0; b < 16; ++b) {
                const int64_t k = kbase + b;
                if (k < K) w[b >> 2] |= static_cast<uint32_t>(static_cast<uint8_t>(q[k * N + n])) << (8 * (b & 3));
            }
        }
        wt[idx] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

static int grid_for(int64_t work) {
    int64_t blocks = (work + 255) / 256;
    if (blocks > 148 * 32) blocks = 148 * 32;
    if (blocks < 1) blocks = 1;
    return static_cast<int>(blocks);
}

}  // namespace w4a16

using namespace w4a16;

extern "C" int w4a16_pack(const int8_t* q_dev, uint8_t* wp_dev, int64_t K, int64_t N, void* stream) {
    if (!q_dev || !wp_dev || K <= 0 || N <= 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc) return rc;
    const int64_t total = ((K + 1) / 2) * N;
    pack_kernel<<<grid_for(total), 256, 0, static_cast<cudaStream_t>(stream)>>>(q_dev, wp_dev, K, N);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

extern "C" int w4a16_unpack(const uint8_t* wp_dev, int8_t* q_dev, int64_t K, int64_t N, void* stream) {
    if (!q_dev || !wp_dev || K <= 0 || N <= 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc) return rc;
    unpack_kernel<<<grid_for(K * N), 256, 0, static_cast<cudaStream_t>(stream)>>>(wp_dev, q_dev, K, N);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

extern "C" int64_t w4a16_tiled_bytes(int64_t K, int64_t N) {
    if (K <= 0 || N <= 0) return 0;
    return ((N + 127) / 128) * ((K + 63) / 64) * 4096;
}

extern "C" int w4a16_repack(const uint8_t* wp_dev, uint8_t* wt_dev, int64_t K, int64_t N, void* stream) {
    if (!wp_dev || !wt_dev || K <= 0 || N <= 0) return W4A16_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(wt_dev) & 15) return W4A16_ERR_MISALIGNED;
    int rc = check_device();
    if (rc) return rc;
    const int64_t KT = (K + 63) / 64;
    const int64_t words = w4a16_tiled_bytes(K, N) / 4;
    repack_kernel<<<grid_for(words), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        wp_dev, reinterpret_cast<uint32_t*>(wt_dev), K, N, KT, words);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

extern "C" int64_t w8a16_tiled_bytes(int64_t K, int64_t N) {
    if (K <= 0 || N <= 0) return 0;
    return ((N + 127) / 128) * ((K + 63) / 64) * 8192;
}

extern "C" int w8a16_repack(const int8_t* q_dev, uint8_t* wt_dev, int64_t K, int64_t N, void* stream) {
    if (!q_dev || !wt_dev || K <= 0 || N <= 0) return W4A16_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(wt_dev) & 15) return W4A16_ERR_MISALIGNED;
    int rc = check_device();
    if (rc) return rc;
    const int64_t KT = (K + 63) / 64;
    const int64_t chunks = w8a16_tiled_bytes(K, N) / 16;
    repack8_kernel<<<grid_for(chunks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        q_dev, reinterpret_cast<uint4*>(wt_dev), K, N, KT, chunks);
    return cudaGetLastError() == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}
