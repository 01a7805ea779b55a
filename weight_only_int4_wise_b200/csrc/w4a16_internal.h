// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/w4a16.h"

namespace w4a16 {

// W4A16_OK if the current device is an sm_100 part this library was built for,
// W4A16_ERR_UNSUPPORTED otherwise (including "no CUDA device").
int check_device();

// Streaming multiprocessors of the current device (0 if unknown).
int sm_count();

// Whether the caller declared weights and scales static (w4a16_set_static_weights).
bool static_weights_enabled();

// A tiled tensor map over fp16 elements [outer, inner] (row stride in bytes),
// box [box_outer, box_inner], no swizzle, zero fill outside the tensor.
// W4A16_OK, or W4A16_ERR_CUDA if the driver's encoder is missing or refuses.
int make_half_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                     uint32_t box_inner, uint32_t box_outer);

// A tiled tensor map over activations A [rows, K] fp16 with a {64, box_rows}
// box, the 128-byte swizzle and zero fill past the tensor, as the tensor-core
// kernels stage them. Encoded maps are kept in a small per-thread cache keyed
// by (device, address, rows, K, box_rows), so repeated calls on the same
// buffers skip the encoder.
int activation_map(CUtensorMap* map, const void* A, int64_t rows, int64_t K, int box_rows);

// The grouped-expert GEMM with an activation epilogue (w4a16_grouped_gemm_act).
int grouped_gemm_act(const w4a16_half* A_dev, const uint8_t* const* Wt, const w4a16_half* const* S,
                     const int32_t* offsets_dev, w4a16_half* C_dev, int64_t E, int64_t total_rows, int64_t N,
                     int64_t K, int64_t G, int act, cudaStream_t stream);

// The expert-layer kernels' latched device status (0 = none, -1 if it could not be read).
int moe_device_status(bool clear);

// The quantiser kernel's latched device status (0 = none, -1 if it could not be read).
int quant_device_status(bool clear);

// Decode-sized products (M <= kSkinnyMaxM) run on the skinny kernel.
constexpr int kSkinnyMaxM = 16;

struct SkinnyPlan {
    int mt;             // token tiles of 8 rows (1 or 2)
    int threads;        // threads per CTA (256 per K half)
    int splits;         // CTAs along K in one cluster
    int depth;          // 128-deep K blocks in flight per thread (2 to 8)
    int grid_x, grid_y;
    int act_stride;     // staged activation row, in halves
    int scale_rows;     // staged scale rows
    int smem;           // dynamic shared memory per CTA
    uint32_t g_magic;   // multiply-shift constant for floor(k / G)
    int post_scale;     // 1 when every 128-deep K block lies in one scale group
};

// W4A16_OK and a plan, or W4A16_ERR_UNSUPPORTED if the shape needs the general kernel.
int skinny_plan(int64_t M, int64_t N, int64_t K, int64_t G, SkinnyPlan* plan);

// The skinny plan for a given K split (1..8 CTAs per cluster), K halves per CTA
// (1 or 2; 2 only for one token tile) and ring depth (deep = 0: four blocks in
// flight per CTA, 1: eight). W4A16_ERR_UNSUPPORTED when that form does not
// exist for the shape (more splits than 128-deep K blocks, shared memory).
int skinny_plan_fill(int64_t M, int64_t N, int64_t K, int64_t G, int splits, int kh, int deep, SkinnyPlan* plan);

// The skinny kernel's latched device status (0 = none, -1 if it could not be read).
int skinny_device_status(bool clear);

int skinny_launch(const SkinnyPlan& plan, const void* A, const uint8_t* Wt, const void* S, void* C, int64_t M,
                  int64_t N, int64_t K, int64_t G, cudaStream_t stream);

// The skinny plan of the grouped form: the smallest K split whose staged
// activations fit (the experts' column tiles already fill the grid).
int skinny_plan_grouped(int64_t total_rows, int64_t N, int64_t K, int64_t G, SkinnyPlan* plan);

// Grouped-expert form of the skinny kernel (grid z = expert) for at most 16
// gathered rows in total (plan from skinny_plan_grouped): rows
// [off[e], off[e+1]) of A and C use Wt[e] and S[e] (host arrays of E device
// pointers); the activation act (W4A16_ACT_*) applies to the fp16 result.
// Malformed offsets (or a segment longer than the plan's token tiles) latch
// W4A16_ERR_BAD_OFFSETS in the skinny status word and write nothing.
int skinny_grouped_launch(const SkinnyPlan& plan, const void* A, const uint8_t* const* Wt, const void* const* S,
                          const int32_t* offsets, void* C, int64_t E, int64_t total_rows, int64_t N, int64_t K,
                          int64_t G, int act, cudaStream_t stream);

}  // namespace w4a16
