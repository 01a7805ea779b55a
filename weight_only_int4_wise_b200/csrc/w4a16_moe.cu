// The INT4 mixture-of-experts layer around the grouped W4A16 GEMM.
//
// Int4 Moe Plugin page (constructor parameters numExperts, topK, hiddenSize,
// moeInterSize, activationType, quantizationGroupSize; getWorkspaceSize and
// enqueue with a workspace). The page names the parameters only; the steps
// here are their plain reading:
//   route     one thread per token picks its topK experts by router logit
//             (ties to the lower index) and weights them by the softmax of the
//             selected logits (fp32);
//   dispatch  a stable counting sort of the (token, slot) pairs by expert:
//             every CTA counts the whole batch (so all CTAs agree on the expert
//             offsets and on whether the ids are valid), then ranks its own
//             128 tokens with one warp ballot per expert;
//   gather    the tokens' rows copied into expert order, 16 bytes per thread;
//   up/down   the grouped tensor-core GEMM (w4a16_gemm.cu), the up projection
//             with the activation in its epilogue;
//   combine   one pass over the down projection's rows, fp32 weighted sum in
//             slot order, one rounding to fp16.
// Every kernel is launched with programmatic dependent launch and waits for
// its predecessor before it reads that predecessor's output.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/w4a16.h"
#include "ptx.cuh"
#include "w4a16_internal.h"

namespace w4a16 {

__device__ int g_moe_status;  // latched device-side error of the expert-layer kernels (0 = none)

__device__ __forceinline__ void moe_latch(int code) { atomicCAS(&g_moe_status, 0, code); }

constexpr int kTokBlock = 128;    // tokens per route / dispatch CTA
constexpr int kCopyThreads = 256;  // threads per gather / combine CTA

// ------------------------------------------------------------------ route
__global__ void __launch_bounds__(kTokBlock) moe_route_kernel(const __half* __restrict__ logits,
                                                              int32_t* __restrict__ ids,
                                                              float* __restrict__ weights, int T, int E, int k) {
    extern __shared__ __half slog[];  // the block's logits [kTokBlock][E]
    grid_dependency_wait();           // the logits may come from the previous kernel
    grid_launch_dependents();
    const int t0 = blockIdx.x * kTokBlock;
    const int nt = min(kTokBlock, T - t0);
    const __half* src = logits + static_cast<int64_t>(t0) * E;
    for (int i = threadIdx.x; i < nt * E; i += kTokBlock) slog[i] = src[i];
    __syncthreads();
    if (static_cast<int>(threadIdx.x) >= nt) return;
    const __half* row = slog + threadIdx.x * E;
    uint64_t taken = 0;
    float sel[W4A16_MAX_TOPK];
    int sid[W4A16_MAX_TOPK];
#pragma unroll
    for (int j = 0; j < W4A16_MAX_TOPK; ++j) {
        sel[j] = 0.f;
        sid[j] = 0;
        if (j < k) {
            // the largest remaining logit; a strict comparison in ascending
            // expert order keeps the lower index on ties
            int bi = -1;
            float best = 0.f;
            for (int e = 0; e < E; ++e) {
                if ((taken >> e) & 1ull) continue;
                const float v = __half2float(row[e]);
                if (bi < 0 || v > best) {
                    bi = e;
                    best = v;
                }
            }
            taken |= 1ull << bi;
            sel[j] = best;
            sid[j] = bi;
        }
    }
    // softmax over the selected logits; sel[0] is their maximum
    float ex[W4A16_MAX_TOPK];
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < W4A16_MAX_TOPK; ++j) {
        ex[j] = j < k ? expf(sel[j] - sel[0]) : 0.f;
        sum += ex[j];
    }
    const int64_t o = static_cast<int64_t>(t0 + threadIdx.x) * k;
#pragma unroll
    for (int j = 0; j < W4A16_MAX_TOPK; ++j) {
        if (j < k) {
            ids[o + j] = sid[j];
            weights[o + j] = ex[j] / sum;
        }
    }
}

// --------------------------------------------------------------- dispatch
__global__ void __launch_bounds__(kTokBlock) moe_dispatch_kernel(const int32_t* __restrict__ ids,
                                                                 int32_t* __restrict__ offsets,
                                                                 int32_t* __restrict__ pos,
                                                                 int32_t* __restrict__ src_row, int T, int E,
                                                                 int k) {
    constexpr int kWarps = kTokBlock / 32;
    __shared__ int tot[W4A16_MAX_EXPERTS];     // pairs per expert, whole batch
    __shared__ int before[W4A16_MAX_EXPERTS];  // pairs per expert in tokens before this block
    __shared__ int base[W4A16_MAX_EXPERTS];    // exclusive scan of tot
    __shared__ int wcnt[kWarps][W4A16_MAX_EXPERTS];
    __shared__ int bad;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    for (int e = tid; e < W4A16_MAX_EXPERTS; e += kTokBlock) {
        tot[e] = 0;
        before[e] = 0;
    }
    if (tid == 0) bad = 0;
    grid_dependency_wait();  // the ids may come from the previous kernel
    grid_launch_dependents();
    __syncthreads();
    const int t0 = blockIdx.x * kTokBlock;

    // Pass 1 over the whole batch, one token per lane: validity and the counts.
    // Lanes that hold the same expert add their count once (the lowest lane).
    int my_bad = 0;
    for (int tb = warp * 32; tb < T; tb += kTokBlock) {
        const int t = tb + lane;
        const bool in = t < T;
        const uint32_t early = __ballot_sync(0xffffffffu, in && t < t0);
        uint64_t seen = 0;
        for (int j = 0; j < k; ++j) {
            int e = in ? ids[static_cast<int64_t>(t) * k + j] : -1;
            if (in && (e < 0 || e >= E || ((seen >> e) & 1ull))) {
                my_bad = 1;
                e = -1;
            }
            if (e >= 0) seen |= 1ull << e;
            const uint32_t same = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && (same & ((1u << lane) - 1u)) == 0) {
                atomicAdd(&tot[e], __popc(same));
                const int nb = __popc(same & early);
                if (nb) atomicAdd(&before[e], nb);
            }
        }
    }
    if (my_bad) bad = 1;
    __syncthreads();
    const int nt = T > t0 ? min(kTokBlock, T - t0) : 0;
    if (bad) {
        // Nothing is routed: no rows for any expert, and every index marked invalid.
        if (blockIdx.x == 0) {
            for (int e = tid; e <= E; e += kTokBlock) offsets[e] = 0;
            if (tid == 0) moe_latch(W4A16_ERR_BAD_ROUTING);
        }
        for (int i = tid; i < nt * k; i += kTokBlock) {
            pos[static_cast<int64_t>(t0) * k + i] = -1;
            src_row[static_cast<int64_t>(t0) * k + i] = -1;
        }
        return;
    }
    if (tid == 0) {
        int acc = 0;
        for (int e = 0; e < E; ++e) {
            base[e] = acc;
            acc += tot[e];
        }
        if (blockIdx.x == 0) {
            for (int e = 0; e < E; ++e) offsets[e] = base[e];
            offsets[E] = acc;
        }
    }

    // Pass 2: the stable rank of each of this block's pairs among the pairs of
    // its expert. A token's experts are distinct, so the rank of (t, j) is the
    // number of earlier tokens that chose the same expert.
    const int t = t0 + tid;
    const bool valid = tid < nt;
    int my_e[W4A16_MAX_TOPK];
    int my_r[W4A16_MAX_TOPK];
    uint64_t mask = 0;
#pragma unroll
    for (int j = 0; j < W4A16_MAX_TOPK; ++j) {
        my_e[j] = -1;
        my_r[j] = 0;
        if (valid && j < k) {
            my_e[j] = ids[static_cast<int64_t>(t) * k + j];
            mask |= 1ull << my_e[j];
        }
    }
    const uint32_t lt = (1u << lane) - 1u;
    for (int e = 0; e < E; ++e) {
        const bool has = (mask >> e) & 1ull;
        const uint32_t b = __ballot_sync(0xffffffffu, has);
        if (lane == 0) wcnt[warp][e] = __popc(b);
        if (has) {
#pragma unroll
            for (int j = 0; j < W4A16_MAX_TOPK; ++j)
                if (my_e[j] == e) my_r[j] = __popc(b & lt);
        }
    }
    __syncthreads();
    if (valid) {
#pragma unroll
        for (int j = 0; j < W4A16_MAX_TOPK; ++j) {
            if (j < k) {
                const int e = my_e[j];
                int r = base[e] + before[e] + my_r[j];
                for (int w = 0; w < warp; ++w) r += wcnt[w][e];
                pos[static_cast<int64_t>(t) * k + j] = r;
                src_row[r] = t;
            }
        }
    }
}

// ----------------------------------------------------------------- gather
__global__ void __launch_bounds__(kCopyThreads) moe_gather_kernel(const __half* __restrict__ X,
                                                                  const int32_t* __restrict__ src_row,
                                                                  __half* __restrict__ Xg, int T, int rows,
                                                                  int H) {
    grid_dependency_wait();  // src_row (and X) may come from the previous kernels
    grid_launch_dependents();
    const int vpr = H / 8;  // 16-byte vectors per row
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const int s = src_row[r];
        const bool ok = s >= 0 && s < T;
        if (!ok && threadIdx.x == 0) moe_latch(W4A16_ERR_BAD_ROUTING);
        const uint4* src = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(ok ? s : 0) * H);
        uint4* dst = reinterpret_cast<uint4*>(Xg + static_cast<int64_t>(r) * H);
        for (int c = threadIdx.x; c < vpr; c += kCopyThreads) dst[c] = ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
    }
}

// ---------------------------------------------------------------- combine
__global__ void __launch_bounds__(kCopyThreads) moe_combine_kernel(const __half* __restrict__ Y,
                                                                   const float* __restrict__ weights,
                                                                   const int32_t* __restrict__ pos,
                                                                   __half* __restrict__ out, int T, int k, int H) {
    grid_dependency_wait();  // Y comes from the previous kernel
    grid_launch_dependents();
    const int vpr = H / 8;
    const int64_t rows = static_cast<int64_t>(T) * k;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        float w[W4A16_MAX_TOPK];
        int p[W4A16_MAX_TOPK];
        bool any_bad = false;
#pragma unroll
        for (int j = 0; j < W4A16_MAX_TOPK; ++j) {
            w[j] = 0.f;
            p[j] = -1;
            if (j < k) {
                w[j] = weights[static_cast<int64_t>(t) * k + j];
                p[j] = pos[static_cast<int64_t>(t) * k + j];
                if (p[j] < 0 || p[j] >= rows) {
                    any_bad = true;
                    p[j] = -1;
                }
            }
        }
        if (any_bad && threadIdx.x == 0) moe_latch(W4A16_ERR_BAD_ROUTING);
        for (int c = threadIdx.x; c < vpr; c += kCopyThreads) {
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
            for (int j = 0; j < W4A16_MAX_TOPK; ++j) {
                if (j < k && p[j] >= 0) {
                    const uint4 v = reinterpret_cast<const uint4*>(Y + static_cast<int64_t>(p[j]) * H)[c];
                    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __half22float2(h[e]);
                        acc[2 * e] = fmaf(w[j], f.x, acc[2 * e]);
                        acc[2 * e + 1] = fmaf(w[j], f.y, acc[2 * e + 1]);
                    }
                }
            }
            uint4 o;
            __half2* oh = reinterpret_cast<__half2*>(&o);
#pragma unroll
            for (int e = 0; e < 4; ++e) oh[e] = __floats2half2_rn(acc[2 * e], acc[2 * e + 1]);
            reinterpret_cast<uint4*>(out + static_cast<int64_t>(t) * H)[c] = o;
        }
    }
}

// ================================================================== host
namespace {

template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
               Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(block, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess ? W4A16_OK
                                                                                       : W4A16_ERR_CUDA;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_route_sizes(int64_t T, int64_t E, int64_t k) {
    if (T < 0 || E < 1 || E > W4A16_MAX_EXPERTS || k < 1 || k > E || k > W4A16_MAX_TOPK)
        return W4A16_ERR_INVALID_ARG;
    if (T * k >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    return W4A16_OK;
}

unsigned copy_grid(int64_t units) {
    const int64_t cap = static_cast<int64_t>(sm_count() > 0 ? sm_count() : 148) * 8;
    return static_cast<unsigned>(units < cap ? (units > 0 ? units : 1) : cap);
}

int64_t round256(int64_t b) { return (b + 255) & ~int64_t(255); }

struct MoeWorkspace {
    int32_t* ids;
    float* weights;
    int32_t* pos;
    int32_t* src_row;
    int32_t* offsets;
    __half* xg;
    __half* act;
    __half* y;
    int64_t bytes;
};

MoeWorkspace carve(void* base, int64_t T, int64_t E, int64_t k, int64_t H, int64_t I) {
    MoeWorkspace w{};
    uint8_t* p = static_cast<uint8_t*>(base);
    int64_t off = 0;
    auto take = [&](int64_t bytes) {
        uint8_t* q = p ? p + off : nullptr;
        off += round256(bytes);
        return q;
    };
    const int64_t pairs = T * k;
    w.ids = reinterpret_cast<int32_t*>(take(pairs * 4));
    w.weights = reinterpret_cast<float*>(take(pairs * 4));
    w.pos = reinterpret_cast<int32_t*>(take(pairs * 4));
    w.src_row = reinterpret_cast<int32_t*>(take(pairs * 4));
    w.offsets = reinterpret_cast<int32_t*>(take((E + 1) * 4));
    w.xg = reinterpret_cast<__half*>(take(pairs * H * 2));
    w.act = reinterpret_cast<__half*>(take(pairs * I * 2));
    w.y = reinterpret_cast<__half*>(take(pairs * H * 2));
    w.bytes = off;
    return w;
}

}  // namespace

int moe_device_status(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_moe_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_moe_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

int moe_route(const w4a16_half* logits, int32_t* ids, float* weights, int64_t T, int64_t E, int64_t k,
              cudaStream_t stream) {
    if (T == 0) return W4A16_OK;
    const unsigned grid = static_cast<unsigned>((T + kTokBlock - 1) / kTokBlock);
    const size_t smem = static_cast<size_t>(kTokBlock) * E * sizeof(__half);
    return launch_pdl(moe_route_kernel, grid, kTokBlock, smem, stream, reinterpret_cast<const __half*>(logits), ids,
                      weights, static_cast<int>(T), static_cast<int>(E), static_cast<int>(k));
}

int moe_dispatch(const int32_t* ids, int32_t* offsets, int32_t* pos, int32_t* src_row, int64_t T, int64_t E,
                 int64_t k, cudaStream_t stream) {
    const unsigned grid = static_cast<unsigned>(T > 0 ? (T + kTokBlock - 1) / kTokBlock : 1);
    return launch_pdl(moe_dispatch_kernel, grid, kTokBlock, 0, stream, ids, offsets, pos, src_row,
                      static_cast<int>(T), static_cast<int>(E), static_cast<int>(k));
}

int moe_gather(const w4a16_half* X, const int32_t* src_row, w4a16_half* Xg, int64_t T, int64_t rows, int64_t H,
               cudaStream_t stream) {
    if (rows == 0) return W4A16_OK;
    return launch_pdl(moe_gather_kernel, copy_grid(rows), kCopyThreads, 0, stream,
                      reinterpret_cast<const __half*>(X), src_row, reinterpret_cast<__half*>(Xg),
                      static_cast<int>(T), static_cast<int>(rows), static_cast<int>(H));
}

int moe_combine(const w4a16_half* Y, const float* weights, const int32_t* pos, w4a16_half* out, int64_t T,
                int64_t k, int64_t H, cudaStream_t stream) {
    if (T == 0) return W4A16_OK;
    return launch_pdl(moe_combine_kernel, copy_grid(T), kCopyThreads, 0, stream, reinterpret_cast<const __half*>(Y),
                      weights, pos, reinterpret_cast<__half*>(out), static_cast<int>(T), static_cast<int>(k),
                      static_cast<int>(H));
}

}  // namespace w4a16

using namespace w4a16;

extern "C" int w4a16_moe_route(const w4a16_half* logits_dev, int32_t* ids_dev, float* weights_dev, int64_t T,
                               int64_t E, int64_t top_k, void* stream) {
    if (!logits_dev || !ids_dev || !weights_dev) return W4A16_ERR_INVALID_ARG;
    int rc = check_route_sizes(T, E, top_k);
    if (rc) return rc;
    if (!aligned(logits_dev, 2) || !aligned(ids_dev, 4) || !aligned(weights_dev, 4)) return W4A16_ERR_MISALIGNED;
    if (T == 0) return W4A16_OK;
    rc = check_device();
    if (rc) return rc;
    return moe_route(logits_dev, ids_dev, weights_dev, T, E, top_k, static_cast<cudaStream_t>(stream));
}

extern "C" int w4a16_moe_dispatch(const int32_t* ids_dev, int32_t* offsets_dev, int32_t* pos_dev,
                                  int32_t* src_row_dev, int64_t T, int64_t E, int64_t top_k, void* stream) {
    if (!ids_dev || !offsets_dev || !pos_dev || !src_row_dev) return W4A16_ERR_INVALID_ARG;
    int rc = check_route_sizes(T, E, top_k);
    if (rc) return rc;
    if (!aligned(ids_dev, 4) || !aligned(offsets_dev, 4) || !aligned(pos_dev, 4) || !aligned(src_row_dev, 4))
        return W4A16_ERR_MISALIGNED;
    rc = check_device();
    if (rc) return rc;
    return moe_dispatch(ids_dev, offsets_dev, pos_dev, src_row_dev, T, E, top_k, static_cast<cudaStream_t>(stream));
}

extern "C" int w4a16_moe_gather(const w4a16_half* X_dev, const int32_t* src_row_dev, w4a16_half* Xg_dev,
                                int64_t T, int64_t rows, int64_t H, void* stream) {
    if (!X_dev || !src_row_dev || !Xg_dev || T < 0 || rows < 0 || H <= 0) return W4A16_ERR_INVALID_ARG;
    if (H % 8 || T >= (int64_t(1) << 31) || rows >= (int64_t(1) << 31) || H >= (int64_t(1) << 31))
        return W4A16_ERR_UNSUPPORTED;
    if (!aligned(X_dev, 16) || !aligned(Xg_dev, 16) || !aligned(src_row_dev, 4)) return W4A16_ERR_MISALIGNED;
    if (rows == 0) return W4A16_OK;
    int rc = check_device();
    if (rc) return rc;
    return moe_gather(X_dev, src_row_dev, Xg_dev, T, rows, H, static_cast<cudaStream_t>(stream));
}

extern "C" int w4a16_moe_combine(const w4a16_half* Y_dev, const float* weights_dev, const int32_t* pos_dev,
                                 w4a16_half* out_dev, int64_t T, int64_t top_k, int64_t H, void* stream) {
    if (!Y_dev || !weights_dev || !pos_dev || !out_dev || T < 0 || top_k < 1 || top_k > W4A16_MAX_TOPK || H <= 0)
        return W4A16_ERR_INVALID_ARG;
    if (H % 8 || T * top_k >= (int64_t(1) << 31) || H >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    if (!aligned(Y_dev, 16) || !aligned(out_dev, 16) || !aligned(weights_dev, 4) || !aligned(pos_dev, 4))
        return W4A16_ERR_MISALIGNED;
    if (T == 0) return W4A16_OK;
    int rc = check_device();
    if (rc) return rc;
    return moe_combine(Y_dev, weights_dev, pos_dev, out_dev, T, top_k, H, static_cast<cudaStream_t>(stream));
}

extern "C" int64_t w4a16_moe_workspace_size(int64_t T, int64_t E, int64_t top_k, int64_t H, int64_t I) {
    if (check_route_sizes(T, E, top_k) != W4A16_OK || H <= 0 || I <= 0) return -1;
    return carve(nullptr, T, E, top_k, H, I).bytes;
}

extern "C" int w4a16_moe_layer(const w4a16_half* X_dev, const w4a16_half* logits_dev, const uint8_t* const* Wt_up,
                               const w4a16_half* const* S_up, const uint8_t* const* Wt_down,
                               const w4a16_half* const* S_down, w4a16_half* out_dev, int64_t T, int64_t E,
                               int64_t top_k, int64_t H, int64_t I, int64_t G, int act, void* workspace_dev,
                               int64_t workspace_bytes, void* stream) {
    if (!X_dev || !logits_dev || !Wt_up || !S_up || !Wt_down || !S_down || !out_dev || !workspace_dev)
        return W4A16_ERR_INVALID_ARG;
    int rc = check_route_sizes(T, E, top_k);
    if (rc) return rc;
    if (H <= 0 || I <= 0 || G <= 0) return W4A16_ERR_INVALID_ARG;
    if (act < W4A16_ACT_IDENTITY || act > W4A16_ACT_GELU_TANH) return W4A16_ERR_INVALID_ARG;
    if (H % 8 || I % 8 || G % 16) return W4A16_ERR_UNSUPPORTED;
    const int64_t need = w4a16_moe_workspace_size(T, E, top_k, H, I);
    if (need < 0 || workspace_bytes < need) return W4A16_ERR_INVALID_ARG;
    for (int64_t e = 0; e < E; ++e)
        if (!Wt_up[e] || !S_up[e] || !Wt_down[e] || !S_down[e]) return W4A16_ERR_INVALID_ARG;
    if (!aligned(X_dev, 16) || !aligned(out_dev, 16) || !aligned(logits_dev, 2) || !aligned(workspace_dev, 16))
        return W4A16_ERR_MISALIGNED;
    if (T == 0) return W4A16_OK;
    rc = check_device();
    if (rc) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const MoeWorkspace w = carve(workspace_dev, T, E, top_k, H, I);
    const int64_t rows = T * top_k;
    if ((rc = moe_route(logits_dev, w.ids, w.weights, T, E, top_k, s))) return rc;
    if ((rc = moe_dispatch(w.ids, w.offsets, w.pos, w.src_row, T, E, top_k, s))) return rc;
    if ((rc = moe_gather(X_dev, w.src_row, reinterpret_cast<w4a16_half*>(w.xg), T, rows, H, s))) return rc;
    if ((rc = grouped_gemm_act(reinterpret_cast<const w4a16_half*>(w.xg), Wt_up, S_up, w.offsets,
                               reinterpret_cast<w4a16_half*>(w.act), E, rows, I, H, G, act, s)))
        return rc;
    if ((rc = grouped_gemm_act(reinterpret_cast<const w4a16_half*>(w.act), Wt_down, S_down, w.offsets,
                               reinterpret_cast<w4a16_half*>(w.y), E, rows, H, I, G, W4A16_ACT_IDENTITY, s)))
        return rc;
    return moe_combine(reinterpret_cast<const w4a16_half*>(w.y), w.weights, w.pos, out_dev, T, top_k, H, s);
}

// ------------------------------------------------- no-allocation entry point
// Some callers cannot hand the layer a workspace: an engine whose execute step
// was promised a zero-byte workspace at build time, or C code that owns no
// device memory pool. A cudaMalloc inside the call is no way out for them:
// it synchronizes the device and can fail under memory pressure in the middle
// of a step. w4a16_moe_layer_static therefore runs the same six steps in a
// fixed region of device memory that belongs to this library (one per device,
// created with the module), sized for decode-scale batches.
namespace w4a16 {
namespace {

constexpr int64_t kStaticScratchBytes = int64_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) uint8_t g_moe_scratch[kStaticScratchBytes];

// Device address of g_moe_scratch, looked up once per device with that device
// current; nullptr if the lookup failed.
void* static_scratch() {
    static std::mutex mu;
    static void* ptr[64] = {};
    static bool done[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_moe_scratch) != cudaSuccess) return nullptr;
        ptr[dev] = p;
        done[dev] = true;
    }
    return ptr[dev];
}

}  // namespace
}  // namespace w4a16

extern "C" int64_t w4a16_moe_static_scratch_bytes(void) { return w4a16::kStaticScratchBytes; }

extern "C" int w4a16_moe_layer_static(const w4a16_half* X_dev, const w4a16_half* logits_dev,
                                      const uint8_t* const* Wt_up, const w4a16_half* const* S_up,
                                      const uint8_t* const* Wt_down, const w4a16_half* const* S_down,
                                      w4a16_half* out_dev, int64_t T, int64_t E, int64_t top_k, int64_t H,
                                      int64_t I, int64_t G, int act, void* stream) {
    const int64_t need = w4a16_moe_workspace_size(T, E, top_k, H, I);
    if (need < 0) return W4A16_ERR_INVALID_ARG;
    if (need > w4a16::kStaticScratchBytes) return W4A16_ERR_SCRATCH_TOO_SMALL;
    if (T == 0) return w4a16_moe_layer(X_dev, logits_dev, Wt_up, S_up, Wt_down, S_down, out_dev, T, E, top_k, H,
                                       I, G, act, reinterpret_cast<void*>(uintptr_t(256)), need, stream);
    if (check_device() != W4A16_OK) return W4A16_ERR_UNSUPPORTED;
    void* scratch = w4a16::static_scratch();
    if (!scratch) return W4A16_ERR_CUDA;
    return w4a16_moe_layer(X_dev, logits_dev, Wt_up, S_up, Wt_down, S_down, out_dev, T, E, top_k, H, I, G, act,
                           scratch, w4a16::kStaticScratchBytes, stream);
}
