// Skinny W4A16 GEMM for decode-sized M (1..16): C[M,N] = A[M,K] x dequant(W).
//
// The operation is the Int4GroupwiseGemmPluginV2 page's (class description:
// activations, int4 weights, scales [ceil(K/G),N], fp16 output). At M <= 16 the
// product is bound by streaming the int4 weights from HBM (K*N/2 bytes), so
// this kernel keeps every hop between HBM and the tensor core inside one
// thread:
//   - each thread streams its own two 16-byte int4 chunks per 128-deep K block
//     with cp.async (a ring of kDepth blocks in flight per thread, no barrier
//     between warps);
//   - it decodes them straight into the A fragment of a warp-level
//     m16n8k16 MMA with the weights as the 16-row operand (16 output columns)
//     and the tokens as the 8-column operand (one or two token tiles);
//   - activations and scale rows for the CTA's K range are staged once in
//     shared memory;
//   - K is split over up to 8 CTAs of a thread-block cluster whose fp32 partial
//     tiles are summed in rank order through distributed shared memory.
//
// Fragment mapping. Inside a 16-deep MMA step the k order is free as long as
// both operands use it. Thread (g = lane/4, t = lane%4) holds, for output
// column g (and g + 8), the 32 codes of chunk t of the block, i.e. block
// k in [32t, 32t + 32). Step s (0..7) takes k = 32t + 4s + {0,1} for the
// fragment's first register pair and 32t + 4s + {2,3} for the second, and the
// activation fragment of token g is read from the same four k.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/w4a16.h"
#include "dequant.cuh"
#include "ptx.cuh"
#include "w4a16_internal.h"

namespace w4a16 {

namespace {

constexpr int kSkWarps = 8;                 // 8 warps x 16 columns = one 128-column weight tile
constexpr int kSkThreads = kSkWarps * 32;
constexpr int kDepth = 4;                   // 128-deep K blocks in flight per thread
constexpr int kBlockK = 128;
constexpr int kWbufBytes = kSkWarps * kDepth * 32 * 32;  // per thread: 2 x 16 bytes per block

struct SkinnyParams {
    const uint8_t* wt;      // tiled weights
    const __half* sc;       // scales [ngroups, N]
    const __half* A;        // activations [M, K]
    __half* C;              // output [M, N]
    int32_t M, N, K, G;
    int32_t ngroups, KT, KB;  // groups, 64-deep tiles, 128-deep blocks
    int32_t splits;
    int32_t act_stride;       // halves per staged activation row (max K range + 8)
    int32_t scale_rows;       // rows of the staged scale window
    uint32_t g_magic;         // floor(k / G) == (k * g_magic) >> 32 for every k < K padded
    int32_t post_scale;       // G % 128 == 0: scale fp32 partials once per block
};

template <int MT>
__global__ void __launch_bounds__(kSkThreads, 2) w4a16_skinny_kernel(const __grid_constant__ SkinnyParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int split = blockIdx.x, nt = blockIdx.y;
    const int b0 = static_cast<int>((static_cast<int64_t>(split) * p.KB) / p.splits);
    const int b1 = static_cast<int>((static_cast<int64_t>(split + 1) * p.KB) / p.splits);
    const int nb = b1 - b0;
    const int kr0 = b0 * kBlockK;                   // first k of this CTA
    const int krange = nb * kBlockK;
    constexpr int MP = 8 * MT;                      // token rows, padded to the MMA's 8-column tiles

    __half* act = reinterpret_cast<__half*>(sm);                                     // [MP][act_stride]
    __half* scl = act + MP * p.act_stride;                                           // [scale_rows][128]
    uint8_t* wbuf = reinterpret_cast<uint8_t*>(scl + p.scale_rows * 128);            // per-thread ring
    float* red = reinterpret_cast<float*>(wbuf);                                     // split-K partials

    // ---- stage activations (zero past M and K) and the scale rows of this K range
    const int g_lo = kr0 / p.G;
    const int g_hi = min(p.ngroups - 1, (kr0 + krange - 1) / p.G);
    const int nrows = g_hi - g_lo + 1;
    {
        const int cpr = krange / 8;  // 16-byte chunks per activation row
        for (int idx = threadIdx.x; idx < MP * cpr; idx += kSkThreads) {
            const int r = idx / cpr, c = idx - r * cpr;
            const int k = kr0 + c * 8;
            const bool ok = r < p.M && k < p.K;
            cp_async16(act + r * p.act_stride + c * 8, ok ? p.A + static_cast<int64_t>(r) * p.K + k : p.A, ok ? 16u : 0u);
        }
        const int ncols = min(128, p.N - nt * 128);
        for (int idx = threadIdx.x; idx < nrows * 16; idx += kSkThreads) {
            const int r = idx >> 4, c = idx & 15;
            const bool ok = c * 8 < ncols;
            cp_async16(scl + r * 128 + c * 8,
                       ok ? p.sc + static_cast<int64_t>(g_lo + r) * p.N + nt * 128 + c * 8 : p.sc, ok ? 16u : 0u);
        }
        cp_async_commit();
    }

    // ---- this thread's weight chunks: columns ja, ja + 8 of the tile, chunk t of each block
    const int ja = warp * 16 + g;
    const uint8_t* wtile = p.wt + static_cast<int64_t>(nt) * p.KT * 4096 + (t & 1) * 2048 + ja * 16;
    uint8_t* myslot = wbuf + (warp * kDepth * 32 + lane) * 32;  // + (block % kDepth) * 32 * 32
    auto issue_block = [&](int i) {
        if (i < nb) {
            const int kt = 2 * (b0 + i) + (t >> 1);
            const bool ok = kt < p.KT;
            const uint8_t* src = wtile + static_cast<int64_t>(kt) * 4096;
            uint8_t* dst = myslot + (i % kDepth) * 32 * 32;
            cp_async16(dst, ok ? src : p.wt, ok ? 16u : 0u);
            cp_async16(dst + 16, ok ? src + 128 : p.wt, ok ? 16u : 0u);
        }
        cp_async_commit();  // one group per block, empty past the end, so the counts stay uniform
    };
#pragma unroll
    for (int i = 0; i < kDepth; ++i) issue_block(i);
    cp_async_wait<kDepth>();  // activations and scales have landed
    __syncthreads();

    float acc[MT][4];
#pragma unroll
    for (int j = 0; j < MT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

    const __half* arow[MT];
#pragma unroll
    for (int j = 0; j < MT; ++j) arow[j] = act + (8 * j + g) * p.act_stride + 32 * t;

    for (int i = 0; i < nb; ++i) {
        cp_async_wait<kDepth - 1>();  // block i is in this thread's slot
        const uint8_t* slot = myslot + (i % kDepth) * 32 * 32;
        const uint4 wa = *reinterpret_cast<const uint4*>(slot);
        const uint4 wb = *reinterpret_cast<const uint4*>(slot + 16);
        const int kb = i * kBlockK;  // block offset inside the staged K range
        const uint32_t wa_w[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t wb_w[4] = {wb.x, wb.y, wb.z, wb.w};

        if (p.post_scale) {
            // One group covers the whole block: accumulate the exact codes, scale once.
            float part[MT][4];
#pragma unroll
            for (int j = 0; j < MT; ++j) part[j][0] = part[j][1] = part[j][2] = part[j][3] = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint4 qa = decode_word(wa_w[w]);
                const uint4 qb = decode_word(wb_w[w]);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t afr[4] = {u ? qa.z : qa.x, u ? qb.z : qb.x, u ? qa.w : qa.y, u ? qb.w : qb.y};
                    const int s = 2 * w + u;
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint2 bfr = *reinterpret_cast<const uint2*>(arow[j] + kb + 4 * s);
                        mma_m16n8k16(part[j], afr, bfr.x, bfr.y);
                    }
                }
            }
            const int gr = (kr0 + kb) / p.G - g_lo;
            const float sa = __half2float(scl[gr * 128 + ja]);
            const float sb = __half2float(scl[gr * 128 + ja + 8]);
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                acc[j][0] = fmaf(part[j][0], sa, acc[j][0]);
                acc[j][1] = fmaf(part[j][1], sa, acc[j][1]);
                acc[j][2] = fmaf(part[j][2], sb, acc[j][2]);
                acc[j][3] = fmaf(part[j][3], sb, acc[j][3]);
            }
        } else {
            // Groups finer than the block: scale each decoded word (rounded to fp16).
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t kk = static_cast<uint32_t>(kr0 + kb + 32 * t + 8 * w);
                const int gr = min(static_cast<int>((static_cast<uint64_t>(kk) * p.g_magic) >> 32), p.ngroups - 1) - g_lo;
                const uint4 qa = dequant_word(wa_w[w], __half2half2(scl[gr * 128 + ja]));
                const uint4 qb = dequant_word(wb_w[w], __half2half2(scl[gr * 128 + ja + 8]));
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t afr[4] = {u ? qa.z : qa.x, u ? qb.z : qb.x, u ? qa.w : qa.y, u ? qb.w : qb.y};
                    const int s = 2 * w + u;
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint2 bfr = *reinterpret_cast<const uint2*>(arow[j] + kb + 4 * s);
                        mma_m16n8k16(acc[j], afr, bfr.x, bfr.y);
                    }
                }
            }
        }
        issue_block(i + kDepth);  // this slot's contents are consumed
    }
    cp_async_wait<0>();

    const int na = nt * 128 + ja;
    if (p.splits == 1) {
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            const int m0 = 8 * j + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = m0 + (e & 1);
                const int n = na + ((e >> 1) << 3);
                if (m < p.M && n < p.N) p.C[static_cast<int64_t>(m) * p.N + n] = __float2half_rn(acc[j][e]);
            }
        }
        return;
    }

    // ---- split-K: partial tiles through distributed shared memory, summed in rank order
    __syncthreads();  // every warp is done with its weight ring, which now holds the partials
#pragma unroll
    for (int j = 0; j < MT; ++j) {
        const int m0 = 8 * j + 2 * t;
#pragma unroll
        for (int e = 0; e < 4; ++e) red[(m0 + (e & 1)) * 128 + ja + ((e >> 1) << 3)] = acc[j][e];
    }
    cluster_sync_all();
    const int S = p.splits;
    const int rank = static_cast<int>(cluster_ctarank());
    const int c0 = (rank * 128) / S, c1 = ((rank + 1) * 128) / S, cw = c1 - c0;
    for (int o = threadIdx.x; o < cw * p.M; o += kSkThreads) {
        const int m = o / cw, col = c0 + (o - m * cw);
        const int n = nt * 128 + col;
        if (n < p.N) {
            float part[8];
#pragma unroll
            for (int r = 0; r < 8; ++r)
                part[r] = r < S ? ld_dsmem_f32(&red[m * 128 + col], static_cast<uint32_t>(r)) : 0.f;
            float sum = 0.f;
#pragma unroll
            for (int r = 0; r < 8; ++r) sum += part[r];
            p.C[static_cast<int64_t>(m) * p.N + n] = __float2half_rn(sum);
        }
    }
    cluster_sync_all();
}

int smem_bytes(int mt, int act_stride, int scale_rows) {
    return 8 * mt * act_stride * 2 + scale_rows * 256 + kWbufBytes;
}

}  // namespace

int skinny_plan(int64_t M, int64_t N, int64_t K, int64_t G, SkinnyPlan* plan) {
    if (M < 1 || M > kSkinnyMaxM) return W4A16_ERR_UNSUPPORTED;
    const int64_t NT = (N + 127) / 128;
    const int64_t KT = (K + 63) / 64;
    const int64_t KB = (KT + 1) / 2;
    const int mt = M <= 8 ? 1 : 2;
    int sms = sm_count();
    if (sms <= 0) sms = 148;
    // Enough CTAs for about two per SM, never more than the cluster limit or the K blocks.
    int64_t splits = (2 * sms + NT - 1) / NT;
    if (splits > 8) splits = 8;
    if (splits > KB) splits = KB;
    if (splits < 1) splits = 1;
    for (;;) {
        const int64_t krange = ((KB + splits - 1) / splits) * kBlockK;
        const int64_t stride = krange + 8;
        const int64_t rows = krange / G + 2;
        const int64_t bytes = smem_bytes(mt, static_cast<int>(stride), static_cast<int>(rows));
        if (bytes <= 200 * 1024) {
            plan->splits = static_cast<int>(splits);
            plan->act_stride = static_cast<int>(stride);
            plan->scale_rows = static_cast<int>(rows < (K + G - 1) / G ? rows : (K + G - 1) / G);
            plan->smem = smem_bytes(mt, plan->act_stride, plan->scale_rows);
            plan->mt = mt;
            plan->grid_x = static_cast<int>(splits);
            plan->grid_y = static_cast<int>(NT);
            break;
        }
        if (splits >= 8 || splits >= KB) return W4A16_ERR_UNSUPPORTED;
        ++splits;
    }
    if (NT > 65535) return W4A16_ERR_UNSUPPORTED;
    // floor(k / G) as a multiply-shift, checked exhaustively over the padded K range.
    const uint64_t magic = ((uint64_t(1) << 32) + static_cast<uint64_t>(G) - 1) / static_cast<uint64_t>(G);
    if (magic > 0xFFFFFFFFull) return W4A16_ERR_UNSUPPORTED;
    for (int64_t k = 0; k < KB * kBlockK; k += 8)
        if (static_cast<int64_t>((static_cast<uint64_t>(k) * magic) >> 32) != k / G) return W4A16_ERR_UNSUPPORTED;
    plan->g_magic = static_cast<uint32_t>(magic);
    plan->post_scale = (G % kBlockK) == 0 ? 1 : 0;
    return W4A16_OK;
}

int skinny_launch(const SkinnyPlan& plan, const void* A, const uint8_t* Wt, const void* S, void* C, int64_t M,
                  int64_t N, int64_t K, int64_t G, cudaStream_t stream) {
    static bool attr_done[2][64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return W4A16_ERR_CUDA;
    const void* fn = plan.mt == 1 ? reinterpret_cast<const void*>(&w4a16_skinny_kernel<1>)
                                  : reinterpret_cast<const void*>(&w4a16_skinny_kernel<2>);
    if (!attr_done[plan.mt - 1][dev]) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess)
            return W4A16_ERR_CUDA;
        attr_done[plan.mt - 1][dev] = true;
    }
    SkinnyParams p;
    p.wt = Wt;
    p.sc = reinterpret_cast<const __half*>(S);
    p.A = reinterpret_cast<const __half*>(A);
    p.C = reinterpret_cast<__half*>(C);
    p.M = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.G = static_cast<int32_t>(G);
    p.ngroups = static_cast<int32_t>((K + G - 1) / G);
    p.KT = static_cast<int32_t>((K + 63) / 64);
    p.KB = (p.KT + 1) / 2;
    p.splits = plan.splits;
    p.act_stride = plan.act_stride;
    p.scale_rows = plan.scale_rows;
    p.g_magic = plan.g_magic;
    p.post_scale = plan.post_scale;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(plan.grid_x), static_cast<unsigned>(plan.grid_y), 1);
    cfg.blockDim = dim3(kSkThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    cfg.numAttrs = 0;
    if (plan.splits > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(plan.splits);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cudaError_t e = plan.mt == 1 ? cudaLaunchKernelEx(&cfg, w4a16_skinny_kernel<1>, p)
                                 : cudaLaunchKernelEx(&cfg, w4a16_skinny_kernel<2>, p);
    return e == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

}  // namespace w4a16
