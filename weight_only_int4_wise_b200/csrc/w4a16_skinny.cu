// Skinny W4A16 GEMM for decode-sized M (1..16): C[M,N] = A[M,K] x dequant(W).
//
// The operation is the Int4GroupwiseGemmPluginV2 page's (class description:
// activations, int4 weights, scales [ceil(K/G),N], fp16 output). At M <= 16 the
// product is bound by streaming the int4 weights from HBM (K*N/2 bytes):
//   - a producer warp moves each 128-deep K block of a 128-column weight tile
//     (8 KB, contiguous in the tiled layout) with one bulk copy into a ring of
//     kDepth shared-memory stages, completing on that stage's mbarrier;
//   - eight compute warps (16 output columns each) read their fragments from a
//     stage, release it at once, and decode them straight into the A operand
//     of a warp-level m16n8k16 MMA (weights as the 16-row operand, tokens as
//     the 8-column operand: one or two token tiles);
//   - scale rows ride on the first stage; activations are staged after the
//     previous kernel in the stream has finished (programmatic dependent
//     launch lets the weight copies start before that);
//   - K is split over up to 8 CTAs of a thread-block cluster whose fp32 partial
//     tiles are summed in rank order in the owning CTA's shared memory.
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

constexpr int kSkWarps = 8;                       // compute warps: 8 x 16 columns = one 128-column tile
constexpr int kSkThreads = (kSkWarps + 1) * 32;   // plus one producer warp
constexpr int kBlockK = 128;
constexpr int kBlockBytes = 8192;                 // int4 codes of a 128-column x 128-deep block
constexpr long long kSkTimeoutCycles = 4000000000ll;

__device__ int g_skinny_status;  // latched device-side error of this kernel (0 = none)

// Bounded wait on an mbarrier phase (SM-clock bound). False on timeout, which is latched.
__device__ __forceinline__ bool sk_wait(uint64_t* bar, uint32_t parity) {
    long long start = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 15u) {
            const long long now = clock64();
            if (start == 0) {
                start = now;
            } else if (now - start > kSkTimeoutCycles) {
                atomicCAS(&g_skinny_status, 0, W4A16_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

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
    int32_t prefetch;         // weights/scales may be read before the previous kernel finishes
};

template <int MT, int kDepth>
__global__ void __launch_bounds__(kSkThreads, 2) w4a16_skinny_kernel(const __grid_constant__ SkinnyParams p) {
    extern __shared__ __align__(1024) uint8_t sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int split = blockIdx.x, nt = blockIdx.y;
    const int b0 = static_cast<int>((static_cast<int64_t>(split) * p.KB) / p.splits);
    const int b1 = static_cast<int>((static_cast<int64_t>(split + 1) * p.KB) / p.splits);
    const int nb = b1 - b0;
    const int kr0 = b0 * kBlockK;                   // first k of this CTA
    const int krange = nb * kBlockK;
    constexpr int MP = 8 * MT;                      // token rows, padded to the MMA's 8-column tiles
    const int S = p.splits;
    const int cwm = (128 + S - 1) / S;              // widest output-column slice of one cluster rank

    uint8_t* ring = sm;                                                   // [kDepth][8 KB]
    __half* act = reinterpret_cast<__half*>(ring + kDepth * kBlockBytes); // [MP][act_stride]
    __half* scl = act + MP * p.act_stride;                                // [scale_rows][128]
    float* red = reinterpret_cast<float*>(scl + p.scale_rows * 128);      // [S][MP][cwm] split-K partials
    uint64_t* full = reinterpret_cast<uint64_t*>(red + (S > 1 ? S * MP * cwm : 0));
    uint64_t* empty = full + kDepth;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDepth);

    const int g_lo = kr0 / p.G;
    const int g_hi = min(p.ngroups - 1, (kr0 + krange - 1) / p.G);
    const int nrows = g_hi - g_lo + 1;
    const uint32_t srow_bytes = static_cast<uint32_t>(min(128, p.N - nt * 128)) * 2u;
    const uint8_t* wsrc = p.wt + (static_cast<int64_t>(nt) * p.KT + 2 * b0) * 4096;
    // Block i holds tiles 2(b0+i) and 2(b0+i)+1; the second is missing at an odd end of K.
    auto block_bytes = [&](int i) { return 2 * (b0 + i) + 1 < p.KT ? kBlockBytes : kBlockBytes / 2; };
    auto issue = [&](int i) {  // producer lane only
        const int s = i % kDepth;
        uint32_t bytes = static_cast<uint32_t>(block_bytes(i));
        if (i == 0) bytes += nrows * srow_bytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(ring + s * kBlockBytes, wsrc + static_cast<int64_t>(i) * kBlockBytes, block_bytes(i), &full[s]);
        if (i == 0)
            for (int r = 0; r < nrows; ++r)
                bulk_g2s(scl + r * 128, p.sc + static_cast<int64_t>(g_lo + r) * p.N + nt * 128, srow_bytes, &full[0]);
    };

    // ---- with static weights (set by the caller) the weight and scale copies
    // start before the previous kernel in the stream has finished
    const bool producer = warp == kSkWarps;
    if (producer && lane == 0) {
        for (int s = 0; s < kDepth; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kSkWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
        if (p.prefetch)
            for (int i = 0; i < min(kDepth, nb); ++i) issue(i);
    }

    // ---- everything else may come from the previous kernel: wait for it, then
    // stage the activations with plain loads (zero past M and K)
    grid_launch_dependents();
    grid_dependency_wait();
    if (producer && lane == 0 && !p.prefetch)
        for (int i = 0; i < min(kDepth, nb); ++i) issue(i);
    {
        const int cpr = krange / 8;  // 16-byte chunks per activation row
        for (int idx = threadIdx.x; idx < MP * cpr; idx += kSkThreads) {
            const int r = idx / cpr, c = idx - r * cpr;
            const int k = kr0 + c * 8;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < p.M && k < p.K) v = *reinterpret_cast<const uint4*>(p.A + static_cast<int64_t>(r) * p.K + k);
            *reinterpret_cast<uint4*>(act + r * p.act_stride + c * 8) = v;
        }
    }
    __syncthreads();  // staged activations and the barrier initialisation are visible

    float acc[MT][4];
#pragma unroll
    for (int j = 0; j < MT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    const int ja = (warp < kSkWarps ? warp : 0) * 16 + g;  // this thread's columns: ja and ja + 8

    if (producer) {
        // ------------------------------------------------ refill freed stages
        if (lane == 0) {
            int issued = min(kDepth, nb);
            for (int i = kDepth; i < nb && !*abort_flag; ++i) {
                const int s = i % kDepth;
                if (!sk_wait(&empty[s], static_cast<uint32_t>((i / kDepth) - 1) & 1u)) {
                    *abort_flag = 1;
                    break;
                }
                fence_proxy_async_smem();  // the warps' reads of the stage precede the copy's writes
                issue(i);
                issued = i + 1;
            }
            // every issued copy lands before the CTA's shared memory is released
            for (int i = max(0, issued - kDepth); i < issued; ++i)
                if (!sk_wait(&full[i % kDepth], static_cast<uint32_t>(i / kDepth) & 1u)) *abort_flag = 1;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ compute
        uint32_t arow[MT];
#pragma unroll
        for (int j = 0; j < MT; ++j) arow[j] = smem_addr(act + (8 * j + g) * p.act_stride + 32 * t);
        // chunk t of column ja: tile t/2 of the block, half t%2
        const uint32_t frag0 = smem_addr(ring) + (t >> 1) * 4096 + (t & 1) * 2048 + ja * 16;
        for (int i = 0; i < nb; ++i) {
            const int s = i % kDepth;
            int ok = 1;
            if (lane == 0) ok = sk_wait(&full[s], static_cast<uint32_t>(i / kDepth) & 1u) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                *abort_flag = 1;
                break;
            }
            mbar_try_wait(&full[s], static_cast<uint32_t>(i / kDepth) & 1u);  // completed: acquire for every lane
            uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = wa;
            if (!(t >> 1) || block_bytes(i) == kBlockBytes) {
                wa = lds128(frag0 + s * kBlockBytes);
                wb = lds128(frag0 + s * kBlockBytes + 128);
            }
            const uint32_t kb2 = static_cast<uint32_t>(i * kBlockK * 2);  // block offset in the staged range, bytes
            const uint32_t wa_w[4] = {wa.x, wa.y, wa.z, wa.w};
            const uint32_t wb_w[4] = {wb.x, wb.y, wb.z, wb.w};
            if (p.post_scale) {
                // One group covers the whole block: one MMA chain over the exact codes,
                // started from a zero accumulator, then one scaled add per element.
                uint4 qa_all[4], qb_all[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    qa_all[w] = decode_word(wa_w[w]);
                    qb_all[w] = decode_word(wb_w[w]);
                }
                // The stage's bytes are all decoded (so both loads have completed):
                // it may be refilled while this warp runs its MMAs.
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                float part[MT][4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint4 qa = qa_all[w];
                    const uint4 qb = qb_all[w];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint32_t afr[4] = {u ? qa.z : qa.x, u ? qb.z : qb.x, u ? qa.w : qa.y, u ? qb.w : qb.y};
                        const int st = 2 * w + u;
#pragma unroll
                        for (int j = 0; j < MT; ++j) {
                            const uint2 bfr = lds64(arow[j] + kb2 + 8 * st);
                            if (st == 0)
                                mma_m16n8k16_zc(part[j], afr, bfr.x, bfr.y);
                            else
                                mma_m16n8k16(part[j], afr, bfr.x, bfr.y);
                        }
                    }
                }
                const int gr = (kr0 + i * kBlockK) / p.G - g_lo;
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
                uint4 qa_all[4], qb_all[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint32_t kk = static_cast<uint32_t>(kr0 + i * kBlockK + 32 * t + 8 * w);
                    const int gr =
                        min(static_cast<int>((static_cast<uint64_t>(kk) * p.g_magic) >> 32), p.ngroups - 1) - g_lo;
                    qa_all[w] = dequant_word(wa_w[w], __half2half2(scl[gr * 128 + ja]));
                    qb_all[w] = dequant_word(wb_w[w], __half2half2(scl[gr * 128 + ja + 8]));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint4 qa = qa_all[w];
                    const uint4 qb = qb_all[w];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint32_t afr[4] = {u ? qa.z : qa.x, u ? qb.z : qb.x, u ? qa.w : qa.y, u ? qb.w : qb.y};
                        const int st = 2 * w + u;
#pragma unroll
                        for (int j = 0; j < MT; ++j) {
                            const uint2 bfr = lds64(arow[j] + kb2 + 8 * st);
                            mma_m16n8k16(acc[j], afr, bfr.x, bfr.y);
                        }
                    }
                }
            }
        }
    }

    const int na = nt * 128 + ja;
    if (S == 1) {
        if (!producer) {
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
        }
        return;
    }

    // ---- split-K: every CTA stores its partials straight into the shared memory
    // of the CTA that owns those output columns (owner q holds columns
    // [ceil(q*128/S), ceil((q+1)*128/S))), one cluster barrier publishes them,
    // and each owner sums its S slices in rank order.
    const int rank = static_cast<int>(cluster_ctarank());
    if (!producer) {
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            const int m0 = 8 * j + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = m0 + (e & 1);
                const int col = ja + ((e >> 1) << 3);
                const int q = (col * S) >> 7;          // owner of this column
                const int cq = (q * 128 + S - 1) / S;  // owner's first column
                if (m < p.M) st_dsmem_f32(&red[(rank * MP + m) * cwm + (col - cq)], static_cast<uint32_t>(q), acc[j][e]);
            }
        }
    }
    cluster_sync_all();
    const int c0 = (rank * 128 + S - 1) / S, c1 = ((rank + 1) * 128 + S - 1) / S, cw = c1 - c0;
    for (int o = threadIdx.x; o < cw * p.M; o += kSkThreads) {
        const int m = o / cw, c = o - m * cw;
        const int n = nt * 128 + c0 + c;
        if (n < p.N) {
            float sum = 0.f;
            for (int r = 0; r < S; ++r) sum += red[(r * MP + m) * cwm + c];
            p.C[static_cast<int64_t>(m) * p.N + n] = __float2half_rn(sum);
        }
    }
}

int smem_bytes(int mt, int depth, int splits, int act_stride, int scale_rows) {
    const int ring = depth * kBlockBytes;
    const int red = splits > 1 ? splits * 8 * mt * ((128 + splits - 1) / splits) * 4 : 0;
    return ring + 8 * mt * act_stride * 2 + scale_rows * 256 + red + 2 * depth * 8 + 16;
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
        const int64_t nbmax = (KB + splits - 1) / splits;
        const int depth = nbmax <= 4 ? 4 : 8;  // keep every block of short K ranges in flight at once
        const int64_t krange = nbmax * kBlockK;
        const int64_t stride = krange + 8;
        const int64_t rows = krange / G + 2;
        const int64_t bytes = smem_bytes(mt, depth, static_cast<int>(splits), static_cast<int>(stride),
                                         static_cast<int>(rows));
        if (bytes <= 200 * 1024) {
            plan->splits = static_cast<int>(splits);
            plan->depth = depth;
            plan->act_stride = static_cast<int>(stride);
            plan->scale_rows = static_cast<int>(rows < (K + G - 1) / G ? rows : (K + G - 1) / G);
            plan->smem = smem_bytes(mt, depth, plan->splits, plan->act_stride, plan->scale_rows);
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

int skinny_device_status(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_skinny_status, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_skinny_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

int skinny_launch(const SkinnyPlan& plan, const void* A, const uint8_t* Wt, const void* S, void* C, int64_t M,
                  int64_t N, int64_t K, int64_t G, cudaStream_t stream) {
    static bool attr_done[4][64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return W4A16_ERR_CUDA;
    const int vi = (plan.mt - 1) * 2 + (plan.depth == 8 ? 1 : 0);
    // (shared-memory carve-out: the largest, so two CTAs fit per SM)
    void (*kernels[4])(SkinnyParams) = {w4a16_skinny_kernel<1, 4>, w4a16_skinny_kernel<1, 8>,
                                        w4a16_skinny_kernel<2, 4>, w4a16_skinny_kernel<2, 8>};
    if (!attr_done[vi][dev]) {
        if (cudaFuncSetAttribute(reinterpret_cast<const void*>(kernels[vi]),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess ||
            cudaFuncSetAttribute(reinterpret_cast<const void*>(kernels[vi]),
                                 cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
                cudaSuccess)
            return W4A16_ERR_CUDA;
        attr_done[vi][dev] = true;
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
    p.prefetch = static_weights_enabled() ? 1 : 0;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(plan.grid_x), static_cast<unsigned>(plan.grid_y), 1);
    cfg.blockDim = dim3(kSkThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (plan.splits > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = static_cast<unsigned>(plan.splits);
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernels[vi], p);
    return e == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

}  // namespace w4a16
