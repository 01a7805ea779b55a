// Skinny W4A16 GEMM for decode-sized M (1..16): C[M,N] = A[M,K] x dequant(W).
//
// The operation is the Int4GroupwiseGemmPluginV2 page's (class description:
// activations, int4 weights, scales [ceil(K/G),N], fp16 output). At M <= 16 the
// product is bound by streaming the int4 weights from HBM (K*N/2 bytes):
//   - each thread streams its own two 16-byte int4 chunks per 128-deep K block
//     with cp.async into a private ring of kDepth blocks (per-thread copies
//     keep more requests in flight per SM than one bulk engine does, and no
//     thread ever reads another thread's slot, so stages need no barrier);
//   - it decodes them straight into the A operand of a warp-level m16n8k16
//     MMA (weights as the 16-row operand, 16 output columns per warp; tokens
//     as the 8-column operand: one or two token tiles);
//   - scale rows ride on the first stage; activations are staged after the
//     previous kernel in the stream has finished (programmatic dependent
//     launch lets the weight copies start before that);
//   - K is split over up to 8 CTAs of a thread-block cluster whose fp32 partial
//     tiles are summed in rank order in the owning CTA's shared memory (one
//     token tile: sized for one CTA per SM; two token tiles: up to two).
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
#include <cstring>

#include "../../include/w4a16.h"
#include "dequant.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"
#include "w4a16_internal.h"

namespace w4a16 {

namespace {

constexpr int kSkWarps = 8;                       // 8 warps x 16 columns = one 128-column weight tile
constexpr int kSkThreads = kSkWarps * 32;         // threads of one K half
constexpr int kBlockK = 128;
constexpr int kSlotBytes = 32;                    // per thread and block: two 16-byte chunks

// No wait in this kernel can fail to end (cp.async groups and cluster barriers
// only); its status word latches malformed expert offsets in grouped mode.
__device__ int g_skinny_status;

struct SkinnyParams {
    const uint8_t* wt;      // tiled weights
    const __half* sc;       // scales [ngroups, N]
    const __half* A;        // activations [M, K]
    __half* C;              // output [M, N]
    int32_t M, N, K, G;
    int32_t ngroups, KT, KB;  // groups, 64-deep tiles, 128-deep blocks
    int32_t splits;
    int32_t act_stride;       // halves per staged activation row (max K range + 16)
    int32_t scale_rows;       // rows of the staged scale window
    uint32_t g_magic;         // floor(k / G) == (k * g_magic) >> 32 for every k < K padded
    int32_t post_scale;       // G % 128 == 0: scale fp32 partials once per block
    int32_t prefetch;         // weights/scales may be read before the previous kernel finishes
    // Grouped-expert mode (grid z = expert): rows [off[e], off[e+1]) of A and C
    // use expert e's weights and scales; M is then the total row count.
    int32_t grouped, E, act;  // act: W4A16_ACT_* applied to the fp16 result
    const int32_t* offsets;
    const uint8_t* wte[W4A16_MAX_EXPERTS];
    const __half* sce[W4A16_MAX_EXPERTS];
};

// KH = 2 runs two sets of 8 warps over the same 128 columns, the first taking
// the even 128-deep blocks of the CTA's K range and the second the odd ones, and
// adds the two partial tiles in shared memory (first + second) after the loop.
// GROUPED: the grouped-expert form (a separate instantiation, so that the
// dense kernels keep their register budget).
template <int MT, int kDepth, int KH, bool GROUPED>
__global__ void __launch_bounds__(KH * kSkThreads, 2)
    w4a16_skinny_kernel(const __grid_constant__ SkinnyParams p) {
    extern __shared__ __align__(1024) uint8_t sm[];
    constexpr int kThreads = KH * kSkThreads;
    // This CTA's operands: the whole product, or in grouped mode its expert's
    // row segment (every CTA of a cluster has the same expert, so a cluster
    // leaves together).
    const uint8_t* Wt = p.wt;
    const __half* Sc = p.sc;
    const __half* Ap = p.A;
    __half* Cp = p.C;
    int Mrows = p.M;
    if constexpr (GROUPED) {
        grid_dependency_wait();  // the offsets come from the previous kernel
        const int32_t* off = p.offsets;
        bool ok = off[0] == 0 && off[p.E] == p.M;
        for (int x = 0; x < p.E && ok; ++x) ok = off[x + 1] >= off[x] && off[x + 1] - off[x] <= 8 * MT;
        if (!ok) {
            if (threadIdx.x == 0) atomicCAS(&g_skinny_status, 0, W4A16_ERR_BAD_OFFSETS);
            return;
        }
        const int e = blockIdx.z;
        const int m0 = off[e];
        Mrows = off[e + 1] - m0;
        if (Mrows == 0) return;
        Wt = p.wte[e];
        Sc = p.sce[e];
        Ap = p.A + static_cast<int64_t>(m0) * p.K;
        Cp = p.C + static_cast<int64_t>(m0) * p.N;
    }
    const int warp = (threadIdx.x >> 5) & (kSkWarps - 1), lane = threadIdx.x & 31;
    const int kh = static_cast<int>(threadIdx.x) / kSkThreads;  // K half: blocks i with i % KH == kh
    const int g = lane >> 2, t = lane & 3;
    const int split = blockIdx.x, nt = blockIdx.y;
    const int b0 = (split * p.KB) / p.splits;  // (32-bit: K < 2^31, so KB < 2^24)
    const int b1 = ((split + 1) * p.KB) / p.splits;
    const int nb = b1 - b0;
    const int kr0 = b0 * kBlockK;                   // first k of this CTA
    const int krange = nb * kBlockK;
    constexpr int MP = 8 * MT;                      // token rows, padded to the MMA's 8-column tiles
    const int S = p.splits;
    const int cwm = (128 + S - 1) / S;              // widest output-column slice of one cluster rank

    __half* act = reinterpret_cast<__half*>(sm);                          // [MP][act_stride]
    __half* scl = act + MP * p.act_stride;                                // [scale_rows][128]
    uint8_t* ring = reinterpret_cast<uint8_t*>(scl + p.scale_rows * 128); // [kDepth][2][threads][16 B]
    float* red = reinterpret_cast<float*>(ring + kDepth * kThreads * kSlotBytes);  // [S][MP][cwm] partials

    const int g_lo = kr0 / p.G;
    const int g_hi = min(p.ngroups - 1, (kr0 + krange - 1) / p.G);
    const int nrows = g_hi - g_lo + 1;
    const int ja = warp * 16 + g;  // this thread's columns: ja and ja + 8

    // This thread's chunk t of columns ja and ja + 8 in block i: tile 2(b0+i) + t/2,
    // half t%2. A missing second tile at an odd end of K reads as zeros.
    const uint8_t* wsrc = Wt + (static_cast<int64_t>(nt) * p.KT + 2 * b0 + (t >> 1)) * 4096 + (t & 1) * 2048 + ja * 16;
    const int kt_last_ok = p.KT - 1 - (t >> 1);
    uint8_t* myslot = ring + threadIdx.x * 16;  // chunk of column ja; column ja + 8's is kThreads * 16 further
    // Local block li of this half is block i = li * KH + kh, in slot li % kDepth.
    auto issue_block = [&](int li) {
        const int i = li * KH + kh;
        if (i < nb) {
            const bool ok = 2 * (b0 + i) <= kt_last_ok;
            const uint8_t* src = wsrc + static_cast<int64_t>(i) * 8192;
            uint8_t* dst = myslot + (li % kDepth) * kThreads * kSlotBytes;
            cp_async16(dst, ok ? src : Wt, ok ? 16u : 0u);
            cp_async16(dst + kThreads * 16, ok ? src + 128 : Wt, ok ? 16u : 0u);
        }
        cp_async_commit();  // one group per block, empty past the end, so the counts stay uniform
    };
    auto issue_scales = [&]() {
        const int ncols = min(128, p.N - nt * 128);
        for (int idx = threadIdx.x; idx < nrows * 16; idx += kThreads) {
            const int r = idx >> 4, c = idx & 15;
            const bool ok = c * 8 < ncols;
            cp_async16(scl + r * 128 + c * 8,
                       ok ? Sc + static_cast<int64_t>(g_lo + r) * p.N + nt * 128 + c * 8 : Sc, ok ? 16u : 0u);
        }
        cp_async_commit();  // the oldest group: complete by the time block 0 is
    };

    // ---- with static weights (declared by the caller) the scale and weight
    // copies start before the previous kernel in the stream has finished
    if (p.prefetch) {
        issue_scales();
#pragma unroll
        for (int i = 0; i < kDepth; ++i) issue_block(i);
    }

    // ---- everything else may come from the previous kernel: wait for it, then
    // stage the activations with plain loads (zero past M and K)
    grid_launch_dependents();
    grid_dependency_wait();
    if (!p.prefetch) {
        issue_scales();
#pragma unroll
        for (int i = 0; i < kDepth; ++i) issue_block(i);
    }
    {
        // 16-byte chunks (row r, chunk c) of the CTA's K range, kThreads apart per
        // thread, walked without a division per chunk; each batch's loads go out
        // together, so a batch costs one memory round trip on this critical path.
        const int cpr = krange / 8;  // 16-byte chunks per activation row
        const int total = MP * cpr;
        int r = static_cast<int>(threadIdx.x) / cpr;
        int c = static_cast<int>(threadIdx.x) - r * cpr;
        const int rstep = kThreads / cpr, cstep = kThreads - rstep * cpr;
        constexpr int kBatch = 4;
        for (int idx0 = threadIdx.x; idx0 < total; idx0 += kBatch * kThreads) {
            uint4 v[kBatch];
            int rr[kBatch], cc[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                rr[u] = r;
                cc[u] = c;
                const int k = kr0 + c * 8;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (idx0 + u * kThreads < total && r < Mrows && k < p.K)
                    v[u] = *reinterpret_cast<const uint4*>(Ap + static_cast<int64_t>(r) * p.K + k);
                c += cstep;
                r += rstep;
                if (c >= cpr) {
                    c -= cpr;
                    ++r;
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                if (idx0 + u * kThreads < total) {
                    // Within each 128-deep block the 4-wide k groups are interleaved: group
                    // (t, s) (k = 32t + 4s .. +3, thread column t's step s) sits at halves
                    // 16s + 4t. With rows 16 halves (32 bytes mod 128) apart, the 32 lanes'
                    // 8-byte fragment loads of one step then hit distinct banks.
                    const int q = cc[u] & 3, t4 = (cc[u] >> 2) & 3;
                    __half* rowp = act + rr[u] * p.act_stride + (cc[u] >> 4) * 128 + 32 * q + 4 * t4;
                    *reinterpret_cast<uint2*>(rowp) = make_uint2(v[u].x, v[u].y);
                    *reinterpret_cast<uint2*>(rowp + 16) = make_uint2(v[u].z, v[u].w);
                }
            }
        }
    }
    cp_async_wait<kDepth - 1>();  // the scale rows (and this thread's first block) have landed
    __syncthreads();              // staged activations and scale rows are visible to all threads
    // Distributed shared memory may be written only once every CTA of the cluster
    // has started: arrive here, and wait for the others before the first remote store.
    if (p.splits > 1) cluster_arrive_relaxed();

    float acc[MT][4], acc2[MT][4];  // (acc2: the odd-step chain when groups are finer than a block)
#pragma unroll
    for (int j = 0; j < MT; ++j) {
        acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
        acc2[j][0] = acc2[j][1] = acc2[j][2] = acc2[j][3] = 0.f;
    }
    uint32_t arow[MT];
#pragma unroll
    for (int j = 0; j < MT; ++j) arow[j] = smem_addr(act + (8 * j + g) * p.act_stride + 4 * t);
    const uint32_t slot0 = smem_addr(myslot);

    const int nbh = (nb - kh + KH - 1) / KH;  // blocks of this half
    for (int li = 0; li < nbh; ++li) {
        cp_async_wait<kDepth - 1>();  // local block li is in this thread's slot
        const int i = li * KH + kh;
        const uint32_t slot = slot0 + (li % kDepth) * kThreads * kSlotBytes;
        const uint4 wa = lds128(slot);
        const uint4 wb = lds128(slot + kThreads * 16);
        const uint32_t kb2 = static_cast<uint32_t>(i * kBlockK * 2);  // block offset in the staged range, bytes
        const uint32_t wa_w[4] = {wa.x, wa.y, wa.z, wa.w};
        const uint32_t wb_w[4] = {wb.x, wb.y, wb.z, wb.w};
        if (p.post_scale) {
            // One group covers the whole block: MMA chains over the exact codes,
            // started from zero accumulators, then one scaled add per element.
            // Two chains (even and odd 16-deep steps) halve the dependent MMA
            // latency; their sum is taken in a fixed order.
            float part[2][MT][4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint4 qa = decode_word(wa_w[w]);
                const uint4 qb = decode_word(wb_w[w]);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t afr[4] = {u ? qa.z : qa.x, u ? qb.z : qb.x, u ? qa.w : qa.y, u ? qb.w : qb.y};
                    const int st = 2 * w + u;
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint2 bfr = lds64(arow[j] + kb2 + 32 * st);
                        if (w == 0)
                            mma_m16n8k16_zc(part[u][j], afr, bfr.x, bfr.y);
                        else
                            mma_m16n8k16(part[u][j], afr, bfr.x, bfr.y);
                    }
                }
            }
            const int gr =
                static_cast<int>((static_cast<uint64_t>(kr0 + i * kBlockK) * p.g_magic) >> 32) - g_lo;  // floor(k / G)
            const float sa = __half2float(scl[gr * 128 + ja]);
            const float sb = __half2float(scl[gr * 128 + ja + 8]);
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                acc[j][0] = fmaf(part[0][j][0] + part[1][j][0], sa, acc[j][0]);
                acc[j][1] = fmaf(part[0][j][1] + part[1][j][1], sa, acc[j][1]);
                acc[j][2] = fmaf(part[0][j][2] + part[1][j][2], sb, acc[j][2]);
                acc[j][3] = fmaf(part[0][j][3] + part[1][j][3], sb, acc[j][3]);
            }
        } else {
            // Groups finer than the block: scale each decoded word (rounded to fp16).
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t kk = static_cast<uint32_t>(kr0 + i * kBlockK + 32 * t + 8 * w);
                const int gr =
                    min(static_cast<int>((static_cast<uint64_t>(kk) * p.g_magic) >> 32), p.ngroups - 1) - g_lo;
                const uint4 qa = dequant_word(wa_w[w], __half2half2(scl[gr * 128 + ja]));
                const uint4 qb = dequant_word(wb_w[w], __half2half2(scl[gr * 128 + ja + 8]));
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t afr[4] = {u ? qa.z : qa.x, u ? qb.z : qb.x, u ? qa.w : qa.y, u ? qb.w : qb.y};
                    const int st = 2 * w + u;
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint2 bfr = lds64(arow[j] + kb2 + 32 * st);
                        mma_m16n8k16(u ? acc2[j] : acc[j], afr, bfr.x, bfr.y);  // two chains
                    }
                }
            }
        }
        issue_block(li + kDepth);  // this thread's slot for local block li is consumed (values decoded above)
    }
    cp_async_wait<0>();
    if (!p.post_scale) {
#pragma unroll
        for (int j = 0; j < MT; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[j][e] += acc2[j][e];
        }
    }
    if (KH == 2) {
        // The second half's partials go through the (drained) ring; the first half adds them.
        float* xr = reinterpret_cast<float*>(ring);
        const int lt = threadIdx.x & (kSkThreads - 1);
        __syncthreads();  // every thread's copies into the ring have completed
        if (kh == 1) {
#pragma unroll
            for (int j = 0; j < MT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) xr[(j * 4 + e) * kSkThreads + lt] = acc[j][e];
        }
        __syncthreads();
        if (kh == 0) {
#pragma unroll
            for (int j = 0; j < MT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[j][e] += xr[(j * 4 + e) * kSkThreads + lt];
        }
    }

    const int na = nt * 128 + ja;
    if (S == 1) {
        if (kh != 0) return;
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            const int m0 = 8 * j + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = m0 + (e & 1);
                const int n = na + ((e >> 1) << 3);
                if (m < Mrows && n < p.N)
                    Cp[static_cast<int64_t>(m) * p.N + n] =
                        GROUPED ? epilogue_value(acc[j][e], p.act) : __float2half_rn(acc[j][e]);
            }
        }
        return;
    }

    // ---- split-K: every CTA stores its partials straight into the shared memory
    // of the CTA that owns those output columns (owner q holds columns
    // [ceil(q*128/S), ceil((q+1)*128/S))), one cluster barrier publishes them,
    // and each owner sums its S slices in rank order.
    const int rank = static_cast<int>(cluster_ctarank());
    cluster_wait();
    if (kh == 0) {
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            const int m0 = 8 * j + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = m0 + (e & 1);
                const int col = ja + ((e >> 1) << 3);
                const int q = (col * S) >> 7;          // owner of this column
                const int cq = (q * 128 + S - 1) / S;  // owner's first column
                if (m < Mrows)
                    st_dsmem_f32(&red[(rank * MP + m) * cwm + (col - cq)], static_cast<uint32_t>(q), acc[j][e]);
            }
        }
    }
    cluster_sync_all();
    const int c0 = (rank * 128 + S - 1) / S, c1 = ((rank + 1) * 128 + S - 1) / S, cw = c1 - c0;
    for (int o = threadIdx.x; o < cw * Mrows; o += kThreads) {
        const int m = o / cw, c = o - m * cw;
        const int n = nt * 128 + c0 + c;
        if (n < p.N) {
            float sum = 0.f;
            for (int r = 0; r < S; ++r) sum += red[(r * MP + m) * cwm + c];
            Cp[static_cast<int64_t>(m) * p.N + n] = GROUPED ? epilogue_value(sum, p.act) : __float2half_rn(sum);
        }
    }
}

// K halves per CTA: two for one token tile over a long K range (16 or more
// 128-deep blocks per CTA), else one. (Two halves take 512 threads and 32K
// registers per CTA: at short K ranges the extra warps gain little, and the
// CTA no longer fits beside a neighbouring launch's CTAs on the SM.)
int k_halves(int mt, int64_t nbmax) { return (mt == 1 && nbmax >= 16) ? 2 : 1; }

int smem_bytes(int kh, int depth, int mt, int splits, int act_stride, int scale_rows) {
    const int ring = depth * kh * kSkThreads * kSlotBytes;
    const int red = splits > 1 ? splits * 8 * mt * ((128 + splits - 1) / splits) * 4 : 0;
    return 8 * mt * act_stride * 2 + scale_rows * 256 + ring + red;
}

}  // namespace

int skinny_plan_fill(int64_t M, int64_t N, int64_t K, int64_t G, int splits, int kh, int deep, SkinnyPlan* plan) {
    if (M < 1 || M > kSkinnyMaxM) return W4A16_ERR_UNSUPPORTED;
    const int64_t NT = (N + 127) / 128;
    const int64_t KT = (K + 63) / 64;
    const int64_t KB = (KT + 1) / 2;
    const int mt = M <= 8 ? 1 : 2;
    if (NT > 65535 || splits < 1 || splits > 8 || splits > KB) return W4A16_ERR_UNSUPPORTED;
    if (kh < 1 || kh > 2 || (kh == 2 && mt != 1)) return W4A16_ERR_UNSUPPORTED;  // compiled forms only
    const int64_t nbmax = (KB + splits - 1) / splits;
    const int dmax = 8 / kh;  // 128-deep blocks in flight per thread: 8 per CTA
    const int depth = deep ? dmax : dmax / 2;
    const int64_t krange = nbmax * kBlockK;
    const int64_t stride = krange + 16;  // 32 bytes mod 128 between rows (see the staging loop)
    const int64_t rows = krange / G + 2;
    const int64_t bytes =
        smem_bytes(kh, depth, mt, splits, static_cast<int>(stride), static_cast<int>(rows));
    if (bytes > 200 * 1024) return W4A16_ERR_UNSUPPORTED;
    // floor(k / G) as a multiply-shift over the padded K range. With
    // magic = (2^32 + e) / G, 0 <= e < G, k * magic / 2^32 = k / G + k * e / (G * 2^32),
    // which floors to floor(k / G) whenever k * e < 2^32 (the fractional part of
    // k / G is at most (G - 1) / G). Otherwise every k is checked.
    const uint64_t magic = ((uint64_t(1) << 32) + static_cast<uint64_t>(G) - 1) / static_cast<uint64_t>(G);
    if (magic > 0xFFFFFFFFull) return W4A16_ERR_UNSUPPORTED;
    const uint64_t e = magic * static_cast<uint64_t>(G) - (uint64_t(1) << 32);
    const uint64_t kend = static_cast<uint64_t>(KB * kBlockK);
    if (e != 0 && kend > ((uint64_t(1) << 32) - 1) / e) {
        for (int64_t k = 0; k < KB * kBlockK; k += 8)
            if (static_cast<int64_t>((static_cast<uint64_t>(k) * magic) >> 32) != k / G) return W4A16_ERR_UNSUPPORTED;
    }
    plan->splits = splits;
    plan->depth = depth;
    plan->act_stride = static_cast<int>(stride);
    plan->scale_rows = static_cast<int>(rows < (K + G - 1) / G ? rows : (K + G - 1) / G);
    plan->smem = smem_bytes(kh, depth, mt, plan->splits, plan->act_stride, plan->scale_rows);
    plan->mt = mt;
    plan->threads = kh * kSkThreads;
    plan->grid_x = splits;
    plan->grid_y = static_cast<int>(NT);
    plan->g_magic = static_cast<uint32_t>(magic);
    plan->post_scale = (G % kBlockK) == 0 ? 1 : 0;
    return W4A16_OK;
}

int skinny_plan(int64_t M, int64_t N, int64_t K, int64_t G, SkinnyPlan* plan) {
    if (M < 1 || M > kSkinnyMaxM) return W4A16_ERR_UNSUPPORTED;
    const int64_t NT = (N + 127) / 128;
    const int64_t KT = (K + 63) / 64;
    const int64_t KB = (KT + 1) / 2;
    const int mt = M <= 8 ? 1 : 2;
    int sms = sm_count();
    if (sms <= 0) sms = 148;
    // One wave (a second wave of clusters would double the time), never more
    // than the cluster limit or the K blocks. One token tile: one CTA per SM,
    // so that every SM does the same share (with two per SM on some SMs and
    // one on others, the clusters wait for the doubly loaded ones: measured
    // 6.7 against 7.6 us at K = N = 4096). Two token tiles, with twice the
    // MMA work per weight, spread over up to two CTAs per SM.
    int64_t splits = (mt == 1 ? sms : 2 * sms) / NT;
    if (splits > 8) splits = 8;
    if (splits > KB) splits = KB;
    if (splits < 1) splits = 1;
    for (;;) {
        const int64_t nbmax = (KB + splits - 1) / splits;
        // All eight blocks in flight per CTA for long K ranges, half of them
        // for short ones.
        const int kh = k_halves(mt, nbmax);
        const int64_t nbh = (nbmax + kh - 1) / kh;  // blocks of one K half
        const int deep = nbh <= (8 / kh) / 2 ? 0 : 1;
        if (skinny_plan_fill(M, N, K, G, static_cast<int>(splits), kh, deep, plan) == W4A16_OK) return W4A16_OK;
        if (splits >= 8 || splits >= KB) return W4A16_ERR_UNSUPPORTED;
        ++splits;
    }
}

int skinny_plan_grouped(int64_t total_rows, int64_t N, int64_t K, int64_t G, SkinnyPlan* plan) {
    // The experts' column tiles already give E x ceil(N/128) CTAs, so K is split
    // only as far as the staged activations need to fit in shared memory.
    if (total_rows < 1 || total_rows > kSkinnyMaxM) return W4A16_ERR_UNSUPPORTED;
    const int64_t KB = ((K + 63) / 64 + 1) / 2;
    const int mt = total_rows <= 8 ? 1 : 2;
    for (int64_t splits = 1; splits <= 8 && splits <= KB; ++splits) {
        const int64_t nbmax = (KB + splits - 1) / splits;
        const int kh = k_halves(mt, nbmax);
        const int64_t nbh = (nbmax + kh - 1) / kh;
        const int deep = nbh <= (8 / kh) / 2 ? 0 : 1;
        if (skinny_plan_fill(total_rows, N, K, G, static_cast<int>(splits), kh, deep, plan) == W4A16_OK)
            return W4A16_OK;
    }
    return W4A16_ERR_UNSUPPORTED;
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

namespace {

// Launch with filled parameters; grid z = 1 (dense) or the number of experts.
int skinny_launch_params(const SkinnyPlan& plan, SkinnyParams& p, int64_t N, int64_t K, int64_t G, unsigned grid_z,
                         cudaStream_t stream) {
    static bool attr_done[12][64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return W4A16_ERR_CUDA;
    const int kh = plan.threads / kSkThreads;
    const int vi = (p.grouped ? 6 : 0) + (plan.mt == 2 ? 4 : (kh == 2 ? 2 : 0)) + (plan.depth == 8 / kh ? 1 : 0);
    // (shared-memory carve-out: the largest, so two CTAs fit per SM)
    void (*kernels[12])(SkinnyParams) = {
        w4a16_skinny_kernel<1, 4, 1, false>, w4a16_skinny_kernel<1, 8, 1, false>,
        w4a16_skinny_kernel<1, 2, 2, false>, w4a16_skinny_kernel<1, 4, 2, false>,
        w4a16_skinny_kernel<2, 4, 1, false>, w4a16_skinny_kernel<2, 8, 1, false>,
        w4a16_skinny_kernel<1, 4, 1, true>,  w4a16_skinny_kernel<1, 8, 1, true>,
        w4a16_skinny_kernel<1, 2, 2, true>,  w4a16_skinny_kernel<1, 4, 2, true>,
        w4a16_skinny_kernel<2, 4, 1, true>,  w4a16_skinny_kernel<2, 8, 1, true>};
    if (!attr_done[vi][dev]) {
        if (cudaFuncSetAttribute(reinterpret_cast<const void*>(kernels[vi]),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024) != cudaSuccess ||
            cudaFuncSetAttribute(reinterpret_cast<const void*>(kernels[vi]),
                                 cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
                cudaSuccess)
            return W4A16_ERR_CUDA;
        attr_done[vi][dev] = true;
    }
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
    cfg.gridDim = dim3(static_cast<unsigned>(plan.grid_x), static_cast<unsigned>(plan.grid_y), grid_z);
    cfg.blockDim = dim3(static_cast<unsigned>(plan.threads), 1, 1);
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

}  // namespace

int skinny_launch(const SkinnyPlan& plan, const void* A, const uint8_t* Wt, const void* S, void* C, int64_t M,
                  int64_t N, int64_t K, int64_t G, cudaStream_t stream) {
    SkinnyParams p;
    std::memset(&p, 0, sizeof(p));
    p.wt = Wt;
    p.sc = reinterpret_cast<const __half*>(S);
    p.A = reinterpret_cast<const __half*>(A);
    p.C = reinterpret_cast<__half*>(C);
    p.M = static_cast<int32_t>(M);
    p.prefetch = static_weights_enabled() ? 1 : 0;
    return skinny_launch_params(plan, p, N, K, G, 1, stream);
}

int skinny_grouped_launch(const SkinnyPlan& plan, const void* A, const uint8_t* const* Wt, const void* const* S,
                          const int32_t* offsets, void* C, int64_t E, int64_t total_rows, int64_t N, int64_t K,
                          int64_t G, int act, cudaStream_t stream) {
    SkinnyParams p;
    std::memset(&p, 0, sizeof(p));
    for (int64_t e = 0; e < E; ++e) {
        p.wte[e] = Wt[e];
        p.sce[e] = reinterpret_cast<const __half*>(S[e]);
    }
    p.wt = Wt[0];
    p.sc = reinterpret_cast<const __half*>(S[0]);
    p.A = reinterpret_cast<const __half*>(A);
    p.C = reinterpret_cast<__half*>(C);
    p.M = static_cast<int32_t>(total_rows);
    p.grouped = 1;
    p.E = static_cast<int32_t>(E);
    p.act = act;
    p.offsets = offsets;
    p.prefetch = 0;  // the expert of a CTA is known only after the offsets, which follow the wait
    return skinny_launch_params(plan, p, N, K, G, static_cast<unsigned>(E), stream);
}

}  // namespace w4a16
