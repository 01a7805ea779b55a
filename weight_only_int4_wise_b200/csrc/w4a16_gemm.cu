// W4A16 group-wise GEMM on sm_100a: C[M,N] = A[M,K] x dequant(W)[K,N].
//
// The operation is the one the Int4GroupwiseGemmPluginV2 page describes
// (class description: activations [b,seq,K] fp16, int4 weights, scales
// [ceil(K/G),N] fp16, output [b,seq,N] fp16; constructor: N columns, K rows,
// groupSize G). The grouped-expert entry point applies it per expert segment
// of gathered rows (Int4MoePlugin page, constructor parameters).
//
// One kernel template serves M > 16 (decode-sized M runs on the skinny
// kernel) and the grouped-expert form. It computes the transposed product
//     D[n, m] = sum_k W[k, n] * A[m, k]
// on the 5th-generation tensor core: each CTA owns 128 weight columns (the MMA
// M extent, one TMEM lane per column) and a tile of BN activation rows (the
// MMA N extent, 16..256), so that small token counts cost no padding of the
// weight side. Warp roles inside a CTA (320 or 576 threads):
//   warp 0      producer: per 64-deep K stage, one TMA tile load of the
//               activations (128-byte swizzle, zero fill past M and K) into a
//               ring of stages, and an L2 prefetch of the column tile's int4
//               stages well ahead of use.
//   warp 1      TMEM allocation and the single MMA-issuing thread
//               (tcgen05.mma kind::f16, A = weights from TMEM, B = activations
//               from shared memory, fp32 accumulator in TMEM); it waits on one
//               barrier per pair of stages.
//   warps 2..   dequantisation, in groups of four warps (one per TMEM lane
//               quadrant; group g takes stages g, g + groups, ...): each thread
//               loads its column's 64 int4 codes of a stage (two 16-byte halves
//               of the tiled layout) and their scale straight into registers,
//               two of its stages ahead, turns them into fp16 (magic-exponent
//               decode, times the group scale) and stores them into the
//               stage's tensor-memory slot; then the epilogue (tcgen05.ld ->
//               fp16 tile in shared memory -> 16-byte row stores).
// Small-M shapes split K across up to 8 CTAs of one thread-block cluster; the
// fp32 partial tiles are summed in rank order through distributed shared
// memory (deterministic, no global workspace).
//
// Every wait is bounded: a wait that runs out latches W4A16_ERR_TIMEOUT in the
// device status word, and the CTA drains its copies, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <unordered_map>

#include "../../include/w4a16.h"
#include "dequant.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"
#include "w4a16_internal.h"

namespace w4a16 {

__device__ int g_status;  // latched device-side error (0 = none)

constexpr int kTileN = 128;                 // weight columns per CTA (MMA M)
constexpr int kTileK = 64;                  // K per pipeline stage
constexpr int kRawBytes = 4096;             // int4 codes of one 128 x 64 tile (8-bit codes: twice that)
constexpr int kSlotCols = kTileK / 2;       // TMEM columns of one dequantised 128 x 64 fp16 tile
constexpr int kGroupWarps = 4;             // one dequantisation group: the 4 TMEM lane quadrants
constexpr int kAhead = 2;                  // stages of its own a dequantising thread loads ahead
constexpr int kPrefetchStages = 12;        // int4 tile stages the producer pulls into L2 ahead of use
// Threads of a CTA with DQ dequantisation groups (each group takes every
// DQ-th stage, so DQ groups keep DQ stages in flight).
__host__ __device__ constexpr int threads_for(int dq) { return (2 + kGroupWarps * dq) * 32; }
static_assert(threads_for(4) <= 1024, "the 256-row tile's four dequantisation groups fit a CTA");
constexpr long long kTimeoutCycles = 4000000000ll;  // about 2 s per wait at the boost clock

struct Params {
    const uint8_t* wt[W4A16_MAX_EXPERTS];   // tiled weights (dense: [0])
    const __half* sc[W4A16_MAX_EXPERTS];    // scales [ceil(K/G), N]
    const int32_t* offsets;                 // grouped: [E+1] on the device
    __half* C;
    int32_t rows;       // dense: M; grouped: total gathered rows
    int32_t N, K, G;
    int32_t ngroups;    // ceil(K/G)
    int32_t KT;         // ceil(K/64)
    int32_t E;          // grouped: number of experts; dense: 1
    int32_t splits;     // CTAs along K (cluster size along x)
    int32_t grouped;
    int32_t prefetch;   // weights/scales may be read before the previous kernel finishes
    int32_t vec_out;    // C rows start on 16-byte boundaries (16-byte output stores)
    long long wait_limit;   // bound of every device wait, in SM clock cycles
    int32_t stall_stage;    // test aid: the dequantising warps withhold this stage's ready signal (< 0: never)
    int32_t act;            // W4A16_ACT_*: elementwise activation of the fp16 result (no K split)
};

// One ring of LS stages. Stage s owns, in shared memory, an activation tile
// and, in tensor memory, a 32-column slot for the dequantised fp16 weights;
// TMEM also holds the fp32 accumulator (BN columns). The int4 codes and the
// scales go straight from global memory into the dequantising threads'
// registers, a few stages ahead, so the copy engine only moves activations.
template <int BN, int LS, int TMEM_COLS>
struct Layout {
    static constexpr int kActBytes = BN * 128;
    static constexpr int kAct = 0;
    static constexpr int kBar = kAct + LS * kActBytes;
    static constexpr int kNumBars = LS + LS / 2 + LS + 1;  // full, afull (per stage pair), done, accfull
    static constexpr int kMisc = kBar + kNumBars * 8;  // tmem base, abort flag, tile info
    static constexpr int kTotal = kMisc + 32;
    static constexpr int kAlloc = kTotal + 1024;       // slack for aligning the base to 1024
    static constexpr int kAccCols = BN < 32 ? 32 : BN;
    static constexpr int kRedBytes = BN * kTileN * 4;  // split-K partials, alias the load ring
    static_assert(kAccCols + LS * kSlotCols <= TMEM_COLS, "TMEM ring does not fit the allocation");
    static_assert(TMEM_COLS == 32 || TMEM_COLS == 64 || TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512,
                  "TMEM allocations are powers of two");
    static_assert(kRedBytes <= kBar, "split-K buffer must fit in the activation ring");
    static_assert((kActBytes % 1024) == 0, "activation tiles need 1024-byte alignment");
    static_assert((LS % 2) == 0, "the MMA thread takes the ring two stages at a time");
};

__device__ __forceinline__ void latch_status(int code) { atomicCAS(&g_status, 0, code); }


// Bounded wait on an mbarrier phase. Returns false if the CTA is aborting or
// the wait ran out (which starts the abort). The bound is counted in SM clock
// cycles (clock64 is a cheap, SM-local register; the global timer is far slower
// to read and would add its latency to every pipeline hand-off).
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort_flag, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    long long start = 0;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0) {
            if (*abort_flag) return false;
            const long long now = clock64();
            if (start == 0) {
                start = now;
            } else if (now - start > limit) {
                *abort_flag = 1;
                latch_status(W4A16_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Bounded wait that ignores the abort flag: used where in-flight asynchronous
// work must finish before its resources are released.
__device__ __forceinline__ bool drain_phase(uint64_t* bar, uint32_t parity) {
    const long long limit = kTimeoutCycles;  // drains keep the long bound whatever the wait bound is
    long long start = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 15u) {
            const long long now = clock64();
            if (start == 0) {
                start = now;
            } else if (now - start > limit) {
                latch_status(W4A16_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Warp-collective forms: lane 0 polls (so the timeout decision is the same for
// the whole warp), then every lane observes the completed phase itself, which
// gives each lane acquire ordering on the data the phase guards. The phase
// cannot move on before this warp arrives elsewhere, so that check is immediate.
__device__ __forceinline__ bool warp_wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                long long limit) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = wait_phase(bar, parity, abort_flag, limit) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) mbar_try_wait(bar, parity);
    return ok != 0;
}

__device__ __forceinline__ bool warp_drain_phase(uint64_t* bar, uint32_t parity) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = drain_phase(bar, parity) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) mbar_try_wait(bar, parity);
    return ok != 0;
}

// OG: G is a multiple of 64, so a stage lies inside one scale group.
// BITS: 4 for the int4 tiled layout, 8 for the 8-bit code layout (W8A16): a
// stage's tile is 4 or 8 KB, and a thread loads 2 or 4 16-byte chunks of its
// column per stage; everything after the decode is the same.
template <int BN, int LS, int TMEM_COLS, int MINB, int DQ, bool OG, int BITS>
__global__ void __launch_bounds__(threads_for(DQ), MINB)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ Params p) {
    using L = Layout<BN, LS, TMEM_COLS>;
    static_assert(BITS == 4 || BITS == 8, "int4 or 8-bit codes");
    constexpr int kTileBytes = BITS == 4 ? kRawBytes : 2 * kRawBytes;  // one 128 x 64 tile of codes
    constexpr int kChunks = BITS / 2;                                  // 16-byte chunks per column and stage
    constexpr int kScales = OG ? 1 : 8;  // scale registers per stage and thread
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (base_addr & 1023u)) & 1023u);

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);   // stage's copies landed
    uint64_t* afull = full + LS;                                     // stage pair ready for the MMAs
    uint64_t* done = afull + LS / 2;                                 // stage's MMAs completed
    uint64_t* accfull = done + LS;                                   // accumulator complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    int* tile_info = reinterpret_cast<int*>(smem + L::kMisc + 8);  // has_tile, expert, m0, rows, staged

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nt = blockIdx.y;

    // ---------------------------------------------------------------- tile
    if (threadIdx.x == 0) {
        int has = 1, expert = 0, m0 = 0, rows = 0;
        if (p.grouped) {
            grid_dependency_wait();  // the offsets may come from the previous kernel
            const int32_t* off = p.offsets;
            bool ok = off[0] == 0 && off[p.E] == p.rows;
            for (int e = 0; e < p.E && ok; ++e) ok = off[e + 1] >= off[e];
            has = 0;
            if (!ok) {
                latch_status(W4A16_ERR_BAD_OFFSETS);
            } else {
                int z = blockIdx.z;
                for (int e = 0; e < p.E; ++e) {
                    const int cnt = off[e + 1] - off[e];
                    const int tiles = (cnt + BN - 1) / BN;
                    if (z < tiles) {
                        has = 1;
                        expert = e;
                        m0 = off[e] + z * BN;
                        rows = min(BN, off[e + 1] - m0);
                        break;
                    }
                    z -= tiles;
                }
            }
        } else {
            m0 = blockIdx.z * BN;
            rows = min(BN, p.rows - m0);
        }
        tile_info[0] = has;
        tile_info[1] = expert;
        tile_info[2] = m0;
        tile_info[3] = rows;
    }
    __syncthreads();
    if (!tile_info[0]) return;  // grouped slot beyond the routed tiles (no cluster in that mode)
    const int expert = tile_info[1];
    const int m0 = tile_info[2];
    const int rows = tile_info[3];
    const int split = p.grouped ? 0 : static_cast<int>(blockIdx.x);
    const int kb = static_cast<int>((static_cast<int64_t>(split) * p.KT) / p.splits);
    const int ke = static_cast<int>((static_cast<int64_t>(split + 1) * p.KT) / p.splits);
    const int nst = ke - kb;
    const int n_mma = min(BN, (rows + 15) & ~15);
    const uint32_t idesc = idesc_f16_f32(128, static_cast<uint32_t>(n_mma));

    auto issue_act = [&](int i) {
        const int s = i % LS;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(L::kActBytes));
        tma_load_2d(smem + L::kAct + s * L::kActBytes, &tmA, (kb + i) * kTileK, m0, &full[s]);
    };

    // ---- dequantisation threads' state (warps 2..). Their first look-ahead
    // loads go out before the barrier and TMEM setup below, so that the
    // first stage's memory latency overlaps it.
    const int dw = warp - 2;
    const int grp = dw >> 2;          // dequantisation group: stages grp, grp + DQ, ...
    const int quad = warp & 3;        // TMEM lane quadrant this warp may access
    const int j = quad * 32 + lane;   // weight column inside the tile = TMEM lane
    const int n = nt * kTileN + j;
    const bool col_ok = n < p.N;
    const uint32_t tlane = static_cast<uint32_t>(quad * 32) << 16;
    // Codes and scales of this thread's stages (i = grp, grp + DQ, ...) are
    // loaded kAhead of its stages ahead into registers: the two 16-byte
    // halves (k 0..31 and 32..63) of the column's stage and its scales (one
    // when G is a multiple of 64, else one per 8-deep word). Loaded values
    // are left exactly as loaded until the stage is decoded: any instruction
    // that reads a register whose load is in flight waits for that load.
    // kk is the first k of the next stage to load, gk = floor(kk / G).
    // (A padded column past N reads column 0's scales; its codes are 0.)
    const uint8_t* wcol = p.wt[expert] + static_cast<int64_t>(nt) * p.KT * kTileBytes + j * 16;
    const __half* scol = p.sc[expert] + (col_ok ? n : 0);
    int li = grp;
    int kk = (kb + grp) * kTileK;
    int gk = kk / p.G;
    auto load_next = [&](uint4 (&r)[kChunks], __half (&sv)[kScales]) {
        if (li < nst) {
            const uint8_t* src = wcol + static_cast<int64_t>(kb + li) * kTileBytes;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) r[c] = ld_nc_v4(src + c * 2048);
            if constexpr (OG) {
                sv[0] = __ldg(scol + static_cast<int64_t>(min(gk, p.ngroups - 1)) * p.N);
            } else {
                const int rem = kk - gk * p.G;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    int g = gk, r2 = rem + 8 * q;
                    while (r2 >= p.G) {
                        r2 -= p.G;
                        ++g;
                    }
                    sv[q] = __ldg(scol + static_cast<int64_t>(min(g, p.ngroups - 1)) * p.N);
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) r[c] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int q = 0; q < kScales; ++q) sv[q] = __float2half(0.f);
        }
        li += DQ;
        kk += kTileK * DQ;
        while ((gk + 1) * p.G <= kk) ++gk;
    };
    uint4 rq0[kChunks], rq1[kChunks];
    __half sq0[kScales], sq1[kScales];
    if (warp >= 2) {
        if (!p.prefetch) grid_dependency_wait();  // weights and scales may come from the previous kernel
        load_next(rq0, sq0);
        load_next(rq1, sq1);
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < LS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&done[s], 1);
        }
        for (int q = 0; q < LS / 2; ++q) mbar_init(&afull[q], 2 * kGroupWarps);
        mbar_init(accfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensor_map(&tmA);
        grid_launch_dependents();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_acc = *tmem_slot;                 // accumulator: columns [0, BN)
    const uint32_t tmem_ring = tmem_acc + L::kAccCols;    // weight slots: kSlotCols columns each

    if (warp == 0) {
        // ------------------------------------------------------ producer
        // A stage's slot is free again once the MMAs that read it completed
        // (which also means the dequantisation warps finished reading it).
        if (lane == 0) {
            grid_dependency_wait();  // the activations may be written by the previous kernel
            // The int4 tile of a stage is one contiguous 4 KB block: pull it into
            // L2 kPrefetchStages ahead, so that the dequantising threads' own
            // loads (issued only kAhead of their stages ahead) find it there.
            // (The ring's first LS activation tiles go out before the prefetches.)
            const uint8_t* wtile = p.wt[expert] + (static_cast<int64_t>(nt) * p.KT + kb) * kTileBytes;
            const int first = min(nst, LS);
            for (int i = 0; i < first; ++i) issue_act(i);
            for (int i = 0; i < min(nst, kPrefetchStages + first); ++i)
                bulk_prefetch_l2(wtile + static_cast<int64_t>(i) * kTileBytes, kTileBytes);
            int issued = first;
            for (; issued < nst; ++issued) {
                const int i = issued;
                if (i >= LS &&
                    !wait_phase(&done[i % LS], static_cast<uint32_t>((i / LS) - 1) & 1u, abort_flag, p.wait_limit))
                    break;
                issue_act(i);
                if (i + kPrefetchStages < nst)
                    bulk_prefetch_l2(wtile + static_cast<int64_t>(i + kPrefetchStages) * kTileBytes, kTileBytes);
            }
            // Every issued copy must land before the CTA's shared memory is released.
            for (int i = max(0, issued - LS); i < issued; ++i)
                drain_phase(&full[i % LS], static_cast<uint32_t>(i / LS) & 1u);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // One barrier per pair of stages covers both operands of both stages:
            // the dequantised weights and, through each group's first warp, the
            // landed activation tiles. (Each wait costs the single issuing thread
            // about as long as an MMA, so it is paid once per eight MMAs.)
            // (The ring is unrolled: each slot's descriptors are constants.)
            const uint64_t bdesc0 = smem_desc_k_sw128(smem_addr(smem + L::kAct));
            bool stop = false;
            for (int base = 0; base < nst && !stop; base += LS) {
                const uint32_t par = static_cast<uint32_t>(base / LS) & 1u;
#pragma unroll
                for (int qq = 0; qq < LS / 2; ++qq) {
                    const int i = base + 2 * qq;
                    if (i >= nst) break;
                    if (!wait_phase(&afull[qq], par, abort_flag, p.wait_limit)) {
                        stop = true;
                        break;
                    }
                    tc_fence_after_sync();
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (i + t < nst) {
                            constexpr uint64_t kStep = static_cast<uint64_t>(L::kActBytes >> 4);
                            const int s = 2 * qq + t;
                            const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(s) * kStep;
                            const uint32_t a0 = tmem_ring + static_cast<uint32_t>(s * kSlotCols);
                            mma_f16_ts(tmem_acc, a0, bdesc, idesc, (i + t) > 0 ? 1u : 0u);
                            mma_f16_ts(tmem_acc, a0 + 8, bdesc + 2, idesc, 1u);
                            mma_f16_ts(tmem_acc, a0 + 16, bdesc + 4, idesc, 1u);
                            mma_f16_ts(tmem_acc, a0 + 24, bdesc + 6, idesc, 1u);
                            mma_commit(&done[s]);
                        }
                    }
                }
            }
            mma_commit(accfull);  // fires once every MMA issued above has completed
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ dequant + epilogue
        // One stage: decode the codes and scales held in (r, sv), refill them
        // with the thread's stage kAhead of its stages later, store the fp16
        // weights into the stage's TMEM slot and arrive. False when aborting.
        auto stage = [&](int i, uint4 (&r)[kChunks], __half (&sv)[kScales]) -> bool {
            const int s = i % LS;
            uint32_t v[2][16];  // (k, k+1) pairs: k 0..31, k 32..63
            if constexpr (BITS == 4) {
                const uint32_t raw[8] = {r[0].x, r[0].y, r[0].z, r[0].w, r[1].x, r[1].y, r[1].z, r[1].w};
#pragma unroll
                for (int q = 0; q < 8; ++q) {  // word q: k 8q .. 8q+7
                    const uint4 o = dequant_word(raw[q], __half2half2(sv[OG ? 0 : q]));
                    v[q >> 2][4 * (q & 3)] = o.x;
                    v[q >> 2][4 * (q & 3) + 1] = o.y;
                    v[q >> 2][4 * (q & 3) + 2] = o.z;
                    v[q >> 2][4 * (q & 3) + 3] = o.w;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {  // chunk c: k 16c .. 16c+15
                    const uint32_t raw[4] = {r[c].x, r[c].y, r[c].z, r[c].w};
#pragma unroll
                    for (int w = 0; w < 4; ++w) {  // word w: k 16c+4w .. +3, scale word (16c+4w)/8
                        const uint2 o = dequant_word8(raw[w], __half2half2(sv[OG ? 0 : 2 * c + (w >> 1)]));
                        const int pr = 8 * c + 2 * w;  // index of the pair (k, k+1) with k = 16c+4w
                        v[pr >> 4][pr & 15] = o.x;
                        v[pr >> 4][(pr & 15) + 1] = o.y;
                    }
                }
            }
            load_next(r, sv);
            // (Columns past N hold code 0 in the tiled layout and get scale 0: v is 0.)
            if (i >= LS &&
                !warp_wait_phase(&done[s], static_cast<uint32_t>((i / LS) - 1) & 1u, abort_flag, p.wait_limit))
                return false;
            tc_fence_after_sync();
            tmem_st_32x32b_x16(tmem_ring + tlane + s * kSlotCols, v[0]);
            tmem_st_32x32b_x16(tmem_ring + tlane + s * kSlotCols + 16, v[1]);
            tmem_st_wait();
            tc_fence_before_sync();
            // The group's first warp also sees the stage's activation tile land,
            // so that the MMA thread waits on one barrier per stage pair. The
            // last stage of an odd count arrives for its missing partner too.
            if ((dw & 3) == 0 &&
                !warp_wait_phase(&full[s], static_cast<uint32_t>(i / LS) & 1u, abort_flag, p.wait_limit))
                return false;
            __syncwarp();
            if (lane == 0 && i != p.stall_stage)
                mbar_arrive_cnt(&afull[(i >> 1) % (LS / 2)], ((i & 1) == 0 && i + 1 == nst) ? 2u : 1u);
            return true;
        };
        // kAhead = 2 register slots, used alternately: a stage's codes stay in
        // the registers they were loaded into (moving a register whose load is
        // still in flight would wait for that load).
        static_assert(kAhead == 2, "the stage loop below alternates two register slots");
        for (int i = grp; i < nst; i += 2 * DQ) {
            if (!stage(i, rq0, sq0)) break;
            if (i + DQ < nst && !stage(i + DQ, rq1, sq1)) break;
        }

        // -------------------------------------------------- epilogue
        // The accumulator is complete (or the CTA is aborting) once accfull fires;
        // either way no MMA may still run when TMEM is released.
        const bool drained = warp_drain_phase(accfull, 0);
        tc_fence_after_sync();
        grid_dependency_wait();  // the output may still be read by the previous kernel
        const int aborted = __shfl_sync(0xffffffffu, *abort_flag, 0);
        const bool have_acc = drained && !aborted && nst > 0;
        if (dw == 0 && lane == 0) tile_info[4] = have_acc ? 1 : 0;
        if (p.splits == 1) {
            // Stage the fp16 tile, row-major [token][128 columns], in the idle
            // activation ring (every copy into it was consumed by a completed
            // MMA), so that the global stores below are whole 16-byte vectors.
            // Two 16-token chunks per TMEM wait.
            if (have_acc) {
                __half* stile = reinterpret_cast<__half*>(smem + L::kAct);
                const int nch = n_mma / 16;
                for (int c = grp; c < nch; c += 2 * DQ) {
                    const bool two = c + DQ < nch;
                    uint32_t v[16], w[16];
                    tmem_ld_32x32b_x16(tmem_acc + tlane + c * 16, v);
                    if (two) tmem_ld_32x32b_x16(tmem_acc + tlane + (c + DQ) * 16, w);
                    tmem_ld_wait();
                    const int act = p.act;
                    if (act == W4A16_ACT_IDENTITY) {
#pragma unroll
                        for (int t = 0; t < 16; ++t)
                            stile[(c * 16 + t) * kTileN + j] = __float2half_rn(__uint_as_float(v[t]));
                        if (two) {
#pragma unroll
                            for (int t = 0; t < 16; ++t)
                                stile[((c + DQ) * 16 + t) * kTileN + j] = __float2half_rn(__uint_as_float(w[t]));
                        }
                    } else {
                        for (int t = 0; t < 16; ++t)
                            stile[(c * 16 + t) * kTileN + j] = epilogue_value(__uint_as_float(v[t]), act);
                        if (two) {
                            for (int t = 0; t < 16; ++t)
                                stile[((c + DQ) * 16 + t) * kTileN + j] = epilogue_value(__uint_as_float(w[t]), act);
                        }
                    }
                }
            }
        } else {
            float* red = reinterpret_cast<float*>(smem + L::kAct);
            for (int c = grp; c < BN / 16; c += DQ) {
                uint32_t v[16];
                if (have_acc && c * 16 < n_mma) {
                    tmem_ld_32x32b_x16(tmem_acc + tlane + c * 16, v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int t = 0; t < 16; ++t) v[t] = 0u;
                }
#pragma unroll
                for (int t = 0; t < 16; ++t) red[(c * 16 + t) * kTileN + j] = __uint_as_float(v[t]);
            }
        }
        tc_fence_before_sync();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_acc, TMEM_COLS);
    }

    if (p.splits == 1 && tile_info[4]) {
        // Row r of the tile is 16 chunks of 8 columns; a warp writes two rows
        // per instruction.
        const __half* stile = reinterpret_cast<const __half*>(smem + L::kAct);
        const int n0 = nt * kTileN;
        for (int o = threadIdx.x; o < rows * 16; o += static_cast<int>(blockDim.x)) {
            const int r = o >> 4;
            const int cc = (o & 15) * 8;
            __half* dst = p.C + static_cast<int64_t>(m0 + r) * p.N + n0 + cc;
            if (p.vec_out && n0 + cc + 8 <= p.N) {
                *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(stile + r * kTileN + cc);
            } else {
                for (int e = 0; e < 8 && n0 + cc + e < p.N; ++e) dst[e] = stile[r * kTileN + cc + e];
            }
        }
    }

    if (p.splits > 1) {
        // Sum the cluster's partial tiles in rank order; rank r writes columns
        // [r*128/S, (r+1)*128/S) of the tile.
        cluster_sync_all();
        const int S = p.splits;
        const int cw = kTileN / S;
        const int rank = static_cast<int>(cluster_ctarank());
        const float* red = reinterpret_cast<const float*>(smem + L::kAct);
        // A CTA that stopped early left its partial tile incomplete: if any CTA of
        // the cluster did, none writes the tile.
        bool aborted = false;
        for (int src = 0; src < S; ++src)
            aborted |= __float_as_int(ld_dsmem_f32(const_cast<int*>(abort_flag), static_cast<uint32_t>(src))) != 0;
        for (int o = threadIdx.x; o < cw * rows; o += static_cast<int>(blockDim.x)) {
            const int col = rank * cw + (o % cw);
            const int tok = o / cw;
            const int nn = nt * kTileN + col;
            if (nn < p.N && !aborted) {
                float part[8];
#pragma unroll
                for (int src = 0; src < 8; ++src)
                    part[src] = src < S ? ld_dsmem_f32(&red[tok * kTileN + col], static_cast<uint32_t>(src)) : 0.f;
                float acc = 0.f;
#pragma unroll
                for (int src = 0; src < 8; ++src) acc += part[src];  // rank order
                p.C[static_cast<int64_t>(m0 + tok) * p.N + nn] = __float2half_rn(acc);
            }
        }
        cluster_sync_all();
    }
}

// ====================================================================== host

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

struct Variant {
    int bn;
    int threads;
    int nominal_per_sm;  // the residency the variant is sized for (used when no device is present)
    int tmem_cols;       // TMEM columns each resident CTA allocates
    int smem;
    // [2 * (8-bit codes) + (any G)]: forms for int4 / 8-bit codes, with G a multiple
    // of 64 (one scale per stage) or any G
    const void* fn[4];
    int (*launch[4])(const CUtensorMap&, const Params&, dim3, int, int, cudaStream_t);
};

template <int BN, int LS, int TC, int MINB, int DQ, bool OG, int BITS>
int launch_variant(const CUtensorMap& map, const Params& p, dim3 grid, int cluster_x, int smem, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads_for(DQ), 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (cluster_x > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = static_cast<unsigned>(cluster_x);
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, w4a16_gemm_kernel<BN, LS, TC, MINB, DQ, OG, BITS>, map, p);
    return e == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}

template <int BN, int LS, int TC, int MINB, int DQ>
Variant make_variant() {
    return Variant{BN,
                   threads_for(DQ),
                   MINB,
                   TC,
                   Layout<BN, LS, TC>::kAlloc,
                   {reinterpret_cast<const void*>(&w4a16_gemm_kernel<BN, LS, TC, MINB, DQ, true, 4>),
                    reinterpret_cast<const void*>(&w4a16_gemm_kernel<BN, LS, TC, MINB, DQ, false, 4>),
                    reinterpret_cast<const void*>(&w4a16_gemm_kernel<BN, LS, TC, MINB, DQ, true, 8>),
                    reinterpret_cast<const void*>(&w4a16_gemm_kernel<BN, LS, TC, MINB, DQ, false, 8>)},
                   {&launch_variant<BN, LS, TC, MINB, DQ, true, 4>, &launch_variant<BN, LS, TC, MINB, DQ, false, 4>,
                    &launch_variant<BN, LS, TC, MINB, DQ, true, 8>, &launch_variant<BN, LS, TC, MINB, DQ, false, 8>}};
}

// Token tiles and their pipeline depths: small tiles keep two CTAs per SM; the
// 256-row tile (one CTA per SM) runs four dequantisation groups of four warps
// (576 threads): each group has four stage periods to decode and store its
// stage. More groups (more warps competing for issue slots, and register
// spills above five) and fewer groups (too little time per stage) both ran
// slower on the prefill and grouped-expert shapes.
// <token tile, ring stages, TMEM columns, CTAs per SM, dequantisation groups>
const Variant kVariants[] = {
    make_variant<16, 6, 256, 2, 2>(),  make_variant<32, 6, 256, 2, 2>(),  make_variant<64, 6, 256, 2, 2>(),
    make_variant<128, 4, 256, 2, 2>(), make_variant<192, 8, 512, 1, 4>(), make_variant<256, 6, 512, 1, 4>(),
};
constexpr int kNumVariants = sizeof(kVariants) / sizeof(kVariants[0]);

const Variant& variant_for(int bn) {
    for (const Variant& v : kVariants)
        if (v.bn == bn) return v;
    return kVariants[kNumVariants - 1];
}

struct DeviceState {
    bool ready = false;
    int ctas_per_sm[2][kNumVariants] = {};  // [8-bit codes][variant]
};

int prepare_device(DeviceState** out) {
    static DeviceState states[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return W4A16_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    DeviceState& st = states[dev];
    if (!st.ready) {
        for (int i = 0; i < 2 * kNumVariants; ++i) {
            const Variant& v = kVariants[i % kNumVariants];
            const int b8 = i / kNumVariants;
            int n = 1 << 30;
            for (int f = 2 * b8; f < 2 * b8 + 2; ++f) {
                const void* fn = v.fn[f];
                if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem) != cudaSuccess ||
                    cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         cudaSharedmemCarveoutMaxShared) != cudaSuccess)
                    return W4A16_ERR_CUDA;
                // Residency from the SM's limits (shared memory with its per-block
                // reservation, registers per warp, threads, TMEM columns); the
                // smaller of the variant's two forms.
                cudaFuncAttributes fa;
                if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return W4A16_ERR_CUDA;
                int smem_sm = 0, resv = 0, regs_sm = 0, threads_sm = 0;
                cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
                cudaDeviceGetAttribute(&resv, cudaDevAttrReservedSharedMemoryPerBlock, dev);
                cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
                cudaDeviceGetAttribute(&threads_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev);
                const int per_warp_regs = ((fa.numRegs * 32 + 255) / 256) * 256;
                n = std::min(n, smem_sm / (v.smem + static_cast<int>(fa.sharedSizeBytes) + resv));
                n = std::min(n, regs_sm / (per_warp_regs * (v.threads / 32)));
                n = std::min(n, threads_sm / v.threads);
                n = std::min(n, 512 / v.tmem_cols);  // every resident CTA holds its TMEM columns
            }
            if (n < 1) return W4A16_ERR_UNSUPPORTED;
            st.ctas_per_sm[b8][i % kNumVariants] = n;
        }
        st.ready = true;
    }
    *out = &st;
    return W4A16_OK;
}

int variant_index(int bn) {
    for (int i = 0; i < kNumVariants; ++i)
        if (kVariants[i].bn == bn) return i;
    return kNumVariants - 1;
}

int token_tile_for(int64_t rows_per_tile) {
    if (rows_per_tile <= 16) return 16;
    if (rows_per_tile <= 32) return 32;
    if (rows_per_tile <= 64) return 64;
    if (rows_per_tile <= 128) return 128;
    if (rows_per_tile <= 192) return 192;
    return 256;
}

int check_shape(int64_t N, int64_t K, int64_t G) {
    if (N <= 0 || K <= 0 || G <= 0) return W4A16_ERR_INVALID_ARG;
    if (N % 8 || K % 8 || G % 16) return W4A16_ERR_UNSUPPORTED;
    if (N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    return W4A16_OK;
}

struct Plan {
    int bn;
    int splits;
    dim3 grid;
    int smem;
    int ctas_per_sm;
};

// bn_force / splits_force > 0 select a tactic's token tile and K split (the
// split only with a single token tile, a power of two that leaves every
// cluster rank at least two K stages); 0 takes the heuristic.
int plan_dense(int64_t M, int64_t N, int64_t K, Plan* plan, bool need_device, int bn_force = 0,
               int splits_force = 0, int bits = 4) {
    const int bn = bn_force > 0 ? bn_force : token_tile_for(M);
    if (variant_for(bn).bn != bn) return W4A16_ERR_UNSUPPORTED;
    const int vi = variant_index(bn);
    int per_sm = kVariants[vi].nominal_per_sm, sms = 148;
    if (need_device) {
        DeviceState* st = nullptr;
        int rc = prepare_device(&st);
        if (rc) return rc;
        per_sm = st->ctas_per_sm[bits == 8 ? 1 : 0][vi];
        sms = sm_count();
    }
    const int64_t NT = (N + kTileN - 1) / kTileN;
    const int64_t MT = (M + bn - 1) / bn;
    const int64_t KT = (K + kTileK - 1) / kTileK;
    if (NT > 65535 || MT > 65535) return W4A16_ERR_UNSUPPORTED;
    int splits = 1;
    if (splits_force > 0) {
        if ((splits_force & (splits_force - 1)) || splits_force > 8 ||
            (splits_force > 1 && (MT != 1 || KT < 2 * splits_force)))
            return W4A16_ERR_UNSUPPORTED;
        splits = splits_force;
    } else if (MT == 1) {
        const int64_t slots = static_cast<int64_t>(sms) * per_sm;
        while (splits < 8 && NT * splits * 2 <= slots && KT >= splits * 4) splits *= 2;
    }
    plan->bn = bn;
    plan->splits = splits;
    plan->grid = dim3(static_cast<unsigned>(splits), static_cast<unsigned>(NT), static_cast<unsigned>(MT));
    plan->smem = kVariants[vi].smem;
    plan->ctas_per_sm = per_sm;
    return W4A16_OK;
}

int plan_grouped(int64_t E, int64_t total_rows, int64_t N, int64_t K, Plan* plan, bool need_device) {
    // Token tile sized for an expert's average row count with headroom, so that
    // most experts need one tile; each tile's MMA covers only its valid rows
    // rounded up to 16.
    const int64_t avg = (total_rows + E - 1) / E;
    const int bn = token_tile_for(avg + avg / 4);
    const int vi = variant_index(bn);
    int per_sm = kVariants[vi].nominal_per_sm;
    if (need_device) {
        DeviceState* st = nullptr;
        int rc = prepare_device(&st);
        if (rc) return rc;
        per_sm = st->ctas_per_sm[0][vi];
    }
    const int64_t NT = (N + kTileN - 1) / kTileN;
    const int64_t slots = total_rows / bn + E;  // >= sum over experts of ceil(rows_e / bn)
    if (NT > 65535 || slots > 65535) return W4A16_ERR_UNSUPPORTED;
    (void)K;
    plan->bn = bn;
    plan->splits = 1;
    plan->grid = dim3(1, static_cast<unsigned>(NT), static_cast<unsigned>(slots));
    plan->smem = kVariants[vi].smem;
    plan->ctas_per_sm = per_sm;
    return W4A16_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void fill_info(const Plan& plan, w4a16_launch_info* info) {
    info->token_tile = plan.bn;
    info->k_splits = plan.splits;
    info->grid_x = static_cast<int32_t>(plan.grid.x);
    info->grid_y = static_cast<int32_t>(plan.grid.y);
    info->grid_z = static_cast<int32_t>(plan.grid.z);
    info->threads_per_cta = variant_for(plan.bn).threads;
    info->smem_bytes = plan.smem;
    info->ctas_per_sm = plan.ctas_per_sm;
}

// ---------------------------------------------------------------- tactics
// A tactic is one launch form of w4a16_gemm for a shape (the plugin page's
// getValidTactics / setTactic): the skinny kernel with a given K split, K
// halves and ring depth (M <= 16 only), or the tensor-core kernel with a given
// token tile and K split. Ids are 1-based positions in the shape's list of
// valid forms, skinny forms first; 0 means the built-in heuristic.
struct Choice {
    bool skinny;
    SkinnyPlan sk;
    Plan tc;
};

constexpr int kTileChoices[] = {16, 32, 64, 128, 192, 256};

void enumerate_tactics(int64_t M, int64_t N, int64_t K, int64_t G, bool need_device, Choice* out, int* count,
                       int capacity) {
    int n = 0;
    auto push = [&](const Choice& c) {
        if (n < capacity) out[n] = c;
        ++n;
    };
    if (M <= kSkinnyMaxM) {
        for (int kh = 1; kh <= 2; ++kh)
            for (int splits = 1; splits <= 8; ++splits)
                for (int deep = 0; deep <= 1; ++deep) {
                    Choice c{};
                    c.skinny = true;
                    if (skinny_plan_fill(M, N, K, G, splits, kh, deep, &c.sk) == W4A16_OK) push(c);
                }
    }
    for (int bn : kTileChoices)
        for (int splits = 1; splits <= 8; splits *= 2) {
            Choice c{};
            c.skinny = false;
            if (plan_dense(M, N, K, &c.tc, need_device, bn, splits) == W4A16_OK) push(c);
        }
    *count = n;
}

constexpr int kMaxTactics = 96;

int tactic_choice(int64_t M, int64_t N, int64_t K, int64_t G, int tactic, bool need_device, Choice* out) {
    Choice all[kMaxTactics];
    int n = 0;
    enumerate_tactics(M, N, K, G, need_device, all, &n, kMaxTactics);
    if (tactic < 1 || tactic > n || tactic > kMaxTactics) return W4A16_ERR_INVALID_ARG;
    *out = all[tactic - 1];
    return W4A16_OK;
}

struct TacticKey {
    int dev;
    int64_t M, N, K, G;
    bool operator==(const TacticKey& o) const {
        return dev == o.dev && M == o.M && N == o.N && K == o.K && G == o.G;
    }
};
struct TacticKeyHash {
    size_t operator()(const TacticKey& k) const {
        uint64_t h = static_cast<uint64_t>(k.dev) * 0x9E3779B97F4A7C15ull;
        for (int64_t v : {k.M, k.N, k.K, k.G}) h = (h ^ static_cast<uint64_t>(v)) * 0x100000001B3ull;
        return static_cast<size_t>(h);
    }
};
struct TacticEntry {
    int tactic;
    Choice choice;
};

std::mutex g_tactic_mu;
std::unordered_map<TacticKey, TacticEntry, TacticKeyHash> g_tactics;
std::atomic<int> g_tactic_count{0};  // lets the GEMM skip the lookup while the table is empty

int current_device() {
    int dev = 0;
    return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

// The table's choice for a shape on the current device, if it holds one.
bool lookup_tactic(int64_t M, int64_t N, int64_t K, int64_t G, Choice* out, int* tactic) {
    if (g_tactic_count.load(std::memory_order_acquire) == 0) return false;
    const TacticKey key{current_device(), M, N, K, G};
    std::lock_guard<std::mutex> lock(g_tactic_mu);
    auto it = g_tactics.find(key);
    if (it == g_tactics.end()) return false;
    *out = it->second.choice;
    if (tactic) *tactic = it->second.tactic;
    return true;
}

void store_tactic(int64_t M, int64_t N, int64_t K, int64_t G, int tactic, const Choice& c) {
    const TacticKey key{current_device(), M, N, K, G};
    std::lock_guard<std::mutex> lock(g_tactic_mu);
    if (tactic == 0) {
        g_tactics.erase(key);
    } else {
        g_tactics[key] = TacticEntry{tactic, c};
    }
    g_tactic_count.store(static_cast<int>(g_tactics.size()), std::memory_order_release);
}

// The table's tactic for the shape, else the heuristic: the skinny kernel for
// decode-sized M, the tensor-core kernel otherwise.
int choose(int64_t M, int64_t N, int64_t K, int64_t G, bool need_device, Choice* c) {
    if (lookup_tactic(M, N, K, G, c, nullptr)) return W4A16_OK;
    c->skinny = skinny_plan(M, N, K, G, &c->sk) == W4A16_OK;
    if (c->skinny) return W4A16_OK;
    return plan_dense(M, N, K, &c->tc, need_device);
}

void fill_info_skinny(const SkinnyPlan& sk, w4a16_launch_info* info) {
    info->token_tile = 8 * sk.mt;
    info->k_splits = sk.splits;
    info->grid_x = sk.grid_x;
    info->grid_y = sk.grid_y;
    info->grid_z = 1;
    info->threads_per_cta = sk.threads;
    info->smem_bytes = sk.smem;
    info->ctas_per_sm = (228 * 1024) / (sk.smem + 1024) < 2 ? (228 * 1024) / (sk.smem + 1024) : 2;
}

}  // namespace

int launch_choice(const Choice& c, const w4a16_half* A_dev, const uint8_t* Wt_dev, const w4a16_half* S_dev,
                  w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G, cudaStream_t stream);
int dense_launch(const Plan& plan, int bits, const w4a16_half* A_dev, const uint8_t* Wt_dev,
                 const w4a16_half* S_dev, w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G,
                 cudaStream_t stream);

int activation_map(CUtensorMap* map, const void* A, int64_t rows, int64_t K, int box_rows) {
    // A small per-thread cache: the encoder costs more than the rest of a
    // decode-sized call on the host, and the same activation buffers recur.
    struct Entry {
        const void* A;
        int64_t rows, K;
        int box, dev;
        CUtensorMap map;
    };
    constexpr int kEntries = 16;
    thread_local Entry cache[kEntries];
    thread_local int used = 0, next = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W4A16_ERR_CUDA;
    for (int i = 0; i < used; ++i) {
        const Entry& e = cache[i];
        if (e.A == A && e.rows == rows && e.K == K && e.box == box_rows && e.dev == dev) {
            *map = e.map;
            return W4A16_OK;
        }
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return W4A16_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(A), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return W4A16_ERR_CUDA;
    Entry& e = cache[next];
    e.A = A;
    e.rows = rows;
    e.K = K;
    e.box = box_rows;
    e.dev = dev;
    e.map = *map;
    next = (next + 1) % kEntries;
    if (used < kEntries) ++used;
    return W4A16_OK;
}

int make_half_map_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                     uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return W4A16_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? W4A16_OK : W4A16_ERR_CUDA;
}

int check_device() {
    // per device: 0 unknown, 1 supported, 2 not (cached: this runs on every call)
    static std::atomic<int> state[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return W4A16_ERR_UNSUPPORTED;
    }
    if (dev < 0 || dev >= 64) return W4A16_ERR_UNSUPPORTED;
    int st = state[dev].load(std::memory_order_acquire);
    if (st == 0) {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return W4A16_ERR_UNSUPPORTED;
        }
        st = (major == 10) ? 1 : 2;
        state[dev].store(st, std::memory_order_release);
    }
    return st == 1 ? W4A16_OK : W4A16_ERR_UNSUPPORTED;
}

namespace {
std::atomic<int> g_static_weights{0};
std::atomic<long long> g_wait_limit{kTimeoutCycles};  // test aid: w4a16_set_fault_injection
std::atomic<int> g_stall_stage{-1};
}

// Set by w4a16_gemm_ex for the duration of one call on this host thread.
thread_local int t_call_static_weights = 0;

bool static_weights_enabled() {
    return t_call_static_weights != 0 || g_static_weights.load(std::memory_order_relaxed) != 0;
}

int sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    n = cached[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace w4a16

using namespace w4a16;

extern "C" const char* w4a16_status_string(int status) {
    switch (status) {
        case W4A16_OK: return "ok";
        case W4A16_ERR_INVALID_ARG: return "invalid argument";
        case W4A16_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case W4A16_ERR_UNSUPPORTED: return "unsupported shape or device";
        case W4A16_ERR_CUDA: return "CUDA runtime error";
        case W4A16_ERR_TIMEOUT: return "bounded device wait ran out";
        case W4A16_ERR_BAD_OFFSETS: return "malformed expert offsets";
        case W4A16_ERR_BAD_ROUTING: return "expert id or gathered-row index out of range";
        case W4A16_ERR_SCRATCH_TOO_SMALL: return "shape needs more than the static scratch of the no-allocation entry point";
        default: return "unknown status";
    }
}

extern "C" int w4a16_set_static_weights(int enable) {
    const int previous = g_static_weights.exchange(enable ? 1 : 0);
    return previous;
}

extern "C" int w4a16_gemm_launch_info(int64_t M, int64_t N, int64_t K, int64_t G, w4a16_launch_info* info) {
    if (!info || M <= 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (M >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    const bool dev = check_device() == W4A16_OK;
    Choice c;
    rc = choose(M, N, K, G, dev, &c);
    if (rc) return rc;
    if (c.skinny)
        fill_info_skinny(c.sk, info);
    else
        fill_info(c.tc, info);
    return W4A16_OK;
}

extern "C" int w4a16_grouped_launch_info(int64_t E, int64_t total_rows, int64_t N, int64_t K, int64_t G,
                                         w4a16_launch_info* info) {
    if (!info || E <= 0 || E > W4A16_MAX_EXPERTS || total_rows <= 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (total_rows >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    const bool dev = check_device() == W4A16_OK;
    SkinnyPlan sk;
    if (skinny_plan_grouped(total_rows, N, K, G, &sk) == W4A16_OK) {
        fill_info_skinny(sk, info);
        info->grid_z = static_cast<int32_t>(E);
        return W4A16_OK;
    }
    Plan plan;
    rc = plan_grouped(E, total_rows, N, K, &plan, dev);
    if (rc) return rc;
    fill_info(plan, info);
    return W4A16_OK;
}

extern "C" int w4a16_gemm(const w4a16_half* A_dev, const uint8_t* Wt_dev, const w4a16_half* S_dev,
                          w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G, void* stream) {
    if (!A_dev || !Wt_dev || !S_dev || !C_dev || M < 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (M >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    if (!aligned16(A_dev) || !aligned16(Wt_dev) || !aligned16(S_dev) ||
        (reinterpret_cast<uintptr_t>(C_dev) & 1u))
        return W4A16_ERR_MISALIGNED;
    if (M == 0) return W4A16_OK;
    rc = check_device();
    if (rc) return rc;
    Choice c;
    rc = choose(M, N, K, G, true, &c);
    if (rc) return rc;
    return launch_choice(c, A_dev, Wt_dev, S_dev, C_dev, M, N, K, G, static_cast<cudaStream_t>(stream));
}

namespace w4a16 {

int launch_choice(const Choice& c, const w4a16_half* A_dev, const uint8_t* Wt_dev, const w4a16_half* S_dev,
                  w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G, cudaStream_t stream) {
    if (c.skinny) return skinny_launch(c.sk, A_dev, Wt_dev, S_dev, C_dev, M, N, K, G, stream);
    return dense_launch(c.tc, 4, A_dev, Wt_dev, S_dev, C_dev, M, N, K, G, stream);
}

// The tensor-core kernel on a dense product, int4 (bits = 4) or 8-bit codes.
int dense_launch(const Plan& plan, int bits, const w4a16_half* A_dev, const uint8_t* Wt_dev,
                 const w4a16_half* S_dev, w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G,
                 cudaStream_t stream) {
    int rc;
    Params p;
    std::memset(&p, 0, sizeof(p));
    p.wt[0] = Wt_dev;
    p.sc[0] = reinterpret_cast<const __half*>(S_dev);
    p.offsets = nullptr;
    p.C = reinterpret_cast<__half*>(C_dev);
    p.rows = static_cast<int32_t>(M);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.G = static_cast<int32_t>(G);
    p.ngroups = static_cast<int32_t>((K + G - 1) / G);
    p.KT = static_cast<int32_t>((K + kTileK - 1) / kTileK);
    p.E = 1;
    p.splits = plan.splits;
    p.grouped = 0;
    p.prefetch = static_weights_enabled() ? 1 : 0;
    p.vec_out = (N % 8) == 0 && aligned16(C_dev);
    p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
    p.stall_stage = g_stall_stage.load(std::memory_order_relaxed);

    CUtensorMap map;
    rc = activation_map(&map, A_dev, M, K, plan.bn);
    if (rc) return rc;
    const Variant& v = variant_for(plan.bn);
    return v.launch[(bits == 8 ? 2 : 0) + ((G % kTileK) ? 1 : 0)](map, p, plan.grid, plan.splits, v.smem, stream);
}

}  // namespace w4a16

namespace w4a16 {

int grouped_gemm_act(const w4a16_half* A_dev, const uint8_t* const* Wt, const w4a16_half* const* S,
                     const int32_t* offsets_dev, w4a16_half* C_dev, int64_t E, int64_t total_rows, int64_t N,
                     int64_t K, int64_t G, int act, cudaStream_t stream) {
    if (!A_dev || !Wt || !S || !offsets_dev || !C_dev || E <= 0 || E > W4A16_MAX_EXPERTS || total_rows < 0)
        return W4A16_ERR_INVALID_ARG;
    if (act < W4A16_ACT_IDENTITY || act > W4A16_ACT_GELU_TANH) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (total_rows >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    for (int64_t e = 0; e < E; ++e) {
        if (!Wt[e] || !S[e]) return W4A16_ERR_INVALID_ARG;
        if (!aligned16(Wt[e]) || !aligned16(S[e])) return W4A16_ERR_MISALIGNED;
    }
    if (!aligned16(A_dev) || (reinterpret_cast<uintptr_t>(C_dev) & 1u) ||
        (reinterpret_cast<uintptr_t>(offsets_dev) & 3u))
        return W4A16_ERR_MISALIGNED;
    if (total_rows == 0) return W4A16_OK;
    rc = check_device();
    if (rc) return rc;
    SkinnyPlan sk;
    if (skinny_plan_grouped(total_rows, N, K, G, &sk) == W4A16_OK)  // decode-sized batches: at most 16 rows in all
        return skinny_grouped_launch(sk, A_dev, Wt, reinterpret_cast<const void* const*>(S), offsets_dev, C_dev, E,
                                     total_rows, N, K, G, act, stream);
    Plan plan;
    rc = plan_grouped(E, total_rows, N, K, &plan, true);
    if (rc) return rc;

    Params p;
    std::memset(&p, 0, sizeof(p));
    for (int64_t e = 0; e < E; ++e) {
        p.wt[e] = Wt[e];
        p.sc[e] = reinterpret_cast<const __half*>(S[e]);
    }
    p.offsets = offsets_dev;
    p.C = reinterpret_cast<__half*>(C_dev);
    p.rows = static_cast<int32_t>(total_rows);
    p.N = static_cast<int32_t>(N);
    p.K = static_cast<int32_t>(K);
    p.G = static_cast<int32_t>(G);
    p.ngroups = static_cast<int32_t>((K + G - 1) / G);
    p.KT = static_cast<int32_t>((K + kTileK - 1) / kTileK);
    p.E = static_cast<int32_t>(E);
    p.splits = 1;
    p.grouped = 1;
    p.vec_out = (N % 8) == 0 && aligned16(C_dev);
    p.prefetch = 0;  // expert weights are read only after the offsets, which follow the wait
    p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
    p.stall_stage = g_stall_stage.load(std::memory_order_relaxed);
    p.act = act;

    CUtensorMap map;
    rc = activation_map(&map, A_dev, total_rows, K, plan.bn);
    if (rc) return rc;
    const Variant& v = variant_for(plan.bn);
    return v.launch[(G % kTileK) ? 1 : 0](map, p, plan.grid, 1, v.smem, stream);  // int4 forms
}

}  // namespace w4a16

extern "C" int w4a16_grouped_gemm(const w4a16_half* A_dev, const uint8_t* const* Wt, const w4a16_half* const* S,
                                  const int32_t* offsets_dev, w4a16_half* C_dev, int64_t E, int64_t total_rows,
                                  int64_t N, int64_t K, int64_t G, void* stream) {
    return grouped_gemm_act(A_dev, Wt, S, offsets_dev, C_dev, E, total_rows, N, K, G, W4A16_ACT_IDENTITY,
                            static_cast<cudaStream_t>(stream));
}

extern "C" int w4a16_grouped_gemm_act(const w4a16_half* A_dev, const uint8_t* const* Wt,
                                      const w4a16_half* const* S, const int32_t* offsets_dev, w4a16_half* C_dev,
                                      int64_t E, int64_t total_rows, int64_t N, int64_t K, int64_t G, int act,
                                      void* stream) {
    return grouped_gemm_act(A_dev, Wt, S, offsets_dev, C_dev, E, total_rows, N, K, G, act,
                            static_cast<cudaStream_t>(stream));
}

extern "C" int w4a16_device_status(int clear) {
    if (check_device() != W4A16_OK) return W4A16_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return W4A16_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return W4A16_ERR_CUDA;
    if (clear && v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return W4A16_ERR_CUDA;
    }
    const int vs = skinny_device_status(clear != 0);
    const int vq = quant_device_status(clear != 0);
    const int vm = moe_device_status(clear != 0);
    if (vs < 0 || vq < 0 || vm < 0) return W4A16_ERR_CUDA;
    return v != 0 ? v : (vs != 0 ? vs : (vq != 0 ? vq : vm));
}

extern "C" int w4a16_set_fault_injection(int64_t stall_stage, int64_t wait_limit_cycles) {
    g_stall_stage.store(stall_stage < 0 || stall_stage > (1 << 30) ? -1 : static_cast<int>(stall_stage));
    g_wait_limit.store(wait_limit_cycles > 0 ? static_cast<long long>(wait_limit_cycles) : kTimeoutCycles);
    return W4A16_OK;
}

// ---------------------------------------------------------------- tactics
extern "C" int w4a16_get_valid_tactics(int64_t M, int64_t N, int64_t K, int64_t G, int32_t* tactics,
                                       int32_t capacity, int32_t* count) {
    if (!count || M <= 0 || capacity < 0 || (capacity > 0 && !tactics)) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (M >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    Choice all[kMaxTactics];
    int n = 0;
    enumerate_tactics(M, N, K, G, check_device() == W4A16_OK, all, &n, kMaxTactics);
    n = std::min(n, kMaxTactics);
    for (int i = 0; i < n && i < capacity; ++i) tactics[i] = i + 1;
    *count = n;
    return W4A16_OK;
}

extern "C" int w4a16_tactic_launch_info(int64_t M, int64_t N, int64_t K, int64_t G, int32_t tactic,
                                        w4a16_launch_info* info) {
    if (!info || M <= 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (M >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    Choice c;
    rc = tactic_choice(M, N, K, G, tactic, check_device() == W4A16_OK, &c);
    if (rc) return rc;
    if (c.skinny)
        fill_info_skinny(c.sk, info);
    else
        fill_info(c.tc, info);
    return W4A16_OK;
}

extern "C" int w4a16_set_tactic(int64_t M, int64_t N, int64_t K, int64_t G, int32_t tactic) {
    if (M <= 0 || tactic < 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (M >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    Choice c{};
    if (tactic > 0) {
        rc = tactic_choice(M, N, K, G, tactic, check_device() == W4A16_OK, &c);
        if (rc) return rc;
    }
    store_tactic(M, N, K, G, tactic, c);
    return W4A16_OK;
}

extern "C" int w4a16_get_tactic(int64_t M, int64_t N, int64_t K, int64_t G, int32_t* tactic) {
    if (!tactic) return W4A16_ERR_INVALID_ARG;
    Choice c;
    int t = 0;
    *tactic = lookup_tactic(M, N, K, G, &c, &t) ? t : 0;
    return W4A16_OK;
}

extern "C" int w4a16_clear_tactics(void) {
    std::lock_guard<std::mutex> lock(g_tactic_mu);
    g_tactics.clear();
    g_tactic_count.store(0, std::memory_order_release);
    return W4A16_OK;
}

extern "C" int w4a16_autotune(const w4a16_half* A_dev, const uint8_t* const* Wt, const w4a16_half* const* S,
                              int32_t copies, w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G,
                              int32_t reps, int32_t* best_tactic, float* best_us, float* times_us,
                              int32_t times_capacity, void* stream) {
    if (!A_dev || !Wt || !S || !C_dev || !best_tactic || M <= 0 || copies < 1 || copies > 1024 || reps < 1 ||
        reps > 10000 || times_capacity < 0 || (times_capacity > 0 && !times_us))
        return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (M >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    for (int32_t c = 0; c < copies; ++c) {
        if (!Wt[c] || !S[c]) return W4A16_ERR_INVALID_ARG;
        if (!aligned16(Wt[c]) || !aligned16(S[c])) return W4A16_ERR_MISALIGNED;
    }
    if (!aligned16(A_dev) || (reinterpret_cast<uintptr_t>(C_dev) & 1u)) return W4A16_ERR_MISALIGNED;
    rc = check_device();
    if (rc) return rc;
    Choice all[kMaxTactics];
    int n = 0;
    enumerate_tactics(M, N, K, G, true, all, &n, kMaxTactics);
    n = std::min(n, kMaxTactics);
    if (n == 0) return W4A16_ERR_UNSUPPORTED;

    // Each tactic's `reps` launches, rotating over the weight copies, are
    // recorded on a private stream into a CUDA graph and replayed on the
    // caller's stream: back to back, as a model's layers run them, with the
    // launch overlap that programmatic dependent launch gives.
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t cap = nullptr;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    if (cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking) != cudaSuccess) return W4A16_ERR_CUDA;
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
        if (e0) cudaEventDestroy(e0);
        cudaStreamDestroy(cap);
        return W4A16_ERR_CUDA;
    }
    float best = 0.f;
    int best_id = 0;
    for (int i = 0; i < n && rc == W4A16_OK; ++i) {
        rc = launch_choice(all[i], A_dev, Wt[0], S[0], C_dev, M, N, K, G, st);  // first use outside the graph
        if (rc == W4A16_OK && cudaStreamSynchronize(st) != cudaSuccess) rc = W4A16_ERR_CUDA;
        if (rc) break;
        cudaGraph_t graph = nullptr;
        cudaGraphExec_t exec = nullptr;
        if (cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
            rc = W4A16_ERR_CUDA;
            break;
        }
        int lrc = W4A16_OK;
        for (int r = 0; r < reps && lrc == W4A16_OK; ++r)
            lrc = launch_choice(all[i], A_dev, Wt[r % copies], S[r % copies], C_dev, M, N, K, G, cap);
        const cudaError_t ce = cudaStreamEndCapture(cap, &graph);
        if (lrc != W4A16_OK || ce != cudaSuccess || cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
            rc = lrc != W4A16_OK ? lrc : W4A16_ERR_CUDA;
        } else {
            float ms = 0.f, best_ms = 0.f;
            // one warm replay, then the fastest of three timed ones
            if (cudaGraphLaunch(exec, st) != cudaSuccess) rc = W4A16_ERR_CUDA;
            for (int t = 0; t < 3 && rc == W4A16_OK; ++t) {
                if (cudaEventRecord(e0, st) != cudaSuccess || cudaGraphLaunch(exec, st) != cudaSuccess ||
                    cudaEventRecord(e1, st) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess ||
                    cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess) {
                    rc = W4A16_ERR_CUDA;
                    break;
                }
                if (t == 0 || ms < best_ms) best_ms = ms;
            }
            const float us = best_ms * 1000.f / static_cast<float>(reps);
            if (i < times_capacity) times_us[i] = us;
            if (rc == W4A16_OK && (best_id == 0 || us < best)) {
                best = us;
                best_id = i + 1;
            }
        }
        if (exec) cudaGraphExecDestroy(exec);
        if (graph) cudaGraphDestroy(graph);
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cudaStreamDestroy(cap);
    if (rc) return rc;
    store_tactic(M, N, K, G, best_id, all[best_id - 1]);
    *best_tactic = best_id;
    if (best_us) *best_us = best;
    return W4A16_OK;
}

// ---------------------------------------------------------------- W8A16
extern "C" int w8a16_gemm_launch_info(int64_t M, int64_t N, int64_t K, int64_t G, w4a16_launch_info* info) {
    if (!info || M <= 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (M >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    Plan plan;
    rc = plan_dense(M, N, K, &plan, check_device() == W4A16_OK, 0, 0, 8);
    if (rc) return rc;
    fill_info(plan, info);
    return W4A16_OK;
}

extern "C" int w8a16_gemm(const w4a16_half* A_dev, const uint8_t* Wt8_dev, const w4a16_half* S_dev,
                          w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G, void* stream) {
    if (!A_dev || !Wt8_dev || !S_dev || !C_dev || M < 0) return W4A16_ERR_INVALID_ARG;
    int rc = check_shape(N, K, G);
    if (rc) return rc;
    if (M >= (int64_t(1) << 31)) return W4A16_ERR_UNSUPPORTED;
    if (!aligned16(A_dev) || !aligned16(Wt8_dev) || !aligned16(S_dev) ||
        (reinterpret_cast<uintptr_t>(C_dev) & 1u))
        return W4A16_ERR_MISALIGNED;
    if (M == 0) return W4A16_OK;
    rc = check_device();
    if (rc) return rc;
    Plan plan;
    rc = plan_dense(M, N, K, &plan, true, 0, 0, 8);
    if (rc) return rc;
    return dense_launch(plan, 8, A_dev, Wt8_dev, S_dev, C_dev, M, N, K, G, static_cast<cudaStream_t>(stream));
}

extern "C" int w4a16_gemm_ex(const w4a16_half* A_dev, const uint8_t* Wt_dev, const w4a16_half* S_dev,
                             w4a16_half* C_dev, int64_t M, int64_t N, int64_t K, int64_t G, uint32_t flags,
                             void* stream) {
    if (flags & ~static_cast<uint32_t>(W4A16_FLAG_STATIC_WEIGHTS)) return W4A16_ERR_INVALID_ARG;
    struct CallScope {
        explicit CallScope(int v) { t_call_static_weights = v; }
        ~CallScope() { t_call_static_weights = 0; }
    } scope((flags & W4A16_FLAG_STATIC_WEIGHTS) ? 1 : 0);
    return w4a16_gemm(A_dev, Wt_dev, S_dev, C_dev, M, N, K, G, stream);
}
