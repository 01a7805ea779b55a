"""CUDA path against the CPU oracle on the same seeded inputs, through the C ABI.

Integer work (pack, unpack, repack) must be bit-exact; the GEMM must satisfy
|gpu - ref| <= 1e-2 + 5e-3 * |ref| element by element. Small cases are compared
in full; the full-size workloads in the launch configuration the benchmark uses
are compared in full as well."""
import numpy as np
import pytest
import torch

import oracle
import pins
import workloads
import weight_only_int4_wise_b200 as w
from gpu_util import dev, device_weights, guarded_output, guards_intact, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def o():
    return oracle.load()


@pytest.fixture(autouse=True)
def clean_status():
    w.device_status(clear=True)
    yield
    assert w.device_status(clear=True) == w.OK


# ------------------------------------------------------------------ packing

@pytest.mark.parametrize("K,N", [(1, 8), (7, 24), (512, 512), (4096, 4096), (4095, 136)])
def test_pack_bit_exact(o, K, N):
    q = workloads.dense(1, K, N, 16, seed=K + N).q
    wp = w.pack(dev(q))
    torch.cuda.synchronize()
    assert np.array_equal(wp.cpu().numpy(), o.pack(q))
    assert np.array_equal(w.unpack(wp, K).cpu().numpy(), q)


def test_pack_all_byte_values(o):
    wp = torch.arange(256, dtype=torch.uint8, device="cuda").view(1, 256)
    q = w.unpack(wp, 2)
    assert np.array_equal(q.cpu().numpy(), o.unpack(wp.cpu().numpy(), 2))
    assert np.array_equal(w.pack(q).cpu().numpy(), wp.cpu().numpy())


@pytest.mark.parametrize("K,N", [(64, 128), (72, 136), (200, 520), (4096, 4096), (4100, 264)])
def test_repack_bit_exact(o, K, N):
    q = workloads.dense(1, K, N, 16, seed=3 * K + N).q
    _, wt = device_weights(q)
    torch.cuda.synchronize()
    assert np.array_equal(wt.cpu().numpy(), o.tile(q))


# --------------------------------------------------------------- small GEMMs

def run_dense(o, M, K, N, G, seed, a_scale=1.0, pad=64):
    c = workloads.dense(M, K, N, G, seed, a_scale=a_scale)
    _, wt = device_weights(c.q)
    flat, C, pad = guarded_output(M, N, pad)
    w.gemm(dev(c.A), wt, dev(c.S), N, G, out=C)
    torch.cuda.synchronize()
    got = C.cpu().numpy()
    ref = o.gemm(c.A, pins.python_pack(c.q), c.S, K, G)
    ok, err, rel = within_tolerance(got, ref)
    assert ok, f"M={M} K={K} N={N} G={G}: max abs err {err}, max rel err {rel}"
    assert guards_intact(flat, pad, M * N), "the kernel wrote outside C"
    return got, ref


def test_tiny_config(o):
    cfg = workloads.CONFIGS["tiny"]
    run_dense(o, cfg["M"], cfg["K"], cfg["N"], cfg["G"], cfg["seed"])


@pytest.mark.parametrize("M", [1, 2, 3, 5, 16, 17, 33, 64, 65, 127, 129, 200, 256, 257, 300])
def test_ragged_rows(o, M):
    # several column tiles with a ragged last one, several K stages, every token-tile size
    run_dense(o, M, 200, 392, 64, seed=100 + M)


@pytest.mark.parametrize("K,N,G", [
    (64, 8, 64), (72, 136, 16), (96, 128, 32), (208, 264, 48), (200, 520, 80), (520, 256, 128),
    (512, 384, 512), (256, 128, 4096), (1024, 256, 64), (1032, 136, 16),
])
def test_shapes_and_group_sizes(o, K, N, G):
    for M in (1, 8, 40):
        run_dense(o, M, K, N, G, seed=K * 7 + N + G + M)


@pytest.mark.parametrize("M,K,N,G", [
    (5, 2176, 9480, 48),   # 17 blocks in one CTA: halves of 9 and 8; ragged last column tile
    (8, 4160, 12288, 16),  # odd number of 64-deep tiles: the last block's second tile reads as zeros
    (7, 8320, 4096, 32),   # 4-CTA cluster, 16-17 blocks per CTA; groups finer than a block
    (3, 4096, 14336, 80),  # one CTA per column tile, no cluster
])
def test_two_k_halves_per_cta(o, M, K, N, G):
    # G not a multiple of 64 runs the warp-MMA skinny kernel; one token tile over long
    # K ranges: two sets of 8 warps split the CTA's blocks
    rc, info = w.w4a16_gemm_launch_info(M, N, K, G)
    assert rc == w.OK and info.threads_per_cta == 512
    run_dense(o, M, K, N, G, seed=M + K + N + G)


@pytest.mark.parametrize("M,K,N,G", [
    (1, 4096, 4096, 128),   # 4-CTA clusters, 16 stages per CTA (more than the 14-stage ring)
    (16, 4096, 4096, 64),   # one scale group per stage
    (3, 1000, 392, 128),    # K % 64 != 0 (zero-padded last stage), ragged last column tile
    (8, 8192, 1024, 256),   # 8-CTA clusters; groups of four stages
    (5, 2048, 136, 2048),   # one group per CTA range; 8 CTAs per cluster
    (16, 960, 8, 64),       # a single 8-column tile, 15 stages split 8 ways
    (2, 192, 264, 4096),    # G > K: one group
    (12, 14336, 256, 128),  # long K ranges: every ring wraps several times
    (7, 4160, 12288, 128),  # 96 column tiles, one CTA per tile: 65 stages per CTA
])
def test_skinny_kernel_more_shapes(o, M, K, N, G):
    # decode-sized M with G a multiple of 64: clusters of 1 to 8 CTAs, ragged K and N,
    # one group per CTA range, long K ranges that wrap every ring
    rc, info = w.w4a16_gemm_launch_info(M, N, K, G)
    assert rc == w.OK and info.token_tile in (8, 16)  # the skinny kernel
    run_dense(o, M, K, N, G, seed=M * 31 + K + N + G)


def test_skinny_long_k_with_large_activations(o):
    # |A| ~ 8 over K = 14336: partial sums of tens of units stay within tolerance
    run_dense(o, 16, 14336, 256, 128, seed=78, a_scale=8.0)


@pytest.mark.parametrize("M", [2, 9, 16])
def test_skinny_kernel_two_token_tiles(o, M):
    # G = 48: the warp-MMA skinny kernel, one and two 8-row token tiles, ragged tiles
    run_dense(o, M, 1040, 392, 48, seed=900 + M)


@pytest.mark.parametrize("K,N,G", [(520, 264, 48), (1032, 136, 16), (200, 392, 80)])
def test_group_sizes_not_multiple_of_64_on_the_largest_tile(o, K, N, G):
    # 300 rows: one full 256-row tile and a ragged one; per-word scales in a stage
    run_dense(o, 300, K, N, G, seed=K + N + G)


@pytest.mark.parametrize("M", [1, 17, 300])
def test_output_rows_off_16_byte_boundaries(o, M):
    # C starts 2 bytes past a 16-byte boundary: the row stores cannot be 16-byte vectors
    run_dense(o, M, 200, 392, 64, seed=500 + M, pad=65)


def test_large_activations_stay_in_tolerance(o):
    # |A| ~ 8: outputs of tens of units exercise the relative part of the bound
    run_dense(o, 16, 2048, 256, 128, seed=77, a_scale=8.0)


def test_deterministic(o):
    c = workloads.dense(5, 4096, 512, 128, 5)
    _, wt = device_weights(c.q)
    A, S = dev(c.A), dev(c.S)
    r1 = w.gemm(A, wt, S, 512, 128).cpu().numpy()
    r2 = w.gemm(A, wt, S, 512, 128).cpu().numpy()
    assert np.array_equal(r1.view(np.uint16), r2.view(np.uint16))


# --------------------------------------------------------------- grouped

def run_grouped(o, case):
    _ = [device_weights(case.q[e]) for e in range(case.E)]
    wts = [x[1] for x in _]
    Ss = [dev(case.S[e]) for e in range(case.E)]
    flat, C, pad = guarded_output(case.total_rows, case.N)
    w.grouped_gemm(dev(case.A), wts, Ss, dev(case.offsets), case.N, case.G, out=C)
    torch.cuda.synchronize()
    got = C.cpu().numpy()
    ref = o.grouped_gemm(case.A, [pins.python_pack(case.q[e]) for e in range(case.E)], list(case.S),
                         case.offsets, case.K, case.G)
    ok, err, rel = within_tolerance(got, ref)
    assert ok, f"grouped: max abs err {err}, max rel err {rel}"
    assert guards_intact(flat, pad, case.total_rows * case.N)
    return got, ref


def test_grouped_small_with_empty_expert(o):
    run_grouped(o, workloads.grouped(E=6, top_k=2, tokens=100, K=256, N=392, G=64, seed=31, empty_experts=[1, 4]))


def test_grouped_uneven_segments(o):
    # 300 tokens routed top-1 over 3 experts: segments of about 100 rows, several token tiles
    run_grouped(o, workloads.grouped(E=3, top_k=1, tokens=300, K=512, N=256, G=128, seed=32))


def test_grouped_single_expert_equals_dense(o):
    c = workloads.dense(70, 512, 256, 128, 33)
    _, wt = device_weights(c.q)
    A, S = dev(c.A), dev(c.S)
    dense = w.gemm(A, wt, S, 256, 128)
    off = torch.tensor([0, 70], dtype=torch.int32, device="cuda")
    grouped = w.grouped_gemm(A, [wt], [S], off, 256, 128)
    torch.cuda.synchronize()
    ok, err, _ = within_tolerance(grouped.cpu().numpy(), dense.cpu().numpy())
    assert ok, err


def test_grouped_rejects_malformed_offsets_on_device():
    c = workloads.dense(8, 128, 128, 64, 34)
    _, wt = device_weights(c.q)
    A, S = dev(c.A), dev(c.S)
    for bad in ([0, 5, 3], [1, 4, 8], [0, 4, 7]):  # decreasing, nonzero start, wrong end
        flat, C, pad = guarded_output(8, 128)
        w.grouped_gemm(A, [wt, wt], [S, S], torch.tensor(bad, dtype=torch.int32, device="cuda"), 128, 64, out=C)
        assert w.device_status(clear=True) == w.ERR_BAD_OFFSETS
        assert guards_intact(flat, pad, 0) and np.all(C.cpu().numpy().view(np.uint16) == 0x7BAD)


@pytest.mark.parametrize("tokens,E,k,K,N,G", [
    (1, 8, 1, 512, 256, 128),    # one row: seven experts without rows
    (4, 8, 2, 1024, 392, 128),   # 8 rows, one token tile, ragged column tile
    (8, 6, 2, 1024, 264, 48),    # 16 rows, two token tiles, groups straddling blocks
    (3, 4, 3, 4096, 512, 64),    # 9 rows, a K split over a cluster
    (16, 8, 1, 256, 128, 32),
])
def test_grouped_decode_batches_run_on_the_skinny_kernel(o, tokens, E, k, K, N, G):
    # at most 16 gathered rows in all: the grouped product runs on the skinny kernel, one
    # grid slice per expert, experts without rows skipped
    c = workloads.grouped(E=E, top_k=k, tokens=tokens, K=K, N=N, G=G, seed=tokens * 11 + K)
    rc, info = w.w4a16_grouped_launch_info(c.E, c.total_rows, c.N, c.K, c.G)
    assert rc == w.OK and info.token_tile in (8, 16) and info.grid_z == E
    run_grouped(o, c)


def test_misaligned_pointer_is_refused():
    c = workloads.dense(4, 128, 128, 64, 35)
    _, wt = device_weights(c.q)
    A = dev(c.A)
    buf = torch.empty(4 * 128 + 8, dtype=torch.float16, device="cuda")
    rc = w.w4a16_gemm(A.data_ptr() + 2, wt, dev(c.S), buf, 4, 128, 128, 64)
    assert rc == w.ERR_MISALIGNED


# --------------------------------------------------------------- quantiser

def quant_case(K, N, G, seed, lo=0.01, hi=3.0, special=True):
    g = np.random.Generator(np.random.PCG64(seed))
    W = (g.standard_normal((K, N)) * g.uniform(lo, hi, size=(1, N))).astype(np.float16)
    if special and K > G:  # one all-zero group in column 0 and a group of exact ties (max 3.5, w = 1.25 -> 2.5)
        W[:G, 0] = 0
        W[G:min(K, 2 * G), 1] = 1.25
        W[G, 1] = 3.5
    return W


@pytest.mark.parametrize("K,N,G", [(200, 24, 64), (4096, 4096, 128), (7, 10, 2), (131, 66, 132), (1000, 520, 16),
                                   (131, 264, 64), (257, 520, 128)])
def test_quantize_bit_exact(o, K, N, G):
    # (131, 264, 64) and (257, 520, 128) take the staged kernel with K odd and not a
    # multiple of G: an odd last row pair and rows past K in the last group
    W = quant_case(K, N, G, seed=K + N + G)
    wp, S = w.quantize(dev(W), G)
    torch.cuda.synchronize()
    ref_wp, ref_S = o.quantize(W, G)
    assert np.array_equal(S.cpu().numpy().view(np.uint16), ref_S.view(np.uint16))
    assert np.array_equal(wp.cpu().numpy(), ref_wp)


def rounding_boundary_case(K, N, G, top):
    """Weights on and next to every rounding boundary of the code range: in each
    group of each column the maximum |w| is top * s with s a power of two, so the
    fp16 scale is exactly s and w / s is exact. The other rows cycle through the
    half-integers of the range (ties, rounded away from zero), their fp16
    neighbours on both sides, and the integers."""
    halves = np.arange(-top, top) + 0.5  # (|w| <= top * s, so the maximum stays top * s)
    base = np.concatenate([halves, np.arange(-top, top + 1).astype(np.float64)])
    W = np.zeros((K, N), dtype=np.float16)
    for n in range(N):
        s = 2.0 ** (-(n % 6) - 3)
        vals = (base * s).astype(np.float16)
        up = np.nextafter(vals[:len(halves)], np.float16(np.inf))
        down = np.nextafter(vals[:len(halves)], np.float16(-np.inf))
        cyc = np.concatenate([vals, up, down])
        cyc = np.roll(cyc, n)
        for g0 in range(0, K, G):
            rows = min(G, K - g0)
            col = np.resize(cyc, rows)
            col[0] = np.float16((top if (g0 // G + n) % 2 == 0 else -top) * s)
            W[g0:g0 + rows, n] = col
    return W


@pytest.mark.parametrize("K,N,G", [(512, 264, 64), (130, 24, 128)])
def test_quantize_rounding_boundaries(o, K, N, G):
    # every tie and its neighbours, on the staged (N % 8 == 0) and fallback forms
    W = rounding_boundary_case(K, N, G, top=7)
    wp, S = w.quantize(dev(W), G)
    torch.cuda.synchronize()
    ref_wp, ref_S = o.quantize(W, G)
    assert np.all(ref_S.astype(np.float32) > 0)
    assert np.array_equal(S.cpu().numpy().view(np.uint16), ref_S.view(np.uint16))
    assert np.array_equal(wp.cpu().numpy(), ref_wp)


def subnormal_scale_case(K, N, G, lo, hi, seed):
    """Weights that are small multiples of 2^-24 (fp16 subnormals): the group
    scales are subnormal too, their rounding is coarse, and quotients beyond the
    code range occur, so the clamp decides codes."""
    g = np.random.Generator(np.random.PCG64(seed))
    units = g.integers(lo, hi + 1, size=(1, N))
    k = np.rint(g.uniform(-1.0, 1.0, size=(K, N)) * units)
    return (k * 2.0 ** -24).astype(np.float16)


@pytest.mark.parametrize("K,N,G", [(256, 264, 64), (130, 24, 128)])
def test_quantize_subnormal_scales(o, K, N, G):
    W = subnormal_scale_case(K, N, G, lo=3, hi=40, seed=K + N)
    wp, S = w.quantize(dev(W), G)
    torch.cuda.synchronize()
    ref_wp, ref_S = o.quantize(W, G)
    q = o.unpack(ref_wp, K)
    assert np.any(q == 7) and np.any(q == -8)  # the clamp is reached
    assert np.array_equal(S.cpu().numpy().view(np.uint16), ref_S.view(np.uint16))
    assert np.array_equal(wp.cpu().numpy(), ref_wp)


def test_quantize_worked_example():
    # the hand-worked example (tests/golden/quantize_example.txt), one zero column added (N even)
    dims, t = pins._read_quantize_example()
    W = np.zeros((dims["K"], dims["N"] + 1), dtype=np.float16)
    W[:, :dims["N"]] = t["W"]
    wp, S = w.quantize(dev(W), dims["G"])
    q = w.unpack(wp, dims["K"]).cpu().numpy()
    torch.cuda.synchronize()
    assert np.array_equal(q[:, :dims["N"]], t["Q"].astype(np.int8)) and np.all(q[:, -1] == 0)
    expect = t["S"].astype(np.float16).view(np.uint16)
    assert np.array_equal(S.cpu().numpy()[:, :dims["N"]].view(np.uint16), expect)


def test_quantize_then_gemm(o):
    # export path: fp16 weights -> codes and scales -> tiled layout -> GEMM. Weights of
    # trained-model size (std 0.005-0.05 per column, scales about 0.002-0.02 as in the
    # workloads): the GPU rounds every dequantised weight to fp16, an error that grows
    # with |q s| and that the tolerance is sized for at these magnitudes.
    K, N, G, M = 1024, 640, 128, 24
    W = quant_case(K, N, G, seed=90, lo=0.005, hi=0.05, special=False)
    A = np.random.Generator(np.random.PCG64(91)).standard_normal((M, K)).astype(np.float16)
    wp, S = w.quantize(dev(W), G)
    wt = w.repack(wp, K)
    C = w.gemm(dev(A), wt, S, N, G)
    torch.cuda.synchronize()
    ref_wp, ref_S = o.quantize(W, G)
    ref = o.gemm(A, ref_wp, ref_S, K, G)
    ok, err, rel = within_tolerance(C.cpu().numpy(), ref)
    assert ok, f"max abs err {err}, max rel err {rel}"


# ------------------------------------------------- full-size workloads

DENSE_FULL = ["decode_m1", "decode_m16", "mlp_up", "mlp_down", "mlp_up_g64"]


@pytest.mark.parametrize("name", DENSE_FULL)
def test_full_size_skinny_configs(o, name):
    c = workloads.make(name)
    _, wt = device_weights(c.q)
    flat, C, pad = guarded_output(c.M, c.N)
    w.gemm(dev(c.A), wt, dev(c.S), c.N, c.G, out=C)
    torch.cuda.synchronize()
    got = C.cpu().numpy()
    ref = o.gemm(c.A, pins.python_pack(c.q), c.S, c.K, c.G)
    ok, err, rel = within_tolerance(got, ref)
    assert ok, f"{name}: max abs err {err}, max rel err {rel}"
    assert guards_intact(flat, pad, c.M * c.N)


def test_full_size_prefill(o):
    # every element of the 2048 x 4096 output against the oracle
    c = workloads.make("prefill")
    _, wt = device_weights(c.q)
    flat, C, pad = guarded_output(c.M, c.N)
    w.gemm(dev(c.A), wt, dev(c.S), c.N, c.G, out=C)
    torch.cuda.synchronize()
    got = C.cpu().numpy()
    assert guards_intact(flat, pad, c.M * c.N)
    ref = o.gemm(c.A, pins.python_pack(c.q), c.S, c.K, c.G)
    ok, err, rel = within_tolerance(got, ref)
    assert ok, f"prefill: max abs err {err}, max rel err {rel}"


def test_full_size_grouped(o):
    # every element of the 1024 x 14336 gathered output against the oracle
    c = workloads.make("grouped")
    rc, info = w.w4a16_grouped_launch_info(c.E, c.total_rows, c.N, c.K, c.G)
    assert rc == w.OK
    got, _ = run_grouped(o, c)
    assert np.all(np.isfinite(got))


@pytest.mark.parametrize("G", [128, 48])
def test_grouped_on_the_192_row_tile(o, G):
    # Experts of about 130 rows: the plan picks the 192-row token tile (8-stage ring,
    # four dequantisation groups), which the full grouped workload also uses.
    c = workloads.grouped(E=4, top_k=1, tokens=520, K=1024, N=392, G=G, seed=60 + G)
    rc, info = w.w4a16_grouped_launch_info(c.E, c.total_rows, c.N, c.K, c.G)
    assert rc == w.OK and info.token_tile == 192
    run_grouped(o, c)


def test_static_weights_mode(o):
    # Weights prepared (and synchronised) well before the GEMMs: with static weights
    # declared the kernels may stream them before the previous kernel finishes.
    cases = [workloads.make("decode_m16"), workloads.dense(8, 4096, 2048, 128, 51), workloads.dense(40, 1024, 640, 64, 52)]
    prepared = [(c, device_weights(c.q)[1], dev(c.A), dev(c.S)) for c in cases]
    torch.cuda.synchronize()
    previous = w.w4a16_set_static_weights(True)
    try:
        outs = [w.gemm(A, wt, S, c.N, c.G) for c, wt, A, S in prepared for _ in range(2)]
        torch.cuda.synchronize()
    finally:
        w.w4a16_set_static_weights(previous)
    for idx, (c, _, _, _) in enumerate(prepared):
        ref = o.gemm(c.A, pins.python_pack(c.q), c.S, c.K, c.G)
        for got in outs[2 * idx:2 * idx + 2]:
            ok, err, rel = within_tolerance(got.cpu().numpy(), ref)
            assert ok, f"static weights, case {idx}: max abs err {err}"


def test_static_weights_per_call(o):
    # The same promise scoped to single calls (w4a16_gemm_ex): calls with and without
    # the flag interleaved on one stream, the process-wide setting left off.
    assert w.w4a16_set_static_weights(False) == 0
    cases = [workloads.make("decode_m1"), workloads.dense(40, 1024, 640, 64, 55)]
    prepared = [(c, device_weights(c.q)[1], dev(c.A), dev(c.S)) for c in cases]
    torch.cuda.synchronize()
    outs = []
    for c, wt, A, S in prepared:
        for flags in (w.FLAG_STATIC_WEIGHTS, 0, w.FLAG_STATIC_WEIGHTS):
            C = torch.empty((c.M, c.N), dtype=torch.float16, device="cuda")
            assert w.w4a16_gemm_ex(A, wt, S, C, c.M, c.N, c.K, c.G, flags) == w.OK
            outs.append(C)
    torch.cuda.synchronize()
    assert w.w4a16_set_static_weights(False) == 0  # the call scope did not leak into the global setting
    for idx, (c, _, _, _) in enumerate(prepared):
        ref = o.gemm(c.A, pins.python_pack(c.q), c.S, c.K, c.G)
        for got in outs[3 * idx:3 * idx + 3]:
            ok, err, rel = within_tolerance(got.cpu().numpy(), ref)
            assert ok, f"per-call static weights, case {idx}: max abs err {err}"


def test_repack_then_gemm_back_to_back(o):
    # The GEMM right after the repack kernel that produced its weights, on one stream.
    for c in (workloads.dense(8, 4096, 14336, 128, 53), workloads.dense(16, 14336, 1024, 128, 54)):
        _, wt = device_weights(c.q)
        got = w.gemm(dev(c.A), wt, dev(c.S), c.N, c.G).cpu().numpy()
        ref = o.gemm(c.A, pins.python_pack(c.q), c.S, c.K, c.G)
        ok, err, rel = within_tolerance(got, ref)
        assert ok, f"repack then gemm: max abs err {err}"


def test_stage_refill_is_race_free(o):
    # K ranges longer than the skinny kernel's ring (so stages are refilled while
    # other warps still compute) must give the same bits on every run.
    for c in (workloads.dense(8, 4096, 14336, 128, 55), workloads.dense(16, 14336, 4096, 64, 56)):
        _, wt = device_weights(c.q)
        A, S = dev(c.A), dev(c.S)
        runs = [w.gemm(A, wt, S, c.N, c.G).cpu().numpy() for _ in range(4)]
        for r in runs[1:]:
            assert np.array_equal(r.view(np.uint16), runs[0].view(np.uint16))
        ok, err, _ = within_tolerance(runs[0], o.gemm(c.A, pins.python_pack(c.q), c.S, c.K, c.G))
        assert ok, f"max abs err {err}"
