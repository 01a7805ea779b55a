"""W8A16 (8-bit codes) on the GPU against the oracle: the repack into the 8-bit
tiled layout bit for bit, and the product element by element within the GEMM
tolerance 1e-2 + 5e-3 |ref|, on ragged shapes, every group size form, decode
and prefill sizes."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import weight_only_int4_wise_b200 as w
from gpu_util import dev, guarded_output, guards_intact, within_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def o():
    return oracle.load()


@pytest.mark.parametrize("K,N", [(64, 128), (72, 136), (130, 200), (4096, 264)])
def test_repack_w8_bit_exact(o, K, N):
    q = np.random.Generator(np.random.PCG64(K + N)).integers(-128, 128, size=(K, N), dtype=np.int8)
    wt = w.repack_w8(dev(q))
    torch.cuda.synchronize()
    assert np.array_equal(wt.cpu().numpy(), o.tile_w8(q))


def run_w8(o, c):
    wt = w.repack_w8(dev(c.q))
    A, S = dev(c.A), dev(c.S)
    flat, C, pad = guarded_output(c.M, c.N)
    assert w.w8a16_gemm(A, wt, S, C, c.M, c.N, c.K, c.G) == w.OK
    torch.cuda.synchronize()
    got = C.cpu().numpy()
    ref = o.gemm_w8(c.A, c.q, c.S, c.K, c.G)
    ok, err, rel = within_tolerance(got, ref)
    assert ok, f"W8 {c.M}x{c.K}x{c.N} G={c.G}: max abs err {err}, max rel err {rel}"
    assert guards_intact(flat, pad, c.M * c.N)
    assert w.device_status() == w.OK


@pytest.mark.parametrize("M,K,N,G", [
    (1, 4096, 4096, 128),    # decode: one 16-row token tile, K split over a cluster
    (16, 1024, 512, 64),
    (5, 136, 264, 32),       # per-word scales (G not a multiple of 64), ragged column tile
    (40, 1024, 512, 48),     # groups straddling the 64-deep stages
    (300, 512, 392, 128),    # several token tiles
    (33, 4096, 256, 8192),   # G > K: one group
])
def test_w8_gemm_matches_oracle(o, M, K, N, G):
    run_w8(o, workloads.dense8(M, K, N, G, seed=M * 3 + N))


@pytest.mark.parametrize("name", ["w8_decode_m16", "w8_prefill"])
def test_w8_full_size(o, name):
    run_w8(o, workloads.make(name))


@pytest.mark.parametrize("K,N,G", [(192, 256, 64), (131, 264, 64), (300, 40, 128), (4096, 1024, 128), (64, 520, 256)])
def test_w8_quantize_bit_exact(o, K, N, G):
    # staged (N % 8 == 0, G <= 256) and fallback forms, odd K and a partial last group
    g = np.random.Generator(np.random.PCG64(K * 7 + N))
    W = (g.standard_normal((K, N)) * g.uniform(0.005, 2.0, size=(1, N))).astype(np.float16)
    q8, S = w.quantize_w8(dev(W), G)
    torch.cuda.synchronize()
    ref_q, ref_S = o.quantize_w8(W, G)
    assert np.array_equal(S.cpu().numpy().view(np.uint16), ref_S.view(np.uint16))
    assert np.array_equal(q8.cpu().numpy(), ref_q)
    assert w.device_status() == w.OK


@pytest.mark.parametrize("K,N,G", [(1024, 264, 256), (300, 40, 128)])
def test_w8_quantize_rounding_boundaries(o, K, N, G):
    # every tie of the 8-bit range and its fp16 neighbours, staged and fallback forms
    from test_gpu_parity import rounding_boundary_case
    W = rounding_boundary_case(K, N, G, top=127)
    q8, S = w.quantize_w8(dev(W), G)
    torch.cuda.synchronize()
    ref_q, ref_S = o.quantize_w8(W, G)
    assert np.array_equal(S.cpu().numpy().view(np.uint16), ref_S.view(np.uint16))
    assert np.array_equal(q8.cpu().numpy(), ref_q)
    assert w.device_status() == w.OK


@pytest.mark.parametrize("K,N,G", [(256, 264, 64), (300, 40, 128)])
def test_w8_quantize_subnormal_scales(o, K, N, G):
    # subnormal scales, coarsely rounded: the clamp to [-128, 127] decides codes
    from test_gpu_parity import subnormal_scale_case
    W = subnormal_scale_case(K, N, G, lo=100, hi=260, seed=K * 3 + N)
    q8, S = w.quantize_w8(dev(W), G)
    torch.cuda.synchronize()
    ref_q, ref_S = o.quantize_w8(W, G)
    assert np.any(ref_q == 127) and np.any(ref_q == -128)
    assert np.array_equal(S.cpu().numpy().view(np.uint16), ref_S.view(np.uint16))
    assert np.array_equal(q8.cpu().numpy(), ref_q)
    assert w.device_status() == w.OK


def test_w8_quantize_then_gemm(o):
    # the export chain: fp16 weights -> 8-bit codes and scales -> tiled layout -> product
    M, K, N, G = 24, 1024, 512, 128
    g = np.random.Generator(np.random.PCG64(77))
    W = (g.standard_normal((K, N)) * 0.02).astype(np.float16)
    A = g.standard_normal((M, K), dtype=np.float32).astype(np.float16)
    q8, S = w.quantize_w8(dev(W), G)
    C = w.gemm_w8(dev(A), w.repack_w8(q8), S, N, G).cpu().numpy()
    ref_q, ref_S = o.quantize_w8(W, G)
    ok, err, _ = within_tolerance(C, o.gemm_w8(A, ref_q, ref_S, K, G))
    assert ok, err
