"""The failure path of the bounded device waits, made to run on the GPU without a fault.

The test aid w4a16_set_fault_injection makes the tensor-core GEMM kernel's
dequantising warps withhold the ready signal of one K stage and shortens every
bounded wait, so the MMA thread's wait for that stage runs out. The kernel must
then latch W4A16_ERR_TIMEOUT, drain its copies and MMAs, free its tensor memory
and write no output tile the stalled stage contributes to; the context must stay
usable and the next normal call must be correct."""
import numpy as np
import pytest
import torch

import oracle
import pins
import workloads
import weight_only_int4_wise_b200 as w
from gpu_util import dev, device_weights, guarded_output, guards_intact, within_tolerance, SENTINEL

pytestmark = pytest.mark.gpu

SHORT_WAIT = 200_000  # SM cycles, about 0.1 ms


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def with_injection(stall_stage, fn):
    w.device_status(clear=True)
    w.w4a16_set_fault_injection(stall_stage, SHORT_WAIT)
    try:
        rc = fn()
        torch.cuda.synchronize()
    finally:
        w.w4a16_set_fault_injection(-1, 0)
    return rc


@pytest.mark.parametrize("M,K,N,G,stall,splits", [
    (40, 1024, 512, 64, 1, 8),    # 8-CTA clusters of 2 stages each: every CTA stops
    (40, 1088, 512, 64, 2, 8),    # 17 stages over 8 ranks: only the rank with 3 stages stops, its peers write nothing
    (300, 512, 392, 128, 5, 1),   # two token tiles, no cluster, ragged last column tile
])
def test_bounded_wait_runs_out_and_is_reported(o, M, K, N, G, stall, splits):
    c = workloads.dense(M, K, N, G, seed=K + N + stall)
    rc, info = w.w4a16_gemm_launch_info(M, N, K, G)
    assert rc == w.OK and info.k_splits == splits and info.token_tile >= 32  # the tensor-core kernel
    _, wt = device_weights(c.q)
    A, S = dev(c.A), dev(c.S)
    torch.cuda.synchronize()
    flat, C, pad = guarded_output(M, N)
    rc = with_injection(stall, lambda: w.w4a16_gemm(A, wt, S, C, M, N, K, G))
    assert rc == w.OK
    assert w.device_status(clear=True) == w.ERR_TIMEOUT
    # every CTA's K range holds the stalled stage, or a cluster peer's does: nothing is written
    assert guards_intact(flat, pad, M * N)
    assert np.all(C.cpu().numpy().view(np.uint16) == SENTINEL)
    # the context is still usable and the next normal call is right
    got = w.gemm(A, wt, S, N, G).cpu().numpy()
    assert w.device_status(clear=True) == w.OK
    ok, err, _ = within_tolerance(got, o.gemm(c.A, pins.python_pack(c.q), c.S, K, G))
    assert ok, f"after the timeout: max abs err {err}"


def test_grouped_bounded_wait_runs_out(o):
    c = workloads.grouped(E=3, top_k=1, tokens=200, K=512, N=256, G=128, seed=72)
    wts = [device_weights(c.q[e])[1] for e in range(c.E)]
    Ss = [dev(c.S[e]) for e in range(c.E)]
    A, off = dev(c.A), dev(c.offsets)
    torch.cuda.synchronize()
    flat, C, pad = guarded_output(c.total_rows, c.N)
    rc = with_injection(3, lambda: w.w4a16_grouped_gemm(A, wts, Ss, off, C, c.E, c.total_rows, c.N, c.K, c.G))
    assert rc == w.OK and w.device_status(clear=True) == w.ERR_TIMEOUT
    assert guards_intact(flat, pad, c.total_rows * c.N)
    assert np.all(C.cpu().numpy().view(np.uint16) == SENTINEL)
    got = w.grouped_gemm(A, wts, Ss, off, c.N, c.G).cpu().numpy()
    assert w.device_status(clear=True) == w.OK
    ref = o.grouped_gemm(c.A, [pins.python_pack(c.q[e]) for e in range(c.E)], list(c.S), c.offsets, c.K, c.G)
    ok, err, _ = within_tolerance(got, ref)
    assert ok, err


def test_short_wait_bound_alone_changes_nothing(o):
    # The short bound without a stalled stage: no wait comes near it.
    c = workloads.dense(64, 2048, 1024, 128, seed=71)
    _, wt = device_weights(c.q)
    A, S = dev(c.A), dev(c.S)
    torch.cuda.synchronize()
    flat, C, pad = guarded_output(c.M, c.N)
    rc = with_injection(-1, lambda: w.w4a16_gemm(A, wt, S, C, c.M, c.N, c.K, c.G))
    assert rc == w.OK and w.device_status(clear=True) == w.OK
    ok, err, _ = within_tolerance(C.cpu().numpy(), o.gemm(c.A, pins.python_pack(c.q), c.S, c.K, c.G))
    assert ok, err
