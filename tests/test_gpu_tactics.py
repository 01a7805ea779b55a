"""Every tactic of w4a16_gemm against the oracle, and the autotuner's table.

A tactic is one launch form of the product for a shape (skinny kernel with a K
split, K halves and ring depth; tensor-core kernel with a token tile and K
split). Each must give the oracle's result within the GEMM tolerance, write
nothing outside C, and the tuned entry must be the one the next call uses."""
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
def empty_table():
    w.w4a16_clear_tactics()
    yield
    w.w4a16_clear_tactics()


@pytest.mark.parametrize("M,K,N,G", [
    (1, 4096, 4096, 128),    # the decode shape: every skinny and tensor-core form
    (16, 1024, 512, 64),     # two token tiles on the skinny kernel
    (5, 136, 264, 32),       # a K range shorter than most splits, ragged column tile
    (8, 2048, 1024, 48),     # groups that straddle the 128-deep blocks
    (40, 1024, 512, 64),     # the tensor-core kernel with K splits over one token tile
    (300, 512, 392, 128),    # several token tiles, ragged last column tile
    (5, 1000, 4696, 48),     # 37 column tiles, groups finer than a block, ragged K and N
    (13, 960, 4696, 64),     # two token tiles, an odd count of 64-deep K tiles
    (1, 2048, 4696, 256),    # one group per two blocks (scaled once per block)
    (8, 4096, 14336, 128),   # the MLP up projection at full size
])
def test_every_tactic_matches_the_oracle(o, M, K, N, G):
    c = workloads.dense(M, K, N, G, seed=M + K + N)
    _, wt = device_weights(c.q)
    A, S = dev(c.A), dev(c.S)
    ref = o.gemm(c.A, pins.python_pack(c.q), c.S, K, G)
    rc, ids = w.w4a16_get_valid_tactics(M, N, K, G)
    assert rc == w.OK and ids
    for t in ids:
        assert w.w4a16_set_tactic(M, N, K, G, t) == w.OK
        _, info = w.w4a16_gemm_launch_info(M, N, K, G)
        assert info.as_dict() == w.w4a16_tactic_launch_info(M, N, K, G, t)[1].as_dict()
        flat, C, pad = guarded_output(M, N)
        assert w.w4a16_gemm(A, wt, S, C, M, N, K, G) == w.OK
        torch.cuda.synchronize()
        ok, err, rel = within_tolerance(C.cpu().numpy(), ref)
        assert ok, f"tactic {t} ({info.as_dict()}): max abs err {err}, max rel err {rel}"
        assert guards_intact(flat, pad, M * N), f"tactic {t} wrote outside C"
    assert w.device_status() == w.OK


@pytest.mark.parametrize("copies", [1, 3])
def test_autotune_stores_the_fastest_and_the_gemm_uses_it(o, copies):
    M, K, N, G = 16, 4096, 4096, 128
    c = workloads.dense(M, K, N, G, seed=33)
    _, wt = device_weights(c.q)
    A, S = dev(c.A), dev(c.S)
    C = torch.empty((M, N), dtype=torch.float16, device="cuda")
    wts, Ss = [wt] + [wt.clone() for _ in range(copies - 1)], [S] + [S.clone() for _ in range(copies - 1)]
    rc, best, us, times = w.w4a16_autotune(A, wts, Ss, C, M, N, K, G, reps=8, with_times=True)
    assert rc == w.OK
    _, ids = w.w4a16_get_valid_tactics(M, N, K, G)
    assert best in ids and 0 < us < 1e4 and len(times) == len(ids)
    assert us == pytest.approx(min(times)) and all(x > 0 for x in times)
    assert w.w4a16_get_tactic(M, N, K, G) == best
    assert w.w4a16_gemm_launch_info(M, N, K, G)[1].as_dict() == w.w4a16_tactic_launch_info(M, N, K, G, best)[1].as_dict()
    got = w.gemm(A, wt, S, N, G).cpu().numpy()
    ok, err, _ = within_tolerance(got, o.gemm(c.A, pins.python_pack(c.q), c.S, K, G))
    assert ok, err
    assert w.device_status() == w.OK
