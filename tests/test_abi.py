"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

import oracle
import weight_only_int4_wise_b200 as w
from weight_only_int4_wise_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")

FAKE = 0x10000  # a non-null, 16-byte aligned address that is never dereferenced on these paths


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(w[48]a16_\w+)\s*\(", text, re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("w4a16_pack", "w4a16_unpack", "w4a16_repack", "w4a16_gemm", "w4a16_grouped_gemm",
                     "w4a16_status_string", "w4a16_tiled_bytes", "w4a16_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in w4a16.h but not exported"
    assert sorted(_lib.EXPORTED) == declared_functions()


def test_status_strings(lib):
    for code in range(9):
        assert w.status_string(code) != "unknown status"
    assert w.status_string(99) == "unknown status"


def test_tiled_bytes_matches_layout_definition(lib):
    o = oracle.load()
    for K, N in [(1, 1), (64, 128), (65, 129), (4096, 4096), (4096, 14336), (14336, 4096), (72, 200)]:
        assert w.w4a16_tiled_bytes(K, N) == o.tiled_bytes(K, N)
    assert w.w4a16_tiled_bytes(0, 5) == 0 and w.w4a16_tiled_bytes(5, -1) == 0


def test_gemm_rejects_bad_arguments_on_host(lib):
    g = lambda **kw: w.w4a16_gemm(kw.get("A", FAKE), kw.get("Wt", FAKE), kw.get("S", FAKE), kw.get("C", FAKE),
                                  kw.get("M", 4), kw.get("N", 128), kw.get("K", 128), kw.get("G", 64), stream=0)
    assert g(A=None) == w.ERR_INVALID_ARG
    assert g(Wt=None) == w.ERR_INVALID_ARG
    assert g(C=None) == w.ERR_INVALID_ARG
    assert g(M=-1) == w.ERR_INVALID_ARG
    assert g(N=0) == w.ERR_INVALID_ARG
    assert g(K=0) == w.ERR_INVALID_ARG
    assert g(G=0) == w.ERR_INVALID_ARG
    assert g(N=100) == w.ERR_UNSUPPORTED   # N % 8
    assert g(K=100) == w.ERR_UNSUPPORTED   # K % 8
    assert g(G=24) == w.ERR_UNSUPPORTED    # G % 16
    assert g(A=FAKE + 8) == w.ERR_MISALIGNED
    assert g(Wt=FAKE + 4) == w.ERR_MISALIGNED
    assert g(S=FAKE + 2) == w.ERR_MISALIGNED
    assert g(C=FAKE + 1) == w.ERR_MISALIGNED
    assert g(M=0) == w.OK  # empty batch: nothing to do, nothing launched


def test_grouped_rejects_bad_arguments_on_host(lib):
    def g(E=2, rows=8, wts=None, ss=None, off=FAKE, A=FAKE, C=FAKE, N=128, K=128, G=64):
        wts = [FAKE] * E if wts is None else wts
        ss = [FAKE] * E if ss is None else ss
        return w.w4a16_grouped_gemm(A, wts, ss, off, C, E, rows, N, K, G, stream=0)
    assert g(E=0, wts=[FAKE], ss=[FAKE]) == w.ERR_INVALID_ARG
    assert g(E=w.MAX_EXPERTS + 1) == w.ERR_INVALID_ARG
    assert g(off=None) == w.ERR_INVALID_ARG
    assert g(rows=-1) == w.ERR_INVALID_ARG
    assert g(wts=[FAKE, 0]) == w.ERR_INVALID_ARG
    assert g(wts=[FAKE, FAKE + 8]) == w.ERR_MISALIGNED
    assert g(off=FAKE + 2) == w.ERR_MISALIGNED
    assert g(G=40) == w.ERR_UNSUPPORTED
    assert g(rows=0) == w.OK


def test_pack_rejects_bad_arguments_on_host(lib):
    assert w.w4a16_pack(None, FAKE, 4, 4, stream=0) == w.ERR_INVALID_ARG
    assert w.w4a16_pack(FAKE, FAKE, 0, 4, stream=0) == w.ERR_INVALID_ARG
    assert w.w4a16_unpack(FAKE, None, 4, 4, stream=0) == w.ERR_INVALID_ARG
    assert w.w4a16_repack(FAKE, FAKE + 4, 4, 4, stream=0) == w.ERR_MISALIGNED
    assert w.w4a16_repack(FAKE, FAKE, 4, -4, stream=0) == w.ERR_INVALID_ARG


def test_quantize_rejects_bad_arguments_on_host(lib):
    q = lambda **kw: w.w4a16_quantize(kw.get("W", FAKE), kw.get("wp", FAKE), kw.get("S", FAKE), kw.get("K", 64),
                                      kw.get("N", 64), kw.get("G", 32), stream=0)
    assert q(W=None) == w.ERR_INVALID_ARG
    assert q(S=None) == w.ERR_INVALID_ARG
    assert q(K=0) == w.ERR_INVALID_ARG and q(G=-2) == w.ERR_INVALID_ARG
    assert q(N=63) == w.ERR_UNSUPPORTED and q(G=33) == w.ERR_UNSUPPORTED
    assert q(W=FAKE + 2) == w.ERR_MISALIGNED and q(S=FAKE + 2) == w.ERR_MISALIGNED and q(wp=FAKE + 1) == w.ERR_MISALIGNED


def test_launch_plan_on_host(lib):
    # Nominal plans (no device here): decode runs the skinny kernel with K split across a
    # cluster (8-row token tiles for M <= 8, 16 for M <= 16); prefill tiles M on the tensor-core kernel.
    rc, info = w.w4a16_gemm_launch_info(1, 4096, 4096, 128)
    assert rc == w.OK and info.token_tile == 8 and info.k_splits > 1 and info.grid_y == 32
    assert info.threads_per_cta == 256  # decode keeps one set of 8 warps per CTA
    rc, info = w.w4a16_gemm_launch_info(8, 14336, 4096, 128)
    assert rc == w.OK and info.token_tile == 8 and info.threads_per_cta == 512  # MLP up: two K halves
    rc, info = w.w4a16_gemm_launch_info(8, 4096, 14336, 128)
    assert rc == w.OK and info.k_splits == 4 and info.threads_per_cta == 512  # MLP down: 28 blocks per CTA
    rc, info = w.w4a16_gemm_launch_info(16, 4096, 4096, 128)
    assert rc == w.OK and info.token_tile == 16 and info.threads_per_cta == 256
    rc, info = w.w4a16_gemm_launch_info(17, 4096, 4096, 128)
    assert rc == w.OK and info.token_tile == 32 and info.threads_per_cta == 320
    rc, info = w.w4a16_gemm_launch_info(2048, 4096, 4096, 128)
    assert rc == w.OK and info.token_tile == 256 and info.k_splits == 1 and info.grid_z == 8
    rc, info = w.w4a16_grouped_launch_info(8, 1024, 14336, 4096, 128)
    assert rc == w.OK and info.grid_y == 112 and info.grid_z >= 8
    rc, _ = w.w4a16_gemm_launch_info(0, 4096, 4096, 128)
    assert rc == w.ERR_INVALID_ARG


def test_valid_call_without_a_gpu_is_refused_not_crashed(lib):
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("a GPU is present")
    except ImportError:
        pass
    rc = w.w4a16_gemm(FAKE, FAKE, FAKE, FAKE, 4, 128, 128, 64, stream=0)
    assert rc == w.ERR_UNSUPPORTED


def test_moe_entry_points_reject_bad_arguments_on_host(lib):
    assert w.w4a16_moe_route(None, FAKE, FAKE, 4, 8, 2, stream=0) == w.ERR_INVALID_ARG
    assert w.w4a16_moe_route(FAKE, FAKE, FAKE, 4, 8, 9, stream=0) == w.ERR_INVALID_ARG       # k > E
    assert w.w4a16_moe_route(FAKE, FAKE, FAKE, 4, 80, 9, stream=0) == w.ERR_INVALID_ARG      # E > 64
    assert w.w4a16_moe_route(FAKE, FAKE, FAKE, 4, 16, w.MAX_TOPK + 1, stream=0) == w.ERR_INVALID_ARG
    assert w.w4a16_moe_route(FAKE, FAKE + 2, FAKE, 4, 8, 2, stream=0) == w.ERR_MISALIGNED
    assert w.w4a16_moe_route(FAKE, FAKE, FAKE, 0, 8, 2, stream=0) == w.OK                    # no tokens
    assert w.w4a16_moe_dispatch(FAKE, None, FAKE, FAKE, 4, 8, 2, stream=0) == w.ERR_INVALID_ARG
    assert w.w4a16_moe_dispatch(FAKE, FAKE, FAKE, FAKE, -1, 8, 2, stream=0) == w.ERR_INVALID_ARG
    assert w.w4a16_moe_gather(FAKE, FAKE, FAKE, 4, 8, 100, stream=0) == w.ERR_UNSUPPORTED   # H % 8
    assert w.w4a16_moe_gather(FAKE + 8, FAKE, FAKE, 4, 8, 128, stream=0) == w.ERR_MISALIGNED
    assert w.w4a16_moe_gather(FAKE, FAKE, FAKE, 4, 0, 128, stream=0) == w.OK
    assert w.w4a16_moe_combine(FAKE, FAKE, FAKE, FAKE, 4, 0, 128, stream=0) == w.ERR_INVALID_ARG
    assert w.w4a16_moe_combine(FAKE, FAKE, FAKE, FAKE + 8, 4, 2, 128, stream=0) == w.ERR_MISALIGNED
    assert w.w4a16_grouped_gemm_act(FAKE, [FAKE] * 2, [FAKE] * 2, FAKE, FAKE, 2, 8, 128, 128, 64, 4,
                                    stream=0) == w.ERR_INVALID_ARG  # unknown activation


def moe_workspace_layout(T, E, k, H, I):
    """The workspace layout the header describes, recomputed: eight regions on 256-byte boundaries."""
    r = lambda b: (b + 255) // 256 * 256
    pairs = T * k
    return 4 * r(pairs * 4) + r((E + 1) * 4) + r(pairs * H * 2) + r(pairs * I * 2) + r(pairs * H * 2)


def test_moe_workspace_size(lib):
    for T, E, k, H, I in [(512, 8, 2, 4096, 14336), (1, 8, 2, 64, 64), (3, 5, 5, 8, 16), (0, 4, 1, 64, 64)]:
        assert w.w4a16_moe_workspace_size(T, E, k, H, I) == moe_workspace_layout(T, E, k, H, I)
    assert w.w4a16_moe_workspace_size(4, 8, 9, 64, 64) == -1
    assert w.w4a16_moe_workspace_size(4, 8, 2, 0, 64) == -1


def test_moe_layer_rejects_bad_arguments_on_host(lib):
    T, E, k, H, I = 4, 4, 2, 128, 256
    need = w.w4a16_moe_workspace_size(T, E, k, H, I)

    def g(**kw):
        ws = [FAKE] * E
        return w.w4a16_moe_layer(kw.get("X", FAKE), kw.get("logits", FAKE), kw.get("up", ws), ws, ws, ws,
                                 kw.get("out", FAKE), kw.get("T", T), E, kw.get("k", k), kw.get("H", H), I,
                                 kw.get("G", 64), kw.get("act", w.ACT_GELU_ERF), kw.get("ws", FAKE),
                                 kw.get("ws_bytes", need), stream=0)
    assert g(X=None) == w.ERR_INVALID_ARG
    assert g(ws=None) == w.ERR_INVALID_ARG
    assert g(ws_bytes=need - 1) == w.ERR_INVALID_ARG
    assert g(act=7) == w.ERR_INVALID_ARG
    assert g(k=5) == w.ERR_INVALID_ARG
    assert g(up=[FAKE, FAKE, 0, FAKE]) == w.ERR_INVALID_ARG
    assert g(H=100) == w.ERR_UNSUPPORTED
    assert g(G=24) == w.ERR_UNSUPPORTED
    assert g(out=FAKE + 8) == w.ERR_MISALIGNED
    assert g(T=0) == w.OK


def test_tactic_lists_on_host(lib):
    # Decode shape: the skinny forms (K split 1..8, one or two K halves, two ring
    # depths) first, then the tensor-core forms (token tiles 16..256, K split 1/2/4/8).
    rc, ids = w.w4a16_get_valid_tactics(1, 4096, 4096, 128)
    assert rc == w.OK and ids == list(range(1, len(ids) + 1)) and 32 < len(ids) <= 96
    infos = [w.w4a16_tactic_launch_info(1, 4096, 4096, 128, t) for t in ids]
    assert all(rc == w.OK for rc, _ in infos)
    kinds = [i.threads_per_cta in (256, 512) and i.token_tile == 8 for _, i in infos]
    assert kinds == sorted(kinds, reverse=True)  # skinny forms precede the tensor-core forms
    assert {(i.k_splits, i.threads_per_cta) for _, i in infos if i.token_tile == 8} >= {(s, 256) for s in range(1, 9)}
    assert w.w4a16_tactic_launch_info(1, 4096, 4096, 128, len(ids) + 1)[0] == w.ERR_INVALID_ARG
    assert w.w4a16_tactic_launch_info(1, 4096, 4096, 128, 0)[0] == w.ERR_INVALID_ARG
    # prefill: one token tile per form, no K split across several token tiles
    rc, ids = w.w4a16_get_valid_tactics(2048, 4096, 4096, 128)
    assert rc == w.OK
    tiles = [w.w4a16_tactic_launch_info(2048, 4096, 4096, 128, t)[1] for t in ids]
    assert [i.token_tile for i in tiles] == [16, 32, 64, 128, 192, 256] and all(i.k_splits == 1 for i in tiles)
    assert w.w4a16_get_valid_tactics(1, 100, 4096, 128)[0] == w.ERR_UNSUPPORTED


def test_tactic_table_round_trip_on_host(lib):
    w.w4a16_clear_tactics()
    shape = (16, 4096, 4096, 128)
    _, default = w.w4a16_gemm_launch_info(*shape)
    _, ids = w.w4a16_get_valid_tactics(*shape)
    assert w.w4a16_get_tactic(*shape) == 0
    pick = ids[-1]  # the 256-row tensor-core tile with an 8-way K split
    assert w.w4a16_set_tactic(*shape, pick) == w.OK
    assert w.w4a16_get_tactic(*shape) == pick
    _, now = w.w4a16_gemm_launch_info(*shape)
    assert now.as_dict() == w.w4a16_tactic_launch_info(*shape, pick)[1].as_dict() != default.as_dict()
    assert w.w4a16_get_tactic(32, 4096, 4096, 128) == 0  # exact shapes only
    assert w.w4a16_set_tactic(*shape, len(ids) + 1) == w.ERR_INVALID_ARG
    assert w.w4a16_set_tactic(*shape, 0) == w.OK and w.w4a16_get_tactic(*shape) == 0
    assert w.w4a16_gemm_launch_info(*shape)[1].as_dict() == default.as_dict()
    w.w4a16_set_tactic(*shape, pick)
    assert w.w4a16_clear_tactics() == w.OK and w.w4a16_get_tactic(*shape) == 0


def test_autotune_rejects_bad_arguments_on_host(lib):
    t = lambda **kw: w.w4a16_autotune(kw.get("A", FAKE), kw.get("wts", [FAKE]), kw.get("ss", [FAKE]), FAKE,
                                      kw.get("M", 4), 128, 128, 64, reps=kw.get("reps", 5), stream=0)[0]
    assert t(A=None) == w.ERR_INVALID_ARG
    assert t(M=0) == w.ERR_INVALID_ARG
    assert t(reps=0) == w.ERR_INVALID_ARG
    assert t(wts=[FAKE, 0], ss=[FAKE, FAKE]) == w.ERR_INVALID_ARG
    assert t(wts=[FAKE + 8]) == w.ERR_MISALIGNED
    assert t(A=FAKE + 8) == w.ERR_MISALIGNED
    try:
        import torch
        if torch.cuda.is_available():
            return
    except ImportError:
        pass
    assert t() == w.ERR_UNSUPPORTED  # a valid call without a GPU


def test_w8_tiled_bytes_and_host_checks(lib):
    o = oracle.load()
    for K, N in [(1, 1), (64, 128), (65, 129), (4096, 14336), (72, 200)]:
        assert w.w8a16_tiled_bytes(K, N) == o.tiled_bytes_w8(K, N) == 2 * w.w4a16_tiled_bytes(K, N)
    g = lambda **kw: w.w8a16_gemm(kw.get("A", FAKE), kw.get("Wt", FAKE), FAKE, kw.get("C", FAKE), kw.get("M", 4),
                                  kw.get("N", 128), 128, kw.get("G", 64), stream=0)
    assert g(A=None) == w.ERR_INVALID_ARG and g(M=-1) == w.ERR_INVALID_ARG
    assert g(N=100) == w.ERR_UNSUPPORTED and g(G=24) == w.ERR_UNSUPPORTED
    assert g(Wt=FAKE + 4) == w.ERR_MISALIGNED and g(C=FAKE + 1) == w.ERR_MISALIGNED
    assert g(M=0) == w.OK
    assert w.w8a16_repack(FAKE, FAKE + 8, 4, 4, stream=0) == w.ERR_MISALIGNED
    assert w.w8a16_repack(None, FAKE, 4, 4, stream=0) == w.ERR_INVALID_ARG
    rc, info = w.w8a16_gemm_launch_info(16, 4096, 4096, 128)
    assert rc == w.OK and info.token_tile == 16 and info.threads_per_cta == 320  # the tensor-core kernel


def test_static_scratch_layer_host_checks(lib):
    # the no-allocation expert layer refuses shapes beyond its static scratch before touching CUDA
    assert w.w4a16_moe_static_scratch_bytes() == 8 << 20
    ptrs = [FAKE] * 8
    call = lambda T, H, I: w.w4a16_moe_layer_static(FAKE, FAKE, ptrs, ptrs, ptrs, ptrs, FAKE, T, 8, 2, H, I, 128,
                                                     w.ACT_RELU, stream=0)
    assert call(512, 4096, 14336) == w.ERR_SCRATCH_TOO_SMALL
    assert call(4, 4096, 0) == w.ERR_INVALID_ARG
    assert call(0, 4096, 14336) == w.OK


def test_gemm_ex_flags_on_host(lib):
    g = lambda flags, M=4: w.w4a16_gemm_ex(FAKE, FAKE, FAKE, FAKE, M, 128, 128, 64, flags, stream=0)
    assert g(2) == w.ERR_INVALID_ARG and g(0x80000000) == w.ERR_INVALID_ARG
    assert g(w.FLAG_STATIC_WEIGHTS, M=0) == w.OK and g(0, M=0) == w.OK
    assert g(w.FLAG_STATIC_WEIGHTS, M=-1) == w.ERR_INVALID_ARG


def test_w8_quantize_rejects_bad_arguments_on_host(lib):
    q = lambda **kw: w.w8a16_quantize(kw.get("W", FAKE), kw.get("q8", FAKE), kw.get("S", FAKE), kw.get("K", 64),
                                      kw.get("N", 64), kw.get("G", 32), stream=0)
    assert q(W=None) == w.ERR_INVALID_ARG and q(K=0) == w.ERR_INVALID_ARG
    assert q(N=63) == w.ERR_UNSUPPORTED and q(G=33) == w.ERR_UNSUPPORTED
    assert q(W=FAKE + 2) == w.ERR_MISALIGNED and q(q8=FAKE + 1) == w.ERR_MISALIGNED
