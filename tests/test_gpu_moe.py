"""The INT4 mixture-of-experts layer on the GPU against the oracle (oracle/moe.py).

Every step is checked on its own, on the same seeded inputs the oracle sees:
routing ids bit-exact and weights within fp32 rounding of the float64 softmax;
the dispatch (offsets, positions, gathered-row tokens) and the gather bit-exact;
the up projection with each activation against the oracle's activation of the
GPU's own pre-activation values (at most one fp16 ulp apart, where fp32 and
float64 evaluation straddle a rounding boundary); the combine within one fp16
ulp of the float64 weighted sum. The whole layer is compared element by element
with the GEMM tolerance 1e-2 + 5e-3 |ref| on a small case and on the full
512-token, 8-expert, 4096 -> 14336 -> 4096 layer."""
import numpy as np
import pytest
import torch

import oracle
from oracle import moe
import pins
import workloads
import weight_only_int4_wise_b200 as w
from gpu_util import dev, device_weights, within_tolerance

pytestmark = pytest.mark.gpu

ACTS = [moe.ACT_IDENTITY, moe.ACT_RELU, moe.ACT_GELU_ERF, moe.ACT_GELU_TANH]


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def ordered(h: np.ndarray) -> np.ndarray:
    """fp16 values mapped to integers whose differences count ulps (sign-magnitude -> two's complement)."""
    b = h.view(np.uint16).astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(ordered(np.ascontiguousarray(a)) - ordered(np.ascontiguousarray(b)))


def logits_case(T, E, seed, ties=False):
    g = np.random.Generator(np.random.PCG64(seed))
    if ties:  # few distinct values: many equal logits inside a token
        return (g.integers(-4, 5, size=(T, E)) / 4.0).astype(np.float16)
    return g.standard_normal((T, E), dtype=np.float32).astype(np.float16)


def gpu_route(logits, k):
    T, E = logits.shape
    ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    wts = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    assert w.w4a16_moe_route(dev(logits), ids, wts, T, E, k) == w.OK
    torch.cuda.synchronize()
    return ids.cpu().numpy(), wts.cpu().numpy()


@pytest.mark.parametrize("T,E,k,ties", [(1, 8, 2, False), (300, 8, 2, False), (300, 8, 2, True), (129, 64, 8, True),
                                        (77, 5, 5, False), (40, 16, 1, True)])
def test_route_matches_oracle(T, E, k, ties):
    lg = logits_case(T, E, seed=T * 7 + E + k, ties=ties)
    ids, wts = gpu_route(lg, k)
    rids, rw = moe.route(lg, k)
    assert np.array_equal(ids, rids)
    assert np.allclose(wts.astype(np.float64), rw, rtol=2e-6, atol=0)
    assert w.device_status() == w.OK


def gpu_dispatch(ids, E):
    T, k = ids.shape
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    pos = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    src = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
    assert w.w4a16_moe_dispatch(dev(ids.astype(np.int32)), off, pos, src, T, E, k) == w.OK
    torch.cuda.synchronize()
    return off.cpu().numpy(), pos.cpu().numpy(), src.cpu().numpy()[:T * k]


def random_ids(T, E, k, seed, skew=False):
    g = np.random.Generator(np.random.PCG64(seed))
    p = None
    if skew:  # most pairs on a few experts, some experts empty
        p = np.zeros(E)
        p[: max(1, E // 4)] = 1.0
        p[-1] = 0.05
        p /= p.sum()
        k = min(k, int(np.count_nonzero(p)))
    ids = np.stack([g.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    return ids


@pytest.mark.parametrize("T,E,k,skew", [(1, 8, 2, False), (512, 8, 2, False), (300, 64, 8, True), (1000, 3, 2, True),
                                        (128, 8, 2, False), (129, 8, 1, False), (700, 64, 2, False)])
def test_dispatch_matches_oracle(T, E, k, skew):
    ids = random_ids(T, E, k, seed=T + E, skew=skew)
    off, pos, src = gpu_dispatch(ids, E)
    order, roff, rpos = moe.dispatch(ids, E)
    assert np.array_equal(off, roff)
    assert np.array_equal(pos, rpos)
    assert np.array_equal(src, order // ids.shape[1])
    assert w.device_status() == w.OK


def test_dispatch_of_no_tokens_writes_empty_offsets():
    off = torch.full((9,), -7, dtype=torch.int32, device="cuda")
    dummy = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert w.w4a16_moe_dispatch(dummy, off, dummy, dummy, 0, 8, 2) == w.OK
    torch.cuda.synchronize()
    assert np.all(off.cpu().numpy() == 0)


@pytest.mark.parametrize("bad", ["range", "repeat"])
def test_dispatch_rejects_bad_ids_on_device(bad):
    ids = random_ids(300, 8, 2, seed=5)
    if bad == "range":
        ids[250, 1] = 8
    else:
        ids[3, 1] = ids[3, 0]
    w.device_status(clear=True)
    off, pos, src = gpu_dispatch(ids, 8)
    assert w.device_status(clear=True) == w.ERR_BAD_ROUTING
    assert np.all(off == 0) and np.all(pos == -1) and np.all(src == -1)


def test_gather_bit_exact():
    g = np.random.Generator(np.random.PCG64(3))
    X = g.standard_normal((50, 264), dtype=np.float32).astype(np.float16)
    src = g.integers(0, 50, size=173).astype(np.int32)
    Xg = torch.zeros((173, 264), dtype=torch.float16, device="cuda")
    assert w.w4a16_moe_gather(dev(X), dev(src), Xg, 50, 173, 264) == w.OK
    torch.cuda.synchronize()
    assert np.array_equal(Xg.cpu().numpy().view(np.uint16), X[src].view(np.uint16))
    # an index out of range writes zeros and latches the status
    src[7] = 50
    w.device_status(clear=True)
    assert w.w4a16_moe_gather(dev(X), dev(src), Xg, 50, 173, 264) == w.OK
    assert w.device_status(clear=True) == w.ERR_BAD_ROUTING
    got = Xg.cpu().numpy()
    assert np.all(got[7] == 0) and np.array_equal(got[8], X[src[8]])


@pytest.mark.parametrize("act", ACTS)
def test_up_projection_with_activation(o, act):
    # gathered rows of three experts (one empty) through the grouped GEMM, with and without the activation
    c = workloads.grouped(E=4, top_k=1, tokens=260, K=512, N=392, G=64, seed=90 + act, empty_experts=[2])
    wts = [device_weights(c.q[e])[1] for e in range(c.E)]
    Ss = [dev(c.S[e]) for e in range(c.E)]
    A, off = dev(c.A), dev(c.offsets)
    h = torch.empty((c.total_rows, c.N), dtype=torch.float16, device="cuda")
    a = torch.empty_like(h)
    assert w.w4a16_grouped_gemm_act(A, wts, Ss, off, h, c.E, c.total_rows, c.N, c.K, c.G, moe.ACT_IDENTITY) == w.OK
    assert w.w4a16_grouped_gemm_act(A, wts, Ss, off, a, c.E, c.total_rows, c.N, c.K, c.G, act) == w.OK
    torch.cuda.synchronize()
    h, a = h.cpu().numpy(), a.cpu().numpy()
    ref_h = o.grouped_gemm(c.A, [pins.python_pack(c.q[e]) for e in range(c.E)], list(c.S), c.offsets, c.K, c.G)
    ok, err, _ = within_tolerance(h, ref_h)
    assert ok, err
    ref_a = moe.activation(h, act)
    d = ulp_diff(a, ref_a)
    if act in (moe.ACT_IDENTITY, moe.ACT_RELU):
        assert d.max() == 0
    else:
        assert d.max() <= 1 and np.count_nonzero(d) <= max(4, d.size // 1000)


@pytest.mark.parametrize("act", ACTS)
def test_up_projection_activation_on_the_skinny_kernel(o, act):
    # 12 gathered rows: the grouped product with its activation runs on the skinny kernel
    c = workloads.grouped(E=4, top_k=2, tokens=6, K=1024, N=264, G=128, seed=95 + act)
    wts = [device_weights(c.q[e])[1] for e in range(c.E)]
    Ss = [dev(c.S[e]) for e in range(c.E)]
    A, off = dev(c.A), dev(c.offsets)
    assert w.w4a16_grouped_launch_info(c.E, c.total_rows, c.N, c.K, c.G)[1].token_tile == 16
    h = torch.empty((c.total_rows, c.N), dtype=torch.float16, device="cuda")
    a = torch.empty_like(h)
    assert w.w4a16_grouped_gemm_act(A, wts, Ss, off, h, c.E, c.total_rows, c.N, c.K, c.G, moe.ACT_IDENTITY) == w.OK
    assert w.w4a16_grouped_gemm_act(A, wts, Ss, off, a, c.E, c.total_rows, c.N, c.K, c.G, act) == w.OK
    torch.cuda.synchronize()
    h, a = h.cpu().numpy(), a.cpu().numpy()
    ref_h = o.grouped_gemm(c.A, [pins.python_pack(c.q[e]) for e in range(c.E)], list(c.S), c.offsets, c.K, c.G)
    ok, err, _ = within_tolerance(h, ref_h)
    assert ok, err
    d = ulp_diff(a, moe.activation(h, act))
    assert d.max() <= (0 if act in (moe.ACT_IDENTITY, moe.ACT_RELU) else 1)
    assert w.device_status() == w.OK


def test_combine_within_one_ulp():
    T, k, H = 333, 2, 512
    g = np.random.Generator(np.random.PCG64(8))
    ids = random_ids(T, 8, k, seed=9)
    _, _, pos = moe.dispatch(ids, 8)
    Y = (g.standard_normal((T * k, H), dtype=np.float32) * 4).astype(np.float16)
    _, wts = moe.route(logits_case(T, 8, seed=10), k)
    wts32 = wts.astype(np.float32)
    out = torch.zeros((T, H), dtype=torch.float16, device="cuda")
    assert w.w4a16_moe_combine(dev(Y), dev(wts32), dev(pos.astype(np.int32)), out, T, k, H) == w.OK
    torch.cuda.synchronize()
    ref = moe.combine(Y, wts32.astype(np.float64), pos)
    d = ulp_diff(out.cpu().numpy(), ref)
    assert d.max() <= 1 and np.count_nonzero(d) <= d.size // 1000


def layer_inputs(c):
    up = [device_weights(c.q_up[e])[1] for e in range(c.E)]
    down = [device_weights(c.q_down[e])[1] for e in range(c.E)]
    return up, [dev(s) for s in c.S_up], down, [dev(s) for s in c.S_down]


def oracle_layer(o, c, act):
    return moe.moe_layer(o, c.X, c.logits, [pins.python_pack(q) for q in c.q_up], list(c.S_up),
                         [pins.python_pack(q) for q in c.q_down], list(c.S_down), c.top_k, c.G, act)


def check_layer(o, c, act):
    up, su, down, sd = layer_inputs(c)
    X, lg = dev(c.X), dev(c.logits)
    ws = torch.empty(w.w4a16_moe_workspace_size(c.tokens, c.E, c.top_k, c.H, c.I), dtype=torch.uint8, device="cuda")
    out = w.moe_layer(X, lg, up, su, down, sd, c.top_k, c.I, c.G, act, workspace=ws)
    torch.cuda.synchronize()
    assert w.device_status() == w.OK
    got = out.cpu().numpy()
    ref = oracle_layer(o, c, act)
    ok, err, rel = within_tolerance(got, ref["out"])
    assert ok, f"layer: max abs err {err}, max rel err {rel}"
    return got, ref, (X, lg, up, su, down, sd, ws)


@pytest.mark.parametrize("T,E,k,H,I,G,act", [
    (37, 4, 2, 256, 384, 64, moe.ACT_GELU_ERF),
    (1, 8, 2, 512, 1024, 128, moe.ACT_RELU),       # one decode token: 16-row tiles, most experts empty
    (5, 6, 3, 264, 136, 32, moe.ACT_GELU_TANH),    # ragged column tiles in both projections
    (300, 8, 2, 512, 768, 48, moe.ACT_IDENTITY),   # groups that straddle K stages
])
def test_layer_matches_oracle(o, T, E, k, H, I, G, act):
    c = workloads.moe(tokens=T, E=E, top_k=k, H=H, I=I, G=G, seed=T + E + H)
    check_layer(o, c, act)


def test_layer_equals_its_steps(o):
    # the layer entry point is exactly the six steps run one by one
    c = workloads.moe(tokens=70, E=4, top_k=2, H=256, I=256, G=64, seed=77)
    got, _, (X, lg, up, su, down, sd, ws) = check_layer(o, c, moe.ACT_GELU_ERF)
    T, E, k = c.tokens, c.E, c.top_k
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    off = torch.empty((E + 1,), dtype=torch.int32, device="cuda")
    pos = torch.empty((T, k), dtype=torch.int32, device="cuda")
    src = torch.empty((T * k,), dtype=torch.int32, device="cuda")
    xg = torch.empty((T * k, c.H), dtype=torch.float16, device="cuda")
    a = torch.empty((T * k, c.I), dtype=torch.float16, device="cuda")
    y = torch.empty((T * k, c.H), dtype=torch.float16, device="cuda")
    out = torch.empty((T, c.H), dtype=torch.float16, device="cuda")
    assert w.w4a16_moe_route(lg, ids, wts, T, E, k) == w.OK
    assert w.w4a16_moe_dispatch(ids, off, pos, src, T, E, k) == w.OK
    assert w.w4a16_moe_gather(X, src, xg, T, T * k, c.H) == w.OK
    assert w.w4a16_grouped_gemm_act(xg, up, su, off, a, E, T * k, c.I, c.H, c.G, moe.ACT_GELU_ERF) == w.OK
    assert w.w4a16_grouped_gemm(a, down, sd, off, y, E, T * k, c.H, c.I, c.G) == w.OK
    assert w.w4a16_moe_combine(y, wts, pos, out, T, k, c.H) == w.OK
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16), got.view(np.uint16))


def test_full_size_layer(o):
    # the 512-token layer: 8 experts, top-2, 4096 -> 14336 -> 4096, G = 128, every output element
    c = workloads.make("moe_layer")
    got, ref, _ = check_layer(o, c, moe.ACT_GELU_ERF)
    assert np.all(np.isfinite(got))
