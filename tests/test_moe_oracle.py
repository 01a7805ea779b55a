"""Pins of the mixture-of-experts oracle (oracle/moe.py) against what the reading of
the Int4 Moe Plugin page and plain mathematics fix: a hand-derived routing example,
closed-form activation values, a single expert (the layer is then the plain chain of
two GEMMs), identical experts (routing weights sum to one), exact brute force on a
tiny layer, and token permutation. Planted mistakes in each step fail a pin."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import exact, moe
import pins
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def read_route_example():
    rows = []
    for line in open(os.path.join(HERE, "golden", "moe_route_example.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lg, k, ids, w = [p.strip() for p in line.split("|")]
        rows.append((np.array([float(x) for x in lg.split()], dtype=np.float16), int(k),
                     [int(x) for x in ids.split()], [float(x) for x in w.split()]))
    return rows


def check_route_example(route_fn):
    for lg, k, ids, w in read_route_example():
        got_ids, got_w = route_fn(lg.reshape(1, -1), k)
        if list(got_ids[0]) != ids or not np.allclose(got_w[0], w, rtol=1e-12, atol=0):
            return False
    return True


def test_route_worked_example():
    assert check_route_example(moe.route)


def test_dispatch_worked_example():
    ids = np.array([[1, 3], [1, 3], [0, 1], [3, 2]], dtype=np.int32)
    order, offsets, pos = moe.dispatch(ids, 4)
    # flat (token*2 + slot) experts: 1 3 1 3 0 1 3 2; stable grouping by expert
    assert list(order) == [4, 0, 2, 5, 7, 1, 3, 6]
    assert list(offsets) == [0, 1, 4, 5, 8]
    assert pos.tolist() == [[1, 5], [2, 6], [0, 3], [7, 4]]


def test_activation_closed_forms():
    x = np.array([-2.0, -1.0, 0.0, 1.0, 2.0, 3.0], dtype=np.float16)
    assert moe.activation(x, moe.ACT_RELU).tolist() == [0.0, 0.0, 0.0, 1.0, 2.0, 3.0]
    assert moe.activation(x, moe.ACT_IDENTITY).tolist() == x.tolist()
    g = moe.activation(x, moe.ACT_GELU_ERF)
    # GELU(x) = x * Phi(x): Phi(1) = 0.8413447460685429, Phi(2) = 0.9772498680518208
    assert g[3] == np.float16(0.8413447460685429) and g[1] == np.float16(-0.15865525393145707)
    assert g[4] == np.float16(1.9544997361036416) and g[2] == 0.0
    t = moe.activation(x, moe.ACT_GELU_TANH)
    # 0.5 (1 + tanh(sqrt(2/pi) (1 + 0.044715))) = 0.8411919906082768
    assert t[3] == np.float16(0.8411919906082768)


def test_numpy_half_rounding_matches_the_oracle(o):
    # the module rounds float64 to fp16 with numpy: the same round-to-nearest-even as the C oracle
    g = np.random.Generator(np.random.PCG64(5))
    xs = np.concatenate([g.standard_normal(2000) * 10.0 ** g.integers(-6, 4, 2000),
                         (np.arange(-300, 300) + 0.5) * 2.0 ** -10])  # ties between fp16 neighbours
    for x in xs:
        assert np.float16(x).view(np.uint16) == o.double_to_half(float(x))


def layer_case(T, E, k, H, I, G, seed, identical=False):
    c = workloads.moe(tokens=T, E=E, top_k=k, H=H, I=I, G=G, seed=seed)
    if identical:
        for e in range(1, E):
            c.q_up[e] = c.q_up[0]
            c.S_up[e] = c.S_up[0]
            c.q_down[e] = c.q_down[0]
            c.S_down[e] = c.S_down[0]
    return c


def run_layer(o, c, act):
    return moe.moe_layer(o, c.X, c.logits, [pins.python_pack(q) for q in c.q_up], list(c.S_up),
                         [pins.python_pack(q) for q in c.q_down], list(c.S_down), c.top_k, c.G, act)


@pytest.mark.parametrize("act", [moe.ACT_RELU, moe.ACT_GELU_ERF])
def test_single_expert_is_the_dense_chain(o, act):
    c = layer_case(T=5, E=1, k=1, H=64, I=96, G=32, seed=11)
    r = run_layer(o, c, act)
    h = o.gemm(c.X, pins.python_pack(c.q_up[0]), c.S_up[0], c.H, c.G)
    y = o.gemm(moe.activation(h, act), pins.python_pack(c.q_down[0]), c.S_down[0], c.I, c.G)
    assert np.array_equal(r["out"].view(np.uint16), y.view(np.uint16))


def test_identical_experts_weights_sum_to_one(o):
    c = layer_case(T=6, E=4, k=2, H=64, I=64, G=32, seed=12, identical=True)
    r = run_layer(o, c, moe.ACT_GELU_TANH)
    h = o.gemm(c.X, pins.python_pack(c.q_up[0]), c.S_up[0], c.H, c.G)
    y = o.gemm(moe.activation(h, moe.ACT_GELU_TANH), pins.python_pack(c.q_down[0]), c.S_down[0], c.I, c.G)
    assert np.array_equal(r["out"].view(np.uint16), y.view(np.uint16))


def fp16_exact(v: Fraction) -> np.float16:
    """Round an exact rational to fp16 (round to nearest, ties to even) by brute force."""
    f = float(v)
    cand = np.float16(f)
    best = None
    bits = int(cand.view(np.uint16))
    for b in (bits - 1, bits, bits + 1):
        c = np.uint16(b & 0xFFFF).view(np.float16)
        if not np.isfinite(c):
            continue
        d = abs(Fraction(float(c)) - v)
        key = (d, int(np.uint16(b & 0xFFFF)) & 1)  # ties: even mantissa
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_tiny_layer_brute_force(o):
    # every step in exact rational arithmetic (routing weights in float64, as the oracle)
    c = layer_case(T=3, E=3, k=2, H=16, I=24, G=8, seed=13)
    r = run_layer(o, c, moe.ACT_RELU)
    ids, w = moe.route(c.logits, 2)
    out = np.zeros((3, 16), dtype=np.float16)
    for t in range(3):
        acc = [Fraction(0)] * 16
        for j in range(2):
            e = int(ids[t, j])
            h = exact.gemm_exact(c.X[t:t + 1], c.q_up[e], c.S_up[e], c.G)
            a = np.maximum(h.astype(np.float64), 0.0).astype(np.float16)
            y = exact.gemm_exact(a, c.q_down[e], c.S_down[e], c.G)
            for n in range(16):
                acc[n] += Fraction(float(w[t, j])) * Fraction(float(y[0, n]))
        for n in range(16):
            out[t, n] = fp16_exact(acc[n])
    assert np.array_equal(r["out"].view(np.uint16), out.view(np.uint16))


def test_token_permutation_permutes_the_output(o):
    c = layer_case(T=12, E=4, k=2, H=64, I=64, G=32, seed=14)
    r = run_layer(o, c, moe.ACT_GELU_ERF)
    perm = np.random.Generator(np.random.PCG64(1)).permutation(12)
    c.X, c.logits = c.X[perm], c.logits[perm]
    r2 = run_layer(o, c, moe.ACT_GELU_ERF)
    assert np.array_equal(r2["out"].view(np.uint16), r["out"][perm].view(np.uint16))


def test_planted_mistakes_are_caught(o):
    # routing: no renormalisation over the selected experts (softmax over all experts)
    def route_unnormalised(lg, k):
        ids, _ = moe.route(lg, k)
        x = lg.astype(np.float64)
        full = np.exp(x - x.max(axis=1, keepdims=True))
        full /= full.sum(axis=1, keepdims=True)
        return ids, np.take_along_axis(full, ids.astype(np.int64), axis=1)
    assert not check_route_example(route_unnormalised)

    # routing: ties to the higher expert index
    def route_ties_high(lg, k):
        x = np.asarray(lg, dtype=np.float64)
        ids = np.argsort(-x - 1e-9 * np.arange(x.shape[1]), axis=1, kind="stable")[:, :k].astype(np.int32)
        sel = np.take_along_axis(x, ids.astype(np.int64), axis=1)
        ex = np.exp(sel - sel.max(axis=1, keepdims=True))
        return ids, ex / ex.sum(axis=1, keepdims=True)
    assert not check_route_example(route_ties_high)

    # combine: weights applied to the wrong slot
    c = layer_case(T=8, E=4, k=2, H=32, I=32, G=16, seed=15)
    r = run_layer(o, c, moe.ACT_RELU)
    swapped = moe.combine(r["y"], r["weights"][:, ::-1], r["pos"])
    assert not np.array_equal(swapped.view(np.uint16), r["out"].view(np.uint16))

    # activation: GELU with the tanh form where the erf form is asked for (and back)
    # (the forms differ by ~4e-4 at x = -3: -3 Phi(-3) = -0.00404969409489028)
    x = np.array([-3.0], dtype=np.float16)
    assert moe.activation(x, moe.ACT_GELU_ERF)[0] == np.float16(-0.00404969409489028)
    assert moe.activation(x, moe.ACT_GELU_TANH)[0] != np.float16(-0.00404969409489028)
