"""The expert layer's no-allocation entry point, w4a16_moe_layer_static, against the
workspace form, w4a16_moe_layer. Both run the same six kernels; only where the
intermediates live differs (a region of device memory the library owns, against a
caller buffer), so the outputs must be bit-identical, also on a second call in a
row that finds the scratch as the first call left it. Kept last in collection
order so that it also runs after every other test has used the device."""
import numpy as np
import pytest
import torch

import workloads
import weight_only_int4_wise_b200 as w
from gpu_util import dev, device_weights

pytestmark = pytest.mark.gpu


def layer_args(c):
    up = [device_weights(c.q_up[e])[1] for e in range(c.E)]
    down = [device_weights(c.q_down[e])[1] for e in range(c.E)]
    return (dev(c.X), dev(c.logits), up, [dev(s) for s in c.S_up], down, [dev(s) for s in c.S_down])


@pytest.mark.parametrize("T,E,k,H,I,G,act", [
    (4, 8, 2, 1024, 2048, 128, w.ACT_GELU_ERF),   # a decode batch
    (37, 4, 2, 512, 768, 64, w.ACT_RELU),
])
def test_static_scratch_matches_workspace(T, E, k, H, I, G, act):
    c = workloads.moe(tokens=T, E=E, top_k=k, H=H, I=I, G=G, seed=T + H)
    X, lg, up, su, down, sd = layer_args(c)
    need = w.w4a16_moe_workspace_size(T, E, k, H, I)
    assert 0 < need <= w.w4a16_moe_static_scratch_bytes()
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ref = torch.empty((T, H), dtype=torch.float16, device="cuda")
    outs = [torch.full((T, H), float("nan"), dtype=torch.float16, device="cuda") for _ in range(2)]
    assert w.w4a16_moe_layer(X, lg, up, su, down, sd, ref, T, E, k, H, I, G, act, ws, need) == w.OK
    for out in outs:  # two calls in a row on the same static scratch
        assert w.w4a16_moe_layer_static(X, lg, up, su, down, sd, out, T, E, k, H, I, G, act) == w.OK
    torch.cuda.synchronize()
    assert w.device_status() == w.OK
    r = ref.cpu().numpy().view(np.uint16)
    for out in outs:
        assert np.array_equal(out.cpu().numpy().view(np.uint16), r)


def test_static_scratch_refuses_larger_shapes():
    # the 512-token layer needs about 45 MB of intermediates: more than the static region
    T, E, k, H, I = 512, 8, 2, 4096, 14336
    assert w.w4a16_moe_workspace_size(T, E, k, H, I) > w.w4a16_moe_static_scratch_bytes()
    x = torch.empty(16, dtype=torch.uint8, device="cuda")
    ptrs = [x] * E
    rc = w.w4a16_moe_layer_static(x, x, ptrs, ptrs, ptrs, ptrs, x, T, E, k, H, I, 128, w.ACT_RELU)
    assert rc == w.ERR_SCRATCH_TOO_SMALL
    assert "static scratch" in w.status_string(rc)
