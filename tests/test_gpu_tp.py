"""GPU parity: edge-free channelwise tensor product (batch 1000, mult 128)."""
import numpy as np
import pytest

from equivariant_mlip_tensor_b200 import synthetic
from oracle import cg as ocg
from oracle import tp as otp
from tests.gpu_common import FWD_TOL, GRAD_TOL, cuda, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from equivariant_mlip_tensor_b200 import api as a
    return a


def test_tp_batch_workload(api):
    w = synthetic.tp_batch()
    L = (w.lmax_in, w.lmax_sh, w.lmax_out)
    plan = api.Plan(*L, w.mult)
    z = plan.tp_forward(cuda(w.x), cuda(w.y), cuda(w.w))
    assert rel_err(host(z), otp.tp_forward(w.x, w.y, w.w, *L)) < FWD_TOL
    gx, gy, gw = plan.tp_backward(cuda(w.x), cuda(w.y), cuda(w.w), cuda(w.grad_z))
    rx, ry, rw = otp.tp_backward(w.x, w.y, w.w, w.grad_z, *L)
    assert rel_err(host(gx), rx) < GRAD_TOL
    assert rel_err(host(gy), ry) < GRAD_TOL
    assert rel_err(host(gw), rw) < GRAD_TOL
    # deterministic: the batch reduction has a fixed order
    _, _, gw2 = plan.tp_backward(cuda(w.x), cuda(w.y), cuda(w.w), cuda(w.grad_z))
    assert np.array_equal(host(gw), host(gw2))


@pytest.mark.parametrize("L,mult,batch", [((1, 1, 1), 8, 3), ((2, 2, 2), 96, 77), ((2, 4, 2), 32, 130),
                                          ((3, 3, 3), 64, 9), ((0, 0, 0), 4, 1), ((3, 4, 3), 32, 19),
                                          ((0, 3, 3), 16, 5), ((2, 1, 0), 8, 11)])
def test_tp_shapes(api, L, mult, batch):
    rng = np.random.default_rng(40 + batch)
    P = len(ocg.paths(*L))
    x = rng.standard_normal((batch, (L[0] + 1) ** 2, mult)).astype(np.float32)
    y = rng.standard_normal((batch, (L[1] + 1) ** 2, mult)).astype(np.float32)
    wt = rng.standard_normal((P, mult)).astype(np.float32)
    g = rng.standard_normal((batch, (L[2] + 1) ** 2, mult)).astype(np.float32)
    plan = api.Plan(*L, mult)
    z = plan.tp_forward(cuda(x), cuda(y), cuda(wt))
    assert rel_err(host(z), otp.tp_forward(x, y, wt, *L)) < FWD_TOL
    gx, gy, gw = plan.tp_backward(cuda(x), cuda(y), cuda(wt), cuda(g))
    rx, ry, rw = otp.tp_backward(x, y, wt, g, *L)
    assert rel_err(host(gx), rx) < GRAD_TOL
    assert rel_err(host(gy), ry) < GRAD_TOL
    assert rel_err(host(gw), rw) < GRAD_TOL
