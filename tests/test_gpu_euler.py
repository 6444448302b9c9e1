"""Euler update on the GPU against the fp64 oracle (blog chapter 5, UniPC)."""
import numpy as np
import pytest
import torch

from gpu_common import f64
from oracle import euler
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu
FRAME = 48 * 44 * 80  # 168,960 latent values per frame


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


@pytest.mark.parametrize("n,offset", [(1, 0), (7, 0), (1000, 1), (FRAME, 0), (FRAME + 3, 1),
                                      (248 * FRAME, 0)])
def test_euler_step_matches_oracle(pv, n, offset):
    x = synth.normal_f32(101, (n + offset,), "cuda")
    v = synth.normal_f32(102, (n + offset,), "cuda")
    x_host = f64(x)[offset:]
    v_host = f64(v)[offset:]
    for sigma, nxt in zip(euler.SIGMAS_4[:-1], euler.SIGMAS_4[1:]):
        ref = euler.euler_step(x_host, v_host, sigma, nxt)
        pv.pv_euler_step(x[offset:], v[offset:], n, float(nxt - sigma))
        torch.cuda.synchronize()
        got = f64(x)[offset:]
        err = np.abs(got - ref)
        assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
        assert np.all(err <= 1e-5 * (np.abs(x_host) + np.abs((nxt - sigma) * v_host)) + 1e-30)
        x_host = ref
    if offset:
        assert float(x[0]) == float(synth.normal_f32(101, (1,))[0])  # untouched prefix


def test_euler_straight_line_closed_form(pv):
    # v = x1 - x0 constant: four steps from sigma = 1 reach x0 (blog chapter 1)
    n = 3 * FRAME
    x0 = synth.normal_f32(103, (n,), "cuda")
    x1 = synth.normal_f32(104, (n,), "cuda")
    v = x1 - x0
    x = x1.clone()
    s = euler.SIGMAS_4
    for i in range(4):
        pv.pv_euler_step(x, v, n, float(s[i + 1] - s[i]))
    torch.cuda.synchronize()
    assert torch.max(torch.abs(x - x0)).item() <= 4e-6 * torch.max(torch.abs(x1) + torch.abs(x0)).item()


def test_euler_rejects_bad_arguments(pv):
    x = torch.zeros(8, device="cuda")
    with pytest.raises(pv.PVError):
        pv.pv_euler_step(x, 0, 8, -0.25)
    with pytest.raises(pv.PVError):
        pv.pv_euler_step(x, x, 8, float("nan"))
    pv.pv_euler_step(x, x, 0, -0.25)  # empty is a no-op


@pytest.mark.parametrize("n,offset,w", [(1, 0, 5.0), (13, 1, 5.0), (FRAME + 3, 1, 4.0),
                                        (31 * FRAME, 0, 5.0), (31 * FRAME, 0, 1.0),
                                        (31 * FRAME, 0, 0.0)])
def test_euler_cfg_step_matches_oracle(pv, n, offset, w):
    x = synth.normal_f32(111, (n + offset,), "cuda")
    vc = synth.normal_f32(112, (n + offset,), "cuda")
    vu = synth.normal_f32(113, (n + offset,), "cuda")
    xh, ch, uh = f64(x)[offset:], f64(vc)[offset:], f64(vu)[offset:]
    sig = euler.shifted_schedule(40, 12.0)
    for i in (0, 17, 39):
        ref = euler.euler_cfg_step(xh, ch, uh, w, sig[i], sig[i + 1])
        d = float(sig[i + 1] - sig[i])
        pv.pv_euler_cfg_step(x[offset:], vc[offset:], vu[offset:], n, w, d)
        torch.cuda.synchronize()
        got = f64(x)[offset:]
        # f32 terms: |x|, |d| (|vu| + |w| (|vc| + |vu|)), each a few ulps
        bound = 2e-6 * (np.abs(xh) + abs(d) * (np.abs(uh) + abs(w) * (np.abs(ch) + np.abs(uh))))
        assert np.all(np.abs(got - ref) <= bound + 1e-30)
        xh = ref
    if offset:
        assert float(x[0]) == float(synth.normal_f32(111, (1,))[0])


def test_euler_cfg_special_cases(pv):
    n = 2 * FRAME
    x = synth.normal_f32(114, (n,), "cuda")
    vc = synth.normal_f32(115, (n,), "cuda")
    vu = synth.normal_f32(116, (n,), "cuda")
    # w = 1 is the conditional step, w = 0 the unconditional one
    for w, v in ((1.0, vc), (0.0, vu)):
        a, b = x.clone(), x.clone()
        pv.pv_euler_cfg_step(a, vc, vu, n, w, -0.125)
        pv.pv_euler_step(b, v, n, -0.125)
        torch.cuda.synchronize()
        assert torch.max(torch.abs(a - b)).item() <= 1e-6 * torch.max(torch.abs(b)).item()
    # equal velocities: guidance has nothing to amplify
    a, b = x.clone(), x.clone()
    pv.pv_euler_cfg_step(a, vc, vc, n, 5.0, -0.125)
    pv.pv_euler_step(b, vc, n, -0.125)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    with pytest.raises(pv.PVError):
        pv.pv_euler_cfg_step(x, vc, 0, n, 5.0, -0.1)
    with pytest.raises(pv.PVError):
        pv.pv_euler_cfg_step(x, vc, vu, n, float("inf"), -0.1)


@pytest.mark.parametrize("n,offset", [(1, 0), (9, 1), (FRAME + 1, 1), (31 * FRAME, 0)])
def test_x0_estimate_matches_oracle(pv, n, offset):
    x = synth.normal_f32(121, (n + offset,), "cuda")
    v = synth.normal_f32(122, (n + offset,), "cuda")
    out = torch.full((n + offset,), 7.0, device="cuda")
    xh, vh = f64(x)[offset:], f64(v)[offset:]
    for sigma in (1.0, 0.75, 0.3125, 0.0):
        pv.pv_x0_estimate(out[offset:], x[offset:], v[offset:], n, sigma)
        torch.cuda.synchronize()
        ref = euler.x0_prediction(xh, vh, sigma)
        got = f64(out)[offset:]
        assert np.all(np.abs(got - ref) <= 2**-23 * (np.abs(xh) + sigma * np.abs(vh)) + 1e-30)
    if offset:
        assert float(out[0]) == 7.0
    # in place (x0 aliases x), and the straight line: x = (1-s) x0 + s x1, v = x1 - x0
    x0 = synth.normal_f32(123, (n,), "cuda")
    x1 = synth.normal_f32(124, (n,), "cuda")
    s = 0.375
    xs = (1 - s) * x0 + s * x1
    pv.pv_x0_estimate(xs, xs, x1 - x0, n, s)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(xs - x0)).item() <= 4e-6 * torch.max(torch.abs(x0) + torch.abs(x1)).item()
