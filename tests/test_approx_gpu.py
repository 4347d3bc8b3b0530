"""The attention kernel's own device approximations, checked against float64
references: the FMA-pipe 2^x (range reduction + a degree-3 polynomial fitted
on [-1/2, 1/2], stated relative error 7.6e-5), the hardware 2^x, and the
integer bf16 packing of non-negative probabilities."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_exp2_approximations(cuda_lib):
    api = cuda_lib
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001), torch.tensor([0.0, -0.5, 0.5, 7.999])])
    xg = x.float().cuda()
    y_poly, y_mufu, _ = api.selftest_approx(xg)
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    rel_poly = ((y_poly.double().cpu() - ref).abs() / ref).max().item()
    rel_mufu = ((y_mufu.double().cpu() - ref).abs() / ref).max().item()
    assert rel_poly <= 8e-5, rel_poly
    assert rel_mufu <= 1e-6, rel_mufu
    # Below the clamp the polynomial path returns 2^-125 times ~1: far below
    # anything that reaches a probability sum (>= 1).
    y, _, _ = api.selftest_approx(torch.tensor([-1e30, -300.0, -126.0], device="cuda"))
    assert torch.all(y.cpu().double() <= 2.0 ** -124)


def test_probability_packing_is_bf16_rounding(cuda_lib):
    api = cuda_lib
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(0, 300, 200000), 2.0 ** rng.uniform(-40, 8, 200000), [0.0, 1.0, 256.0]])
    xt = torch.from_numpy(x.astype(np.float32))
    _, _, bits = api.selftest_approx(xt.cuda())
    got = bits.cpu().numpy().astype(np.uint32)
    u = xt.numpy().view(np.uint32)
    half_up = ((u + 0x8000) >> 16).astype(np.uint32)
    np.testing.assert_array_equal(got, half_up)
    # Against round-to-nearest-even it differs only on exact ties.
    rne = xt.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).astype(np.uint32)
    diff = got != rne
    assert np.all((u[diff] & 0xFFFF) == 0x8000)
