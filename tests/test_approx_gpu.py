"""The attention kernel's own device approximations, checked against float64
references: the FMA-pipe 2^x (range reduction + a degree-3 polynomial fitted
on [-1/2, 1/2], stated relative error 7.6e-5; both lanes of the paired
version), the hardware 2^x, and the bf16 packing of probabilities."""

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
    """The packing of P is round-to-nearest-even bf16 (what torch does)."""
    api = cuda_lib
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(0, 300, 200000), 2.0 ** rng.uniform(-40, 8, 200000), [0.0, 1.0, 256.0]])
    xt = torch.from_numpy(x.astype(np.float32))
    _, _, bits = api.selftest_approx(xt.cuda())
    got = bits.cpu().numpy().astype(np.uint32)
    rne = xt.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).astype(np.uint32)
    np.testing.assert_array_equal(got, rne)
    # Exact ties go to the even neighbour: 1 + 2^-8 -> 1, 1 + 3 * 2^-8 -> 1 + 2^-6.
    ties = torch.tensor([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8], dtype=torch.float32)
    _, _, tb = api.selftest_approx(ties.cuda())
    got_t = tb.cpu().numpy().astype(np.uint32) << 16
    np.testing.assert_array_equal(got_t.view(np.float32), np.array([1.0, 1 + 2.0 ** -6], np.float32))


def test_bounded_wait_timeout_sets_status_and_context_survives(cuda_lib):
    """The kernels' bounded mbarrier wait, made to run out on purpose (a
    barrier nothing arrives at): the kernel returns, the status word reports
    the timeout once, and the context keeps working."""
    api = cuda_lib
    api.sync_status()  # start clean
    api.selftest_timeout()
    with pytest.raises(api.InfiniError) as e:
        api.sync_status()
    assert e.value.status == api.ERR_TIMEOUT
    api.sync_status()  # the word was cleared
    y, _, _ = api.selftest_approx(torch.tensor([0.0, 1.0, -1.0], device="cuda"))
    assert torch.allclose(y.cpu(), torch.tensor([1.0, 2.0, 0.5]), rtol=1e-4)
