"""Pins for the float64 oracle's backward: central finite differences of the
forward oracle (which shares no code with the backward), torch autograd of
library routines, and closed forms of special cases.  CPU only.

Training through the memory is back-propagation through time over the
segments ("Hugging Face Infini-Attention 再現分析", "重み減衰とロールアウト";
"Leave No Context Behind" explainer, "限界").
"""

import numpy as np
import pytest
import torch

from oracle import (elu_plus_one, elu_plus_one_grad, infini_attention_backward,
                    infini_attention_forward, local_causal_attention_vjp)


def _away_from_zero(rng, shape, gap=1e-2):
    """N(0, 1) samples with |x| >= gap (sigma has a kink in its second
    derivative at 0, which a finite difference straddling it would see)."""
    x = rng.standard_normal(shape)
    return np.where(np.abs(x) < gap, np.sign(x + 1e-30) * gap + x, x)


def _problem(rng, B, H_q, H_kv, L, d_k, d_v):
    q = _away_from_zero(rng, (B, H_q, L, d_k))
    k = _away_from_zero(rng, (B, H_kv, L, d_k))
    v = rng.standard_normal((B, H_kv, L, d_v))
    beta = rng.uniform(-2, 2, size=H_q)
    M_in = rng.standard_normal((B, H_kv, d_k, d_v))
    z_in = rng.uniform(0.5, 1.5, size=(B, H_kv, d_k))  # den, r > 0 everywhere
    return [q, k, v, beta, M_in, z_in]


def _loss(inputs, seg_len, rule, dout, dM_out, dz_out):
    out, M_out, z_out = infini_attention_forward(*inputs, seg_len, rule)
    return float((dout * out).sum() + (dM_out * M_out).sum() + (dz_out * z_out).sum())


def test_elu_plus_one_grad_matches_torch_autograd():
    x = torch.linspace(-20, 20, 4001, dtype=torch.float64, requires_grad=True)
    (torch.nn.functional.elu(x, alpha=1.0) + 1.0).sum().backward()
    np.testing.assert_allclose(elu_plus_one_grad(x.detach().numpy()), x.grad.numpy(),
                               rtol=1e-15, atol=0)


def test_attention_vjp_matches_torch_autograd_sdpa():
    rng = np.random.default_rng(7)
    n, d_k, d_v = 13, 8, 5
    Q, K, V, dA = (rng.standard_normal(s) for s in [(n, d_k), (n, d_k), (n, d_v), (n, d_v)])
    tq, tk, tv = (torch.from_numpy(a).requires_grad_(True) for a in (Q, K, V))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    out.backward(torch.from_numpy(dA))
    dQ, dK, dV = local_causal_attention_vjp(Q, K, V, dA)
    for got, ref in ((dQ, tq.grad), (dK, tk.grad), (dV, tv.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("rule", ["linear", "delta"])
@pytest.mark.parametrize("shape", [
    # GQA (two query heads per KV head), a ragged last segment (3, 3, 1)
    dict(B=1, H_q=2, H_kv=1, L=7, d_k=3, d_v=2, S=3),
    # two batch rows, two KV heads, one query head each, segments (2, 2, 2, 1)
    dict(B=2, H_q=2, H_kv=2, L=7, d_k=2, d_v=3, S=2),
])
def test_backward_matches_central_differences(rule, shape):
    rng = np.random.default_rng(11 if rule == "linear" else 12)
    S = shape.pop("S")
    inputs = _problem(rng, **shape)
    shape["S"] = S
    B, H_q, H_kv, L, d_k, d_v = (shape[n] for n in ("B", "H_q", "H_kv", "L", "d_k", "d_v"))
    dout = rng.standard_normal((B, H_q, L, d_v))
    dM_out = rng.standard_normal((B, H_kv, d_k, d_v))
    dz_out = rng.standard_normal((B, H_kv, d_k))
    grads = infini_attention_backward(*inputs, S, rule, dout, dM_out, dz_out)
    h = 1e-6
    for idx, (x, gx) in enumerate(zip(inputs, grads)):
        assert gx.shape == x.shape
        fd = np.zeros_like(x)
        for pos in np.ndindex(x.shape):
            keep = x[pos]
            x[pos] = keep + h
            jp = _loss(inputs, S, rule, dout, dM_out, dz_out)
            x[pos] = keep - h
            jm = _loss(inputs, S, rule, dout, dM_out, dz_out)
            x[pos] = keep
            fd[pos] = (jp - jm) / (2 * h)
        np.testing.assert_allclose(gx, fd, rtol=2e-6, atol=2e-6, err_msg=f"input {idx}")


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_gate_closed_at_local_attention_only(rule):
    """g = 0 (beta = -inf): the output ignores the memory, so nothing flows
    from dout into M_in, z_in or beta; for the linear rule the state
    gradients pass straight through (dM_in = dM_out, dz_in = dz_out)."""
    rng = np.random.default_rng(3)
    q, k, v, beta, M_in, z_in = _problem(rng, 1, 2, 1, 9, 3, 4)
    beta[:] = -np.inf
    dout = rng.standard_normal((1, 2, 9, 4))
    dM_out = rng.standard_normal((1, 1, 3, 4))
    dz_out = rng.standard_normal((1, 1, 3))
    dq, dk, dv, db, dM_in, dz_in = infini_attention_backward(
        q, k, v, beta, M_in, z_in, 4, rule, dout, dM_out, dz_out)
    assert np.all(db == 0.0)
    if rule == "linear":
        np.testing.assert_array_equal(dM_in, dM_out)
        np.testing.assert_array_equal(dz_in, dz_out)
    # dout alone moves none of the state gradients
    _, _, _, db0, dM0, dz0 = infini_attention_backward(
        q, k, v, beta, M_in, z_in, 4, rule, dout, np.zeros_like(dM_out), np.zeros_like(dz_out))
    assert np.all(dM0 == 0.0) and np.all(dz0 == 0.0) and np.all(db0 == 0.0)


def test_linear_update_gradient_closed_form():
    """dout = 0, linear rule: only the update path carries gradient, and the
    state gradient is constant over the segments, so
    dk_t = (v_t dM^T + dz) * sigma'(k_t) and dv_t = sigma(k_t) dM."""
    rng = np.random.default_rng(5)
    q, k, v, beta, M_in, z_in = _problem(rng, 1, 1, 1, 10, 4, 3)
    dM = rng.standard_normal((1, 1, 4, 3))
    dz = rng.standard_normal((1, 1, 4))
    dq, dk, dv, db, dM_in, dz_in = infini_attention_backward(
        q, k, v, beta, M_in, z_in, 3, "linear", np.zeros((1, 1, 10, 3)), dM, dz)
    kk, vv = k[0, 0], v[0, 0]
    np.testing.assert_allclose(dk[0, 0], (vv @ dM[0, 0].T + dz[0, 0]) * elu_plus_one_grad(kk),
                               rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dv[0, 0], elu_plus_one(kk) @ dM[0, 0], rtol=1e-13, atol=1e-13)
    assert np.all(dq == 0.0) and np.all(db == 0.0)
    np.testing.assert_array_equal(dM_in, dM)
    np.testing.assert_array_equal(dz_in, dz)
