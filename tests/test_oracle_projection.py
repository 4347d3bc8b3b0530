"""Pins for the float64 oracle's prologue (Q/K/V projections and the rotary
embedding), each against something other than the oracle's own formula:
brute-force loops, complex-number arithmetic, and invariants the rotation
must satisfy.  CPU only.

Sources: "Как работает Infini-attention", section 9 (linear Q/K/V layers);
"Leave No Context Behind" explainer, "メモリ構造" (the memory reuses the
attention's Q/K/V); the rotary embedding of RoFormer with the rotate-half
pairing (a reading: the pages do not define the position encoding).
"""

import cmath
import math

import numpy as np
import pytest

from oracle import apply_rope, qkv_project_rope, qkv_projection, rope_angles, rope_tables


def test_projection_matches_brute_force_loops():
    """Every output element as an explicit sum over the input features, with
    the head order q heads, then k heads, then v heads."""
    rng = np.random.default_rng(7)
    B, L, dm, H_q, H_kv, d = 2, 3, 5, 2, 1, 2
    x = rng.standard_normal((B, L, dm))
    w = rng.standard_normal(((H_q + 2 * H_kv) * d, dm))
    bias = rng.standard_normal((H_q + 2 * H_kv) * d)
    q, k, v = qkv_projection(x, w, bias, H_q, H_kv, d)
    assert q.shape == (B, H_q, L, d) and k.shape == (B, H_kv, L, d) and v.shape == (B, H_kv, L, d)
    for b in range(B):
        for t in range(L):
            for name, out, H, first_row in (("q", q, H_q, 0), ("k", k, H_kv, H_q * d),
                                            ("v", v, H_kv, (H_q + H_kv) * d)):
                for h in range(H):
                    for j in range(d):
                        row = first_row + h * d + j
                        ref = bias[row]
                        for c in range(dm):
                            ref += x[b, t, c] * w[row, c]
                        assert abs(out[b, h, t, j] - ref) < 1e-12, (name, b, t, h, j)


def test_projection_without_bias_is_the_plain_product():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((1, 4, 6))
    w = rng.standard_normal((4 * 3, 6))  # H_q = 2, H_kv = 1, d = 3
    q0, k0, v0 = qkv_projection(x, w, None, 2, 1, 3)
    q1, k1, v1 = qkv_projection(x, w, np.zeros(12), 2, 1, 3)
    for a, b in ((q0, q1), (k0, k1), (v0, v1)):
        assert np.array_equal(a, b)
    assert q0[0, 1, 2, 0] == pytest.approx(float(np.dot(x[0, 2], w[3])), abs=1e-12)


def test_rope_angles_closed_form():
    a = rope_angles(5, 8, base=10000.0)
    assert a.shape == (5, 4)
    assert np.all(a[0] == 0.0)
    # theta_i = 10000^(-2i/8): 1, 0.1, 0.01, 0.001
    assert np.allclose(a[1], [1.0, 0.1, 0.01, 0.001], rtol=1e-14, atol=0)
    assert a[4, 2] == pytest.approx(4 * 0.01, rel=1e-14)
    c, s = rope_tables(3, 2, base=10000.0)
    assert c[2, 0] == pytest.approx(math.cos(2.0), abs=1e-15)
    assert s[2, 0] == pytest.approx(math.sin(2.0), abs=1e-15)


def test_rope_is_complex_multiplication():
    """Pair (x_i, x_{i+d/2}) as x_i + j x_{i+d/2}, rotated by e^{j p theta_i}."""
    rng = np.random.default_rng(9)
    d, L, base = 6, 7, 500.0
    x = rng.standard_normal((L, d))
    c, s = rope_tables(L, d, base)
    y = apply_rope(x, c, s)
    half = d // 2
    for t in range(L):
        for i in range(half):
            theta = base ** (-2.0 * i / d)
            z = complex(x[t, i], x[t, i + half]) * cmath.exp(1j * t * theta)
            assert y[t, i] == pytest.approx(z.real, abs=1e-12)
            assert y[t, i + half] == pytest.approx(z.imag, abs=1e-12)


def test_rope_position_zero_is_identity_and_norms_are_kept():
    rng = np.random.default_rng(10)
    d, L = 16, 9
    x = rng.standard_normal((2, L, d))
    c, s = rope_tables(L, d)
    y = apply_rope(x, c, s)
    assert np.allclose(y[:, 0], x[:, 0], atol=0, rtol=0)
    half = d // 2
    n_x = x[..., :half] ** 2 + x[..., half:] ** 2
    n_y = y[..., :half] ** 2 + y[..., half:] ** 2
    assert np.allclose(n_x, n_y, rtol=1e-13, atol=1e-13)


def test_rope_inverse_rotation_restores_the_input():
    rng = np.random.default_rng(11)
    d, L = 8, 12
    x = rng.standard_normal((L, d))
    c, s = rope_tables(L, d, base=77.0)
    assert np.allclose(apply_rope(apply_rope(x, c, s), c, -s), x, rtol=0, atol=1e-13)


def test_rotated_dot_products_depend_on_relative_position_only():
    """<R(m) q, R(n) k> is a function of m - n: the property the rotary
    embedding exists for."""
    rng = np.random.default_rng(12)
    d = 32
    qv, kv = rng.standard_normal(d), rng.standard_normal(d)
    c, s = rope_tables(300, d)

    def dot(m, n):
        xq = np.zeros((300, d))
        xk = np.zeros((300, d))
        xq[m], xk[n] = qv, kv
        return float(np.dot(apply_rope(xq, c, s)[m], apply_rope(xk, c, s)[n]))

    for m, n in ((7, 3), (4, 0), (104, 100), (299, 295)):
        assert dot(m, n) == pytest.approx(dot(4, 0), rel=1e-11, abs=1e-11)
    assert dot(9, 3) != pytest.approx(dot(4, 0), rel=1e-3)


def test_project_rope_rotates_queries_and_keys_not_values():
    rng = np.random.default_rng(13)
    B, L, dm, H_q, H_kv, d = 1, 6, 8, 4, 2, 4
    x = rng.standard_normal((B, L, dm))
    w = rng.standard_normal(((H_q + 2 * H_kv) * d, dm))
    bias = rng.standard_normal((H_q + 2 * H_kv) * d)
    c, s = rope_tables(L, d)
    q, k, v = qkv_projection(x, w, bias, H_q, H_kv, d)
    qr, kr, vr = qkv_project_rope(x, w, bias, c, s, H_q, H_kv, d)
    assert np.array_equal(v, vr)
    assert np.array_equal(q[:, :, 0], qr[:, :, 0]) and np.array_equal(k[:, :, 0], kr[:, :, 0])
    assert not np.allclose(q[:, :, 1:], qr[:, :, 1:])
    # Bias enters before the rotation: rotating (xW^T) and the bias separately
    # and adding gives the same result (the rotation is linear).
    q0, _, _ = qkv_projection(x, w, None, H_q, H_kv, d)
    bq = np.broadcast_to(bias[: H_q * d].reshape(H_q, 1, d), (H_q, L, d))[None]
    assert np.allclose(apply_rope(q0, c, s) + apply_rope(bq, c, s), qr, atol=1e-12)
    q2, _, _ = qkv_project_rope(x, w, bias, None, None, H_q, H_kv, d)
    assert np.array_equal(q2, q)
