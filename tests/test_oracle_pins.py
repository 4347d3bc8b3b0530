"""Pins for the float64 oracle: each check compares it with something other
than itself -- a library routine, a closed form, brute force, exact rational
arithmetic or an invariant of the method.  CPU only.

Sources: "Hugging Face Infini-Attention 再現分析", section
"Infini-Attention メカニズム" (six steps); "Leave No Context Behind" explainer,
sections "メモリの読み出し", "メモリの更新", "長期情報と短期情報の統合",
"実装上の流れ", FAQ "delta rule".
"""

from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

from oracle import (elu_plus_one, gate_sigmoid, local_causal_attention,
                    memory_retrieval, memory_update, infini_attention_forward,
                    segment_bounds, scan_states)

TOL = 1e-10  # float64 self-consistency bar


def rand_problem(rng, B=2, H_q=4, H_kv=2, L=40, d_k=8, d_v=6):
    q = rng.standard_normal((B, H_q, L, d_k))
    k = rng.standard_normal((B, H_kv, L, d_k))
    v = rng.standard_normal((B, H_kv, L, d_v))
    beta = rng.uniform(-3, 3, size=H_q)
    M0 = np.zeros((B, H_kv, d_k, d_v))
    z0 = np.zeros((B, H_kv, d_k))
    return q, k, v, beta, M0, z0


def sdpa_causal(q, k, v):
    """torch's scaled_dot_product_attention, causal, float64 on CPU."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), is_causal=True).numpy()


# ---------------------------------------------------------------- elementwise

def test_elu_plus_one_matches_torch_elu():
    x = np.concatenate([np.linspace(-30, 30, 2001), [0.0, -0.0, 1e-300, -1e-300]])
    ref = torch.nn.functional.elu(torch.from_numpy(x), alpha=1.0).numpy() + 1.0
    # torch forms expm1(x) + 1, which cancels for x << 0: compare absolutely.
    np.testing.assert_allclose(elu_plus_one(x), ref, rtol=1e-15, atol=2e-16)
    assert np.all(elu_plus_one(x) > 0)


def test_gate_sigmoid_matches_scipy_expit_and_infinities():
    b = np.array([-np.inf, -800, -40, -6, -1e-3, 0.0, 1e-3, 2.5, 40, 800, np.inf])
    np.testing.assert_allclose(gate_sigmoid(b), scipy.special.expit(b), rtol=1e-15, atol=0)
    assert gate_sigmoid(np.array([-np.inf]))[0] == 0.0
    assert gate_sigmoid(np.array([np.inf]))[0] == 1.0


# ---------------------------------------------------------------- A_dot

def test_local_attention_matches_library_sdpa():
    rng = np.random.default_rng(1)
    for n, d in [(1, 4), (7, 8), (33, 16)]:
        Q, K, V = (rng.standard_normal((n, d)) * 3 for _ in range(3))
        np.testing.assert_allclose(local_causal_attention(Q, K, V),
                                   sdpa_causal(Q, K, V), rtol=0, atol=TOL)


def test_beta_minus_inf_is_per_segment_causal_sdpa():
    """beta -> -inf: out equals causal SDPA run on each segment separately."""
    rng = np.random.default_rng(2)
    q, k, v, beta, M0, z0 = rand_problem(rng, L=48)
    beta[:] = -np.inf
    S = 16
    for rule in ("linear", "delta"):
        out, _, _ = infini_attention_forward(q, k, v, beta, M0, z0, S, rule)
        B, H_q, L, d = q.shape
        g = H_q // k.shape[1]
        kr = np.repeat(k, g, axis=1)
        vr = np.repeat(v, g, axis=1)
        # [B, H, T, S, d] -> [B*T, H, S, d]
        T = L // S
        seg = lambda a: a.reshape(B, H_q, T, S, a.shape[-1]).transpose(0, 2, 1, 3, 4).reshape(
            B * T, H_q, S, a.shape[-1])
        ref = sdpa_causal(seg(q), seg(kr), seg(vr))
        ref = ref.reshape(B, T, H_q, S, -1).transpose(0, 2, 1, 3, 4).reshape(B, H_q, L, -1)
        np.testing.assert_allclose(out, ref, rtol=0, atol=TOL)


def test_single_segment_is_gated_causal_sdpa():
    """T = 1 (S = L): out = (1 - sg(beta)) SDPA, and exactly SDPA at beta = -inf."""
    rng = np.random.default_rng(3)
    q, k, v, beta, M0, z0 = rand_problem(rng, H_q=2, H_kv=2, L=25)
    out, _, _ = infini_attention_forward(q, k, v, beta, M0, z0, 25, "linear")
    ref = sdpa_causal(q, k, v)
    w = 1.0 - scipy.special.expit(beta)
    np.testing.assert_allclose(out, ref * w[None, :, None, None], rtol=0, atol=TOL)
    beta[:] = -np.inf
    out, _, _ = infini_attention_forward(q, k, v, beta, M0, z0, 25, "delta")
    np.testing.assert_allclose(out, ref, rtol=0, atol=TOL)


def test_ragged_last_segment_is_causal_within_itself():
    rng = np.random.default_rng(4)
    q, k, v, beta, M0, z0 = rand_problem(rng, B=1, H_q=1, H_kv=1, L=23)
    beta[:] = -np.inf
    out, _, _ = infini_attention_forward(q, k, v, beta, M0, z0, 10, "linear")
    for r0, r1 in segment_bounds(23, 10):
        ref = sdpa_causal(q[:, :, r0:r1], k[:, :, r0:r1], v[:, :, r0:r1])
        np.testing.assert_allclose(out[:, :, r0:r1], ref, rtol=0, atol=TOL)
    assert segment_bounds(23, 10) == [(0, 10), (10, 20), (20, 23)]


# ---------------------------------------------------------------- A_mem, gate

def brute_force_linear_retrieval(q, k, v, S):
    """Kernelised linear attention over all earlier segments, by explicit sums.

    For token i of segment s (zero initial memory, linear rule):
    A_mem[i] = sum_{j < s*S} (sq_i . sk_j) v_j / sum_{j < s*S} (sq_i . sk_j).
    """
    L, d_v = v.shape
    out = np.zeros((L, d_v))
    for i in range(L):
        start = (i // S) * S
        if start == 0:
            continue
        sq = np.where(q[i] > 0, q[i] + 1, np.exp(np.minimum(q[i], 0)))
        num = np.zeros(d_v)
        den = 0.0
        for j in range(start):
            sk = np.where(k[j] > 0, k[j] + 1, np.exp(np.minimum(k[j], 0)))
            w = float(np.dot(sq, sk))
            num += w * v[j]
            den += w
        out[i] = num / den
    return out


def test_beta_plus_inf_is_linear_attention_over_past_segments():
    rng = np.random.default_rng(5)
    q, k, v, beta, M0, z0 = rand_problem(rng, B=1, H_q=2, H_kv=1, L=30, d_k=5, d_v=7)
    beta[:] = np.inf
    S = 8
    out, _, _ = infini_attention_forward(q, k, v, beta, M0, z0, S, "linear")
    for h in range(2):
        ref = brute_force_linear_retrieval(q[0, h], k[0, 0], v[0, 0], S)
        np.testing.assert_allclose(out[0, h], ref, rtol=0, atol=TOL)
    assert np.all(out[0, :, :S] == 0.0)  # first segment: empty memory retrieves 0


def test_finite_gate_mixes_closed_forms():
    """Finite beta: out = expit(beta) * brute-force A_mem + (1 - expit(beta)) * SDPA."""
    rng = np.random.default_rng(6)
    q, k, v, beta, M0, z0 = rand_problem(rng, B=1, H_q=2, H_kv=1, L=24, d_k=4, d_v=4)
    S = 8
    out, _, _ = infini_attention_forward(q, k, v, beta, M0, z0, S, "linear")
    for h in range(2):
        a_mem = brute_force_linear_retrieval(q[0, h], k[0, 0], v[0, 0], S)
        a_dot = np.concatenate([sdpa_causal(q[0, h, r0:r1], k[0, 0, r0:r1], v[0, 0, r0:r1])
                                for r0, r1 in segment_bounds(24, S)])
        gs = scipy.special.expit(beta[h])
        np.testing.assert_allclose(out[0, h], gs * a_mem + (1 - gs) * a_dot, rtol=0, atol=TOL)


def test_retrieval_zero_denominator_gives_zero_and_uses_previous_state():
    sQ = np.ones((3, 4))
    assert np.all(memory_retrieval(sQ, np.ones((4, 2)), np.zeros(4)) == 0.0)
    # A nonzero initial state is read by the first segment.
    M = np.arange(8.0).reshape(4, 2)
    z = np.array([1.0, 2.0, 3.0, 4.0])
    got = memory_retrieval(sQ, M, z)
    np.testing.assert_allclose(got, np.tile(M.sum(0) / z.sum(), (3, 1)), atol=TOL)


# ---------------------------------------------------------------- update

def brute_force_state(k, v):
    M = np.zeros((k.shape[1], v.shape[1]))
    z = np.zeros(k.shape[1])
    for t in range(k.shape[0]):
        sk = np.where(k[t] > 0, k[t] + 1, np.exp(np.minimum(k[t], 0)))
        M += np.outer(sk, v[t])
        z += sk
    return M, z


def test_linear_state_is_brute_force_sum_and_independent_of_segment_length():
    rng = np.random.default_rng(7)
    q, k, v, beta, M0, z0 = rand_problem(rng, L=32)
    refs = [brute_force_state(k[b, j], v[b, j]) for b in range(2) for j in range(2)]
    for S in (32, 16, 8, 4, 2, 1, 5, 7):
        _, M, z = infini_attention_forward(q, k, v, beta, M0, z0, S, "linear")
        for n, (Mr, zr) in enumerate(refs):
            b, j = divmod(n, 2)
            np.testing.assert_allclose(M[b, j], Mr, rtol=0, atol=TOL)
            np.testing.assert_allclose(z[b, j], zr, rtol=0, atol=TOL)


def test_linear_state_invariant_to_token_order_within_segment():
    rng = np.random.default_rng(8)
    k = rng.standard_normal((16, 6))
    v = rng.standard_normal((16, 5))
    sK = elu_plus_one(k)
    M, z = memory_update(np.zeros((6, 5)), np.zeros(6), sK, v, "linear")
    p = rng.permutation(16)
    M2, z2 = memory_update(np.zeros((6, 5)), np.zeros(6), sK[p], v[p], "linear")
    np.testing.assert_allclose(M, M2, atol=TOL)
    np.testing.assert_allclose(z, z2, atol=TOL)


def test_delta_equals_linear_on_first_update():
    rng = np.random.default_rng(9)
    sK = elu_plus_one(rng.standard_normal((12, 6)))
    V = rng.standard_normal((12, 5))
    Ml, zl = memory_update(np.zeros((6, 5)), np.zeros(6), sK, V, "linear")
    Md, zd = memory_update(np.zeros((6, 5)), np.zeros(6), sK, V, "delta")
    np.testing.assert_array_equal(Ml, Md)
    np.testing.assert_array_equal(zl, zd)
    # Through the whole layer: a single-segment stream gives the same state.
    q, k, v, beta, M0, z0 = rand_problem(rng, L=16)
    a = infini_attention_forward(q, k, v, beta, M0, z0, 16, "linear")
    b = infini_attention_forward(q, k, v, beta, M0, z0, 16, "delta")
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_delta_fixed_point():
    """If every value equals what the memory already returns for its key,
    the delta rule leaves M unchanged (z still grows)."""
    rng = np.random.default_rng(10)
    d_k, d_v = 6, 5
    # A prior state left by a real segment of 20 tokens.
    sK0 = elu_plus_one(rng.standard_normal((20, d_k)))
    M, z = memory_update(np.zeros((d_k, d_v)), np.zeros(d_k), sK0,
                         rng.standard_normal((20, d_v)), "linear")
    sK = elu_plus_one(rng.standard_normal((9, d_k)))
    V = (sK @ M) / (sK @ z)[:, None]
    M1, z1 = memory_update(M, z, sK, V, "delta")
    np.testing.assert_allclose(M1, M, rtol=0, atol=1e-12)
    np.testing.assert_allclose(z1, z + sK.sum(0), rtol=0, atol=1e-12)
    # The linear rule does move: the pin above is not vacuous.
    M2, _ = memory_update(M, z, sK, V, "linear")
    assert np.abs(M2 - M).max() > 1e-3


def test_delta_one_hot_keys_slot_recurrence():
    """Keys whose sigma is a unit vector e_i (one coordinate 0, the rest -60)
    turn the memory into slots: z_i counts writes and row i of M holds
    m_i.  The delta rule then gives, per segment and slot,
    m_i <- m_i + sum(v) - n_i * m_i / c_i (c_i > 0), m_i <- m_i + sum(v) (c_i = 0),
    c_i <- c_i + n_i -- derived by hand from the rule, no matrices involved."""
    rng = np.random.default_rng(11)
    d_k, d_v, S, T = 4, 3, 5, 6
    slots = rng.integers(0, d_k, size=S * T)
    k = np.full((S * T, d_k), -60.0)
    k[np.arange(S * T), slots] = 0.0
    v = rng.standard_normal((S * T, d_v))
    m = np.zeros((d_k, d_v))
    c = np.zeros(d_k)
    for s in range(T):
        rows = range(s * S, (s + 1) * S)
        new_m = m.copy()
        for i in range(d_k):
            mine = [t for t in rows if slots[t] == i]
            if not mine:
                continue
            new_m[i] += v[mine].sum(0)
            if c[i] > 0:
                new_m[i] -= len(mine) * m[i] / c[i]
        for t in rows:
            c[slots[t]] += 1
        m = new_m
    q = rng.standard_normal((1, 1, S * T, d_k))
    _, M, z = infini_attention_forward(q, k[None, None], v[None, None], np.zeros(1),
                                       np.zeros((1, 1, d_k, d_v)), np.zeros((1, 1, d_k)), S, "delta")
    np.testing.assert_allclose(M[0, 0], m, rtol=0, atol=1e-9)
    np.testing.assert_allclose(z[0, 0], c, rtol=0, atol=1e-9)


def test_exact_rational_worked_example():
    """Positive q and k make sigma(x) = x + 1 rational, and beta = +inf makes
    out = A_mem, so the whole memory path has an exact rational answer.
    Computed here with Fractions by brute force over past tokens (linear) and
    by the slotless per-token sums; compared to the float64 oracle."""
    q = [[Fraction(1, 2), Fraction(1, 4)], [Fraction(3, 2), Fraction(1, 1)],
         [Fraction(1, 8), Fraction(2, 1)], [Fraction(5, 4), Fraction(3, 8)],
         [Fraction(1, 1), Fraction(1, 2)], [Fraction(3, 4), Fraction(7, 4)]]
    k = [[Fraction(1, 4), Fraction(1, 2)], [Fraction(1, 1), Fraction(1, 8)],
         [Fraction(3, 8), Fraction(5, 4)], [Fraction(2, 1), Fraction(1, 4)],
         [Fraction(1, 2), Fraction(3, 2)], [Fraction(1, 8), Fraction(1, 1)]]
    v = [[Fraction(1, 1), Fraction(-2, 1)], [Fraction(3, 1), Fraction(1, 2)],
         [Fraction(-1, 2), Fraction(5, 4)], [Fraction(2, 1), Fraction(1, 1)],
         [Fraction(-3, 2), Fraction(1, 4)], [Fraction(1, 4), Fraction(-1, 1)]]
    S = 2
    sig = lambda r: [x + 1 for x in r]
    expect = []
    for i in range(6):
        start = (i // S) * S
        if start == 0:
            expect.append([Fraction(0), Fraction(0)])
            continue
        sq = sig(q[i])
        w = [sum(a * b for a, b in zip(sq, sig(k[j]))) for j in range(start)]
        den = sum(w)
        expect.append([sum(w[j] * v[j][c] for j in range(start)) / den for c in range(2)])
    Mexp = [[sum(sig(k[t])[a] * v[t][c] for t in range(6)) for c in range(2)] for a in range(2)]
    zexp = [sum(sig(k[t])[a] for t in range(6)) for a in range(2)]
    f = lambda x: np.array(x, dtype=np.float64)
    out, M, z = infini_attention_forward(f(q)[None, None], f(k)[None, None], f(v)[None, None],
                                         np.array([np.inf]), np.zeros((1, 1, 2, 2)),
                                         np.zeros((1, 1, 2)), S, "linear")
    np.testing.assert_allclose(out[0, 0], f(expect), rtol=1e-14, atol=0)
    np.testing.assert_allclose(M[0, 0], f(Mexp), rtol=1e-14, atol=0)
    np.testing.assert_allclose(z[0, 0], f(zexp), rtol=1e-14, atol=0)
    assert expect[2][0] == Fraction(expect[2][0])  # exact value, not a float


# ---------------------------------------------------------------- layout / state transfer

def test_gqa_equals_mha_with_repeated_kv():
    rng = np.random.default_rng(12)
    q, k, v, beta, M0, z0 = rand_problem(rng, B=2, H_q=6, H_kv=2, L=24)
    for rule in ("linear", "delta"):
        out, M, z = infini_attention_forward(q, k, v, beta, M0, z0, 8, rule)
        kr, vr = np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1)
        out2, M2, z2 = infini_attention_forward(q, kr, vr, beta, np.repeat(M0, 3, 1),
                                                np.repeat(z0, 3, 1), 8, rule)
        np.testing.assert_allclose(out, out2, rtol=0, atol=TOL)
        for h in range(6):
            np.testing.assert_allclose(M2[:, h], M[:, h // 3], rtol=0, atol=TOL)
            np.testing.assert_allclose(z2[:, h], z[:, h // 3], rtol=0, atol=TOL)


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_split_stream_equals_whole_stream(rule):
    """forward(L1) then forward(L2) with the state carried equals forward(L1+L2)
    when L1 is a whole number of segments ([HF] "State Transfer")."""
    rng = np.random.default_rng(13)
    q, k, v, beta, M0, z0 = rand_problem(rng, L=36)
    S, L1 = 6, 18
    out, M, z = infini_attention_forward(q, k, v, beta, M0, z0, S, rule)
    o1, M1, z1 = infini_attention_forward(q[:, :, :L1], k[:, :, :L1], v[:, :, :L1], beta, M0, z0, S, rule)
    o2, M2, z2 = infini_attention_forward(q[:, :, L1:], k[:, :, L1:], v[:, :, L1:], beta, M1, z1, S, rule)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=2), out, rtol=0, atol=TOL)
    np.testing.assert_allclose(M2, M, rtol=0, atol=TOL)
    np.testing.assert_allclose(z2, z, rtol=0, atol=TOL)


def test_scan_states_yields_previous_memory():
    rng = np.random.default_rng(14)
    k = rng.standard_normal((10, 3))
    v = rng.standard_normal((10, 2))
    seen = list(scan_states(k, v, np.zeros((3, 2)), np.zeros(3), 4, "linear"))
    assert [(s, r0, r1) for s, r0, r1, _, _ in seen] == [(0, 0, 4), (1, 4, 8), (2, 8, 10), (3, 10, 10)]
    for s, r0, _, M, z in seen:
        Mr, zr = brute_force_state(k[:r0], v[:r0]) if r0 else (np.zeros((3, 2)), np.zeros(3))
        np.testing.assert_allclose(M, Mr, atol=TOL)
        np.testing.assert_allclose(z, zr, atol=TOL)
