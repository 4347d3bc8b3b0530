"""Plain float64 backward (vector-Jacobian products) of the layer forward in
``infini_oracle``: the gradients of a scalar loss with respect to q, k, v,
beta, M_in and z_in, given its gradients with respect to out, M_out and z_out.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

The forward is the one stated in ``infini_oracle`` (sources [HF] "Hugging Face
Infini-Attention 再現分析", "Infini-Attention メカニズム"; [LNC] "Leave No
Context Behind" explainer, "メモリの読み出し", "メモリの更新", FAQ "delta
rule"; [RU] section 3 eq. 1 for the 1/sqrt(d) scale).  Training through the
memory is back-propagation through time over the segments ([HF] "重み減衰と
ロールアウト": rollout 16 x segment 64; [LNC] "限界": BPTT); the pages give no
gradient formulas, so every step below is the chain rule applied to the
forward's own steps, in reverse order:

  * per KV head, the segments are walked backwards carrying dL/dM_s and
    dL/dz_s (starting from dM_out, dz_out);
  * segment s's update (M_{s-1}, z_{s-1}, sigma(K_s), V_s) -> (M_s, z_s) is
    differentiated first, then every query head's output of segment s, which
    read M_{s-1} and z_{s-1};
  * rows whose retrieval denominator (sigma(q).z or, delta rule, sigma(k).z)
    is exactly 0 take a constant 0 in the forward, so no gradient flows
    through them (the readings of the forward);
  * sigma'(x) = 1 for x > 0 and e^x for x <= 0 (continuous at 0).

Pinned in ``tests/test_oracle_backward.py`` against central finite
differences of ``infini_attention_forward`` (which uses none of this file)
and closed forms of special cases.
"""

import numpy as np

from .infini_oracle import (elu_plus_one, gate_sigmoid, scan_states,
                            segment_bounds)


def elu_plus_one_grad(x):
    """d sigma / dx: 1 for x > 0, e^x for x <= 0."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, 1.0, np.exp(np.minimum(x, 0.0)))


def local_causal_attention_vjp(Qs, Ks, Vs, dA):
    """(dQ, dK, dV) of A = softmax(Q K^T / sqrt(d) + causal mask) V.

    With P the row-softmax: dV = P^T dA, dP = dA V^T, and the softmax's
    Jacobian gives dS = P * (dP - rowsum(dP * P)); the scores' scale carries
    into dQ = dS K / sqrt(d) and dK = dS^T Q / sqrt(d).
    """
    n, d_k = Qs.shape
    scale = 1.0 / np.sqrt(d_k)
    scores = (Qs @ Ks.T) * scale
    scores[np.triu(np.ones((n, n), dtype=bool), k=1)] = -np.inf
    scores -= scores.max(axis=1, keepdims=True)
    P = np.exp(scores)
    P /= P.sum(axis=1, keepdims=True)
    dV = P.T @ dA
    dP = dA @ Vs.T
    dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
    return (dS @ Ks) * scale, (dS.T @ Qs) * scale, dV


def memory_retrieval_vjp(sQ, M, z, dA):
    """(d sigma(Q), dM, dz) of A = sigma(Q) M / (sigma(Q) z) (0 rows where den = 0).

    num = sQ M, den = sQ z: dnum = dA / den, dden = -rowsum(dA * A) / den on
    rows with den != 0 (0 elsewhere); d sQ = dnum M^T + dden z^T,
    dM = sQ^T dnum, dz = sQ^T dden.
    """
    num = sQ @ M
    den = sQ @ z
    nz = den != 0.0
    A = np.zeros_like(num)
    A[nz] = num[nz] / den[nz, None]
    dnum = np.zeros_like(num)
    dnum[nz] = dA[nz] / den[nz, None]
    dden = np.zeros_like(den)
    dden[nz] = -(dA[nz] * A[nz]).sum(axis=1) / den[nz]
    dsQ = dnum @ M.T + np.outer(dden, z)
    return dsQ, sQ.T @ dnum, sQ.T @ dden


def memory_update_vjp(M, z, sK, Vs, rule, dM_new, dz_new):
    """(dM, dz, d sigma(K), dV) of one segment's update (M, z) -> (M_new, z_new).

    linear: M_new = M + sK^T V.
    delta:  r = sK z, R = (sK M) / r (0 rows where r = 0), U = V - R,
            M_new = M + sK^T U.
    Both:   z_new = z + colsum(sK).
    """
    dM = dM_new.copy()
    dz = dz_new.copy()
    if rule == "linear":
        dsK = Vs @ dM_new.T
        dV = sK @ dM_new
    elif rule == "delta":
        r = sK @ z
        nz = r != 0.0
        N = sK @ M
        R = np.zeros_like(N)
        R[nz] = N[nz] / r[nz, None]
        U = Vs - R
        dU = sK @ dM_new
        dsK = U @ dM_new.T
        dV = dU.copy()
        dR = -dU
        dN = np.zeros_like(N)
        dN[nz] = dR[nz] / r[nz, None]
        dr = np.zeros_like(r)
        dr[nz] = -(dR[nz] * R[nz]).sum(axis=1) / r[nz]
        dsK += dN @ M.T + np.outer(dr, z)
        dM += sK.T @ dN
        dz += sK.T @ dr
    else:
        raise ValueError(f"unknown update rule {rule!r}")
    dsK += dz_new[None, :]
    return dM, dz, dsK, dV


def segment_output_vjp(Qs, Ks, Vs, M_prev, z_prev, beta_h, dout):
    """(dQ, dK, dV, dM_prev, dz_prev, dbeta) of
    out = g A_mem + (1 - g) A_dot, g = sigmoid(beta).

    dA_mem = g dout, dA_dot = (1 - g) dout, dg = sum(dout * (A_mem - A_dot)),
    dbeta = dg g (1 - g); sigma(Q)'s gradient goes through sigma'(Q).
    """
    g = float(gate_sigmoid(np.array([beta_h]))[0])
    sQ = elu_plus_one(Qs)
    num = sQ @ M_prev
    den = sQ @ z_prev
    A_mem = np.zeros_like(num)
    nz = den != 0.0
    A_mem[nz] = num[nz] / den[nz, None]
    n, d_k = Qs.shape
    scores = (Qs @ Ks.T) / np.sqrt(d_k)
    scores[np.triu(np.ones((n, n), dtype=bool), k=1)] = -np.inf
    scores -= scores.max(axis=1, keepdims=True)
    P = np.exp(scores)
    P /= P.sum(axis=1, keepdims=True)
    A_dot = P @ Vs
    dbeta = float((dout * (A_mem - A_dot)).sum()) * g * (1.0 - g)
    dsQ, dM, dz = memory_retrieval_vjp(sQ, M_prev, z_prev, g * dout)
    dQ, dK, dV = local_causal_attention_vjp(Qs, Ks, Vs, (1.0 - g) * dout)
    dQ += dsQ * elu_plus_one_grad(Qs)
    return dQ, dK, dV, dM, dz, dbeta


def infini_attention_backward(q, k, v, beta, M_in, z_in, seg_len, rule,
                              dout, dM_out, dz_out):
    """Gradients (dq, dk, dv, dbeta, dM_in, dz_in), float64, of the loss whose
    gradients with respect to (out, M_out, z_out) are (dout, dM_out, dz_out).

    Shapes as in ``infini_attention_forward``; the returned gradients have
    the shapes of the corresponding inputs.
    """
    B, H_q, L, d_k = q.shape
    H_kv = k.shape[1]
    d_v = v.shape[-1]
    g = H_q // H_kv
    dq = np.zeros((B, H_q, L, d_k))
    dk = np.zeros((B, H_kv, L, d_k))
    dv = np.zeros((B, H_kv, L, d_v))
    dbeta = np.zeros(H_q)
    dM_in = np.zeros((B, H_kv, d_k, d_v))
    dz_in = np.zeros((B, H_kv, d_k))
    bounds = segment_bounds(L, seg_len)
    for b in range(B):
        for j in range(H_kv):
            kc = np.asarray(k[b, j], dtype=np.float64)
            vc = np.asarray(v[b, j], dtype=np.float64)
            # The memory each segment read (M_{s-1}, z_{s-1}), from the forward scan.
            states = [(M, z) for s, r0, r1, M, z in
                      scan_states(kc, vc, M_in[b, j], z_in[b, j], seg_len, rule)]
            gM = np.array(dM_out[b, j], dtype=np.float64)
            gz = np.array(dz_out[b, j], dtype=np.float64)
            for s in reversed(range(len(bounds))):
                r0, r1 = bounds[s]
                M_prev, z_prev = states[s]
                Ks, Vs = kc[r0:r1], vc[r0:r1]
                sK = elu_plus_one(Ks)
                gM, gz, dsK, dVs = memory_update_vjp(M_prev, z_prev, sK, Vs, rule, gM, gz)
                dk[b, j, r0:r1] += dsK * elu_plus_one_grad(Ks)
                dv[b, j, r0:r1] += dVs
                for h in range(j * g, (j + 1) * g):
                    Qs = np.asarray(q[b, h, r0:r1], dtype=np.float64)
                    dQ, dK, dV, dMr, dzr, db = segment_output_vjp(
                        Qs, Ks, Vs, M_prev, z_prev, beta[h],
                        np.asarray(dout[b, h, r0:r1], dtype=np.float64))
                    dq[b, h, r0:r1] = dQ
                    dk[b, j, r0:r1] += dK
                    dv[b, j, r0:r1] += dV
                    gM = gM + dMr
                    gz = gz + dzr
                    dbeta[h] += db
            dM_in[b, j] = gM
            dz_in[b, j] = gz
    return dq, dk, dv, dbeta, dM_in, dz_in
