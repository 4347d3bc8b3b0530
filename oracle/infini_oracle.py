"""Plain, slow, float64 restatement of the Infini-attention layer forward.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

Sources (page title, then section):
  [HF]  "Hugging Face Infini-Attention 再現分析" (agentlenshq blog), section
        "Infini-Attention メカニズム": the six steps Segmentation, Local
        Attention, Memory Retrieval, Integration, Memory Update, State Transfer.
  [LNC] "Leave No Context Behind: Efficient Infinite Context Transformers with
        Infini-attention" explainer (abeam guide), sections "基本アイデア",
        "メモリ構造", "メモリの読み出し", "メモリの更新",
        "長期情報と短期情報の統合", "実装上の流れ", FAQ "delta rule".
  [RU]  "Как работает Infini-attention (Google, 2024)" (aivaro), section 3,
        equation 1: the 1/sqrt(d) softmax scale (only that is taken from it).

The pages state the method in prose only.  The readings taken where they are
silent:
  * sigma(x) = ELU(x) + 1 with alpha = 1, applied to the raw q and k.
  * z is a d_k vector (sum of sigma(k) over past tokens); the retrieval
    denominator is the scalar sigma(q_i) . z per row; a row whose denominator
    is exactly 0 retrieves 0 (no epsilon).
  * Segment s reads and (delta rule) corrects against the memory left by
    segment s-1, before this segment's update.
  * The delta rule is applied once per segment: every key of the segment sees
    M_{s-1}.  Rows whose sigma(k).z_{s-1} is 0 take a retrieval term of 0.
  * z grows by the sum of sigma(k) under both rules.
  * The gate is applied on every segment, including the first (where the
    retrieval is 0).
  * Grouped-query heads: query head h reads KV head floor(h / g), g = H_q/H_kv.
  * Only the last segment may be shorter than S; it is causal within itself.

Everything is computed in float64 from the exact values of the inputs (bf16
or fp32 values upcast without rounding).
"""

import numpy as np


def elu_plus_one(x):
    """sigma(x) = ELU(x) + 1: x + 1 for x > 0 and e^x for x <= 0.

    [HF] "Memory Retrieval" and [LNC] "メモリの読み出し" name ELU + 1 as the
    nonlinearity applied to the query (and, for the normaliser and the
    update, to the keys).  Continuous at 0 and strictly positive.
    """
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def gate_sigmoid(beta):
    """Logistic function of the per-head gate logit beta, exact at +-inf.

    [HF] "Integration" and [LNC] "長期情報と短期情報の統合": a learned scalar
    per head, passed through a sigmoid, weighs memory against local attention.
    """
    b = np.asarray(beta, dtype=np.float64)
    out = np.empty_like(b)
    pos = b >= 0.0
    out[pos] = 1.0 / (1.0 + np.exp(-b[pos]))
    eb = np.exp(b[~pos])
    out[~pos] = eb / (1.0 + eb)
    return out


def local_causal_attention(Qs, Ks, Vs):
    """A_dot = softmax(Q K^T / sqrt(d_k) + causal mask) V inside one segment.

    [HF] "Local Attention": standard causal dot-product attention restricted
    to the current segment.  [RU] section 3 eq. 1 fixes the 1/sqrt(d) scale.
    The mask keeps keys j <= i (diagonal included), so no row is empty.
    """
    Qs = np.asarray(Qs, dtype=np.float64)
    Ks = np.asarray(Ks, dtype=np.float64)
    Vs = np.asarray(Vs, dtype=np.float64)
    n, d_k = Qs.shape
    scores = (Qs @ Ks.T) / np.sqrt(d_k)
    future = np.triu(np.ones((n, n), dtype=bool), k=1)
    scores[future] = -np.inf
    scores -= scores.max(axis=1, keepdims=True)
    p = np.exp(scores)
    p /= p.sum(axis=1, keepdims=True)
    return p @ Vs


def memory_retrieval(sQ, M, z):
    """A_mem = sigma(Q) M / (sigma(Q) z), row-wise; 0 where the denominator is 0.

    [HF] "Memory Retrieval" (the query reads the compressive memory M_{s-1});
    [LNC] "メモリの読み出し" (normalised by the sum of past keys, z).
    sQ: [n, d_k] = sigma(Q_s); M: [d_k, d_v]; z: [d_k].
    """
    num = sQ @ M
    den = sQ @ z
    out = np.zeros_like(num)
    nz = den != 0.0
    out[nz] = num[nz] / den[nz, None]
    return out


def memory_update(M, z, sK, Vs, rule):
    """One segment's memory update; returns (M_s, z_s).

    linear ([HF] "Memory Update", [LNC] "メモリの更新"): the segment's
      key/value pairs are added as outer products, M_s = M_{s-1} + sigma(K)^T V.
    delta  ([LNC] "メモリの更新" and FAQ "delta rule"): only what the memory
      does not already return is written,
      M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1})),
      with the retrieval term 0 on rows whose denominator is 0.
    Both rules: z_s = z_{s-1} + sum over the segment's rows of sigma(K).
    """
    if rule == "linear":
        M_new = M + sK.T @ Vs
    elif rule == "delta":
        rden = sK @ z
        R = np.zeros((sK.shape[0], M.shape[1]), dtype=np.float64)
        nz = rden != 0.0
        R[nz] = (sK[nz] @ M) / rden[nz, None]
        M_new = M + sK.T @ (Vs - R)
    else:
        raise ValueError(f"unknown update rule {rule!r}")
    z_new = z + sK.sum(axis=0)
    return M_new, z_new


def segment_bounds(L, S):
    """Row ranges [(s-1)S, min(sS, L)) of the T = ceil(L/S) segments.

    [HF] "Segmentation": the sequence is cut into fixed-length segments that
    are processed in order; only the last one may be shorter.
    """
    if S < 1 or L < 1:
        raise ValueError("segment length and sequence length must be >= 1")
    T = -(-L // S)
    return [(s * S, min((s + 1) * S, L)) for s in range(T)]


def scan_states(k_chain, v_chain, M0, z0, S, rule):
    """Yield (s, r0, r1, M_{s-1}, z_{s-1}) for every segment of one KV chain.

    The generator hands out the memory each segment reads, then applies that
    segment's update ([HF] "State Transfer": only M and z move on to the next
    segment; [LNC] "実装上の流れ": read first, update last).  After the last
    segment it yields (T, L, L, M_T, z_T).
    k_chain: [L, d_k]; v_chain: [L, d_v]; M0: [d_k, d_v]; z0: [d_k].
    """
    M = np.array(M0, dtype=np.float64, copy=True)
    z = np.array(z0, dtype=np.float64, copy=True)
    L = k_chain.shape[0]
    bounds = segment_bounds(L, S)
    for s, (r0, r1) in enumerate(bounds):
        yield s, r0, r1, M, z
        sK = elu_plus_one(k_chain[r0:r1])
        Vs = np.asarray(v_chain[r0:r1], dtype=np.float64)
        M, z = memory_update(M, z, sK, Vs, rule)
    yield len(bounds), L, L, M, z


def segment_output(Qs, Ks, Vs, M_prev, z_prev, beta_h):
    """out = sg(beta) A_mem + (1 - sg(beta)) A_dot for one head and segment.

    [HF] "Integration" / [LNC] "長期情報と短期情報の統合".
    """
    g = float(gate_sigmoid(np.array([beta_h]))[0])
    A_dot = local_causal_attention(Qs, Ks, Vs)
    A_mem = memory_retrieval(elu_plus_one(Qs), M_prev, z_prev)
    return g * A_mem + (1.0 - g) * A_dot


def infini_attention_forward(q, k, v, beta, M_in, z_in, seg_len, rule,
                             heads=None):
    """The layer forward: returns (out, M_out, z_out) in float64.

    q: [B, H_q, L, d_k]; k: [B, H_kv, L, d_k]; v: [B, H_kv, L, d_v];
    beta: [H_q]; M_in: [B, H_kv, d_k, d_v]; z_in: [B, H_kv, d_k].
    ``heads`` optionally restricts which query heads get an output (the rest
    stay 0); M_out and z_out are always computed for every KV head.

    Per KV head, the segments are scanned in order ([HF] six steps;
    [LNC] "実装上の流れ"): each query head of the group attends locally,
    reads M_{s-1}, z_{s-1} and mixes the two; then the memory is updated with
    the segment's keys and values (the memory reuses the attention's Q, K, V:
    [LNC] "メモリ構造").
    """
    B, H_q, L, d_k = q.shape
    H_kv = k.shape[1]
    d_v = v.shape[-1]
    if H_q % H_kv:
        raise ValueError("H_q must be a multiple of H_kv")
    g = H_q // H_kv
    want = set(range(H_q)) if heads is None else set(heads)
    out = np.zeros((B, H_q, L, d_v), dtype=np.float64)
    M_out = np.zeros((B, H_kv, d_k, d_v), dtype=np.float64)
    z_out = np.zeros((B, H_kv, d_k), dtype=np.float64)
    for b in range(B):
        for j in range(H_kv):
            kc = np.asarray(k[b, j], dtype=np.float64)
            vc = np.asarray(v[b, j], dtype=np.float64)
            for s, r0, r1, M, z in scan_states(kc, vc, M_in[b, j], z_in[b, j],
                                               seg_len, rule):
                if r0 == r1:
                    M_out[b, j] = M
                    z_out[b, j] = z
                    break
                for h in range(j * g, (j + 1) * g):
                    if h not in want:
                        continue
                    Qs = np.asarray(q[b, h, r0:r1], dtype=np.float64)
                    out[b, h, r0:r1] = segment_output(Qs, kc[r0:r1], vc[r0:r1],
                                                      M, z, beta[h])
    return out, M_out, z_out
