"""Plain float64 Q/K/V projections with rotary position embedding: the
prologue that produces the query, key and value heads the layer consumes.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

Sources and readings.
  * The memory reuses the attention's own Q, K and V; no separate features
    are computed for it ("Leave No Context Behind" explainer, "メモリ構造").
  * Each segment's Q, K and V come from linear layers over the layer input
    (d_model -> d_model, with bias) ("Как работает Infini-attention", section
    9, simplified implementation).  Applied to every token of the sequence at
    once, that is one product y = x W^T + b; W stacks the query rows (H_q * d
    of them), then the key rows (H_kv * d), then the value rows (H_kv * d),
    the usual fused-QKV weight; head h of each part is its columns
    [h d, (h + 1) d).
  * The pages name no position encoding beyond noting that the HF reproduction
    starts from Llama models (which use rotary embeddings) and listing RoPE
    scaling as a competing context extension.  Reading taken: the rotary
    embedding of RoFormer (Su et al., 2021), with the pairing of the Llama
    family, dimension i with dimension i + d/2 ("rotate half"):
        x'_i         = x_i cos(a_{t,i}) - x_{i+d/2} sin(a_{t,i})
        x'_{i+d/2}   = x_{i+d/2} cos(a_{t,i}) + x_i sin(a_{t,i})
    for i < d/2, a_{t,i} = p_t * base^(-2i/d), p_t the position of token t.
    Queries and keys are rotated, values are not; the bias is added before
    the rotation.  The rotation is given by cos / sin tables [positions, d/2]
    (one row per token), so a caller may count positions over the whole
    sequence or restart them in each segment.

Pinned in ``tests/test_oracle_projection.py``: brute-force loops on tiny
inputs, the complex-number form of the rotation, the relative-position
property of rotated dot products, norm preservation and inverses.
"""

import numpy as np


def rope_angles(n_pos, d, base=10000.0):
    """a[p, i] = p * base^(-2 i / d) for positions p = 0..n_pos-1, i < d/2."""
    if d % 2:
        raise ValueError("the rotary embedding needs an even head dimension")
    inv = np.asarray(base, dtype=np.float64) ** (-2.0 * np.arange(d // 2, dtype=np.float64) / d)
    return np.outer(np.arange(n_pos, dtype=np.float64), inv)


def rope_tables(n_pos, d, base=10000.0):
    """(cos, sin) of rope_angles, float64 [n_pos, d/2]."""
    a = rope_angles(n_pos, d, base)
    return np.cos(a), np.sin(a)


def apply_rope(x, cos, sin):
    """Rotate x [..., L, d] token by token: row t of x by row t of the tables
    (rotate-half pairing, dimension i with i + d/2)."""
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    c = np.asarray(cos, dtype=np.float64)[: x.shape[-2]]
    s = np.asarray(sin, dtype=np.float64)[: x.shape[-2]]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def qkv_projection(x, w, bias, H_q, H_kv, d):
    """y = x W^T (+ bias), split into heads.

    x [B, L, d_model], w [(H_q + 2 H_kv) d, d_model], bias [(H_q + 2 H_kv) d]
    or None.  Returns q [B, H_q, L, d], k and v [B, H_kv, L, d], float64.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    B, L, _ = x.shape
    if w.shape[0] != (H_q + 2 * H_kv) * d:
        raise ValueError("weight rows must be (H_q + 2 H_kv) * d")
    y = x @ w.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    nq, nk = H_q * d, H_kv * d

    def heads(part, H):
        return part.reshape(B, L, H, d).transpose(0, 2, 1, 3)

    return (heads(y[..., :nq], H_q), heads(y[..., nq:nq + nk], H_kv),
            heads(y[..., nq + nk:], H_kv))


def qkv_project_rope(x, w, bias, cos, sin, H_q, H_kv, d):
    """The prologue: projections, then the rotation of queries and keys.
    cos / sin [>= L, d/2], or None for no rotation."""
    q, k, v = qkv_projection(x, w, bias, H_q, H_kv, d)
    if cos is not None:
        q = apply_rope(q, cos, sin)
        k = apply_rope(k, cos, sin)
    return q, k, v
