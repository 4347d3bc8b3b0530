"""Seeded synthetic inputs for the Infini-attention layer forward.

This module is shared by the tests, the bench and the CPU oracle's callers.  It
holds none of the method's arithmetic: it draws i.i.d. values from a seeded
counter-based generator (NumPy's Philox) and rounds them to bf16 where the
workload asks for bf16.

Streams.  Every (tensor, batch, head) slice has its own Philox key
(seed, stream id), so any slice can be regenerated alone (large workloads are
checked on sampled heads) and generation parallelises over threads without
changing the values.
"""

from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

(_T_Q, _T_K, _T_V, _T_BETA, _T_PAIR, _T_DOUT, _T_DSTATE, _T_STATE, _T_X, _T_W,
 _T_BIAS) = 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11


def _stream(seed, tensor, b=0, h=0):
    return np.random.Generator(
        np.random.Philox(key=[int(seed), (tensor << 40) | (b << 20) | h]))


def round_bf16_bits(x):
    """Round float32 values to bf16 (round to nearest even); return uint16 bits.

    NaN is not produced by the generators, so no NaN handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits):
    """Exact float32 values of bf16 bit patterns."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_slice(seed, tensor, b, h, n, d, bf16):
    x = _stream(seed, tensor, b, h).standard_normal((n, d), dtype=np.float32)
    if bf16:
        return round_bf16_bits(x)
    return x


def normal_tensor(seed, tensor, B, H, L, d, bf16, threads=None, heads=None):
    """[B, H, L, d] i.i.d. N(0, 1): uint16 bf16 bits if ``bf16`` else float32.

    ``heads`` limits generation to the listed head indices (others stay 0).
    """
    out = np.zeros((B, H, L, d), dtype=np.uint16 if bf16 else np.float32)
    jobs = [(b, h) for b in range(B) for h in range(H)
            if heads is None or h in heads]

    def work(bh):
        b, h = bh
        out[b, h] = _normal_slice(seed, tensor, b, h, L, d, bf16)

    n = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=n) as ex:
        list(ex.map(work, jobs))
    return out


_TENSOR_CODES = {"q": _T_Q, "k": _T_K, "v": _T_V}


def _pair(cfg, seed):
    g = _stream(seed, _T_PAIR)
    ks = g.standard_normal(cfg.d_k, dtype=np.float32)
    vs = g.standard_normal(cfg.d_v, dtype=np.float32)
    if cfg.dtype == "bf16":
        ks, vs = round_bf16_bits(ks), round_bf16_bits(vs)
    p = 2 * cfg.seg_len + 1000
    if p >= cfg.L:
        raise ValueError("inserted pair lies beyond the sequence")
    return p, {"k": ks, "v": vs, "q": ks}


def make_head(cfg, name, b, h, seed=None):
    """The [L, d] slice of tensor ``name`` ('q', 'k' or 'v') for batch row b
    and head h, exactly as make_inputs would place it."""
    seed = cfg.seed if seed is None else seed
    d = cfg.d_v if name == "v" else cfg.d_k
    x = _normal_slice(seed, _TENSOR_CODES[name], b, h, cfg.L, d, cfg.dtype == "bf16")
    if cfg.insert_pair:
        p, pair = _pair(cfg, seed)
        if name == "q":
            x[cfg.L - 1] = pair["q"]
        else:
            x[p] = pair[name]
    return x


def make_beta(cfg, seed=None):
    seed = cfg.seed if seed is None else seed
    return _stream(seed, _T_BETA).uniform(-cfg.beta_range, cfg.beta_range,
                                          size=cfg.H_q).astype(np.float32)


def make_inputs(cfg, seed=None, heads_q=None, heads_kv=None):
    """Inputs for one workload configuration (see ``configs.py``).

    Returns a dict with
      q, k, v : uint16 bf16 bits [B,H,L,d] when cfg.dtype == 'bf16', else float32
      beta    : float32 [H_q], U(-beta_range, beta_range)
      M_in    : float32 [B,H_kv,d_k,d_v] zeros;  z_in: float32 [B,H_kv,d_k] zeros
    and, for workloads with an inserted key/value pair, 'pair_pos'.
    ``heads_q`` / ``heads_kv`` restrict which head slices are drawn (others 0).

    Inserted pair: one fixed key/value pair, drawn from its own stream, sits at
    token 2*S + 1000 (inside the third segment) of every (batch, KV head), and
    the query at the last position of every query head is set to that key.
    """
    seed = cfg.seed if seed is None else seed
    bf16 = cfg.dtype == "bf16"
    q = normal_tensor(seed, _T_Q, cfg.B, cfg.H_q, cfg.L, cfg.d_k, bf16, heads=heads_q)
    k = normal_tensor(seed, _T_K, cfg.B, cfg.H_kv, cfg.L, cfg.d_k, bf16, heads=heads_kv)
    v = normal_tensor(seed, _T_V, cfg.B, cfg.H_kv, cfg.L, cfg.d_v, bf16, heads=heads_kv)
    res = dict(q=q, k=k, v=v, beta=make_beta(cfg, seed),
               M_in=np.zeros((cfg.B, cfg.H_kv, cfg.d_k, cfg.d_v), np.float32),
               z_in=np.zeros((cfg.B, cfg.H_kv, cfg.d_k), np.float32))
    if cfg.insert_pair:
        p, pair = _pair(cfg, seed)
        hq = range(cfg.H_q) if heads_q is None else sorted(heads_q)
        hk = range(cfg.H_kv) if heads_kv is None else sorted(heads_kv)
        for h in hk:
            k[:, h, p, :] = pair["k"]
            v[:, h, p, :] = pair["v"]
        for h in hq:
            q[:, h, cfg.L - 1, :] = pair["q"]
        res["pair_pos"] = p
    return res


def as_float64(x, dtype):
    """Exact float64 values of a generated tensor (bf16 bits or float32)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def make_output_grads(cfg, seed=None, scale=1.0):
    """Seeded upstream gradients for the backward: dout [B, H_q, L, d_v]
    (bf16 bits or float32, like the forward's output), and float32 dM_out
    [B, H_kv, d_k, d_v], dz_out [B, H_kv, d_k], all i.i.d. N(0, scale^2)
    (``scale`` a power of two keeps bf16 values exact)."""
    seed = cfg.seed if seed is None else seed
    bf16 = cfg.dtype == "bf16"
    dout = np.zeros((cfg.B, cfg.H_q, cfg.L, cfg.d_v), dtype=np.uint16 if bf16 else np.float32)
    for b in range(cfg.B):
        for h in range(cfg.H_q):
            x = _stream(seed, _T_DOUT, b, h).standard_normal((cfg.L, cfg.d_v), dtype=np.float32)
            x *= np.float32(scale)
            dout[b, h] = round_bf16_bits(x) if bf16 else x
    g = _stream(seed, _T_DSTATE)
    dM = g.standard_normal((cfg.B, cfg.H_kv, cfg.d_k, cfg.d_v), dtype=np.float32) * np.float32(scale)
    dz = g.standard_normal((cfg.B, cfg.H_kv, cfg.d_k), dtype=np.float32) * np.float32(scale)
    return dict(dout=dout, dM_out=dM, dz_out=dz)


def make_state(cfg, seed=None):
    """A seeded nonzero memory state to start from: M_in ~ N(0, 1/d_k) and
    z_in ~ U(0.5, 1.5) (positive, as a sum of ELU+1 values is), float32."""
    seed = cfg.seed if seed is None else seed
    g = _stream(seed, _T_STATE)
    M = g.standard_normal((cfg.B, cfg.H_kv, cfg.d_k, cfg.d_v), dtype=np.float32)
    M *= np.float32(1.0 / np.sqrt(cfg.d_k))
    z = g.uniform(0.5, 1.5, size=(cfg.B, cfg.H_kv, cfg.d_k)).astype(np.float32)
    return M, z


_X_ROWS = 4096  # rows of x per Philox stream (any chunk regenerates alone)


def make_projection_inputs(cfg, d_model=None, seed=None, bias=True, threads=None):
    """Inputs of the Q/K/V projection prologue for a workload.

    Returns a dict with
      x    : uint16 bf16 bits [B, L, d_model], i.i.d. N(0, 1)
      w    : uint16 bf16 bits [(H_q + 2 H_kv) d, d_model], N(0, 1/d_model)
             (query rows, then key rows, then value rows)
      bias : float32 [(H_q + 2 H_kv) d], N(0, 0.1^2), or None
    d_model defaults to H_q * d_k (the model width of the pages' Llama
    shapes).  Needs d_k == d_v.
    """
    seed = cfg.seed if seed is None else seed
    if cfg.d_k != cfg.d_v:
        raise ValueError("the fused projection needs d_k == d_v")
    dm = cfg.H_q * cfg.d_k if d_model is None else d_model
    n_out = (cfg.H_q + 2 * cfg.H_kv) * cfg.d_k
    x = np.empty((cfg.B, cfg.L, dm), dtype=np.uint16)
    jobs = [(b, r0) for b in range(cfg.B) for r0 in range(0, cfg.L, _X_ROWS)]

    def work(job):
        b, r0 = job
        n = min(_X_ROWS, cfg.L - r0)
        g = _stream(seed, _T_X, b, r0 // _X_ROWS)
        x[b, r0:r0 + n] = round_bf16_bits(g.standard_normal((n, dm), dtype=np.float32))

    nt = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=nt) as ex:
        list(ex.map(work, jobs))
    wf = _stream(seed, _T_W).standard_normal((n_out, dm), dtype=np.float32)
    wf *= np.float32(1.0 / np.sqrt(dm))
    res = dict(x=x, w=round_bf16_bits(wf), bias=None)
    if bias:
        res["bias"] = (_stream(seed, _T_BIAS).standard_normal(n_out, dtype=np.float32)
                       * np.float32(0.1))
    return res
