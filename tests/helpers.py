"""Shared test helpers: seeded inputs to torch tensors, error measures, oracle runs."""

import numpy as np
import torch

import oracle
from compressive_memory_transformer_segment_b200 import synth

# Tolerances stated for this layer: bf16 I/O with fp32 accumulation, fp32 I/O,
# and the memory state after the longest stream.
TOL_OUT = {"bf16": 2e-2, "f32": 1e-4}
TOL_STATE = 1e-3


def to_torch(x, dtype, device="cuda"):
    """Generated array (bf16 bits or float32) to a tensor of the workload dtype."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device)


def inputs_f64(inp, dtype):
    return {key: synth.as_float64(inp[key], dtype) for key in ("q", "k", "v")}


def state_rel_errors(M_gpu, z_gpu, M_ref, z_ref):
    """Max over KV heads of ||dM||_F / ||M||_F, and max_i |dz_i| / |z_i|."""
    M_gpu = np.asarray(M_gpu, np.float64)
    z_gpu = np.asarray(z_gpu, np.float64)
    dM = np.linalg.norm((M_gpu - M_ref).reshape(-1, M_ref.shape[-2] * M_ref.shape[-1]), axis=1)
    nM = np.linalg.norm(M_ref.reshape(-1, M_ref.shape[-2] * M_ref.shape[-1]), axis=1)
    em = float(np.max(np.where(nM > 0, dM / np.maximum(nM, 1e-300), dM)))
    dz = np.abs(z_gpu - z_ref)
    ez = float(np.max(np.where(np.abs(z_ref) > 0, dz / np.maximum(np.abs(z_ref), 1e-300), dz)))
    return em, ez


def gpu_forward(api, inp, w, M_in=None, z_in=None, **kw):
    q = to_torch(inp["q"], w.dtype)
    k = to_torch(inp["k"], w.dtype)
    v = to_torch(inp["v"], w.dtype)
    beta = torch.from_numpy(inp["beta"]).cuda()
    M0 = torch.from_numpy(inp["M_in"] if M_in is None else M_in).float().cuda().contiguous()
    z0 = torch.from_numpy(inp["z_in"] if z_in is None else z_in).float().cuda().contiguous()
    out, M, z = api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule, **kw)
    api.sync_status()
    return out.float().cpu().numpy().astype(np.float64), M.cpu().numpy(), z.cpu().numpy()


def oracle_forward(inp, w, M_in=None, z_in=None):
    x = inputs_f64(inp, w.dtype)
    M0 = inp["M_in"] if M_in is None else M_in
    z0 = inp["z_in"] if z_in is None else z_in
    return oracle.infini_attention_forward(x["q"], x["k"], x["v"], inp["beta"].astype(np.float64),
                                           np.asarray(M0, np.float64), np.asarray(z0, np.float64),
                                           w.seg_len, w.rule)
