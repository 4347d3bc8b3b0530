"""Thin Python binding of libinfini_attn.so (argument marshalling only).

Every step of the layer runs in the library's CUDA kernels; this module only
checks tensor metadata, builds the C structs and passes raw pointers and the
current CUDA stream.  PyTorch provides device memory and streams.  There is no
fallback: if the library is missing, every call raises.

Names follow the C ABI in include/infini_attn.h.
"""

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libinfini_attn.so")

RULES = {"linear": 0, "delta": 1}
DTYPES = {torch.bfloat16: 0, torch.float32: 1}
PATHS = {0: "simt", 1: "tcgen05"}

OK = 0
ERR_ARG, ERR_UNSUPPORTED, ERR_ALIAS, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE, ERR_ALIGN = (
    -1, -2, -3, -4, -5, -6, -7)
ERR_SCRATCH_LIMIT = -8


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H_q", ctypes.c_int), ("H_kv", ctypes.c_int),
                ("L", ctypes.c_int), ("d_k", ctypes.c_int), ("d_v", ctypes.c_int),
                ("dtype", ctypes.c_int)]


class Plan(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("launches", ctypes.c_int),
                ("num_segments", ctypes.c_int), ("workspace_bytes", ctypes.c_size_t)]


class InfiniError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"infini_attn status {status}: {message}")
        self.status = status


_lib = None

# (name, restype, argtypes) for every entry point of include/infini_attn.h.
_P = ctypes.c_void_p
_SIGNATURES = [
    ("infini_attn_version", ctypes.c_int, []),
    ("infini_attn_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("infini_attn_init_state", ctypes.c_int, [_P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, _P]),
    ("infini_attn_workspace_bytes", ctypes.c_size_t, [ctypes.POINTER(Dims), ctypes.c_int, ctypes.c_int]),
    ("infini_attn_plan", ctypes.c_int, [ctypes.POINTER(Dims), ctypes.c_int, ctypes.c_int,
                                        ctypes.POINTER(Plan)]),
    ("infini_attn_forward", ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int,
                                           ctypes.POINTER(Dims), _P, _P, _P, _P, ctypes.c_size_t, _P]),
    ("infini_attn_state_update", ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int, ctypes.c_int,
                                                ctypes.POINTER(Dims), _P, _P, _P, ctypes.c_size_t, _P]),
    ("infini_attn_state_sum", ctypes.c_int, [_P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, _P, _P, _P]),
    ("infini_attn_decode_workspace_bytes", ctypes.c_size_t, [ctypes.POINTER(Dims), ctypes.c_int,
                                                              ctypes.c_int]),
    ("infini_attn_decode_step", ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, _P, _P,
                                               ctypes.c_int, ctypes.c_int, ctypes.POINTER(Dims), _P,
                                               _P, ctypes.c_size_t, _P]),
    ("infini_attn_host_arena_bytes", ctypes.c_size_t, [ctypes.POINTER(Dims), ctypes.c_int, ctypes.c_int]),
    ("infini_attn_forward_host", ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int,
                                                ctypes.POINTER(Dims), _P, _P, _P, _P,
                                                ctypes.c_size_t, _P]),
    ("infini_attn_sync_status", ctypes.c_int, [_P]),
    ("infini_attn_set_kernel_timing", ctypes.c_int, [ctypes.c_int]),
    ("infini_attn_kernel_times", ctypes.c_int, [ctypes.POINTER(ctypes.c_double),
                                                ctypes.POINTER(ctypes.c_int), ctypes.c_int,
                                                ctypes.c_int]),
    ("infini_attn_selftest_approx", ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int, _P]),
    ("infini_attn_selftest_timeout", ctypes.c_int, [_P]),
    ("infini_attn_forward_noalloc", ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int,
                                                   ctypes.c_int, ctypes.POINTER(Dims), _P, _P, _P,
                                                   _P]),
    ("infini_attn_noalloc_scratch_limit", ctypes.c_size_t, []),
    ("infini_attn_backward_workspace_bytes", ctypes.c_size_t, [ctypes.POINTER(Dims), ctypes.c_int,
                                                                ctypes.c_int]),
    ("infini_attn_qkv_project", ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.POINTER(Dims), ctypes.c_int,
                                               _P, _P, _P, _P]),
    ("infini_attn_rope_tables", ctypes.c_int, [_P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                               _P]),
    ("infini_attn_backward", ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_int,
                                            ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P,
                                            _P, _P, ctypes.c_size_t, _P]),
]


def load_library(path=None):
    """Load the in-tree CUDA library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} is missing: build it with "
            "`python -m compressive_memory_transformer_segment_b200.build`")
    lib = ctypes.CDLL(path)
    for name, res, args in _SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def exported_symbols():
    return [name for name, _, _ in _SIGNATURES]


def status_string(status):
    return load_library().infini_attn_status_string(int(status)).decode()


def _check(rc):
    if rc != OK:
        raise InfiniError(rc, status_string(rc))


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _one_device(first, *tensors, stream=None):
    """The library launches on the current CUDA device: every tensor (and the
    stream, if given) must be on the device of ``first``, which the call then
    makes current."""
    dev = first.device
    for t in tensors:
        if isinstance(t, torch.Tensor) and t.device != dev:
            raise ValueError(f"all tensors must be on {dev}; got one on {t.device}")
    if stream is not None and stream.device != dev:
        raise ValueError(f"the stream is on {stream.device}, the tensors on {dev}")
    return torch.cuda.device(dev)


def make_dims(B, H_q, H_kv, L, d_k, d_v, dtype):
    return Dims(B, H_q, H_kv, L, d_k, d_v, DTYPES[dtype] if isinstance(dtype, torch.dtype) else dtype)


def _dims_from(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, L, d]")
    B, H_q, L, d_k = q.shape
    H_kv, d_v = k.shape[1], v.shape[-1]
    if tuple(k.shape) != (B, H_kv, L, d_k) or tuple(v.shape) != (B, H_kv, L, d_v):
        raise ValueError("k must be [B, H_kv, L, d_k] and v [B, H_kv, L, d_v]")
    if q.dtype not in DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype, bfloat16 or float32")
    return make_dims(B, H_q, H_kv, L, d_k, d_v, q.dtype)


def _rule(rule):
    return RULES[rule] if isinstance(rule, str) else int(rule)


def workspace_bytes(dims, seg_len, rule):
    return load_library().infini_attn_workspace_bytes(ctypes.byref(dims), int(seg_len), _rule(rule))


def plan(dims, seg_len, rule):
    p = Plan()
    _check(load_library().infini_attn_plan(ctypes.byref(dims), int(seg_len), _rule(rule),
                                           ctypes.byref(p)))
    return {"path": PATHS.get(p.path, p.path), "launches": p.launches,
            "num_segments": p.num_segments, "workspace_bytes": p.workspace_bytes}


def init_state(B, H_kv, d_k, d_v, device=None, stream=None):
    """Allocate and zero (M, z) on the GPU through infini_attn_init_state."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    M = torch.empty((B, H_kv, d_k, d_v), dtype=torch.float32, device=device)
    z = torch.empty((B, H_kv, d_k), dtype=torch.float32, device=device)
    _check(load_library().infini_attn_init_state(
        ctypes.c_void_p(M.data_ptr()), ctypes.c_void_p(z.data_ptr()), B, H_kv, d_k, d_v,
        _stream_handle(stream)))
    return M, z


def _dev(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def forward(q, k, v, beta, M_in, z_in, seg_len, rule, out=None, M_out=None, z_out=None,
            workspace=None, stream=None):
    """infini_attn_forward on CUDA tensors; returns (out, M_out, z_out).

    Outputs are allocated when not given.  ``workspace`` is an optional uint8
    CUDA tensor of at least workspace_bytes(...) bytes; without it the library
    takes stream-ordered scratch itself.
    """
    lib = load_library()
    dims = _dims_from(q, k, v)
    B, H_q, L, H_kv, d_k, d_v = dims.B, dims.H_q, dims.L, dims.H_kv, dims.d_k, dims.d_v
    if out is None:
        out = torch.empty((B, H_q, L, d_v), dtype=q.dtype, device=q.device)
    if M_out is None:
        M_out = torch.empty((B, H_kv, d_k, d_v), dtype=torch.float32, device=q.device)
    if z_out is None:
        z_out = torch.empty((B, H_kv, d_k), dtype=torch.float32, device=q.device)
    args = [_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
            _dev(beta, "beta", torch.float32, (H_q,)),
            _dev(M_in, "M_in", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_in, "z_in", torch.float32, (B, H_kv, d_k))]
    outs = [_dev(out, "out", q.dtype, (B, H_q, L, d_v)),
            _dev(M_out, "M_out", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_out, "z_out", torch.float32, (B, H_kv, d_k))]
    if workspace is not None:
        ws_ptr, ws_n = _dev(workspace, "workspace", torch.uint8), workspace.numel()
    else:
        ws_ptr, ws_n = ctypes.c_void_p(0), 0
    with _one_device(q, k, v, beta, M_in, z_in, out, M_out, z_out, workspace, stream=stream):
        _check(lib.infini_attn_forward(*args, int(seg_len), _rule(rule), ctypes.byref(dims), *outs,
                                       ws_ptr, ws_n, _stream_handle(stream)))
    return out, M_out, z_out


def backward_workspace_bytes(dims, seg_len, rule):
    """infini_attn_backward_workspace_bytes (0 for unsupported shapes)."""
    return load_library().infini_attn_backward_workspace_bytes(ctypes.byref(dims), int(seg_len),
                                                               _rule(rule))


def backward(q, k, v, beta, M_in, z_in, seg_len, rule, dout, dM_out=None, dz_out=None,
             workspace=None, stream=None):
    """infini_attn_backward on CUDA tensors: the gradients of a loss with
    respect to the forward's inputs, given its gradients with respect to
    (out, M_out, z_out) (``dM_out`` / ``dz_out`` may be None for zero).
    Returns (dq, dk, dv, dbeta, dM_in, dz_in), all float32."""
    lib = load_library()
    dims = _dims_from(q, k, v)
    B, H_q, L, H_kv, d_k, d_v = dims.B, dims.H_q, dims.L, dims.H_kv, dims.d_k, dims.d_v
    f32 = dict(dtype=torch.float32, device=q.device)
    dq = torch.empty((B, H_q, L, d_k), **f32)
    dk = torch.empty((B, H_kv, L, d_k), **f32)
    dv = torch.empty((B, H_kv, L, d_v), **f32)
    dbeta = torch.empty((H_q,), **f32)
    dM_in = torch.empty((B, H_kv, d_k, d_v), **f32)
    dz_in = torch.empty((B, H_kv, d_k), **f32)
    args = [_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
            _dev(beta, "beta", torch.float32, (H_q,)),
            _dev(M_in, "M_in", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_in, "z_in", torch.float32, (B, H_kv, d_k))]
    grads_in = [_dev(dout, "dout", q.dtype, (B, H_q, L, d_v)),
                _dev(dM_out, "dM_out", torch.float32, (B, H_kv, d_k, d_v))
                if dM_out is not None else ctypes.c_void_p(0),
                _dev(dz_out, "dz_out", torch.float32, (B, H_kv, d_k))
                if dz_out is not None else ctypes.c_void_p(0)]
    outs = [_dev(t, n) for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (dbeta, "dbeta"),
                                     (dM_in, "dM_in"), (dz_in, "dz_in"))]
    if workspace is not None:
        ws_ptr, ws_n = _dev(workspace, "workspace", torch.uint8), workspace.numel()
    else:
        ws_ptr, ws_n = ctypes.c_void_p(0), 0
    with _one_device(q, k, v, beta, M_in, z_in, dout, dM_out, dz_out, workspace, stream=stream):
        _check(lib.infini_attn_backward(*args, int(seg_len), _rule(rule), ctypes.byref(dims),
                                        *grads_in, *outs, ws_ptr, ws_n, _stream_handle(stream)))
    return dq, dk, dv, dbeta, dM_in, dz_in


def state_update(k, v, M_in, z_in, seg_len, rule, M_out=None, z_out=None, workspace=None,
                 stream=None):
    """infini_attn_state_update on CUDA tensors: the state after the segments
    of k, v from (M_in, z_in); returns (M_out, z_out).  ``workspace``: an
    optional uint8 CUDA tensor of workspace_bytes(make_dims(B, H_kv, H_kv, L,
    d_k, d_v, dtype), seg_len, rule) bytes or more."""
    lib = load_library()
    if k.dim() != 4 or v.dim() != 4:
        raise ValueError("k and v must be [B, H_kv, L, d]")
    B, H_kv, L, d_k = k.shape
    d_v = v.shape[3]
    if tuple(v.shape[:3]) != (B, H_kv, L) or v.dtype != k.dtype:
        raise ValueError("v must match k in batch, heads, length and dtype")
    if k.dtype not in DTYPES:
        raise ValueError("k, v must be bfloat16 or float32")
    dims = make_dims(B, H_kv, H_kv, L, d_k, d_v, k.dtype)
    if M_out is None:
        M_out = torch.empty((B, H_kv, d_k, d_v), dtype=torch.float32, device=k.device)
    if z_out is None:
        z_out = torch.empty((B, H_kv, d_k), dtype=torch.float32, device=k.device)
    args = [_dev(k, "k"), _dev(v, "v"),
            _dev(M_in, "M_in", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_in, "z_in", torch.float32, (B, H_kv, d_k))]
    outs = [_dev(M_out, "M_out", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_out, "z_out", torch.float32, (B, H_kv, d_k))]
    if workspace is not None:
        ws_ptr, ws_n = _dev(workspace, "workspace", torch.uint8), workspace.numel()
    else:
        ws_ptr, ws_n = ctypes.c_void_p(0), 0
    with _one_device(k, v, M_in, z_in, M_out, z_out, workspace, stream=stream):
        _check(lib.infini_attn_state_update(*args, int(seg_len), _rule(rule), ctypes.byref(dims),
                                            *outs, ws_ptr, ws_n, _stream_handle(stream)))
    return M_out, z_out


def state_sum(M_base, z_base, parts, n_parts, M_out=None, z_out=None, stream=None):
    """infini_attn_state_sum: (M_base + the first ``n_parts`` packed states of
    ``parts`` (float32 CUDA tensor [n, B*H_kv*d_k*d_v + B*H_kv*d_k]), z_base
    likewise), summed in part order; returns (M_out, z_out)."""
    lib = load_library()
    B, H_kv, d_k, d_v = M_base.shape
    if M_out is None:
        M_out = torch.empty_like(M_base)
    if z_out is None:
        z_out = torch.empty_like(z_base)
    n_parts = int(n_parts)
    width = B * H_kv * d_k * (d_v + 1)
    if parts.dim() != 2 or parts.shape[1] != width or not 0 <= n_parts <= parts.shape[0]:
        raise ValueError(f"parts must be [n >= n_parts, {width}]")
    args = [_dev(M_base, "M_base", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_base, "z_base", torch.float32, (B, H_kv, d_k)),
            _dev(parts, "parts", torch.float32) if n_parts > 0 else ctypes.c_void_p(0), n_parts,
            B, H_kv, d_k, d_v,
            _dev(M_out, "M_out", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_out, "z_out", torch.float32, (B, H_kv, d_k))]
    with _one_device(M_base, z_base, parts, M_out, z_out, stream=stream):
        _check(lib.infini_attn_state_sum(*args, _stream_handle(stream)))
    return M_out, z_out


def rope_tables(n_pos, d, base=10000.0, device=None, stream=None):
    """infini_attn_rope_tables: float32 (cos, sin) [n_pos, d/2] on the GPU."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    cos = torch.empty((n_pos, d // 2), dtype=torch.float32, device=device)
    sin = torch.empty((n_pos, d // 2), dtype=torch.float32, device=device)
    with _one_device(cos, sin, stream=stream):
        _check(load_library().infini_attn_rope_tables(
            ctypes.c_void_p(cos.data_ptr()), ctypes.c_void_p(sin.data_ptr()), int(n_pos), int(d),
            float(base), _stream_handle(stream)))
    return cos, sin


def qkv_project(x, w_qkv, bias, rope_cos, rope_sin, H_q, H_kv, d, q=None, k=None, v=None,
                stream=None):
    """infini_attn_qkv_project: x bf16 [B, L, d_model], w_qkv bf16
    [(H_q + 2 H_kv) d, d_model], bias float32 [(H_q + 2 H_kv) d] or None,
    rope_cos / rope_sin float32 [L, d/2] or None; returns bf16 (q, k, v) in
    the [B, H, L, d] layout of ``forward``."""
    lib = load_library()
    if x.dim() != 3:
        raise ValueError("x must be [B, L, d_model]")
    B, L, dm = x.shape
    n_out = (H_q + 2 * H_kv) * d
    if q is None:
        q = torch.empty((B, H_q, L, d), dtype=torch.bfloat16, device=x.device)
    if k is None:
        k = torch.empty((B, H_kv, L, d), dtype=torch.bfloat16, device=x.device)
    if v is None:
        v = torch.empty((B, H_kv, L, d), dtype=torch.bfloat16, device=x.device)
    if (rope_cos is None) != (rope_sin is None):
        raise ValueError("give both rotary tables or neither")
    rot = [ctypes.c_void_p(0), ctypes.c_void_p(0)]
    if rope_cos is not None:
        rot = [_dev(rope_cos, "rope_cos", torch.float32, (L, d // 2)),
               _dev(rope_sin, "rope_sin", torch.float32, (L, d // 2))]
    dims = make_dims(B, H_q, H_kv, L, d, d, torch.bfloat16)
    args = [_dev(x, "x", torch.bfloat16), _dev(w_qkv, "w_qkv", torch.bfloat16, (n_out, dm)),
            _dev(bias, "bias", torch.float32, (n_out,)) if bias is not None else ctypes.c_void_p(0),
            *rot, ctypes.byref(dims), int(dm),
            _dev(q, "q", torch.bfloat16, (B, H_q, L, d)), _dev(k, "k", torch.bfloat16, (B, H_kv, L, d)),
            _dev(v, "v", torch.bfloat16, (B, H_kv, L, d))]
    with _one_device(x, w_qkv, bias, rope_cos, rope_sin, q, k, v, stream=stream):
        _check(lib.infini_attn_qkv_project(*args, _stream_handle(stream)))
    return q, k, v


def decode_workspace_bytes(dims, seg_len, rule):
    return int(load_library().infini_attn_decode_workspace_bytes(ctypes.byref(dims), int(seg_len),
                                                                 _rule(rule)))


def decode_step(q_t, k_t, v_t, beta, k_buf, v_buf, pos, M, z, seg_len, rule, out=None,
                workspace=None, stream=None):
    """infini_attn_decode_step on CUDA tensors: q_t [B, H_q, d], k_t, v_t
    [B, H_kv, d], buffers [B, H_kv, seg_len, d]; (M, z) updated in place when
    pos == seg_len - 1.  Returns out [B, H_q, d]."""
    lib = load_library()
    if q_t.dim() != 3 or k_t.dim() != 3 or v_t.dim() != 3 or k_buf.dim() != 4:
        raise ValueError("q_t, k_t, v_t must be [B, heads, d] and the buffers [B, H_kv, S, d]")
    B, H_q, d = q_t.shape
    H_kv = k_t.shape[1]
    if q_t.dtype not in DTYPES:
        raise ValueError("dtype must be bfloat16 or float32")
    dims = make_dims(B, H_q, H_kv, 1, d, d, q_t.dtype)
    if out is None:
        out = torch.empty_like(q_t)
    buf = (B, H_kv, int(seg_len), d)
    args = [_dev(q_t, "q_t", q_t.dtype, (B, H_q, d)), _dev(k_t, "k_t", q_t.dtype, (B, H_kv, d)),
            _dev(v_t, "v_t", q_t.dtype, (B, H_kv, d)), _dev(beta, "beta", torch.float32, (H_q,)),
            _dev(k_buf, "k_buf", q_t.dtype, buf), _dev(v_buf, "v_buf", q_t.dtype, buf), int(pos),
            _dev(M, "M", torch.float32, (B, H_kv, d, d)), _dev(z, "z", torch.float32, (B, H_kv, d)),
            int(seg_len), _rule(rule), ctypes.byref(dims), _dev(out, "out", q_t.dtype, (B, H_q, d))]
    if workspace is not None:
        ws_ptr, ws_n = _dev(workspace, "workspace", torch.uint8), workspace.numel()
    else:
        ws_ptr, ws_n = ctypes.c_void_p(0), 0
    with _one_device(q_t, k_t, v_t, beta, k_buf, v_buf, M, z, out, workspace, stream=stream):
        _check(lib.infini_attn_decode_step(*args, ws_ptr, ws_n, _stream_handle(stream)))
    return out


class DecodeStream:
    """A stream decoded one token at a time: owns the segment buffers, the
    memory state and the position (marshalling around decode_step)."""

    def __init__(self, B, H_q, H_kv, d, seg_len, rule, dtype=torch.bfloat16, device=None,
                 M=None, z=None):
        device = torch.device("cuda") if device is None else device
        self.seg_len, self.rule, self.pos = int(seg_len), rule, 0
        self.k_buf = torch.zeros((B, H_kv, self.seg_len, d), dtype=dtype, device=device)
        self.v_buf = torch.zeros_like(self.k_buf)
        self.M = (torch.zeros((B, H_kv, d, d), dtype=torch.float32, device=device) if M is None
                  else M.clone())
        self.z = (torch.zeros((B, H_kv, d), dtype=torch.float32, device=device) if z is None
                  else z.clone())
        dims = make_dims(B, H_q, H_kv, 1, d, d, dtype)
        # zero-filled: the step's ticket counters start at 0
        self.workspace = torch.zeros(decode_workspace_bytes(dims, self.seg_len, rule),
                                     dtype=torch.uint8, device=device)

    def step(self, q_t, k_t, v_t, beta, out=None, stream=None):
        out = decode_step(q_t, k_t, v_t, beta, self.k_buf, self.v_buf, self.pos, self.M, self.z,
                          self.seg_len, self.rule, out=out, workspace=self.workspace, stream=stream)
        self.pos = (self.pos + 1) % self.seg_len
        return out

    def final_state(self, stream=None):
        """(M, z) after every token so far, counting a partly filled segment
        (the stream itself is left unchanged)."""
        if self.pos == 0:
            return self.M.clone(), self.z.clone()
        n = self.pos
        return state_update(self.k_buf[:, :, :n].contiguous(), self.v_buf[:, :, :n].contiguous(),
                            self.M, self.z, n, self.rule, stream=stream)


def host_arena_bytes(dims, seg_len, rule):
    return load_library().infini_attn_host_arena_bytes(ctypes.byref(dims), int(seg_len), _rule(rule))


def _host(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CPU tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def forward_host(q, k, v, beta, M_in, z_in, seg_len, rule, out, M_out, z_out, arena,
                 stream=None):
    """infini_attn_forward_host: host tensors in and out (pinned for async
    copies), device ``arena`` (uint8 CUDA tensor of host_arena_bytes(...))."""
    lib = load_library()
    dims = _dims_from(q, k, v)
    B, H_q, L, H_kv, d_k, d_v = dims.B, dims.H_q, dims.L, dims.H_kv, dims.d_k, dims.d_v
    args = [_host(q, "q"), _host(k, "k"), _host(v, "v"),
            _host(beta, "beta", torch.float32, (H_q,)),
            _host(M_in, "M_in", torch.float32, (B, H_kv, d_k, d_v)),
            _host(z_in, "z_in", torch.float32, (B, H_kv, d_k))]
    outs = [_host(out, "out", q.dtype, (B, H_q, L, d_v)),
            _host(M_out, "M_out", torch.float32, (B, H_kv, d_k, d_v)),
            _host(z_out, "z_out", torch.float32, (B, H_kv, d_k))]
    _check(lib.infini_attn_forward_host(*args, int(seg_len), _rule(rule), ctypes.byref(dims), *outs,
                                        _dev(arena, "arena", torch.uint8), arena.numel(),
                                        _stream_handle(stream)))
    return out, M_out, z_out


def sync_status(stream=None):
    """Wait for the stream; raise InfiniError(ERR_TIMEOUT) if a kernel gave up."""
    _check(load_library().infini_attn_sync_status(_stream_handle(stream)))


KERNEL_KINDS = ("state_scan", "attention")


def set_kernel_timing(enable):
    _check(load_library().infini_attn_set_kernel_timing(1 if enable else 0))


def kernel_times(reset=True):
    """{kind: (total ms, launches)} of the kernels timed since the last reset."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    _check(load_library().infini_attn_kernel_times(ms, cnt, n, 1 if reset else 0))
    return {KERNEL_KINDS[i]: (ms[i], cnt[i]) for i in range(n)}


def noalloc_scratch_limit():
    return load_library().infini_attn_noalloc_scratch_limit()


def forward_noalloc(q, k, v, beta, M_in, z_in, seg_len, rule, out, M_out, z_out, stream=None):
    """infini_attn_forward_noalloc: the forward for callers that cannot allocate
    GPU memory while they run.  All outputs must be given (this wrapper
    allocates nothing either); scratch comes from the library's static array.
    """
    lib = load_library()
    dims = _dims_from(q, k, v)
    B, H_q, L, H_kv, d_k, d_v = dims.B, dims.H_q, dims.L, dims.H_kv, dims.d_k, dims.d_v
    args = [_dev(q, "q"), _dev(k, "k"), _dev(v, "v"),
            _dev(beta, "beta", torch.float32, (H_q,)),
            _dev(M_in, "M_in", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_in, "z_in", torch.float32, (B, H_kv, d_k))]
    outs = [_dev(out, "out", q.dtype, (B, H_q, L, d_v)),
            _dev(M_out, "M_out", torch.float32, (B, H_kv, d_k, d_v)),
            _dev(z_out, "z_out", torch.float32, (B, H_kv, d_k))]
    with _one_device(q, k, v, beta, M_in, z_in, out, M_out, z_out, stream=stream):
        _check(lib.infini_attn_forward_noalloc(*args, int(seg_len), _rule(rule),
                                               ctypes.byref(dims), *outs, _stream_handle(stream)))
    return out, M_out, z_out


def selftest_approx(x, stream=None):
    """(poly 2^x, hardware 2^x, bf16 bits of |x|) computed on the GPU for the
    CUDA float32 tensor ``x`` by the kernel-side approximations."""
    x = x.contiguous()
    y_poly, y_mufu = torch.empty_like(x), torch.empty_like(x)
    bits = torch.empty(x.shape, dtype=torch.int32, device=x.device)
    _check(load_library().infini_attn_selftest_approx(
        _dev(x, "x", torch.float32), _dev(y_poly, "y_poly"), _dev(y_mufu, "y_mufu"),
        _dev(bits, "bits"), x.numel(), _stream_handle(stream)))
    return y_poly, y_mufu, bits


def selftest_timeout(stream=None):
    """Enqueue the bounded-wait failure-path self-check (one warp whose wait
    on a barrier nothing arrives at gives up after ~2 s and sets the device
    status word); a following sync_status raises InfiniError(ERR_TIMEOUT)."""
    _check(load_library().infini_attn_selftest_timeout(_stream_handle(stream)))
