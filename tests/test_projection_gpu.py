"""GPU parity of the Q/K/V projection prologue (infini_attn_qkv_project and
infini_attn_rope_tables through the C ABI) against the float64 oracle on the
same seeded bf16 inputs.

The memory reuses the attention's Q/K/V ("Leave No Context Behind" explainer,
"メモリ構造"), which come from linear layers over the input ("Как работает
Infini-attention", section 9); the rotation is RoFormer's rotary embedding in
the rotate-half pairing (a reading; the pages define no position encoding).

Tolerance: the kernel accumulates exact bf16 products in fp32 and rounds the
result to bf16 (unit roundoff 2^-8), so every element must satisfy
|got - ref| <= 2^-8 |ref| + 1e-4 max|ref| (the second term covers the fp32
accumulation over d_model and the fp32 rotary tables).  The tables
themselves: fp64 values rounded to fp32, |got - ref| <= 1e-7.
"""

import numpy as np
import pytest
import torch

import oracle
from compressive_memory_transformer_segment_b200 import configs, synth
from helpers import to_torch

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


def check_close(name, got, ref):
    got = np.asarray(got, np.float64)
    scale = max(float(np.max(np.abs(ref))), 1e-6)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4 * scale
    bad = np.abs(got - ref) > bound
    assert not bad.any(), (name, int(bad.sum()), float(np.max(np.abs(got - ref) - bound)))


def to_np(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_case(api, w, d_model, bias=True, rope=True, rows=None):
    """Project on the GPU; compare all rows (rows=None) or the listed (b, t)
    rows of every head with the oracle."""
    inp = synth.make_projection_inputs(w, d_model, bias=bias)
    d = w.d_k
    x = to_torch(inp["x"], "bf16")
    wq = to_torch(inp["w"], "bf16")
    b_t = torch.from_numpy(inp["bias"]).cuda() if bias else None
    cos = sin = None
    if rope:
        cos, sin = api.rope_tables(w.L, d)
    q, k, v = api.qkv_project(x, wq, b_t, cos, sin, w.H_q, w.H_kv, d)
    api.sync_status()
    wf = synth.bf16_bits_to_f32(inp["w"]).astype(np.float64)
    bf = inp["bias"].astype(np.float64) if bias else None
    c64 = s64 = None
    if rope:
        c64, s64 = oracle.rope_tables(w.L, d)
    if rows is None:
        xf = synth.bf16_bits_to_f32(inp["x"]).astype(np.float64)
        rq, rk, rv = oracle.qkv_project_rope(xf, wf, bf, c64, s64, w.H_q, w.H_kv, d)
        for name, g, r in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
            check_close(name, to_np(g), r)
    else:
        for b, t in rows:
            xr = synth.bf16_bits_to_f32(inp["x"][b:b + 1, t:t + 1]).astype(np.float64)
            cr = sr = None
            if rope:  # row t of the tables, placed at position 0 of a 1-token call
                cr, sr = c64[t:t + 1], s64[t:t + 1]
            rq, rk, rv = oracle.qkv_project_rope(xr, wf, bf, cr, sr, w.H_q, w.H_kv, d)
            for name, g, r in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
                check_close(f"{name}[{b},{t}]", to_np(g[b, :, t]), r[0, :, 0])
    return q, k, v


CASES = [
    # name, workload overrides, d_model, bias, rope
    ("d64_ragged_rows_two_col_tiles", dict(B=2, H_q=4, H_kv=2, L=200, d_k=64, d_v=64), 256, True, True),
    ("d128_gqa", dict(B=1, H_q=8, H_kv=2, L=300, d_k=128, d_v=128), 512, False, True),
    ("d64_padded_col_tile_partial_k", dict(B=1, H_q=3, H_kv=1, L=130, d_k=64, d_v=64), 200, True, False),
    ("d128_fewer_rows_than_a_tile", dict(B=1, H_q=2, H_kv=1, L=20, d_k=128, d_v=128), 64, True, True),
    # Many row tiles (1183, eight waves on 148 SMs), the last one ragged,
    # tiles straddling the two batch rows.
    ("d64_many_row_tiles_ragged", dict(B=2, H_q=2, H_kv=1, L=75700, d_k=64, d_v=64), 64, True, True),
]


@pytest.mark.parametrize("name,over,dm,bias,rope", CASES, ids=[c[0] for c in CASES])
def test_projection_parity(cuda_lib, name, over, dm, bias, rope):
    w = W["tiny"].with_(name=name, dtype="bf16", **over)
    run_case(cuda_lib, w, dm, bias, rope)


def test_projection_200m_shape_full(cuda_lib):
    """The 200M training shape in full: 8 x 1024 tokens, d_model 768,
    12 + 2 x 12 heads of 64."""
    run_case(cuda_lib, W["200m-linear"], None)


def test_projection_8b_shape_sampled_rows(cuda_lib):
    """The 8B shape (2 x 32768 tokens, d_model 4096, 32 query and 8 KV heads
    of 128) in the launch configuration the bench times; sampled rows,
    including the first and last of each batch row and rows at tile edges."""
    w = W["8b-delta"]
    rng = np.random.default_rng(5)
    rows = [(0, 0), (0, 127), (0, 128), (1, 0), (1, w.L - 1), (0, w.L - 1)]
    rows += [(int(rng.integers(w.B)), int(rng.integers(w.L))) for _ in range(26)]
    run_case(cuda_lib, w, None, rows=rows)


def test_rope_tables_match_the_oracle(cuda_lib):
    for n_pos, d, base in ((32768, 128, 10000.0), (1000, 64, 500000.0), (7, 2, 10.0)):
        cos, sin = cuda_lib.rope_tables(n_pos, d, base)
        c64, s64 = oracle.rope_tables(n_pos, d, base)
        assert np.max(np.abs(cos.cpu().numpy() - c64)) <= 1e-7
        assert np.max(np.abs(sin.cpu().numpy() - s64)) <= 1e-7


def test_projection_bitwise_repeatable_and_feeds_the_forward(cuda_lib):
    api = cuda_lib
    w = W["tiny"].with_(name="rep", dtype="bf16", B=2, H_q=4, H_kv=2, L=384, d_k=64, d_v=64,
                        seg_len=128, rule="delta")
    inp = synth.make_projection_inputs(w, 256)
    x, wq = to_torch(inp["x"], "bf16"), to_torch(inp["w"], "bf16")
    b_t = torch.from_numpy(inp["bias"]).cuda()
    cos, sin = api.rope_tables(w.L, 64)
    a = api.qkv_project(x, wq, b_t, cos, sin, w.H_q, w.H_kv, 64)
    b = api.qkv_project(x, wq, b_t, cos, sin, w.H_q, w.H_kv, 64)
    for s, t in zip(a, b):
        assert torch.equal(s, t)
    beta = torch.zeros(w.H_q, dtype=torch.float32, device="cuda")
    M0, z0 = api.init_state(w.B, w.H_kv, 64, 64)
    out, M, z = api.forward(*a, beta, M0, z0, w.seg_len, w.rule)
    api.sync_status()
    assert out.shape == (w.B, w.H_q, w.L, 64) and torch.isfinite(out.float()).all()


def test_projection_rejects_unsupported_shapes(cuda_lib):
    api = cuda_lib
    x = torch.zeros((1, 16, 128), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((4 * 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(api.InfiniError) as exc:
        api.qkv_project(x, wq, None, None, None, 2, 1, 32)
    assert exc.value.status == api.ERR_UNSUPPORTED


def test_projection_then_forward_matches_the_oracle_chain(cuda_lib):
    """The prologue feeds the layer: x -> (q, k, v) -> forward on the GPU
    against the oracle's projection (rounded to bf16, the prologue's output
    type) followed by the oracle's forward.  A bf16 rounding tie resolved
    differently on the two sides moves an output by far less than the bf16
    output tolerance."""
    api = cuda_lib
    w = W["tiny"].with_(name="chain", dtype="bf16", B=1, H_q=4, H_kv=2, L=320, d_k=64, d_v=64,
                        seg_len=128, rule="delta")
    inp = synth.make_projection_inputs(w, 256)
    x, wq = to_torch(inp["x"], "bf16"), to_torch(inp["w"], "bf16")
    b_t = torch.from_numpy(inp["bias"]).cuda()
    cos, sin = api.rope_tables(w.L, 64)
    q, k, v = api.qkv_project(x, wq, b_t, cos, sin, w.H_q, w.H_kv, 64)
    beta = torch.from_numpy(synth.make_beta(w)).cuda()
    M0, z0 = api.init_state(w.B, w.H_kv, 64, 64)
    out, M, z = api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule)
    api.sync_status()
    c64, s64 = oracle.rope_tables(w.L, 64)
    rq, rk, rv = oracle.qkv_project_rope(synth.as_float64(inp["x"], "bf16"),
                                         synth.as_float64(inp["w"], "bf16"),
                                         inp["bias"].astype(np.float64), c64, s64, w.H_q, w.H_kv, 64)
    rq, rk, rv = (synth.as_float64(synth.round_bf16_bits(t.astype(np.float32)), "bf16")
                  for t in (rq, rk, rv))
    ro, rM, rz = oracle.infini_attention_forward(
        rq, rk, rv, synth.make_beta(w).astype(np.float64), np.zeros((w.B, w.H_kv, 64, 64)),
        np.zeros((w.B, w.H_kv, 64)), w.seg_len, w.rule)
    assert float(np.max(np.abs(out.float().cpu().numpy() - ro))) <= 2e-2
    scale = float(np.max(np.abs(rM)))
    assert float(np.max(np.abs(M.cpu().numpy() - rM))) <= 1e-3 * scale
