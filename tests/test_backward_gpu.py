"""GPU parity of the backward (infini_attn_backward through the C ABI) against
the float64 oracle's backward on identical seeded inputs and upstream
gradients.

Back-propagation through the segments' memory is what training over a
rollout of segments needs ("Hugging Face Infini-Attention 再現分析",
"重み減衰とロールアウト": rollout 16 x segment 64, the 200M shape).

Tolerance: the kernels compute in fp32 from the exact input values (bf16 or
fp32), so each gradient tensor must match the float64 oracle to
max |got - ref| <= 1e-3 * max |ref| (fp32 rounding through the segments'
sums and the reverse walk over up to 16 segments).
"""

import numpy as np
import pytest
import torch

import oracle
from compressive_memory_transformer_segment_b200 import configs, synth
from helpers import inputs_f64, to_torch

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS
TOL_BWD = 1e-3
NAMES = ("dq", "dk", "dv", "dbeta", "dM_in", "dz_in")


def run_gpu(api, w, inp, grads, M_in, z_in, dM=True):
    q, k, v = (to_torch(inp[n], w.dtype) for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).cuda()
    M0 = torch.from_numpy(M_in).cuda().contiguous()
    z0 = torch.from_numpy(z_in).cuda().contiguous()
    dout = to_torch(grads["dout"], w.dtype)
    dM_out = torch.from_numpy(grads["dM_out"]).cuda() if dM else None
    dz_out = torch.from_numpy(grads["dz_out"]).cuda() if dM else None
    res = api.backward(q, k, v, beta, M0, z0, w.seg_len, w.rule, dout, dM_out, dz_out)
    api.sync_status()
    return [t.cpu().numpy().astype(np.float64) for t in res]


def run_oracle(w, inp, grads, M_in, z_in, dM=True):
    x = inputs_f64(inp, w.dtype)
    dout = synth.as_float64(grads["dout"], w.dtype)
    dM_out = grads["dM_out"].astype(np.float64) if dM else np.zeros(M_in.shape)
    dz_out = grads["dz_out"].astype(np.float64) if dM else np.zeros(z_in.shape)
    return oracle.infini_attention_backward(
        x["q"], x["k"], x["v"], inp["beta"].astype(np.float64), M_in.astype(np.float64),
        z_in.astype(np.float64), w.seg_len, w.rule, dout, dM_out, dz_out)


def check(api, w, state="random", dM=True):
    inp = synth.make_inputs(w)
    grads = synth.make_output_grads(w)
    if state == "random":
        M_in, z_in = synth.make_state(w)
    else:
        M_in, z_in = inp["M_in"], inp["z_in"]
    got = run_gpu(api, w, inp, grads, M_in, z_in, dM)
    ref = run_oracle(w, inp, grads, M_in, z_in, dM)
    errs = {}
    for name, g, r in zip(NAMES, got, ref):
        assert g.shape == r.shape, name
        assert np.all(np.isfinite(g)), name
        scale = max(float(np.max(np.abs(r))), 1e-6)
        errs[name] = float(np.max(np.abs(g - r))) / scale
    assert all(e <= TOL_BWD for e in errs.values()), (w.name, errs)
    return errs


CASES = [
    # name, overrides, initial state
    ("tiny_f32_linear", dict(), "random"),
    ("tiny_f32_delta", dict(rule="delta"), "random"),
    ("tiny_f32_delta_zero_state", dict(rule="delta"), "zero"),
    ("f32_d64_gqa_ragged_delta", dict(d_k=64, d_v=64, B=2, H_q=4, H_kv=2, L=200, rule="delta"),
     "random"),
    ("bf16_d64_S64_linear_ragged", dict(dtype="bf16", d_k=64, d_v=64, L=300, H_q=2, H_kv=2),
     "zero"),
    ("bf16_d64_S32_gqa_delta", dict(dtype="bf16", d_k=64, d_v=64, L=260, seg_len=32, H_q=4,
                                    H_kv=2, rule="delta"), "random"),
    ("f32_S1", dict(L=20, seg_len=1), "random"),
    ("f32_L_lt_S_delta", dict(L=40, seg_len=64, rule="delta"), "random"),
    ("f32_S17_odd", dict(L=100, seg_len=17, rule="delta"), "random"),
]


@pytest.mark.parametrize("name,over,state", CASES, ids=[c[0] for c in CASES])
def test_backward_parity(cuda_lib, name, over, state):
    check(cuda_lib, W["tiny"].with_(name=name, **over), state)


def test_backward_without_state_gradients(cuda_lib):
    """dM_out = dz_out = NULL: the same as passing zeros."""
    check(cuda_lib, W["tiny"].with_(name="no_dstate", rule="delta"), "random", dM=False)


@pytest.mark.parametrize("name", ["200m-linear", "200m-delta"])
def test_backward_rollout_shape(cuda_lib, name):
    """The training shape: rollout 16 x segment 64, d = 64, 8 x 12 heads."""
    check(cuda_lib, W[name], "zero")


def test_backward_bitwise_repeatable(cuda_lib):
    w = W["tiny"].with_(name="repeat", dtype="bf16", d_k=64, d_v=64, rule="delta", H_q=4, H_kv=2)
    inp = synth.make_inputs(w)
    grads = synth.make_output_grads(w)
    M_in, z_in = synth.make_state(w)
    a = run_gpu(cuda_lib, w, inp, grads, M_in, z_in)
    b = run_gpu(cuda_lib, w, inp, grads, M_in, z_in)
    for name, x, y in zip(NAMES, a, b):
        assert np.array_equal(x, y), name


def test_backward_unsupported_shapes(cuda_lib):
    api = cuda_lib
    for d, S in ((128, 64), (64, 128), (32, 65)):
        dims = api.make_dims(1, 2, 2, 256, d, d, torch.float32)
        assert api.backward_workspace_bytes(dims, S, "linear") == 0
    w = W["tiny"].with_(d_k=128, d_v=128)
    inp = synth.make_inputs(w)
    grads = synth.make_output_grads(w)
    with pytest.raises(api.InfiniError) as exc:
        run_gpu(api, w, inp, grads, inp["M_in"], inp["z_in"])
    assert exc.value.status == -2  # INFINI_ERR_UNSUPPORTED


def test_backward_ignores_workspace_contents(cuda_lib):
    """A workspace full of NaN gives the same gradients as a fresh one: every
    byte the backward reads there is written earlier in the same call."""
    api = cuda_lib
    w = W["tiny"].with_(name="ws_nan", dtype="bf16", d_k=64, d_v=64, rule="delta", H_q=4, H_kv=2,
                        L=300)
    inp = synth.make_inputs(w)
    grads = synth.make_output_grads(w)
    M_in, z_in = synth.make_state(w)
    ref = run_gpu(api, w, inp, grads, M_in, z_in)
    q, k, v = (to_torch(inp[n], w.dtype) for n in ("q", "k", "v"))
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, q.dtype)
    nbytes = api.backward_workspace_bytes(dims, w.seg_len, w.rule)
    ws = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device="cuda").view(torch.uint8)
    got = api.backward(q, k, v, torch.from_numpy(inp["beta"]).cuda(), torch.from_numpy(M_in).cuda(),
                       torch.from_numpy(z_in).cuda(), w.seg_len, w.rule, to_torch(grads["dout"], w.dtype),
                       torch.from_numpy(grads["dM_out"]).cuda(), torch.from_numpy(grads["dz_out"]).cuda(),
                       workspace=ws)
    api.sync_status()
    for name, g, r in zip(NAMES, got, ref):
        assert np.array_equal(g.cpu().numpy().astype(np.float64), r), name
