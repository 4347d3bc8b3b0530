"""Streaming decode on the GPU: a sequence decoded one token at a time
(infini_attn_decode_step through api.DecodeStream) gives, token by token, the
outputs of the float64 oracle's layer forward over the whole sequence, and
the same final state; and it agrees with the library's own forward.

Cases cover both rules, bf16 and fp32, d = 32/64/128, GQA groups of 2, 4 and
8 query heads (the last over two query-head chunks of the attention kernel),
segments longer than one 128-row chunk, and a last segment left partly
filled (the final state then comes from the state update of its rows)."""

import numpy as np
import pytest
import torch

from compressive_memory_transformer_segment_b200 import configs, synth
from helpers import TOL_OUT, TOL_STATE, oracle_forward, state_rel_errors, to_torch

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS

CASES = [
    ("f32_d32_S16_delta", dict(dtype="f32", d_k=32, d_v=32, rule="delta", B=2, H_q=4, H_kv=2,
                               L=16 * 3 + 5, seg_len=16)),
    ("bf16_d128_S128_gqa4_linear", dict(dtype="bf16", d_k=128, d_v=128, rule="linear", B=1, H_q=8,
                                        H_kv=2, L=128 * 2 + 40, seg_len=128)),
    ("bf16_d64_S64_gqa8_delta", dict(dtype="bf16", d_k=64, d_v=64, rule="delta", B=2, H_q=8, H_kv=1,
                                     L=64 * 3 + 1, seg_len=64)),
    ("bf16_d128_S256_delta", dict(dtype="bf16", d_k=128, d_v=128, rule="delta", B=1, H_q=2, H_kv=1,
                                  L=256 + 200, seg_len=256)),
]


@pytest.mark.parametrize("name,over", CASES, ids=[c[0] for c in CASES])
def test_decode_token_by_token_equals_forward(cuda_lib, name, over):
    api = cuda_lib
    w = W["tiny"].with_(name=name, **over)
    inp = synth.make_inputs(w)
    q, k, v = (to_torch(inp[n], w.dtype) for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).cuda()
    dt = q.dtype
    st = api.DecodeStream(w.B, w.H_q, w.H_kv, w.d_k, w.seg_len, w.rule, dtype=dt)
    outs = []
    for t in range(w.L):
        outs.append(st.step(q[:, :, t].contiguous(), k[:, :, t].contiguous(), v[:, :, t].contiguous(),
                            beta).clone())
    M_T, z_T = st.final_state()
    api.sync_status()
    out = torch.stack(outs, 2).float().cpu().numpy().astype(np.float64)
    ro, rM, rz = oracle_forward(inp, w)
    err = float(np.max(np.abs(out - ro)))
    assert err <= TOL_OUT[w.dtype], (name, err)
    em, ez = state_rel_errors(M_T.cpu().numpy(), z_T.cpu().numpy(), rM, rz)
    assert em <= TOL_STATE and ez <= TOL_STATE, (name, em, ez)
    # the library's forward over the whole sequence
    M0 = torch.zeros_like(M_T)
    z0 = torch.zeros_like(z_T)
    f_out, f_M, _ = api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule)
    api.sync_status()
    assert float(torch.max(torch.abs(f_out.float() - torch.from_numpy(out).cuda().float()))) <= \
        2 * TOL_OUT[w.dtype]


def test_decode_state_updates_only_at_segment_end(cuda_lib):
    api = cuda_lib
    w = W["tiny"].with_(dtype="bf16", d_k=64, d_v=64, rule="linear", B=1, H_q=2, H_kv=2, L=64,
                        seg_len=32)
    inp = synth.make_inputs(w)
    q, k, v = (to_torch(inp[n], w.dtype) for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).cuda()
    st = api.DecodeStream(w.B, w.H_q, w.H_kv, w.d_k, w.seg_len, w.rule, dtype=q.dtype)
    for t in range(31):
        st.step(q[:, :, t].contiguous(), k[:, :, t].contiguous(), v[:, :, t].contiguous(), beta)
    api.sync_status()
    assert torch.count_nonzero(st.M) == 0 and torch.count_nonzero(st.z) == 0
    st.step(q[:, :, 31].contiguous(), k[:, :, 31].contiguous(), v[:, :, 31].contiguous(), beta)
    api.sync_status()
    assert st.pos == 0
    M_ref, z_ref = api.state_update(k[:, :, :32].contiguous(), v[:, :, :32].contiguous(),
                                    torch.zeros_like(st.M), torch.zeros_like(st.z), 32, "linear")
    api.sync_status()
    assert torch.equal(st.M, M_ref) and torch.equal(st.z, z_ref)
    # the buffer holds the segment's keys and values
    assert torch.equal(st.k_buf, k[:, :, :32]) and torch.equal(st.v_buf, v[:, :, :32])
