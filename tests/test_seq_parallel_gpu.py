"""The state-only entry point and the sequence-parallel linear rule on the GPU.

infini_attn_state_update runs the forward's scan alone: its (M_out, z_out)
must equal the forward's bit for bit (same kernels, same order) and the
oracle's within the state tolerance.  The sequence-parallel forward is
emulated with several virtual ranks on one GPU, through the same host
functions the multi-rank path uses (shard.local_state_update,
shard.prefix_states) with the exchange done by stacking the updates: the
concatenated outputs and the final state are compared with the oracle.
"""

import numpy as np
import pytest
import torch

from compressive_memory_transformer_segment_b200 import configs, shard, synth
from helpers import TOL_OUT, TOL_STATE, oracle_forward, state_rel_errors, to_torch

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS

STATE_CASES = [
    ("f32_linear", dict(dtype="f32", rule="linear", B=2, H_q=4, H_kv=2, L=300, seg_len=64)),
    ("f32_delta", dict(dtype="f32", rule="delta", B=2, H_q=4, H_kv=2, L=300, seg_len=64)),
    ("bf16_d128_linear", dict(dtype="bf16", d_k=128, d_v=128, rule="linear", B=1, H_q=4, H_kv=2,
                              L=1000, seg_len=256)),
    ("bf16_d128_delta", dict(dtype="bf16", d_k=128, d_v=128, rule="delta", B=1, H_q=4, H_kv=2,
                             L=1000, seg_len=256)),
    ("bf16_d64_delta", dict(dtype="bf16", d_k=64, d_v=64, rule="delta", B=2, H_q=2, H_kv=2,
                            L=700, seg_len=128)),
]


def _tensors(w, inp, M_in=None, z_in=None):
    q, k, v = (to_torch(inp[n], w.dtype) for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).cuda()
    M0 = torch.from_numpy(inp["M_in"] if M_in is None else M_in).float().cuda().contiguous()
    z0 = torch.from_numpy(inp["z_in"] if z_in is None else z_in).float().cuda().contiguous()
    return q, k, v, beta, M0, z0


@pytest.mark.parametrize("name,over", STATE_CASES, ids=[c[0] for c in STATE_CASES])
def test_state_update_equals_forward_state(cuda_lib, name, over):
    api = cuda_lib
    w = W["tiny"].with_(name=name, **over)
    inp = synth.make_inputs(w)
    # a nonzero initial state: the state after another stream
    prev = synth.make_inputs(w.with_(seed=w.seed + 17))
    _, Mp, zp = oracle_forward(prev, w)
    Mp, zp = Mp.astype(np.float32), zp.astype(np.float32)
    q, k, v, beta, M0, z0 = _tensors(w, inp, Mp, zp)
    _, M_f, z_f = api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule)
    M_s, z_s = api.state_update(k, v, M0, z0, w.seg_len, w.rule)
    api.sync_status()
    assert torch.equal(M_s, M_f) and torch.equal(z_s, z_f)
    _, rM, rz = oracle_forward(inp, w, Mp, zp)
    em, ez = state_rel_errors(M_s.cpu().numpy(), z_s.cpu().numpy(), rM, rz)
    assert em <= TOL_STATE and ez <= TOL_STATE, (em, ez)


def test_state_update_in_place(cuda_lib):
    api = cuda_lib
    w = W["tiny"].with_(dtype="bf16", d_k=128, d_v=128, rule="linear", B=1, H_q=2, H_kv=2, L=512,
                        seg_len=256)
    inp = synth.make_inputs(w)
    _, k, v, _, M0, z0 = _tensors(w, inp)
    M_ref, z_ref = api.state_update(k, v, M0, z0, w.seg_len, w.rule)
    api.state_update(k, v, M0, z0, w.seg_len, w.rule, M_out=M0, z_out=z0)
    api.sync_status()
    assert torch.equal(M0, M_ref) and torch.equal(z0, z_ref)


SP_CASES = [
    # (name, workload overrides, virtual ranks)
    ("f32_S64_3ranks", dict(dtype="f32", rule="linear", B=2, H_q=4, H_kv=2, L=64 * 7 + 20,
                            seg_len=64), 3),
    ("bf16_d128_S256_2ranks", dict(dtype="bf16", d_k=128, d_v=128, rule="linear", B=1, H_q=4,
                                   H_kv=2, L=256 * 5 + 100, seg_len=256), 2),
    ("bf16_d128_S256_4ranks_one_q_per_kv", dict(dtype="bf16", d_k=128, d_v=128, rule="linear", B=1,
                                                H_q=2, H_kv=2, L=256 * 6, seg_len=256), 4),
]


@pytest.mark.parametrize("name,over,world", SP_CASES, ids=[c[0] for c in SP_CASES])
def test_sequence_parallel_linear_rule(cuda_lib, name, over, world):
    api = cuda_lib
    w = W["tiny"].with_(name=name, **over)
    inp = synth.make_inputs(w)
    q, k, v, beta, M0, z0 = _tensors(w, inp)
    runs = [shard.segment_range(w.L, w.seg_len, world, r) for r in range(world)]
    # each virtual rank's update of its run (the all-gather, stacked here)
    updates = torch.stack([shard.local_state_update(k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(),
                                                    w.seg_len, api.state_update) for a, b in runs])
    outs = []
    for r, (a, b) in enumerate(runs):
        M_in, z_in, M_T, z_T = shard.prefix_states(updates, r, M0, z0, api.state_sum)
        o, _, _ = api.forward(q[:, :, a:b].contiguous(), k[:, :, a:b].contiguous(),
                              v[:, :, a:b].contiguous(), beta, M_in, z_in, w.seg_len, "linear")
        outs.append(o)
    api.sync_status()
    out = torch.cat(outs, 2).float().cpu().numpy().astype(np.float64)
    ro, rM, rz = oracle_forward(inp, w)
    err = float(np.max(np.abs(out - ro)))
    assert err <= TOL_OUT[w.dtype], err
    em, ez = state_rel_errors(M_T.cpu().numpy(), z_T.cpu().numpy(), rM, rz)
    assert em <= TOL_STATE and ez <= TOL_STATE, (em, ez)


def test_state_sum_adds_parts_in_order(cuda_lib):
    """infini_attn_state_sum against the same fp32 additions done one part at a
    time (bitwise: the library adds each element in part order), in place and
    out of place, with zero parts copying the base."""
    api = cuda_lib
    g = torch.Generator(device="cuda").manual_seed(3)
    B, H_kv, d_k, d_v, n = 2, 3, 64, 32, 5
    M0 = torch.randn((B, H_kv, d_k, d_v), generator=g, device="cuda")
    z0 = torch.rand((B, H_kv, d_k), generator=g, device="cuda")
    parts = torch.randn((n, B * H_kv * d_k * (d_v + 1)), generator=g, device="cuda")
    nM = M0.numel()
    for k_ in (0, 1, 3, n):
        M, z = api.state_sum(M0, z0, parts, k_)
        rM, rz = M0.clone(), z0.clone()
        for p in range(k_):
            rM += parts[p, :nM].view_as(M0)
            rz += parts[p, nM:].view_as(z0)
        assert torch.equal(M, rM) and torch.equal(z, rz)
    Mi, zi = M0.clone(), z0.clone()
    api.state_sum(Mi, zi, parts, n, M_out=Mi, z_out=zi)
    assert torch.equal(Mi, rM) and torch.equal(zi, rz)
