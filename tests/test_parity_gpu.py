"""GPU parity: the CUDA library (through the C ABI) against the float64 oracle
on identical seeded inputs.

Small cases are compared element by element in full; the workloads too large
for the oracle are run at full size, in the same launch configuration the
bench times, and compared on sampled heads and segments (heads are independent
of one another, so the other heads only need to exist).

Tolerances: max |out - oracle| <= 2e-2 for bf16 I/O, <= 1e-4 for fp32 I/O;
relative error of M (Frobenius, per KV head) and of z (per entry) <= 1e-3.
"""

import numpy as np
import pytest
import torch

import oracle
from compressive_memory_transformer_segment_b200 import configs, synth
from helpers import (TOL_OUT, TOL_STATE, gpu_forward, oracle_forward, state_rel_errors,
                     to_torch)

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


def check_full(api, w, inp=None, M_in=None, z_in=None):
    inp = synth.make_inputs(w) if inp is None else inp
    out, M, z = gpu_forward(api, inp, w, M_in=M_in, z_in=z_in)
    ro, rM, rz = oracle_forward(inp, w, M_in=M_in, z_in=z_in)
    err = float(np.max(np.abs(out - ro)))
    em, ez = state_rel_errors(M, z, rM, rz)
    assert np.all(np.isfinite(out))
    assert err <= TOL_OUT[w.dtype], (w.name, err)
    assert em <= TOL_STATE and ez <= TOL_STATE, (w.name, em, ez)
    return err, em, ez


# ------------------------------------------------------------ configurations

@pytest.mark.parametrize("name", ["tiny", "200m-linear", "200m-delta"])
def test_workload_full_parity(cuda_lib, name):
    check_full(cuda_lib, W[name])


def test_tiny_delta(cuda_lib):
    check_full(cuda_lib, W["tiny"].with_(rule="delta"))


CASES = [
    # name, overrides
    ("ragged_tail_f32", dict(L=200)),
    ("seg1", dict(L=16, seg_len=1)),
    ("seg63", dict(L=300, seg_len=63)),
    ("seg65_delta", dict(L=300, seg_len=65, rule="delta")),
    ("L_lt_S", dict(L=50, seg_len=64)),
    ("gqa_b2", dict(B=2, H_q=8, H_kv=2, L=192, rule="delta")),
    ("dk64_dv32", dict(d_k=64, d_v=32, L=160)),
    ("dk32_dv128", dict(d_k=32, d_v=128, L=160, rule="delta")),
    ("bf16_d128_S256", dict(dtype="bf16", d_k=128, d_v=128, L=700, seg_len=256, H_q=4, H_kv=2)),
    ("bf16_d64_S128_delta", dict(dtype="bf16", d_k=64, d_v=64, L=512 + 77, seg_len=128, rule="delta")),
    ("bf16_d128_S2048_ragged", dict(dtype="bf16", d_k=128, d_v=128, L=4096 + 300, seg_len=2048,
                                    H_q=4, H_kv=1, rule="delta")),
    ("bf16_S64_odd_L", dict(dtype="bf16", d_k=64, d_v=64, L=64 * 5 + 17, seg_len=64, H_q=2, H_kv=2)),
]


@pytest.mark.parametrize("name,over", CASES, ids=[c[0] for c in CASES])
def test_edge_cases(cuda_lib, name, over):
    check_full(cuda_lib, W["tiny"].with_(name=name, **over))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_extremes(cuda_lib, dtype):
    w = W["tiny"].with_(dtype=dtype, H_q=4, H_kv=2, L=256, seg_len=64)
    inp = synth.make_inputs(w)
    inp["beta"] = np.array([-np.inf, np.inf, -80.0, 80.0], np.float32)
    check_full(cuda_lib, w, inp)
    # beta = +inf: the first segment retrieves from an empty memory -> exactly 0.
    out, _, _ = gpu_forward(cuda_lib, inp, w)
    assert np.all(out[:, 1, :64] == 0.0)


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_nonzero_initial_state(cuda_lib, rule):
    w = W["tiny"].with_(rule=rule, B=2, H_q=4, H_kv=2, L=192)
    prev = synth.make_inputs(w.with_(seed=77))
    _, M0, z0 = oracle_forward(prev, w)
    check_full(cuda_lib, w, M_in=M0.astype(np.float32), z_in=z0.astype(np.float32))


@pytest.mark.parametrize("dtype,rule", [("f32", "linear"), ("bf16", "delta")])
def test_split_stream_in_place_state(cuda_lib, dtype, rule):
    """forward(L1) then forward(L2) with the state updated in place equals
    forward(L1 + L2) when L1 is a whole number of segments."""
    api = cuda_lib
    w = W["tiny"].with_(dtype=dtype, rule=rule, B=2, H_q=4, H_kv=2, L=320, seg_len=64)
    inp = synth.make_inputs(w)
    q, k, v = (to_torch(inp[n], dtype) for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).cuda()
    M, z = api.init_state(2, 2, 32, 32)
    out_full, M_full, z_full = api.forward(q, k, v, beta, M, z, 64, rule)
    L1 = 128
    o1, _, _ = api.forward(q[:, :, :L1].contiguous(), k[:, :, :L1].contiguous(),
                           v[:, :, :L1].contiguous(), beta, M, z, 64, rule, M_out=M, z_out=z)
    o2, _, _ = api.forward(q[:, :, L1:].contiguous(), k[:, :, L1:].contiguous(),
                           v[:, :, L1:].contiguous(), beta, M, z, 64, rule, M_out=M, z_out=z)
    api.sync_status()
    tol = TOL_OUT[dtype]
    assert torch.max(torch.abs(torch.cat([o1, o2], 2).float() - out_full.float())) <= tol
    assert torch.allclose(M, M_full, rtol=1e-5, atol=1e-4)
    assert torch.allclose(z, z_full, rtol=1e-6, atol=1e-5)


def test_gqa_equals_repeated_kv_mha(cuda_lib):
    api = cuda_lib
    w = W["tiny"].with_(dtype="bf16", B=2, H_q=8, H_kv=2, L=256, seg_len=64, rule="delta")
    inp = synth.make_inputs(w)
    q, k, v = (to_torch(inp[n], "bf16") for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).cuda()
    M0, z0 = api.init_state(2, 2, 32, 32)
    out, M, z = api.forward(q, k, v, beta, M0, z0, 64, "delta")
    kr, vr = k.repeat_interleave(4, 1).contiguous(), v.repeat_interleave(4, 1).contiguous()
    M1, z1 = api.init_state(2, 8, 32, 32)
    out2, M2, z2 = api.forward(q, kr, vr, beta, M1, z1, 64, "delta")
    api.sync_status()
    assert torch.equal(out, out2)
    assert torch.equal(M2, M.repeat_interleave(4, 1))
    assert torch.equal(z2, z.repeat_interleave(4, 1))


def test_repeat_calls_bitwise_identical(cuda_lib):
    api = cuda_lib
    w = W["200m-delta"]
    inp = synth.make_inputs(w)
    a = gpu_forward(api, inp, w)
    b = gpu_forward(api, inp, w)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_workspace_given_or_taken_agree(cuda_lib):
    api = cuda_lib
    w = W["200m-linear"]
    inp = synth.make_inputs(w)
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, torch.bfloat16)
    n = api.workspace_bytes(dims, w.seg_len, w.rule)
    ws = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")  # garbage contents
    a = gpu_forward(api, inp, w, workspace=ws)
    b = gpu_forward(api, inp, w)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_host_buffer_entry_point_matches_device(cuda_lib):
    api = cuda_lib
    w = W["200m-delta"]
    inp = synth.make_inputs(w)
    dev = gpu_forward(api, inp, w)
    q, k, v = (to_torch(inp[n], "bf16", "cpu").pin_memory() for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).pin_memory()
    M0 = torch.from_numpy(inp["M_in"]).pin_memory()
    z0 = torch.from_numpy(inp["z_in"]).pin_memory()
    out = torch.empty((w.B, w.H_q, w.L, w.d_v), dtype=torch.bfloat16).pin_memory()
    M = torch.empty_like(M0).pin_memory()
    z = torch.empty_like(z0).pin_memory()
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, torch.bfloat16)
    arena = torch.empty(api.host_arena_bytes(dims, w.seg_len, w.rule), dtype=torch.uint8,
                        device="cuda")
    api.forward_host(q, k, v, beta, M0, z0, w.seg_len, w.rule, out, M, z, arena)
    api.sync_status()
    np.testing.assert_array_equal(out.float().numpy(), dev[0])
    np.testing.assert_array_equal(M.numpy(), dev[1])
    np.testing.assert_array_equal(z.numpy(), dev[2])


def test_gpu_argument_errors(cuda_lib):
    api = cuda_lib
    q = torch.zeros((1, 2, 64, 32), device="cuda")
    k = torch.zeros((1, 2, 64, 32), device="cuda")
    beta = torch.zeros(2, device="cuda")
    M, z = api.init_state(1, 2, 32, 32)
    with pytest.raises(api.InfiniError) as e:
        api.forward(q, k, k, beta, M, z, 64, "linear", out=q)  # out aliases q
    assert e.value.status == api.ERR_ALIAS
    with pytest.raises(api.InfiniError) as e:
        api.forward(q, k, k, beta, M, z, 0, "linear")
    assert e.value.status == api.ERR_ARG
    # In-place state is allowed.
    api.forward(q, k, k, beta, M, z, 64, "linear", M_out=M, z_out=z)
    api.sync_status()


# ------------------------------------------------------------ full size, sampled

SAMPLED = {
    # name: (batch row, KV head, query heads of that group to check, segments)
    "300m-linear": (3, 5, [5], [0, 1, 7]),
    "300m-delta": (1, 15, [15], [0, 4, 7]),
    "8b-delta": (1, 6, [24, 27], [0, 8, 15]),
    "1m-linear": (0, 13, [13], [0, 2, 255, 511]),
}


def sampled_inputs(w, b, j, heads):
    """Full-size GPU tensors whose sampled slices hold the seeded values."""
    t = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q = torch.zeros((w.B, w.H_q, w.L, w.d_k), dtype=t, device="cuda")
    k = torch.zeros((w.B, w.H_kv, w.L, w.d_k), dtype=t, device="cuda")
    v = torch.zeros((w.B, w.H_kv, w.L, w.d_v), dtype=t, device="cuda")
    host = {}
    for h in heads:
        host[("q", h)] = synth.make_head(w, "q", b, h)
        q[b, h] = to_torch(host[("q", h)], w.dtype)
    for name, dst in (("k", k), ("v", v)):
        host[(name, j)] = synth.make_head(w, name, b, j)
        dst[b, j] = to_torch(host[(name, j)], w.dtype)
    return q, k, v, host


@pytest.mark.parametrize("name", list(SAMPLED))
def test_full_size_sampled(cuda_lib, name):
    api = cuda_lib
    w = W[name]
    b, j, heads, segs = SAMPLED[name]
    q, k, v, host = sampled_inputs(w, b, j, heads)
    beta_np = synth.make_beta(w)
    beta = torch.from_numpy(beta_np).cuda()
    M0, z0 = api.init_state(w.B, w.H_kv, w.d_k, w.d_v)
    out, M, z = api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule)
    api.sync_status()
    del q, k, v
    kc = synth.as_float64(host[("k", j)], w.dtype)
    vc = synth.as_float64(host[("v", j)], w.dtype)
    worst = 0.0
    for s, r0, r1, Mp, zp in oracle.scan_states(kc, vc, np.zeros((w.d_k, w.d_v)), np.zeros(w.d_k),
                                                w.seg_len, w.rule):
        if r0 == r1:
            em, ez = state_rel_errors(M[b, j].cpu().numpy(), z[b, j].cpu().numpy(), Mp, zp)
            assert em <= TOL_STATE and ez <= TOL_STATE, (em, ez)
            break
        if s not in segs:
            continue
        for h in heads:
            qs = synth.as_float64(host[("q", h)][r0:r1], w.dtype)
            ref = oracle.segment_output(qs, kc[r0:r1], vc[r0:r1], Mp, zp, float(beta_np[h]))
            got = out[b, h, r0:r1].float().cpu().numpy()
            worst = max(worst, float(np.max(np.abs(got - ref))))
    assert worst <= TOL_OUT[w.dtype], worst


# ------------------------------------------------------------ path selection

TC_CASES = [
    ("tc_d128_S128_linear", dict(dtype="bf16", d_k=128, d_v=128, L=384, seg_len=128, H_q=2, H_kv=2)),
    ("tc_d128_S256_gqa_delta", dict(dtype="bf16", d_k=128, d_v=128, L=1024, seg_len=256, B=2,
                                    H_q=8, H_kv=2, rule="delta")),
    ("tc_d64_S512_ragged", dict(dtype="bf16", d_k=64, d_v=64, L=1500, seg_len=512, H_q=3, H_kv=3)),
    ("tc_d128_L_lt_S", dict(dtype="bf16", d_k=128, d_v=128, L=200, seg_len=256)),
    # Three query heads per KV head and an odd number of query tiles per group:
    # work items pair tiles of different positions, one item has a single tile.
    ("tc_d64_gqa3_S384_ragged", dict(dtype="bf16", d_k=64, d_v=64, L=900, seg_len=384, H_q=6,
                                     H_kv=2, rule="delta")),
    ("tc_d128_gqa2_S256_ragged", dict(dtype="bf16", d_k=128, d_v=128, L=700, seg_len=256, B=2,
                                      H_q=4, H_kv=2)),
    # One query head per KV head at d = 128 (work items pair tiles qt and qt - 1
    # of one head, so the second tile has one key tile less), several items
    # per CTA and a ragged last segment.
    ("tc_d128_mha_S512_ragged", dict(dtype="bf16", d_k=128, d_v=128, L=1500, seg_len=512, B=2,
                                     H_q=3, H_kv=3, rule="delta")),
    # Three query heads per KV head at d = 128: items whose two tiles sit at
    # different positions (unequal key-tile counts) next to items with equal
    # ones, so both orders of the end-of-item retrieval and next scores run.
    ("tc_d128_gqa3_S384_ragged", dict(dtype="bf16", d_k=128, d_v=128, L=1000, seg_len=384, H_q=6,
                                      H_kv=2)),
    # Segments shorter than a query tile (several segments per tile, the
    # short-segment kernel): a ragged last segment and a last tile that ends
    # past the sequence; four segments per tile with GQA, where the last
    # tile's later segments do not exist; d = 128.
    ("tc_small_d64_S64_delta_ragged", dict(dtype="bf16", d_k=64, d_v=64, L=1000, seg_len=64, B=2,
                                           H_q=3, H_kv=3, rule="delta")),
    ("tc_small_d64_S32_gqa_ragged", dict(dtype="bf16", d_k=64, d_v=64, L=1030, seg_len=32, H_q=4,
                                         H_kv=2)),
    ("tc_small_d128_S64_delta", dict(dtype="bf16", d_k=128, d_v=128, L=384, seg_len=64, H_q=2,
                                     H_kv=2, rule="delta")),
    # More (segment, KV head) items than SMs: the persistent products kernel
    # runs several items per CTA (block counters and the accumulator hand-off
    # carry across items), with a ragged last segment.
    ("tc_d64_S256_delta_items", dict(dtype="bf16", d_k=64, d_v=64, L=8292, seg_len=256, B=2,
                                     H_q=3, H_kv=3, rule="delta")),
    ("tc_d128_S128_linear_items", dict(dtype="bf16", d_k=128, d_v=128, L=6405, seg_len=128,
                                       H_q=3, H_kv=3)),
]


def test_path_selection(cuda_lib):
    api = cuda_lib
    for name, over, path in [("8b-delta", {}, "tcgen05"), ("1m-linear", {}, "tcgen05"),
                             ("300m-delta", {}, "tcgen05"), ("tiny", {}, "simt"),
                             ("200m-linear", {}, "tcgen05"), ("200m-delta", {}, "tcgen05"),
                             ("200m-linear", {"seg_len": 63}, "simt")]:
        w = W[name].with_(**over)
        dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, 0 if w.dtype == "bf16" else 1)
        assert api.plan(dims, w.seg_len, w.rule)["path"] == path, name
    for name, over in TC_CASES:
        w = W["tiny"].with_(**over)
        dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, 0)
        assert api.plan(dims, w.seg_len, w.rule)["path"] == "tcgen05", name


@pytest.mark.parametrize("name,over", TC_CASES, ids=[c[0] for c in TC_CASES])
def test_tensor_core_path_cases(cuda_lib, name, over):
    check_full(cuda_lib, W["tiny"].with_(name=name, **over))


def _scale_bf16_bits(bits, factor):
    """bf16 bit patterns times a power of two (exact)."""
    f = (bits.astype(np.uint32) << 16).view(np.float32) * np.float32(factor)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


# Keys of later tiles 8x larger than the rest: their scores exceed the first
# tile's row max by far more than 2^16 / 128 in 2^x terms, so the lazy softmax
# reference moves mid-segment: in the low half of a tile (keys 0..63), in the
# high half (64..127) and in both, with earlier tiles already accumulated in O.
# With one query head per KV head the two halves of a work item take the even
# and the odd key tiles, so spikes there also give the two halves row maxima
# far apart when their softmax states are merged: 8x, 32x (scores ~2^7 apart
# in 2^x terms, so the smaller half's weight would underflow fp32 if the
# retrieval were folded into that half alone), and a spike inside tile 0.
_LATER = (128 + 100, 256 + 10, 384 + 5, 384 + 120)
SPIKE_CASES = [
    ("spike_d128_gqa", dict(dtype="bf16", d_k=128, d_v=128, L=1024, seg_len=512, H_q=4, H_kv=2,
                            rule="delta"), 8.0, _LATER),
    ("spike_d64_gqa", dict(dtype="bf16", d_k=64, d_v=64, L=1024, seg_len=512, H_q=4, H_kv=2), 8.0,
     _LATER),
    ("spike_d128_one_q_per_kv", dict(dtype="bf16", d_k=128, d_v=128, L=1024, seg_len=512, H_q=2,
                                     H_kv=2), 8.0, _LATER),
    ("spike32_d64_one_q_per_kv_odd_tiles", dict(dtype="bf16", d_k=64, d_v=64, L=1024, seg_len=512,
                                               H_q=2, H_kv=2), 32.0, (128 + 100, 384 + 5)),
    ("spike_d128_one_q_per_kv_tile0", dict(dtype="bf16", d_k=128, d_v=128, L=1024, seg_len=512,
                                           H_q=2, H_kv=2, rule="delta"), 8.0, (3, 77)),
]


@pytest.mark.parametrize("name,over,factor,offsets", SPIKE_CASES, ids=[c[0] for c in SPIKE_CASES])
def test_tensor_core_path_softmax_reference_moves(cuda_lib, name, over, factor, offsets):
    w = W["tiny"].with_(name=name, **over)
    inp = synth.make_inputs(w)
    for seg0 in range(0, w.L, w.seg_len):
        for off in offsets:
            if seg0 + off < w.L:
                inp["k"][:, :, seg0 + off, :] = _scale_bf16_bits(inp["k"][:, :, seg0 + off, :], factor)
    check_full(cuda_lib, w, inp)


def test_tensor_core_path_deterministic_and_workspace_independent(cuda_lib):
    api = cuda_lib
    w = W["tiny"].with_(dtype="bf16", d_k=128, d_v=128, L=1024, seg_len=256, B=2, H_q=4, H_kv=2,
                        rule="delta")
    inp = synth.make_inputs(w)
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, torch.bfloat16)
    n = api.workspace_bytes(dims, w.seg_len, w.rule)
    ws = torch.full((n,), 0x7F, dtype=torch.uint8, device="cuda")
    a = gpu_forward(api, inp, w, workspace=ws)
    b = gpu_forward(api, inp, w)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("seg_len", [128, 64])
def test_tensor_core_path_gate_extremes(cuda_lib, seg_len):
    w = W["tiny"].with_(dtype="bf16", d_k=64, d_v=64, H_q=4, H_kv=2, L=512, seg_len=seg_len)
    inp = synth.make_inputs(w)
    inp["beta"] = np.array([-np.inf, np.inf, -80.0, 80.0], np.float32)
    check_full(cuda_lib, w, inp)
    out, _, _ = gpu_forward(cuda_lib, inp, w)
    # beta = +inf: out is the retrieval alone, exactly 0 on the first segment
    assert np.all(out[:, 1, :seg_len] == 0.0)


def test_tensor_core_path_split_stream(cuda_lib):
    api = cuda_lib
    w = W["tiny"].with_(dtype="bf16", rule="delta", B=1, H_q=4, H_kv=2, L=1024, seg_len=256,
                        d_k=128, d_v=128)
    inp = synth.make_inputs(w)
    q, k, v = (to_torch(inp[n], "bf16") for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).cuda()
    M, z = api.init_state(1, 2, 128, 128)
    out_full, M_full, z_full = api.forward(q, k, v, beta, M, z, 256, "delta")
    L1 = 512
    o1, _, _ = api.forward(q[:, :, :L1].contiguous(), k[:, :, :L1].contiguous(),
                           v[:, :, :L1].contiguous(), beta, M, z, 256, "delta", M_out=M, z_out=z)
    o2, _, _ = api.forward(q[:, :, L1:].contiguous(), k[:, :, L1:].contiguous(),
                           v[:, :, L1:].contiguous(), beta, M, z, 256, "delta", M_out=M, z_out=z)
    api.sync_status()
    assert torch.max(torch.abs(torch.cat([o1, o2], 2).float() - out_full.float())) <= 2e-2
    assert torch.allclose(M, M_full, rtol=1e-5, atol=1e-4)


def test_linear_rule_tokens_per_second_does_not_fall_with_length(cuda_lib):
    """The per-token cost is O(S) at fixed S and d: at the 1M-token shape
    (32 heads, d = 128, S = 2048, linear rule) a 1M-token forward keeps at least
    the throughput of a 64K-token slice (device time, CUDA events)."""
    api = cuda_lib
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(7)

    def tokens_per_s(L, reps):
        q = torch.randn(1, 32, L, 128, device=dev, generator=g).to(torch.bfloat16)
        k = torch.randn(1, 32, L, 128, device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn(1, 32, L, 128, device=dev, generator=g).to(torch.bfloat16)
        beta = torch.zeros(32, device=dev)
        M, z = api.init_state(1, 32, 128, 128)
        dims = api.make_dims(1, 32, 32, L, 128, 128, torch.bfloat16)
        ws = torch.empty(api.workspace_bytes(dims, 2048, "linear"), dtype=torch.uint8, device=dev)
        out = torch.empty_like(q)
        Mo, zo = torch.empty_like(M), torch.empty_like(z)
        for _ in range(2):
            api.forward(q, k, v, beta, M, z, 2048, "linear", out, Mo, zo, ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            api.forward(q, k, v, beta, M, z, 2048, "linear", out, Mo, zo, ws)
        e1.record()
        api.sync_status()
        return L * reps / (e0.elapsed_time(e1) / 1e3)

    small = tokens_per_s(65536, 8)
    large = tokens_per_s(1 << 20, 2)
    assert large >= 0.8 * small, (small, large)
