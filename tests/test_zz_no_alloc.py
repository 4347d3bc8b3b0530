"""The no-allocation entry point, infini_attn_forward_noalloc.

It exists for callers that cannot allocate GPU memory while they run (an
allocator's own callback, a loop that must never block on the driver's
allocator, an embedding that owns all device memory): they pass inputs and
outputs only, and the scratch comes from a static device array inside the
library.  These tests call it through the C ABI and compare it with the
regular infini_attn_forward (which takes a workspace) on two calls in a row.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""

import ctypes

import pytest
import torch

from compressive_memory_transformer_segment_b200 import api, configs, synth
from helpers import TOL_OUT, TOL_STATE, to_torch


def test_noalloc_rejects_problems_beyond_its_static_scratch():
    """Host-side check (no CUDA call is made): a 1M-token stream needs far more
    scratch than the static array holds."""
    lib = api.load_library()
    w = configs.WORKLOADS["1m-linear"]
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, 0)
    assert api.workspace_bytes(dims, w.seg_len, w.rule) > api.noalloc_scratch_limit()
    P = ctypes.c_void_p
    MB = 1 << 20
    rc = lib.infini_attn_forward_noalloc(P(MB), P(2 * MB), P(3 * MB), P(4 * MB), P(5 * MB),
                                         P(6 * MB), w.seg_len, 0, ctypes.byref(dims), P(7 * MB),
                                         P(8 * MB), P(9 * MB), P(0))
    assert rc == api.ERR_SCRATCH_LIMIT
    assert "scratch" in api.status_string(rc)


def _problem(w, seed):
    ww = w.with_(seed=seed)
    inp = synth.make_inputs(ww)
    q, k, v = (to_torch(inp[n], w.dtype) for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).cuda()
    M0, z0 = api.init_state(w.B, w.H_kv, w.d_k, w.d_v)
    return q, k, v, beta, M0, z0


def _outputs_like(q, M0, z0, w):
    out = torch.empty((w.B, w.H_q, w.L, w.d_v), dtype=q.dtype, device=q.device)
    return out, torch.empty_like(M0), torch.empty_like(z0)


# The shape whose scratch layout is left in the static array before each
# compared call: a different workload, so that a read of any byte the call
# did not write itself would see another layout's values.
_POISON = {"tiny": "8b-delta", "200m-delta": "8b-delta", "8b-delta": "300m-delta"}


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "200m-delta", "8b-delta"])
def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_lib, name):
    w = configs.WORKLOADS[name]
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, tdt)
    need = api.workspace_bytes(dims, w.seg_len, w.rule)
    assert need <= api.noalloc_scratch_limit()
    # Another workload's call fills the static array with its own layout.
    pw = configs.WORKLOADS[_POISON[name]]
    g = torch.Generator(device="cuda").manual_seed(7)
    pdt = torch.bfloat16 if pw.dtype == "bf16" else torch.float32
    pq = torch.randn((pw.B, pw.H_q, pw.L, pw.d_k), generator=g, device="cuda").to(pdt)
    pk = torch.randn((pw.B, pw.H_kv, pw.L, pw.d_k), generator=g, device="cuda").to(pdt)
    pv = torch.randn((pw.B, pw.H_kv, pw.L, pw.d_v), generator=g, device="cuda").to(pdt)
    pbeta = torch.zeros(pw.H_q, dtype=torch.float32, device="cuda")
    pM0, pz0 = api.init_state(pw.B, pw.H_kv, pw.d_k, pw.d_v)
    api.forward_noalloc(pq, pk, pv, pbeta, pM0, pz0, pw.seg_len, pw.rule,
                        *_outputs_like(pq, pM0, pz0, pw))
    del pq, pk, pv
    outs = []
    for seed_shift in (0, 1):  # two different inputs, back to back
        q, k, v, beta, M0, z0 = _problem(w, w.seed + 100 * seed_shift)
        # The reference forward reads a NaN-filled workspace: any byte it read
        # before writing would turn its results into NaN.
        ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=q.device)
        ref = api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule, workspace=ws)
        got = _outputs_like(q, M0, z0, w)
        api.forward_noalloc(q, k, v, beta, M0, z0, w.seg_len, w.rule, *got)
        outs.append((ref, got))
    api.sync_status()
    for ref, got in outs:
        assert torch.isfinite(ref[0].float()).all() and torch.isfinite(ref[1]).all()
        assert torch.max(torch.abs(got[0].float() - ref[0].float())).item() <= TOL_OUT[w.dtype]
        rel_M = (torch.linalg.vector_norm(got[1] - ref[1]) /
                 torch.linalg.vector_norm(ref[1]).clamp_min(1e-30)).item()
        rel_z = (torch.abs(got[2] - ref[2]) / torch.abs(ref[2]).clamp_min(1e-30)).max().item()
        assert rel_M <= TOL_STATE and rel_z <= TOL_STATE


@pytest.mark.gpu
def test_noalloc_commits_no_device_memory_after_a_warm_up_call(cuda_lib):
    """The first call on a device may load the library's GPU code (lazy module
    loading commits memory for the code and the static array); a second call
    of the same shape must not change the device's free memory."""
    w = configs.WORKLOADS["8b-delta"].with_(L=4096)
    q, k, v, beta, M0, z0 = _problem(w, w.seed)
    got = _outputs_like(q, M0, z0, w)
    api.forward_noalloc(q, k, v, beta, M0, z0, w.seg_len, w.rule, *got)  # warm-up
    api.sync_status()
    free0 = torch.cuda.mem_get_info()[0]
    api.forward_noalloc(q, k, v, beta, M0, z0, w.seg_len, w.rule, *got)
    api.sync_status()
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 == free0
