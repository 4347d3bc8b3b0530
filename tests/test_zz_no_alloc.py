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


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "200m-delta", "8b-delta"])
def test_noalloc_matches_forward_on_two_calls_in_a_row(cuda_lib, name):
    w = configs.WORKLOADS[name]
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, tdt)
    assert api.workspace_bytes(dims, w.seg_len, w.rule) <= api.noalloc_scratch_limit()
    outs = []
    for seed_shift in (0, 1):  # two different inputs, back to back
        ww = w.with_(seed=w.seed + 100 * seed_shift)
        inp = synth.make_inputs(ww)
        q, k, v = (to_torch(inp[n], w.dtype) for n in ("q", "k", "v"))
        beta = torch.from_numpy(inp["beta"]).cuda()
        M0, z0 = api.init_state(w.B, w.H_kv, w.d_k, w.d_v)
        ref = api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule)
        got = (torch.empty_like(ref[0]), torch.empty_like(ref[1]), torch.empty_like(ref[2]))
        api.forward_noalloc(q, k, v, beta, M0, z0, w.seg_len, w.rule, *got)
        outs.append((ref, got))
    api.sync_status()
    for ref, got in outs:
        assert torch.max(torch.abs(got[0].float() - ref[0].float())).item() <= TOL_OUT[w.dtype]
        rel_M = (torch.linalg.vector_norm(got[1] - ref[1]) /
                 torch.linalg.vector_norm(ref[1]).clamp_min(1e-30)).item()
        rel_z = (torch.abs(got[2] - ref[2]) / torch.abs(ref[2]).clamp_min(1e-30)).max().item()
        assert rel_M <= TOL_STATE and rel_z <= TOL_STATE
    # The second call did not return the first call's (stale) results.
    assert not torch.equal(outs[0][1][0], outs[1][1][0])
