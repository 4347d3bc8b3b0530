"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol include/infini_attn.h declares, and rejects bad arguments on the host
before any CUDA call (no compute is launched here)."""

import ctypes
import os
import re

import pytest

from compressive_memory_transformer_segment_b200 import api, configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"INFINI_API\s+[\w\s\*]*?\b(infini_attn_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    return api.load_library()


def test_library_exports_every_declared_symbol(lib):
    declared = header_symbols()
    assert {"infini_attn_init_state", "infini_attn_forward"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(api.exported_symbols())
    assert lib.infini_attn_version() >> 16 == 1


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, 12345):
        assert api.status_string(code)


def dims_of(w):
    return api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, 0 if w.dtype == "bf16" else 1)


@pytest.mark.parametrize("name", sorted(configs.WORKLOADS))
def test_plan_and_workspace_for_every_workload(name):
    w = configs.WORKLOADS[name]
    d = dims_of(w)
    p = api.plan(d, w.seg_len, w.rule)
    assert p["num_segments"] == w.T
    assert p["workspace_bytes"] == api.workspace_bytes(d, w.seg_len, w.rule) > 0
    # The workspace holds at least the z read by every segment.
    assert p["workspace_bytes"] >= w.T * w.B * w.H_kv * w.d_k * 4
    assert api.host_arena_bytes(d, w.seg_len, w.rule) > p["workspace_bytes"]


@pytest.mark.parametrize("bad", [
    dict(B=0), dict(H_q=3, H_kv=2), dict(L=0), dict(d_k=48), dict(d_v=256), dict(dtype=7),
])
def test_plan_rejects_bad_sizes(bad):
    base = dict(B=1, H_q=4, H_kv=2, L=128, d_k=64, d_v=64, dtype=0)
    base.update(bad)
    d = api.Dims(**base)
    with pytest.raises(api.InfiniError) as e:
        api.plan(d, 64, "linear")
    assert e.value.status in (api.ERR_ARG, api.ERR_UNSUPPORTED)
    assert api.workspace_bytes(d, 64, "linear") == 0


def test_plan_rejects_bad_rule_and_segment():
    d = api.Dims(1, 2, 2, 64, 32, 32, 1)
    for seg, rule in ((0, 0), (-3, 1), (16, 2)):
        with pytest.raises(api.InfiniError):
            api.plan(d, seg, rule)


def _fwd(lib, ptrs, dims, seg=64, rule=0, ws=0, ws_n=0):
    P = ctypes.c_void_p
    q, k, v, beta, M, z, out, Mo, zo = (P(x) for x in ptrs)
    return lib.infini_attn_forward(q, k, v, beta, M, z, seg, rule, ctypes.byref(dims), out, Mo, zo,
                                   P(ws), ws_n, P(0))


def test_forward_validates_on_host_before_any_cuda_call(lib):
    """Fake, never-dereferenced addresses: every case below must be rejected
    by the host checks, so no CUDA call happens (this machine has no GPU)."""
    d = api.Dims(1, 2, 2, 128, 32, 32, 1)  # f32: q = k = v = out = 32 KiB
    MB = 1 << 20
    good = [1 * MB, 2 * MB, 3 * MB, 4 * MB, 5 * MB, 6 * MB, 7 * MB, 8 * MB, 9 * MB]
    bad = list(good)
    bad[0] = 0
    assert _fwd(lib, bad, d) == api.ERR_ARG
    bad = list(good)
    bad[2] += 4
    assert _fwd(lib, bad, d) == api.ERR_ALIGN
    bad = list(good)
    bad[6] = good[0] + 1024  # out inside q
    assert _fwd(lib, bad, d) == api.ERR_ALIAS
    bad = list(good)
    bad[7] = good[6]  # M_out == out
    assert _fwd(lib, bad, d) == api.ERR_ALIAS
    bad = list(good)
    bad[8] = good[4] + 16  # z_out overlaps M_in (not the permitted in-place pair)
    assert _fwd(lib, bad, d) == api.ERR_ALIAS
    assert _fwd(lib, good, d, ws=10 * MB, ws_n=16) == api.ERR_WORKSPACE
    assert _fwd(lib, good, d, ws=10 * MB + 16, ws_n=1 << 30) == api.ERR_WORKSPACE
    assert _fwd(lib, good, d, ws=0, ws_n=64) == api.ERR_ARG
    assert _fwd(lib, good, d, ws=good[0], ws_n=1 << 20) == api.ERR_ALIAS
    d_bad = api.Dims(1, 2, 2, 128, 40, 32, 1)
    assert _fwd(lib, good, d_bad) == api.ERR_UNSUPPORTED


def test_state_update_validates_on_host_before_any_cuda_call(lib):
    P = ctypes.c_void_p
    d = api.Dims(1, 2, 2, 128, 32, 32, 1)
    MB = 1 << 20
    k, v, M, z, Mo, zo = 1 * MB, 2 * MB, 3 * MB, 4 * MB, 5 * MB, 6 * MB

    def call(k=k, v=v, M=M, z=z, Mo=Mo, zo=zo, seg=64, rule=0, ws=0, ws_n=0, dims=d):
        return lib.infini_attn_state_update(P(k), P(v), P(M), P(z), seg, rule, ctypes.byref(dims),
                                            P(Mo), P(zo), P(ws), ws_n, P(0))

    assert call(k=0) == api.ERR_ARG
    assert call(v=v + 8) == api.ERR_ALIGN
    assert call(Mo=k + 1024) == api.ERR_ALIAS      # M_out inside k
    assert call(zo=M + 16) == api.ERR_ALIAS        # z_out overlaps M_in
    assert call(rule=7) == api.ERR_ARG
    assert call(seg=0) == api.ERR_ARG
    assert call(ws=10 * MB, ws_n=16) == api.ERR_WORKSPACE
    assert call(dims=api.Dims(1, 2, 2, 128, 40, 32, 1)) == api.ERR_UNSUPPORTED


def test_decode_step_validates_on_host_before_any_cuda_call(lib):
    P = ctypes.c_void_p
    d = api.Dims(1, 4, 2, 1, 32, 32, 1)
    MB = 1 << 20
    good = dict(q=1 * MB, k=2 * MB, v=3 * MB, beta=4 * MB, kb=5 * MB, vb=6 * MB, M=7 * MB, z=8 * MB,
                out=9 * MB)

    def call(pos=0, seg=16, rule=0, ws=0, ws_n=0, dims=d, **over):
        a = dict(good, **over)
        return lib.infini_attn_decode_step(P(a["q"]), P(a["k"]), P(a["v"]), P(a["beta"]), P(a["kb"]),
                                           P(a["vb"]), pos, P(a["M"]), P(a["z"]), seg, rule,
                                           ctypes.byref(dims), P(a["out"]), P(ws), ws_n, P(0))

    assert lib.infini_attn_decode_workspace_bytes(ctypes.byref(d), 16, 0) > 0
    assert lib.infini_attn_decode_workspace_bytes(ctypes.byref(api.Dims(1, 4, 2, 1, 32, 64, 1)),
                                                  16, 0) == 0
    assert call(pos=16) == api.ERR_ARG            # pos must be < seg_len
    assert call(pos=-1) == api.ERR_ARG
    assert call(q=0) == api.ERR_ARG
    assert call(k=good["k"] + 4) == api.ERR_ALIGN
    assert call(out=good["q"]) == api.ERR_ALIAS    # out over q_t
    assert call(kb=good["vb"] + 64) == api.ERR_ALIAS
    assert call(M=good["kb"] + 256) == api.ERR_ALIAS
    assert call(ws=10 * MB, ws_n=16) == api.ERR_WORKSPACE
    assert call(ws=good["M"], ws_n=1 << 22) == api.ERR_ALIAS
    assert call(dims=api.Dims(1, 4, 2, 1, 32, 64, 1)) == api.ERR_UNSUPPORTED


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(api, "_lib", None)
    with pytest.raises(FileNotFoundError):
        api.load_library(str(tmp_path / "missing.so"))


def test_state_sum_rejects_bad_arguments_on_the_host(lib):
    """Argument checks of infini_attn_state_sum return before any CUDA call."""
    P = ctypes.c_void_p
    MB = 1 << 20
    n_M, n_z = 2 * 3 * 8 * 8 * 4, 2 * 3 * 8 * 4
    base = (P(MB), P(2 * MB))
    assert lib.infini_attn_state_sum(P(0), P(2 * MB), P(0), 0, 2, 3, 8, 8, P(3 * MB), P(4 * MB),
                                     P(0)) == api.ERR_ARG
    assert lib.infini_attn_state_sum(*base, P(0), 2, 2, 3, 8, 8, P(3 * MB), P(4 * MB),
                                     P(0)) == api.ERR_ARG  # parts NULL with n_parts > 0
    assert lib.infini_attn_state_sum(*base, P(0), -1, 2, 3, 8, 8, P(3 * MB), P(4 * MB),
                                     P(0)) == api.ERR_ARG
    assert lib.infini_attn_state_sum(*base, P(0), 0, 0, 3, 8, 8, P(3 * MB), P(4 * MB),
                                     P(0)) == api.ERR_ARG
    assert lib.infini_attn_state_sum(*base, P(0), 0, 2, 3, 8, 8, P(3 * MB + 4), P(4 * MB),
                                     P(0)) == api.ERR_ALIGN
    # M_out overlapping z_out, or the parts, or another state's base
    assert lib.infini_attn_state_sum(*base, P(0), 0, 2, 3, 8, 8, P(3 * MB), P(3 * MB + n_M - 16),
                                     P(0)) == api.ERR_ALIAS
    assert lib.infini_attn_state_sum(*base, P(5 * MB), 1, 2, 3, 8, 8, P(5 * MB + 64), P(4 * MB),
                                     P(0)) == api.ERR_ALIAS
    assert lib.infini_attn_state_sum(*base, P(0), 0, 2, 3, 8, 8, P(MB + 16), P(4 * MB),
                                     P(0)) == api.ERR_ALIAS
    assert n_z < n_M


def test_backward_workspace_and_host_checks(lib):
    """The backward's sizing and argument checks run on the host: supported
    shapes (seg_len <= 64, d_k = d_v in {32, 64}) get a workspace that holds
    at least the fp32 states of every segment; others get 0, and the call
    returns INFINI_ERR_UNSUPPORTED (or INFINI_ERR_ARG for NULL pointers)
    before touching a GPU."""
    w = configs.WORKLOADS["200m-delta"]
    d = dims_of(w)
    nbytes = api.backward_workspace_bytes(d, w.seg_len, w.rule)
    assert nbytes >= w.T * w.B * w.H_kv * w.d_k * w.d_k * 4
    for over in (dict(d_k=128, d_v=128), dict(d_k=64, d_v=32)):
        dd = dims_of(w.with_(**over))
        assert api.backward_workspace_bytes(dd, w.seg_len, w.rule) == 0
    assert api.backward_workspace_bytes(d, 65, w.rule) == 0
    null = ctypes.c_void_p(0)
    args = [null] * 6 + [w.seg_len, 1, ctypes.byref(d)] + [null] * 9 + [null, 0, null]
    assert lib.infini_attn_backward(*args) == -1  # INFINI_ERR_ARG
    args[6] = 128
    assert lib.infini_attn_backward(*args) == -2  # INFINI_ERR_UNSUPPORTED


def test_qkv_project_and_rope_tables_check_arguments_on_the_host(lib):
    """The projection prologue's and the rotary tables' argument checks
    return before any CUDA call."""
    P = ctypes.c_void_p
    MB = 1 << 20
    d = api.make_dims(2, 4, 2, 256, 64, 64, 0)
    x, w, bias, cs, sn = P(1 * MB), P(8 * MB), P(12 * MB), P(13 * MB), P(14 * MB)
    q, k, v = P(20 * MB), P(24 * MB), P(28 * MB)

    def call(*a, dims=d, dm=256):
        a = list(a) if a else [x, w, bias, cs, sn]
        return lib.infini_attn_qkv_project(*a, ctypes.byref(dims), dm, q, k, v, P(0))

    assert call(P(0), w, bias, cs, sn) == api.ERR_ARG
    assert call(x, w, bias, cs, P(0)) == api.ERR_ARG         # one table without the other
    assert call(dm=0) == api.ERR_ARG
    assert call(dims=api.make_dims(2, 4, 2, 256, 128, 64, 0)) == api.ERR_UNSUPPORTED
    assert call(dims=api.make_dims(2, 4, 2, 256, 32, 32, 0)) == api.ERR_UNSUPPORTED
    assert call(dims=api.make_dims(2, 4, 2, 256, 64, 64, 1)) == api.ERR_UNSUPPORTED  # f32
    assert call(dm=60) == api.ERR_UNSUPPORTED
    assert call(dm=260) == api.ERR_UNSUPPORTED
    assert call(P(1 * MB + 8), w, bias, cs, sn) == api.ERR_ALIGN
    # q [2, 4, 256, 64] bf16 = 256 KB from 20 MB: an input there overlaps it.
    assert call(x, w, bias, P(20 * MB + 4096), sn) == api.ERR_ALIAS
    assert lib.infini_attn_qkv_project(x, w, bias, cs, sn, ctypes.byref(d), 256, q, P(20 * MB + 64),
                                       v, P(0)) == api.ERR_ALIAS
    assert lib.infini_attn_rope_tables(P(0), P(MB), 16, 64, 10000.0, P(0)) == api.ERR_ARG
    assert lib.infini_attn_rope_tables(P(MB), P(2 * MB), 0, 64, 10000.0, P(0)) == api.ERR_ARG
    assert lib.infini_attn_rope_tables(P(MB), P(2 * MB), 16, 63, 10000.0, P(0)) == api.ERR_ARG
    assert lib.infini_attn_rope_tables(P(MB), P(2 * MB), 16, 64, 0.0, P(0)) == api.ERR_ARG
    assert lib.infini_attn_rope_tables(P(MB), P(MB + 256), 16, 64, 1e4, P(0)) == api.ERR_ALIAS


def test_plain_c_program_uses_the_boundary(tmp_path):
    """The header compiles as C99 and a C program linked against the library
    gets the documented answers from the host-side calls (no GPU needed)."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(api.LIB_PATH)
    exe = tmp_path / "c_abi_check"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), api.LIB_PATH,
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == "c-abi ok"
