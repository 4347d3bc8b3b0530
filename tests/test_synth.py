"""The seeded input module: bf16 rounding, determinism, per-slice streams."""

import numpy as np
import torch

from compressive_memory_transformer_segment_b200 import configs, synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 7,
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40, 1.00390625, 1.01171875],
                                 dtype=np.float32)])
    ours = synth.round_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_inputs_deterministic_and_slices_independent():
    w = configs.WORKLOADS["tiny"].with_(B=2, H_q=4, H_kv=2, dtype="bf16")
    a = synth.make_inputs(w)
    b = synth.make_inputs(w)
    for key in ("q", "k", "v", "beta"):
        np.testing.assert_array_equal(a[key], b[key])
    only = synth.make_inputs(w, heads_q={3}, heads_kv={1})
    np.testing.assert_array_equal(only["q"][:, 3], a["q"][:, 3])
    np.testing.assert_array_equal(only["k"][:, 1], a["k"][:, 1])
    assert not only["q"][:, 0].any()
    assert np.all(np.abs(a["beta"]) <= w.beta_range)


def test_inserted_pair_placement():
    w = configs.WORKLOADS["tiny"].with_(L=2 * 64 + 1000 + 50, insert_pair=True, dtype="bf16")
    x = synth.make_inputs(w)
    p = x["pair_pos"]
    assert p == 2 * 64 + 1000
    np.testing.assert_array_equal(x["k"][0, 0, p], x["k"][0, 1, p])
    np.testing.assert_array_equal(x["q"][0, 0, w.L - 1], x["k"][0, 0, p])


def test_algorithmic_counts_8b():
    w = configs.WORKLOADS["8b-delta"]
    assert abs(configs.algorithmic_flops(w) / 1.204e12 - 1) < 2e-3
    assert abs(configs.algorithmic_bytes(w) / 1.344e9 - 1) < 2e-3


def test_make_head_matches_make_inputs():
    w = configs.WORKLOADS["tiny"].with_(B=2, H_q=4, H_kv=2, L=2 * 64 + 1000 + 8,
                                        insert_pair=True, dtype="bf16")
    x = synth.make_inputs(w)
    for name, H in (("q", 4), ("k", 2), ("v", 2)):
        for b in range(2):
            for h in range(H):
                np.testing.assert_array_equal(synth.make_head(w, name, b, h), x[name][b, h])
    np.testing.assert_array_equal(synth.make_beta(w), x["beta"])


def test_decode_bytes_per_segment_closed_form():
    """The decode roofline's byte count (bench.py) against a sum over the
    positions of one segment, written out call by call."""
    import importlib.util
    import os
    spec = importlib.util.spec_from_file_location(
        "bench_mod", os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    for name, over in (("8b-delta", {}), ("tiny", dict(dtype="bf16", d_k=64, d_v=64, seg_len=48))):
        w = configs.WORKLOADS[name].with_(**over)
        e = 2 if w.dtype == "bf16" else 4
        d, S = w.d_k, w.seg_len
        total = 0
        for pos in range(S):
            per_kv = (pos + 1) * 2 * d * e + d * d * 4 + d * 4 + 2 * d * e + 2 * d * e
            per_q = d * e + d * e + 4
            total += w.B * (w.H_kv * per_kv + w.H_q * per_q)
        assert bench.decode_bytes_per_segment(w) == total


def test_bench_reference_arm_runs_on_the_host():
    """`bench.py --impl reference` (the float64 oracle on the host cores)
    prints one JSON line in the bench's format, with no GPU."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "1",
                          "--reference-budget", "1"],
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["unit"] == "tokens/s" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
