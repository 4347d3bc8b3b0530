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
