"""Properties of the seeded input generator (no GPU)."""
import numpy as np
import torch

import synth


def test_bf16_rounding_is_nearest_even():
    one = np.float32(1.0)
    vals = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9, -2.5, 0.0],
                    dtype=np.float32)
    got = synth.bits_to_f32(synth.bf16_bits(vals))
    # 1+2^-8 is a tie between 1 and 1+2^-7 -> even mantissa (1.0);
    # 1+3*2^-8 is a tie between 1+2^-7 and 1+2^-6 -> even (1+2^-6).
    assert got.tolist() == [1.0, 1.0, 1.0 + 2.0 ** -6, 1.0, -2.5, 0.0]
    assert one == got[0]


def test_uniform_mask_exact_count_and_nested():
    w = synth.WORKLOADS
    masks = {d: synth.make_mask(w[f"enc_train_d{d}"]) for d in ("1.0", "0.5", "0.25", "0.1")}
    assert {d: int(m.sum()) for d, m in masks.items()} == {"1.0": 2304, "0.5": 1152, "0.25": 576, "0.1": 230}
    assert np.all(masks["0.5"] >= masks["0.25"]) and np.all(masks["0.25"] >= masks["0.1"])


def test_zipf_row_profile():
    w = synth.WORKLOADS["large_fwd"]
    m = synth.make_mask(w)
    counts = m.sum(axis=1)
    s = sorted(counts.tolist(), reverse=True)
    assert sum(s) == 1434 and s[:8] == [64, 64, 64, 64, 64, 59, 50, 43]
    assert np.median(counts) == 2 and min(s) >= 1
    # the profile is a property of the rank law, not of the seed
    c2 = synth.zipf_row_counts(w.R, w.C, w.nnz, 1.1, np.random.default_rng(99))
    assert sorted(c2.tolist(), reverse=True) == s


def test_inputs_are_seeded_and_shaped():
    w = synth.WORKLOADS["tiny_fwd"]
    a, b = synth.make_inputs(w), synth.make_inputs(w)
    assert all(np.array_equal(a[k], b[k]) for k in a)
    assert a["X"].shape == (64, 256) and a["W"].shape == (256, 256) and a["mask"].sum() == 16
    Wf = synth.bits_to_f32(a["W"])
    assert abs(Wf.std() - 1 / 16) < 0.01
    t = torch.from_numpy(a["X"].view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(t, synth.bits_to_f32(a["X"]))


def test_semi24_weight_has_at_most_two_nonzeros_per_group():
    rng = np.random.default_rng(0)
    W = synth.semi24_weight(64, 256, rng)
    nz = ((W & 0x7FFF) != 0).reshape(64, 64, 4).sum(axis=2)
    assert (nz == 2).all()  # no normal draw of std 1 rounds to zero in bf16 here
    Wf = synth.semi24_weight(64, 256, np.random.default_rng(0), fewer=0.5)
    nzf = ((Wf & 0x7FFF) != 0).reshape(64, 64, 4).sum(axis=2)
    assert nzf.max() <= 2 and (nzf == 0).any() and (nzf == 1).any()
    assert (Wf == 0x8000).any()  # signed zeros appear
    assert np.array_equal(synth.semi24_weight(8, 16, np.random.default_rng(3)),
                          synth.semi24_weight(8, 16, np.random.default_rng(3)))


def test_semi24_workload_inputs_are_seeded():
    w = synth.SEMI24_WORKLOADS["semi24_fwd"]
    a = synth.make_semi24_inputs(w, M=4)
    b = synth.make_semi24_inputs(w, M=4)
    assert a["X"].shape == (4, w.K) and a["W"].shape == (w.N, w.K)
    assert np.array_equal(a["W"], b["W"]) and np.array_equal(a["X"], b["X"])
    assert w.flops() == 2 * w.M * w.N * (w.K // 2)
