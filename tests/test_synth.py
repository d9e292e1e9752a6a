"""The seeded input generators: determinism, rounding and the stated recipes."""
import numpy as np
import torch

import gh_synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(0, 3, 100000).astype(np.float32),
                        np.array([1.00390625, 1.01171875, -2.0 ** -130, 3.3e38], dtype=np.float32)])
    bits = gh_synth.f32_to_bf16(v)
    expect = torch.tensor(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, expect)
    np.testing.assert_array_equal(gh_synth.bf16_to_f32(bits),
                                  torch.tensor(v).to(torch.bfloat16).float().numpy())


def test_generation_is_deterministic_and_thread_independent(monkeypatch):
    a = gh_synth.ce_normal(300, 20001, 3.0, ignore_frac=0.02, seed=5)
    monkeypatch.setattr(gh_synth, "_threads", lambda: 1)
    b = gh_synth.ce_normal(300, 20001, 3.0, ignore_frac=0.02, seed=5)
    np.testing.assert_array_equal(a.logits, b.logits)
    np.testing.assert_array_equal(a.targets, b.targets)
    c = gh_synth.ce_normal(300, 20001, 3.0, ignore_frac=0.02, seed=6)
    assert not np.array_equal(a.logits, c.logits)


def test_ignore_fraction_is_exact():
    p = gh_synth.ce_normal(1000, 64, 1.0, ignore_frac=0.10, seed=0)
    assert int((p.targets == -100).sum()) == 100
    v = p.targets[p.targets != -100]
    assert v.min() >= 0 and v.max() < 64


def test_small_workload_recipe():
    p = gh_synth.ce_small(z_loss=1e-4)
    assert p.logits.dtype == np.float32 and p.logits.shape == (64, 1024)
    assert int((p.targets == -100).sum()) == 6
    assert abs(p.logits.std() - 2.0) < 0.05 and p.reduction == "mean" and p.z_loss == 1e-4


def test_spiked_student_t_recipe():
    p = gh_synth.ce_student_t_spiked(200, 3000, seed=3, dtype="f32")
    q = gh_synth.ce_student_t_spiked(200, 3000, seed=3, dtype="f32", spike=0.0)
    x, y = p.values_f32(), q.values_f32()
    np.testing.assert_array_equal(p.targets, q.targets)
    assert 2.0 < np.median(np.abs(y)) < 6.0
    # exactly 20 positions (10% of rows) differ by +30, one per row, 10 at the target
    r, c = np.nonzero(x != y)
    assert len(r) == 20 and len(set(r.tolist())) == 20
    np.testing.assert_allclose(x[r, c] - y[r, c], 30.0, atol=1e-4)
    assert int((c == p.targets[r]).sum()) == 10


def test_linear_recipe_shapes_and_scales():
    p = gh_synth.linear_ce_normal(64, 32, 500, chunk=16, ignore_frac=0.05, seed=2)
    X = gh_synth.bf16_to_f32(p.inputs)
    W = gh_synth.bf16_to_f32(p.weight)
    assert X.shape == (64, 32) and W.shape == (500, 32)
    assert abs(X.std() - 1.0) < 0.1 and abs(W.std() - 0.02) < 0.002
    assert int((p.targets == -100).sum()) == 3
