"""The seeded generator: determinism, head-prefix consistency, shapes and dtypes."""
import numpy as np
import torch

from synthetic import CONFIGS, make_inputs, token_grid_features


def test_generator_is_deterministic_and_head_prefix_consistent():
    cfg = CONFIGS["tiny"]
    q1, k1, v1 = make_inputs(cfg, 0)
    q2, k2, v2 = make_inputs(cfg, 0, heads=1)
    assert q1.shape == (1, 2, 1024, 64) and q1.dtype == torch.float32
    assert torch.equal(q1[:, :1], q2) and torch.equal(k1[:, :1], k2) and torch.equal(v1[:, :1], v2)
    q3, _, _ = make_inputs(cfg, 1)
    assert not torch.equal(q1, q3)


def test_generator_bf16_cast_and_scale():
    cfg = CONFIGS["small"].with_(grid=(2, 8, 8), heads=2)
    q, k, v = make_inputs(cfg, 0)
    assert q.dtype == torch.bfloat16 and q.shape == (1, 2, 128, 128)
    q64, _, _ = make_inputs(cfg, 0, dtype=torch.float64)
    assert torch.equal(q64.to(torch.bfloat16), q)
    # latent variance ~ pos (1) + sigma_c^2 + sigma_n^2 -> per-entry std of Q ~ 1.5
    std = float(q64.std())
    assert 1.0 < std < 2.2


def test_positional_features():
    f = token_grid_features((2, 3, 4))
    assert f.shape == (24, 24)
    # token (t=1, y=2, x=3) is the last one; its x-axis f=0 sin feature
    assert np.isclose(f[-1, 16], np.sin(2 * np.pi * 3 / 4))
    assert np.allclose(f[:, 0::2] ** 2 + f[:, 1::2] ** 2, 1.0)
