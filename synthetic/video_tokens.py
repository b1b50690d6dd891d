"""Seeded generator of video-DiT-like attention inputs.

The SparsePR pages measure on four video diffusion transformers whose weights and
prompts are not available here; these synthetic latents stand in for them with the
same token grids, head counts and head dims.  A token's latent is

    latent = pos(t, y, x) @ Wpos + mean[patch(y, x)] + noise

where ``pos`` holds 8 sin/cos features per grid axis (frequencies 2^0..2^3 over the
axis length), ``mean`` is one of C Gaussian cluster means that is constant over p x p
spatial patches and over time (a static scene), and ``noise`` is isotropic Gaussian.
Each head projects the latent with its own Gaussian Wq, Wk, Wv (std 1/sqrt(d)).

Draw order (numpy PCG64 ``default_rng(seed)``, all in float64):
  1. Wpos [24, d] ~ N(0, 1/24)
  2. per batch element: cluster means [C, d] ~ N(0, sigma_c^2);
     patch ids [ceil(Y/p), ceil(X/p)] uniform in [0, C);
     noise [N, d] ~ N(0, sigma_n^2);
     then per head: Wq, Wk, Wv [d, d] ~ N(0, 1/d) in that order.
The fp64 projections are cast to the config dtype (bf16 round-to-nearest-even) once;
both the oracle and the CUDA path read those cast values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class WorkloadConfig:
    name: str
    grid: tuple            # (T, Y, X) token grid, raster order t, y, x
    heads: int
    head_dim: int
    dtype: str             # "bf16" or "f32"
    n_clusters: int
    patch: int
    sigma_c: float
    sigma_n: float
    # attention-call parameters
    block: int             # query-block / key-group capacity B
    n_sampled: int         # S sampled queries for key response profiles
    n_probe: int           # P exact probe rows per head
    density: float         # target executed-pair density (probes counted)
    ridge_lambda: float
    rank: int              # residual subspace rank r
    kmeans_iters: int = 4
    batch: int = 1

    @property
    def n_tokens(self) -> int:
        t, y, x = self.grid
        return t * y * x

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def with_(self, **kw) -> "WorkloadConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": WorkloadConfig("tiny", (4, 16, 16), 2, 64, "f32", 32, 4, 1.0, 0.5,
                           block=64, n_sampled=64, n_probe=32, density=0.25,
                           ridge_lambda=1e-3, rank=8),
    "small": WorkloadConfig("small", (8, 32, 32), 8, 128, "bf16", 32, 4, 1.0, 0.5,
                            block=128, n_sampled=256, n_probe=64, density=0.22,
                            ridge_lambda=1e-3, rank=16),
    "video": WorkloadConfig("video", (21, 45, 80), 40, 128, "bf16", 128, 5, 1.0, 0.5,
                            block=128, n_sampled=512, n_probe=256, density=0.22,
                            ridge_lambda=1e-3, rank=32),
    "long": WorkloadConfig("long", (33, 45, 80), 24, 128, "bf16", 128, 5, 1.0, 0.5,
                           block=128, n_sampled=512, n_probe=256, density=0.22,
                           ridge_lambda=1e-3, rank=32),
    "broad": WorkloadConfig("broad", (13, 36, 70), 16, 128, "bf16", 32, 4, 0.3, 1.0,
                            block=128, n_sampled=512, n_probe=256, density=0.26,
                            ridge_lambda=1e-3, rank=32),
}


def token_grid_features(grid) -> np.ndarray:
    """[N, 24] sin/cos features of each token's (t, y, x) coordinate, raster order."""
    t_len, y_len, x_len = grid
    tt, yy, xx = np.meshgrid(np.arange(t_len), np.arange(y_len), np.arange(x_len),
                             indexing="ij")
    feats = []
    for coord, length in ((tt, t_len), (yy, y_len), (xx, x_len)):
        c = coord.reshape(-1).astype(np.float64)
        for f in range(4):
            ang = 2.0 * math.pi * (2.0 ** f) * c / length
            feats.append(np.sin(ang))
            feats.append(np.cos(ang))
    return np.stack(feats, axis=1)


def make_inputs(cfg: WorkloadConfig, seed: int = 0, heads: Optional[int] = None,
                dtype: Optional[torch.dtype] = None):
    """Draw Q, K, V for ``cfg`` as CPU torch tensors [batch, heads, N, d].

    ``heads`` < cfg.heads keeps only the first heads; because heads are drawn in
    order, those are identical to the first heads of the full draw.
    ``dtype`` overrides the config dtype (the cast is the last step).
    """
    rng = np.random.default_rng(seed)
    t_len, y_len, x_len = cfg.grid
    n, d = cfg.n_tokens, cfg.head_dim
    n_heads = cfg.heads if heads is None else heads
    out_dtype = cfg.torch_dtype if dtype is None else dtype
    pos = token_grid_features(cfg.grid)
    w_pos = rng.normal(0.0, math.sqrt(1.0 / 24.0), size=(24, d))
    pos_proj = pos @ w_pos
    py, px = -(-y_len // cfg.patch), -(-x_len // cfg.patch)
    yy, xx = np.meshgrid(np.arange(y_len), np.arange(x_len), indexing="ij")
    patch_of_pixel = ((yy // cfg.patch) * px + (xx // cfg.patch)).reshape(-1)
    patch_of_token = np.tile(patch_of_pixel, t_len)
    qs, ks, vs = [], [], []
    for _ in range(cfg.batch):
        means = rng.normal(0.0, cfg.sigma_c, size=(cfg.n_clusters, d))
        ids = rng.integers(0, cfg.n_clusters, size=(py, px)).reshape(-1)
        noise = rng.normal(0.0, cfg.sigma_n, size=(n, d))
        latent = pos_proj + means[ids[patch_of_token]] + noise
        qh, kh, vh = [], [], []
        for h in range(cfg.heads):
            wq = rng.normal(0.0, 1.0 / math.sqrt(d), size=(d, d))
            wk = rng.normal(0.0, 1.0 / math.sqrt(d), size=(d, d))
            wv = rng.normal(0.0, 1.0 / math.sqrt(d), size=(d, d))
            if h >= n_heads:
                continue
            qh.append(torch.from_numpy(latent @ wq).to(out_dtype))
            kh.append(torch.from_numpy(latent @ wk).to(out_dtype))
            vh.append(torch.from_numpy(latent @ wv).to(out_dtype))
        qs.append(torch.stack(qh))
        ks.append(torch.stack(kh))
        vs.append(torch.stack(vh))
    return torch.stack(qs), torch.stack(ks), torch.stack(vs)
