"""Element-wise parity of Response-Coupled Partitioning's continuous arithmetic.

The method groups keys "by how their keys respond to sampled queries" and queries "by
their responses to the resulting key-group centroids" (SparsePR abstract).  The GPU runs
both clusterings in the head-dim form tau^2 (x - c)^T Gamma (x - c) on tensor cores; this
file checks every quantity that feeds a decision against the fp64 oracle, each time on
the inputs the GPU itself used (its previous iteration's labels are injected, so every
iteration is compared on identical inputs):

* S1: the sampled query indices, bit-exact against ``midpoint_stride``;
* the metrics Gamma (Q_S^T Q_S for keys, mu^T mu for queries);
* S2/S4: every iteration's distance matrix against ``squared_distances`` of the
  response profiles (keys) or the query coordinates u_i = tau q_i mu^T (queries), within
  a bound derived from the bf16 hi + lo split (below);
* every iteration's labels: the production fill of the GPU's own distances, bit-exact
  against ``fill`` of the same fp32 matrix;
* S3: the key-group means mu and the query-block means qbar against ``group_means``;
* S5: the centroid block scores against ``routing_scores(..., "centroid")``.

Distance bound.  The GPU forms D = tau^2 (x.Gamma.x + c.Gamma.c - 2 x.w) with w = Gamma c
carried as bf16 hi + lo (residual <= 2^-17 |w| per element), products accumulated in
fp32.  The cross term's error is therefore <= 2 (2^-17 + d 2^-24) sum_e |x_e||w_e| and the
norms' and the final sum's rounding a few fp32 ulps of x.Gamma.x + c.Gamma.c, so
|D_gpu - D| <= REL_D tau^2 (x.Gamma.x + c.Gamma.c + 2 sum_e |x_e||w_e|) with
REL_D = 2^-13 (8x the split residual, covering the fp32 Gamma, centroids and w).
"""
import math

import numpy as np
import pytest
import torch

import free_block_sparse_response_b200 as spr
from oracle import sparsepr_oracle as O
from synthetic import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu

REL_D = 2.0 ** -13     # distances, relative to the bound above
TOL_GAMMA = 1e-5       # metrics, relative Frobenius (fp32 sums of <= 591 products)
TOL_MEAN = 1e-5        # group means, relative Frobenius per head (fp32 sums of <= 128 rows)
REL_SC = 1e-5          # block scores, relative to tau sum_e |qbar_e| |mu_e|


@pytest.fixture(scope="module", autouse=True)
def _built():
    from free_block_sparse_response_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    spr.lib()


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _cfg(w, **kw):
    base = dict(block=w.block, n_sampled=w.n_sampled, n_probe=w.n_probe, kmeans_iters=w.kmeans_iters,
                rank=w.rank, density=w.density, ridge_lambda=w.ridge_lambda)
    base.update(kw)
    return spr.SparsePRConfig(**base)


def _dist_bound(x_d, gamma, cent_d, tau):
    """tau^2 (x.Gamma.x + c.Gamma.c + 2 sum_e |x_e||(Gamma c)_e|) for every (row, group)."""
    a = np.einsum("ie,ef,if->i", x_d, gamma, x_d)
    w = cent_d @ gamma
    c = np.einsum("ge,ge->g", w, cent_d)
    return tau * tau * (a[:, None] + c[None, :] + 2.0 * (np.abs(x_d) @ np.abs(w).T))


def _side(name, x_resp, x_d, gamma, tau, dist, labels_gpu, g_count, block, rows, check_fill):
    """One clustering side, iteration by iteration, on the GPU's own previous labels.
    x_resp: the items in the space the oracle clusters (profiles or coordinates);
    x_d: the same items in head dim (for the error bound); dist(t, rows) the GPU's
    fp32 distances of iteration t on those rows (rows None: the whole matrix).
    Returns the largest distance error as a fraction of its bound."""
    n = x_resp.shape[0]
    labels = O.chunk_labels(n, block)
    cent = O.group_means(x_resp, labels, g_count)
    worst = 0.0
    for t in range(labels_gpu.shape[0]):
        cent_d = O.group_means(x_d, labels, g_count)
        d_ref = O.squared_distances(x_resp[rows], cent)
        bound = _dist_bound(x_d[rows], gamma, cent_d, tau)
        err = np.abs(dist(t, rows).astype(np.float64) - d_ref)
        ratio = float(np.max(err / bound))
        worst = max(worst, ratio)
        assert ratio <= REL_D, f"{name} iteration {t}: distance error {ratio:.3g} of the bound"
        new_labels = labels_gpu[t].astype(np.int64)
        if check_fill(t):
            assert np.array_equal(new_labels, O.fill(dist(t, None), block)), f"{name} iteration {t}: fill"
        labels = new_labels
        cent = O.group_means(x_resp, labels, g_count, previous=cent)
    return worst


def _dist_accessor(trace_dist, h):
    """dist(t, rows) over the traced [T, HH, N, G] device tensor of head h."""
    def dist(t, rows):
        m = trace_dist[t, h]
        return (m if rows is None else m[torch.from_numpy(np.asarray(rows)).cuda()]).cpu().numpy()
    return dist


def _check_partition(w, heads, rows_per_head=None, fill_iters=None, mode=spr.PARTITION_RESPONSE):
    """Trace a partition call and compare it with the oracle head by head."""
    q, k, _ = make_inputs(w, 0, heads=heads)
    cfg = _cfg(w, partition_mode=mode)
    part, tr = spr.test_partition_trace(q.cuda(), k.cuda(), cfg)
    n, d, B, S = w.n_tokens, w.head_dim, w.block, w.n_sampled
    g_count = spr.num_groups(n, B)
    tau = 1.0 / math.sqrt(d)
    semantic = mode == spr.PARTITION_SEMANTIC
    if not semantic:
        assert np.array_equal(tr["sample_idx"].cpu().numpy(), O.midpoint_stride(n, S))
    rng = np.random.default_rng(3)
    report = {}
    for h in range(heads):
        qh, kh = (t[0, h].double().numpy() for t in (q, k))
        rows = np.arange(n) if rows_per_head is None else np.sort(rng.choice(n, rows_per_head, replace=False))
        check_fill = (lambda t: True) if fill_iters is None else (lambda t: h == 0 and t in fill_iters)
        # ---- keys: profiles r_j = tau Q_S k_j (semantic: the raw keys)
        if semantic:
            gamma_k, k_resp, tau_k = np.eye(d), kh, 1.0
        else:
            sidx = O.midpoint_stride(n, S)
            qs = qh[sidx]
            gamma_k, k_resp, tau_k = qs.T @ qs, O.key_response_profiles(qh, kh, sidx, tau), tau
        assert _rel(tr["key_gamma"][h].cpu().numpy(), gamma_k) <= TOL_GAMMA
        key_labels = tr["key_labels"][:, h].cpu().numpy()
        worst_k = _side("keys", k_resp, kh, gamma_k, tau_k, _dist_accessor(tr["key_dist"], h), key_labels,
                        g_count, B, rows, check_fill)
        kl = key_labels[-1].astype(np.int64)
        mu = O.group_means(kh, kl, g_count)
        assert _rel(tr["mu"][h].cpu().numpy(), mu) <= TOL_MEAN
        # ---- queries: coordinates u_i = tau q_i mu^T (semantic: the raw queries)
        if semantic:
            gamma_q, q_resp, tau_q = np.eye(d), qh, 1.0
        else:
            gamma_q, q_resp, tau_q = mu.T @ mu, tau * (qh @ mu.T), tau
        assert _rel(tr["query_gamma"][h].cpu().numpy(), gamma_q) <= TOL_GAMMA
        query_labels = tr["query_labels"][:, h].cpu().numpy()
        worst_q = _side("queries", q_resp, qh, gamma_q, tau_q, _dist_accessor(tr["query_dist"], h), query_labels,
                        g_count, B, rows, check_fill)
        ql = query_labels[-1].astype(np.int64)
        qbar = O.group_means(qh, ql, g_count)
        assert _rel(tr["qbar"][h].cpu().numpy(), qbar) <= TOL_MEAN
        # ---- S5: centroid block scores on the GPU's final labels
        sc_ref = O.routing_scores(qh, kh, tau, kl, ql, g_count, "centroid").astype(np.float64)
        sc_gpu = part.block_scores[0, h].cpu().numpy().astype(np.float64)
        sc_bound = tau * (np.abs(qbar) @ np.abs(mu).T)
        assert np.max(np.abs(sc_gpu - sc_ref) / sc_bound) <= REL_SC
        # the call's outputs are the traced final labels
        assert np.array_equal(_perm_labels(part.key_perm[0, h], part.key_gsize[0, h], n, B), kl)
        assert np.array_equal(_perm_labels(part.query_perm[0, h], part.qblock_size[0, h], n, B), ql)
        report[h] = (f"{worst_k:.3g}", f"{worst_q:.3g}")
    print(f"{w.name}: largest distance error / bound per head (keys, queries): {report}")
    return report


def _perm_labels(perm, sizes, n, block):
    perm, sizes = perm.cpu().numpy(), sizes.cpu().numpy()
    labels = np.full(n, -1, dtype=np.int64)
    for g in range(sizes.size):
        labels[perm[g * block: g * block + sizes[g]]] = g
    return labels


def test_partition_trace_tiny_fp32():
    """fp32 SIMT path (d = 64, B = 64): every iteration of both sides, both heads."""
    _check_partition(CONFIGS["tiny"], heads=2)


def test_partition_trace_small_bf16():
    """bf16 tensor-core path (d = 128, B = 128, G = 64): all rows, all iterations."""
    _check_partition(CONFIGS["small"], heads=2)


def test_partition_trace_ragged():
    """N = 1035 (last group of 11 tokens), bf16 d = 128."""
    w = CONFIGS["small"].with_(grid=(5, 9, 23), heads=2, n_sampled=128)
    _check_partition(w, heads=2)


def test_partition_trace_bf16_d64_block64():
    """bf16 d = 64, B = 64 (the mma.sync row-GEMM path), ragged N = 990."""
    w = CONFIGS["tiny"].with_(grid=(3, 15, 22), dtype="bf16")
    _check_partition(w, heads=2)


def test_partition_trace_semantic_small():
    """The semantic baseline's raw-space distances (identity metric, no tau)."""
    _check_partition(CONFIGS["small"], heads=2, mode=spr.PARTITION_SEMANTIC)


def test_partition_trace_video_two_heads():
    """75,600 tokens, G = 591: 1,024 sampled rows of every distance matrix of two heads;
    the fill of head 0's first key and first query iteration on the full matrices."""
    _check_partition(CONFIGS["video"], heads=2, rows_per_head=1024, fill_iters=(0,))
