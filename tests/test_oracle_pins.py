"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed form, a
library routine, a brute-force restatement with different indexing, a hand-worked
fixture, or an invariant that a dropped term, a wrong sign or a transposed operand
would break.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import sparsepr_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _random_partition(rng, n, block):
    """Random labels with capacity `block` and every group non-empty."""
    g = O.n_groups(n, block)
    perm = rng.permutation(n)
    labels = np.empty(n, dtype=np.int64)
    labels[perm] = np.arange(n) // block   # contiguous chunks of a random order
    return labels, g


# ------------------------------------------------------------------ sparse attention

def test_density_full_sparse_equals_dense_for_any_partition():
    """At 100 % density every block routes every group, so the sparse output is
    dense attention, whatever the partition (spec pin)."""
    rng = _rng(1)
    n, d, block = 200, 16, 32
    q, k, v = (rng.normal(size=(n, d)) for _ in range(3))
    tau = 1 / math.sqrt(d)
    kl, g = _random_partition(rng, n, block)
    ql, _ = _random_partition(rng, n, block)
    routes = np.tile(np.arange(g), (g, 1))
    s = O.sparse_attention(q, k, v, tau, kl, ql, routes)
    dense = O.dense_attention_rows(q, k, v, tau, np.arange(n))
    assert np.max(np.abs(s - dense)) <= 1e-12 * np.max(np.abs(dense))


def test_density_full_whole_call_equals_dense():
    """Whole call at k = G: residuals vanish, the map is ~0 and O equals dense."""
    rng = _rng(2)
    n, d = 256, 16
    q, k, v = (rng.normal(size=(n, d)) for _ in range(3))
    out = O.sparsepr_head(q, k, v, block=32, n_sampled=32, n_probe=24, density=4.0,
                          ridge_lambda=1e-3, rank=4, kmeans_iters=2)
    assert out["k"] == O.n_groups(n, 32)
    dense = O.dense_attention_rows(q, k, v, out["tau"], np.arange(n))
    assert np.max(np.abs(out["O"] - dense)) <= 1e-10 * np.max(np.abs(dense))
    assert np.linalg.norm(out["fit"]["M"]) <= 1e-9
    assert np.linalg.norm(out["fit"]["beta"]) <= 1e-9


def test_sparse_matches_bruteforce_mask_64_tokens():
    """64 tokens: build the explicit N x N mask from the routes, masked softmax with
    -inf outside the support, times V: must equal the oracle's per-block gather."""
    rng = _rng(3)
    n, d, block, kk = 64, 8, 16, 2
    q, k, v = (rng.normal(size=(n, d)) for _ in range(3))
    tau = 0.7
    kl, g = _random_partition(rng, n, block)
    ql, _ = _random_partition(rng, n, block)
    routes = np.stack([np.sort(rng.choice(g, size=kk, replace=False)) for _ in range(g)])
    mask = np.zeros((n, n), dtype=bool)
    for i in range(n):
        for j in range(n):
            mask[i, j] = kl[j] in set(routes[ql[i]].tolist())
    logits = tau * q @ k.T
    logits[~mask] = -np.inf
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    ref = (p / p.sum(axis=1, keepdims=True)) @ v
    s = O.sparse_attention(q, k, v, tau, kl, ql, routes)
    assert np.max(np.abs(s - ref)) <= 1e-13


# -------------------------------------------------------------------- dense / probes

def test_dense_attention_matches_torch_sdpa():
    rng = _rng(4)
    n, d = 96, 32
    q, k, v = (rng.normal(size=(n, d)) for _ in range(3))
    tau = 1 / math.sqrt(d)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        scale=tau)[0].numpy()
    out = O.dense_attention_rows(q, k, v, tau, np.arange(n), chunk=40)
    assert np.max(np.abs(out - ref)) <= 1e-13


def test_dense_attention_closed_forms():
    """q = 0 gives uniform weights (the mean of V); one key scaled far above the rest
    gives that key's value row."""
    rng = _rng(5)
    n, d = 50, 8
    k, v = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    out = O.dense_attention_rows(np.zeros((1, d)), k, v, 1.0, np.array([0]))
    assert np.allclose(out[0], v.mean(axis=0), rtol=0, atol=1e-14)
    q = rng.normal(size=(1, d))
    k2 = k.copy()
    k2[17] = 1e3 * q[0] / np.linalg.norm(q[0])
    out = O.dense_attention_rows(q, k2, v, 1.0, np.array([0]))
    assert np.allclose(out[0], v[17], rtol=0, atol=1e-12)


def test_probe_rows_are_exact_copies():
    rng = _rng(6)
    n, d = 128, 8
    q, k, v = (rng.normal(size=(n, d)) for _ in range(3))
    out = O.sparsepr_head(q, k, v, block=32, n_sampled=16, n_probe=10, density=0.4,
                          ridge_lambda=1e-3, rank=3, kmeans_iters=1)
    exact = O.dense_attention_rows(q, k, v, out["tau"], out["probe_idx"])
    assert np.array_equal(out["O"][out["probe_idx"]], exact)


# --------------------------------------------------------------------------- the fit

def _gauss_jordan_solve(a, b):
    """Independent solver: Gauss-Jordan with partial pivoting in long double."""
    a = np.array(a, dtype=np.longdouble)
    b = np.array(b, dtype=np.longdouble)
    n = a.shape[0]
    aug = np.concatenate([a, b], axis=1)
    for col in range(n):
        piv = col + int(np.argmax(np.abs(aug[col:, col])))
        aug[[col, piv]] = aug[[piv, col]]
        aug[col] /= aug[col, col]
        for row in range(n):
            if row != col:
                aug[row] -= aug[row, col] * aug[col]
    return aug[:, n:]


@pytest.mark.parametrize("p,d,r,lam", [(40, 12, 3, 1e-3), (10, 12, 4, 1e-2), (64, 8, 8, 0.5)])
def test_ridge_matches_augmented_normal_equations(p, d, r, lam):
    """Centred Cholesky ridge == augmented normal equations
    ([X 1]^T W [X 1] + diag(lambda I, 0)) theta = [X 1]^T W Z, solved by Gauss-Jordan
    in long double and by numpy.linalg.solve (the bias is unpenalised)."""
    rng = _rng(7)
    x = rng.normal(size=(p, d)) + 0.3
    z = rng.normal(size=(p, r))
    w = rng.uniform(0.2, 2.0, size=p)
    a, b = O.ridge_affine(x, z, w, lam)
    xa = np.concatenate([x, np.ones((p, 1))], axis=1)
    lhs = xa.T @ (w[:, None] * xa)
    lhs[:d, :d] += lam * np.eye(d)
    rhs = xa.T @ (w[:, None] * z)
    theta = _gauss_jordan_solve(lhs, rhs).astype(np.float64)
    assert np.max(np.abs(a - theta[:d].T)) <= 1e-10 * max(1.0, np.max(np.abs(theta)))
    assert np.max(np.abs(b - theta[d])) <= 1e-10 * max(1.0, np.max(np.abs(theta)))
    theta2 = np.linalg.solve(lhs, rhs)
    assert np.max(np.abs(a - theta2[:d].T)) <= 1e-9 * max(1.0, np.max(np.abs(theta2)))


@pytest.mark.parametrize("p,d,r,lam", [(40, 12, 3, 1e-3), (10, 12, 4, 1e-2), (64, 8, 8, 0.5)])
def test_relative_ridge_matches_augmented_normal_equations(p, d, r, lam):
    """The scale-relative reading of lambda (ridge_mode "relative"): the same augmented
    normal equations with lambda_eff = lambda * (sum_p w_p |x_p - xbar|^2) / d, that sum
    (the trace of the centred weighted Gram) formed here row by row in long double."""
    rng = _rng(17)
    x = rng.normal(size=(p, d)) * 3.0 + 0.3
    z = rng.normal(size=(p, r))
    w = rng.uniform(0.2, 2.0, size=p)
    a, b = O.ridge_affine(x, z, w, lam, ridge_mode="relative")
    xl, wl = x.astype(np.longdouble), w.astype(np.longdouble)
    xbar = sum(wl[i] * xl[i] for i in range(p)) / sum(wl)
    spread = sum(wl[i] * sum((xl[i, e] - xbar[e]) ** 2 for e in range(d)) for i in range(p))
    lam_eff = float(lam * spread / d)
    xa = np.concatenate([x, np.ones((p, 1))], axis=1)
    lhs = xa.T @ (w[:, None] * xa)
    lhs[:d, :d] += lam_eff * np.eye(d)
    rhs = xa.T @ (w[:, None] * z)
    theta = _gauss_jordan_solve(lhs, rhs).astype(np.float64)
    assert np.max(np.abs(a - theta[:d].T)) <= 1e-10 * max(1.0, np.max(np.abs(theta)))
    assert np.max(np.abs(b - theta[d])) <= 1e-10 * max(1.0, np.max(np.abs(theta)))


def test_relative_ridge_makes_the_fit_scale_invariant():
    """Scaling the sparse and the dense probe outputs by s leaves M unchanged and scales
    beta by s under the relative lambda (weights, subspace and Gram all scale
    consistently); under the absolute lambda M moves (lambda does not scale)."""
    rng = _rng(18)
    p, d, r, lam, s = 20, 16, 4, 1e-2, 1e-2
    xs = rng.normal(size=(p, d))
    dp = xs + 0.3 * rng.normal(size=(p, d)) @ rng.normal(size=(d, d)) * 0.2 + 0.1
    f1 = O.fit_residual(xs, dp, lam, r, ridge_mode="relative")
    f2 = O.fit_residual(s * xs, s * dp, lam, r, ridge_mode="relative")
    assert np.max(np.abs(f2["M"] - f1["M"])) <= 1e-9 * np.max(np.abs(f1["M"]))
    assert np.max(np.abs(f2["beta"] - s * f1["beta"])) <= 1e-9 * np.max(np.abs(s * f1["beta"]))
    g1 = O.fit_residual(xs, dp, lam, r)
    g2 = O.fit_residual(s * xs, s * dp, lam, r)
    assert np.max(np.abs(g2["M"] - g1["M"])) > 1e-3 * np.max(np.abs(g1["M"]))


@pytest.mark.parametrize("d,rank_c,r", [(12, 12, 4), (24, 6, 8), (32, 32, 32)])
def test_jacobi_subspace_matches_eigh(d, rank_c, r):
    """Top-r projector and eigenvalues of the oracle's Jacobi match numpy.linalg.eigh
    (full-rank and rank-deficient second moments)."""
    rng = _rng(8)
    y = rng.normal(size=(rank_c, d)) * np.linspace(3, 0.2, d)
    c = y.T @ y
    evals, vecs = O.jacobi_eigh(c)
    ref_vals, ref_vecs = np.linalg.eigh(c)
    ref_vals, ref_vecs = ref_vals[::-1], ref_vecs[:, ::-1]
    assert np.max(np.abs(evals - ref_vals)) <= 1e-10 * ref_vals[0]
    assert np.max(np.abs(vecs.T @ vecs - np.eye(d))) <= 1e-12
    rr = min(r, rank_c)
    proj = vecs[:, :rr] @ vecs[:, :rr].T
    ref_proj = ref_vecs[:, :rr] @ ref_vecs[:, :rr].T
    assert np.max(np.abs(proj - ref_proj)) <= 1e-10


def _planted(rng, n_rows, d, r):
    x = rng.normal(size=(n_rows, d))
    u_star, _ = np.linalg.qr(rng.normal(size=(d, r)))
    a_star = rng.normal(size=(r, d)) * 0.3
    b_star = rng.normal(size=r)
    m_star, beta_star = u_star @ a_star, u_star @ b_star
    dense = x + x @ m_star.T + beta_star
    return x, dense, m_star, beta_star, a_star


def test_planted_affine_residual_is_recovered():
    """Residual exactly affine in the sparse output and inside an r-dim subspace:
    with P >= d+1 and a vanishing ridge, the fit recovers M*, beta* and the apply
    step reconstructs the unprobed rows (spec pin)."""
    rng = _rng(9)
    d, r, p, n_un = 16, 5, 40, 200
    x, dense, m_star, beta_star, _ = _planted(rng, p + n_un, d, r)
    fit = O.fit_residual(x[:p], dense[:p], 1e-12, r)
    assert np.linalg.norm(fit["M"] - m_star) <= 1e-8 * np.linalg.norm(m_star)
    assert np.linalg.norm(fit["beta"] - beta_star) <= 1e-8 * np.linalg.norm(beta_star)
    probe_idx = np.arange(p)
    out = O.apply_residual(x, fit["M"], fit["beta"], probe_idx, dense[:p])
    err = O.rel_l2_errors(out, dense, probe_idx)
    assert err["mean"] <= 1e-8


def test_planted_affine_ridge_shrinkage_bound():
    """With lambda > 0 the map shrinks by lambda A* (G + lambda I)^-1, bounded by
    lambda |A*| / sigma_min(X_c^T W X_c)."""
    rng = _rng(10)
    d, r, p = 16, 5, 48
    x, dense, m_star, _, a_star = _planted(rng, p, d, r)
    lam = 1e-3
    fit = O.fit_residual(x, dense, lam, r)
    w = O.probe_weights(dense)
    xc = x - (w @ x) / w.sum()
    gram = xc.T @ (w[:, None] * xc)
    bound = lam * np.linalg.norm(a_star) / np.linalg.eigvalsh(gram)[0]
    gap = np.linalg.norm(fit["M"] - m_star)
    assert gap <= bound
    assert gap > 0.01 * bound          # the ridge does act


def test_weights_make_objective_relative_error():
    """Default weights are 1/|d_p|^2 scaled to sum P."""
    d_probe = np.array([[3.0, 4.0], [0.0, 1.0], [1.0, 0.0]])
    w = O.probe_weights(d_probe)
    raw = np.array([1 / 25, 1.0, 1.0])
    assert np.allclose(w, raw * 3 / raw.sum(), rtol=1e-15)
    assert np.allclose(O.probe_weights(d_probe, "uniform"), 1.0)


# ------------------------------------------------------------------------ the metric

def test_metric_matches_bruteforce_loops_64_tokens():
    rng = _rng(11)
    n, d = 64, 8
    o, o_star = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    probe_idx = np.array([0, 5, 63, 20])
    errs = []
    for i in range(n):
        if i in set(probe_idx.tolist()):
            continue
        num = 0.0
        den = 0.0
        for e in range(d):
            num += (o[i, e] - o_star[i, e]) ** 2
            den += o_star[i, e] ** 2
        errs.append(math.sqrt(num) / math.sqrt(den))
    res = O.rel_l2_errors(o, o_star, probe_idx)
    assert res["errors"].size == n - probe_idx.size
    assert abs(res["mean"] - sum(errs) / len(errs)) <= 1e-14
    srt = sorted(errs)
    assert res["p99"] == pytest.approx(srt[math.ceil(0.99 * len(srt)) - 1], rel=1e-14)
    assert O.rel_l2_errors(o_star, o_star, probe_idx)["mean"] == 0.0


# ------------------------------------------------------------------- clustering: fill

def _fill_reference(dist, cap):
    """Independent restatement of the proposal rule with Python lists and sorted()."""
    n, g_count = len(dist), len(dist[0])
    room = [cap] * g_count
    label = [None] * n
    while any(lbl is None for lbl in label):
        proposals = {}
        for i in range(n):
            if label[i] is not None:
                continue
            best = None
            for g in range(g_count):
                if room[g] == 0:
                    continue
                if best is None or dist[i][g] < dist[i][best]:
                    best = g
            proposals.setdefault(best, []).append(i)
        for g, items in proposals.items():
            items.sort(key=lambda i: (float(dist[i][g]), i))
            for i in items[: room[g]]:
                label[i] = g
            room[g] -= min(room[g], len(items))
    return np.array(label)


def test_fill_hand_worked_fixture():
    fx = json.load(open(os.path.join(GOLDEN, "fill_hand_worked.json")))
    labels = O.fill(np.array(fx["D"], dtype=np.float32), fx["cap"])
    assert labels.tolist() == fx["labels"]


def test_fill_bruteforce_small_instances():
    """All tiny instances with few distinct values (many ties) vs the restatement."""
    rng = _rng(12)
    count = 0
    for n, g_count, cap in [(3, 2, 2), (4, 2, 2), (5, 3, 2), (6, 2, 3), (8, 3, 3), (7, 7, 1)]:
        for _ in range(150):
            dist = rng.integers(0, 3, size=(n, g_count)).astype(np.float32)
            assert O.fill(dist, cap).tolist() == _fill_reference(dist.tolist(), cap).tolist()
            count += 1
    assert count == 900


def test_fill_invariants_and_preferred_groups_full():
    rng = _rng(13)
    n, g_count, cap = 300, 12, 26
    dist = rng.normal(size=(n, g_count)).astype(np.float32) ** 2
    labels = O.fill(dist, cap)
    sizes = np.bincount(labels, minlength=g_count)
    assert sizes.max() <= cap and sizes.sum() == n and (labels >= 0).all()
    # every group an item prefers to its own was full when it was placed, so is full
    for i in range(n):
        own = dist[i, labels[i]]
        better = (dist[i] < own) | ((dist[i] == own) & (np.arange(g_count) < labels[i]))
        assert (sizes[better] == cap).all()


def test_fill_special_cases():
    n, cap = 40, 8
    g_count = 5
    # distance to chunk centres |(i + 1/2)/B - (g + 1/2)| -> contiguous chunks
    dist = np.abs((np.arange(n)[:, None] + 0.5) / cap
                  - (np.arange(g_count)[None, :] + 0.5)).astype(np.float32)
    assert (O.fill(dist, cap) == np.arange(n) // cap).all()
    # capacity never binding -> plain argmin with lower-index ties
    rng = _rng(14)
    dist = rng.integers(0, 4, size=(n, g_count)).astype(np.float32)
    assert (O.fill(dist, n) == np.argmin(dist, axis=1)).all()
    # -0.0 and +0.0 tie: lower group wins
    assert O.fill(np.array([[0.0, -0.0]], dtype=np.float32), 1).tolist() == [0]
    assert O.fill(np.array([[-0.0, 0.0]], dtype=np.float32), 1).tolist() == [0]
    with pytest.raises(O.NonFiniteError):
        O.fill(np.array([[np.nan, 1.0]], dtype=np.float32), 1)


def test_kmeans_zero_iterations_is_chunks_and_planted_clusters_recovered():
    rng = _rng(15)
    g_count, cap, dim = 6, 10, 5
    labels, _ = O.balanced_kmeans(rng.normal(size=(57, dim)), 6, cap, 0)
    assert (labels == np.arange(57) // cap).all()
    centers = rng.normal(size=(g_count, dim)) * 20
    truth = np.repeat(np.arange(g_count), cap)
    order = rng.permutation(g_count * cap)
    x = centers[truth[order]] + 0.1 * rng.normal(size=(g_count * cap, dim))
    labels, _ = O.balanced_kmeans(x, g_count, cap, 4)
    # same partition up to renaming of the groups
    pairs = set(zip(labels.tolist(), truth[order].tolist()))
    assert len(pairs) == g_count
    assert np.bincount(labels).tolist() == [cap] * g_count


def test_profile_distances_equal_head_dim_metric_form():
    """|r_j - c_g|^2 in response space equals tau^2 (k_j - kappa_g)^T (Q_S^T Q_S)
    (k_j - kappa_g) with kappa_g the group's mean key: the response-space centroid is
    tau Q_S kappa_g because responses are linear in the key."""
    rng = _rng(16)
    n, d, s_count, cap = 90, 6, 11, 15
    q, k = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    tau = 0.4
    sidx = O.midpoint_stride(n, s_count)
    prof = O.key_response_profiles(q, k, sidx, tau)
    assert prof.shape == (n, s_count)
    assert prof[7, 3] == pytest.approx(tau * float(q[sidx[3]] @ k[7]), rel=1e-14)
    labels, g = _random_partition(rng, n, cap)
    cent_prof = O.group_means(prof, labels, g)
    kappa = O.group_means(k, labels, g)
    assert np.allclose(cent_prof, tau * kappa @ q[sidx].T, rtol=0, atol=1e-12)
    gamma = q[sidx].T @ q[sidx]
    dist = O.squared_distances(prof, cent_prof)
    for i in (0, 44, 89):
        for gg in range(g):
            diff = k[i] - kappa[gg]
            assert dist[i, gg] == pytest.approx(tau * tau * diff @ gamma @ diff, rel=1e-10)


# --------------------------------------------------------------------------- routing

def test_route_hand_worked_fixture():
    fx = json.load(open(os.path.join(GOLDEN, "route_hand_worked.json")))
    routes = O.route(np.array(fx["Sc"], dtype=np.float32), fx["k"])
    assert routes.tolist() == fx["route"]
    pairs = O.executed_pairs(routes, np.array(fx["key_sizes"]), np.array(fx["block_sizes"]),
                             fx["n_probe"], fx["n_tokens"])
    assert pairs == fx["executed_pairs"]


def test_route_invariants_and_pair_recount():
    rng = _rng(17)
    n, block, probes, rho = 500, 32, 7, 0.3
    g = O.n_groups(n, block)
    kk = O.route_k(n, block, rho, probes)
    assert kk * n * block + probes * n <= rho * n * n < (kk + 1) * n * block + probes * n
    sc = rng.integers(-3, 3, size=(g, g)).astype(np.float32)   # many ties
    routes = O.route(sc, kk)
    for b in range(g):
        rset = set(routes[b].tolist())
        assert len(rset) == kk and list(routes[b]) == sorted(rset)
        inside = [(float(sc[b, x]), -x) for x in rset]
        outside = [(float(sc[b, x]), -x) for x in range(g) if x not in rset]
        assert min(inside) > max(outside)
    kl, _ = _random_partition(rng, n, block)
    ql, _ = _random_partition(rng, n, block)
    ks, bs = np.bincount(kl, minlength=g), np.bincount(ql, minlength=g)
    recount = 0
    for i in range(n):
        allowed = set(routes[ql[i]].tolist())
        recount += sum(1 for j in range(n) if kl[j] in allowed)
    pairs = O.executed_pairs(routes, ks, bs, probes, n)
    assert pairs == recount + probes * n
    assert pairs / n ** 2 <= rho


def test_route_k_matches_config_table():
    """k for the five workloads from the budget inequality (probes counted)."""
    assert O.route_k(1024, 64, 0.25, 32) == 3
    assert O.route_k(8192, 128, 0.22, 64) == 13
    assert O.route_k(75600, 128, 0.22, 256) == 127
    assert O.route_k(118800, 128, 0.22, 256) == 202
    assert [O.route_k(32760, 128, 0.26, p) for p in (32, 64, 128, 256, 512)] == [66, 66, 65, 64, 62]
    assert O.route_k(100, 10, 0.0, 5) == 1          # clamp low
    assert O.route_k(100, 10, 9.0, 5) == 10         # clamp high


def test_midpoint_stride():
    assert O.midpoint_stride(10, 5).tolist() == [1, 3, 5, 7, 9]
    assert O.midpoint_stride(7, 1).tolist() == [3]
    idx = O.midpoint_stride(75600, 256)
    assert len(set(idx.tolist())) == 256 and idx.min() >= 0 and idx.max() < 75600


def test_labels_to_perm_layout():
    labels = np.array([2, 0, 2, 1, 0, 2])
    perm, sizes = O.labels_to_perm(labels, 3, 4)
    assert perm.tolist() == [1, 4, -1, -1, 3, -1, -1, -1, 0, 2, 5, -1]
    assert sizes.tolist() == [2, 1, 3]


def test_partition_and_route_follow_planted_attention():
    """Keys in G tight clusters along orthogonal directions; each query points at one
    cluster.  Response-coupled partitioning must recover the key clusters, group the
    queries by target, and k = 1 routing must send every block to its target group,
    so the sparse output is almost the dense one (a sign or operand slip in the query
    coordinates or the block scores routes to the wrong group and fails)."""
    rng = _rng(18)
    g_count, block, d = 6, 16, 12
    n = g_count * block
    dirs = np.linalg.qr(rng.normal(size=(d, d)))[0][:, :g_count].T * 4.0
    key_cluster = rng.permutation(np.repeat(np.arange(g_count), block))
    query_target = rng.permutation(np.repeat(np.arange(g_count), block))
    k = dirs[key_cluster] + 0.05 * rng.normal(size=(n, d))
    q = 3.0 * dirs[query_target] + 0.05 * rng.normal(size=(n, d))
    v = rng.normal(size=(n, d))
    tau = 1.0 / math.sqrt(d)
    part = O.partition(q, k, tau, block, n_sampled=48, iters=3)
    assert len(set(zip(part["key_labels"].tolist(), key_cluster.tolist()))) == g_count
    assert len(set(zip(part["query_labels"].tolist(), query_target.tolist()))) == g_count
    routes = O.route(part["block_scores"], 1)
    for b in range(g_count):
        members = np.flatnonzero(part["query_labels"] == b)
        target_keys = np.flatnonzero(key_cluster == query_target[members[0]])
        assert set(part["key_labels"][target_keys].tolist()) == {routes[b, 0]}
    s = O.sparse_attention(q, k, v, tau, part["key_labels"], part["query_labels"], routes)
    dense = O.dense_attention_rows(q, k, v, tau, np.arange(n))
    assert O.rel_l2_errors(s, dense, np.array([], dtype=np.int64))["mean"] < 1e-3


# ------------------------------------------------------------ semantic baseline partition

def test_semantic_keys_equal_response_keys_when_sampled_queries_are_a_scaled_basis():
    """With tau = 1/2 and the d sampled queries equal to 2 e_m, every key's response
    profile is the key itself, bit for bit, so Response-Coupled Partitioning and the
    semantic partition (k-means on raw keys) must give identical key labels and mean
    keys; the query sides still differ in general (coordinates u vs raw q)."""
    rng = _rng(31)
    n, d, block = 96, 8, 16
    q, k = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    sidx = O.midpoint_stride(n, d)
    q[sidx] = 2.0 * np.eye(d)
    tau = 0.5
    assert np.array_equal(O.key_response_profiles(q, k, sidx, tau), k)
    resp = O.partition(q, k, tau, block, n_sampled=d, iters=3)
    sem = O.partition_semantic(q, k, tau, block, iters=3)
    assert np.array_equal(resp["key_labels"], sem["key_labels"])
    assert np.array_equal(resp["mu"], sem["mu"])


def test_semantic_partition_recovers_planted_raw_clusters():
    """Keys and queries in tight clusters of their own (in raw space): the semantic
    partition must recover both clusterings, whatever the queries attend to."""
    rng = _rng(32)
    g_count, block, d = 5, 12, 10
    n = g_count * block
    kc = rng.normal(size=(g_count, d)) * 8
    qc = rng.normal(size=(g_count, d)) * 8
    key_truth = rng.permutation(np.repeat(np.arange(g_count), block))
    query_truth = rng.permutation(np.repeat(np.arange(g_count), block))
    k = kc[key_truth] + 0.1 * rng.normal(size=(n, d))
    q = qc[query_truth] + 0.1 * rng.normal(size=(n, d))
    sem = O.partition_semantic(q, k, 1 / math.sqrt(d), block, iters=3)
    assert len(set(zip(sem["key_labels"].tolist(), key_truth.tolist()))) == g_count
    assert len(set(zip(sem["query_labels"].tolist(), query_truth.tolist()))) == g_count
    assert np.bincount(sem["query_labels"]).tolist() == [block] * g_count



# --------------------------------------------------------------- routing score readings

def test_routing_scores_bruteforce_and_jensen_bound():
    """Each score reading against explicit loops over members; LSE >= size-corrected
    everywhere (Jensen: log sum exp >= log n + mean), with equality for a group whose
    keys are all equal; "centroid" equals the partition's block scores."""
    rng = _rng(41)
    n, d, block = 80, 6, 16
    q, k = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    tau = 0.7
    part = O.partition(q, k, tau, block, n_sampled=20, iters=2)
    kl, ql = part["key_labels"], part["query_labels"]
    g = O.n_groups(n, block)
    k2 = k.copy()
    k2[kl == 2] = k2[kl == 2][0]      # group 2: identical keys
    cen = O.routing_scores(q, k, tau, kl, ql, g, "centroid")
    assert np.array_equal(cen, part["block_scores"])
    siz = O.routing_scores(q, k, tau, kl, ql, g, "size_corrected")
    lse = O.routing_scores(q, k, tau, kl, ql, g, "lse")
    for b in range(g):
        qb = q[ql == b].mean(axis=0)
        for gg in range(g):
            members = np.flatnonzero(kl == gg)
            logits = [tau * float(qb @ k[j]) for j in members]
            mu = k[members].mean(axis=0)
            assert siz[b, gg] == pytest.approx(tau * float(qb @ mu) + math.log(len(members)), rel=1e-6, abs=1e-6)
            assert lse[b, gg] == pytest.approx(math.log(sum(math.exp(x) for x in logits)), rel=1e-6, abs=1e-6)
    assert (lse >= siz - 1e-5).all()
    lse2 = O.routing_scores(q, k2, tau, kl, ql, g, "lse")
    siz2 = O.routing_scores(q, k2, tau, kl, ql, g, "size_corrected")
    assert np.allclose(lse2[:, 2], siz2[:, 2], rtol=1e-6, atol=1e-5)


def test_route_global_hand_worked_fixture():
    fx = json.load(open(os.path.join(GOLDEN, "route_global_hand_worked.json")))
    sc = np.array(fx["Sc"], dtype=np.float32)
    ks, bs = np.array(fx["key_sizes"]), np.array(fx["block_sizes"])
    for case in fx["cases"]:
        routes = O.route_global(sc, ks, bs, fx["n_tokens"], fx["n_probe"], case["density"])
        assert [r.tolist() for r in routes] == case["routes"]
        pairs = sum(int(bs[b]) * int(ks[routes[b]].sum()) for b in range(len(routes)))
        assert pairs == case["executed_pairs"]


def test_route_global_invariants():
    """Every block keeps its best group; the pairs stay within the budget (unless the
    kept best groups alone exceed it); the taken pairs precede every left-out pair in
    (descending score, block, group) order; and the first left-out pair would not fit."""
    rng = _rng(23)
    for trial in range(20):
        gq, g = int(rng.integers(2, 9)), int(rng.integers(2, 9))
        sc = rng.integers(-3, 4, size=(gq, g)).astype(np.float32)   # many ties
        ks, bs = rng.integers(0, 6, size=g), rng.integers(1, 6, size=gq)
        n, probes, rho = int(bs.sum()), int(rng.integers(0, 3)), float(rng.uniform(0.05, 1.2))
        routes = O.route_global(sc, ks, bs, n, probes, rho)
        budget = math.floor(rho * n * n - float(probes * n))
        best = [int(np.lexsort((np.arange(g), -sc[b]))[0]) for b in range(gq)]
        spent = sum(int(bs[b]) * int(ks[routes[b]].sum()) for b in range(gq))
        kept = sum(int(bs[b]) * int(ks[best[b]]) for b in range(gq))
        assert all(best[b] in routes[b].tolist() for b in range(gq))
        assert spent <= max(budget, kept)
        key = lambda b, gg: (-float(sc[b, gg]), b, gg)
        taken = [(b, int(x)) for b in range(gq) for x in routes[b] if int(x) != best[b]]
        left = [(b, x) for b in range(gq) for x in range(g) if x not in routes[b].tolist()]
        if taken and left:
            assert max(key(*t) for t in taken) < min(key(*e) for e in left)
        if left:
            first = min(left, key=lambda e: key(*e))
            assert spent + int(bs[first[0]]) * int(ks[first[1]]) > budget


def test_route_global_single_block_is_uniform_topk():
    """One block and equal group sizes: the global allocation takes the floor(budget /
    (n_b B)) best groups, the uniform top-k route with that k."""
    rng = _rng(29)
    for trial in range(10):
        g, nb, blk = int(rng.integers(3, 12)), int(rng.integers(2, 6)), int(rng.integers(2, 6))
        sc = rng.integers(-2, 3, size=(1, g)).astype(np.float32)
        ks, bs = np.full(g, blk), np.array([nb])
        n, rho = 10, float(rng.uniform(0.01, 2.0))
        budget = math.floor(rho * n * n)
        kk = min(g, max(1, budget // (nb * blk)))
        got = O.route_global(sc, ks, bs, n, 0, rho)
        assert got[0].tolist() == O.route(sc, kk)[0].tolist()
