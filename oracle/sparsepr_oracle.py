"""Plain fp64 CPU oracle of one SparsePR attention call.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` may import or run this module.  The CUDA
library never calls it, and it shares no code with the CUDA path.

Sources (all prose; the pages print no equations, listings or worked examples):

* [abs]   SparsePR paper abstract, English text on the arxivdaily.com page for
          arXiv 2608.18484 (the most detailed description of the method).
* [abs-d] the same abstract as reprinted on the peercurrent.com digest page.
* [news]  "Partition the Support, Reconstruct the Residual: Training-Free Sparse
          Attention for Video Generation and World Models", skillfed.io article;
          its paragraph on the method's two components adds that the partition is
          one asymmetric pass and that the correction is confined to the output
          subspace seen in the probe residuals.

Everything is per (batch, head): inputs are 2-D float64 arrays [N, d] that hold the
values both sides read (bf16 or fp32 inputs, upcast).  Steps follow the method in
the order the pages give it:

  1. sample queries; key response profiles r_j[m] = tau * q_{s_m} . k_j   [abs]
  2. balanced k-means of the profiles into G = ceil(N/B) key groups, capacity B,
     K and V move together ("paired K/V groups")                          [abs, abs-d]
  3. key-group centroids mu_g give query coordinates u_i[g] = tau q_i . mu_g [abs-d, news]
  4. balanced k-means of the query coordinates into Gq = ceil(N/B) blocks  [abs]
  5. each query block keeps the k key groups with the largest centroid score,
     k set by the executed-pair density budget with probe rows counted      [abs, news]
  6. softmax attention restricted to the routed groups                       [abs]
     (the semantic baseline partition of the comparisons replaces steps 1-4 by
     balanced k-means on raw K and raw Q: ``partition_semantic``)
  7. exact dense attention for P probe rows                                  [abs, news]
  8. weighted ridge fit of an affine map sparse output -> residual inside the
     top-r subspace of the probe residuals                                   [abs, news]
  9. add the predicted residual to every unprobed row; probe rows are exact   [abs]
 10. metric: per-row relative L2 error against dense, mean over unprobed rows [abs];
     the p99 tail is reported too                                            [news]

Readings taken where the pages are silent:

* sample and probe rows: midpoint stride floor((2m+1) N / (2 count)) in raster order;
* response = scaled logit tau q.k (a per-query shift would not change k-means);
* balanced k-means: init = means of contiguous chunks of B tokens, T Lloyd
  iterations, each assignment is the capacity-B proposal rule ``fill`` below,
  distances computed in fp64 and rounded to fp32 before the decision;
* k = clamp(floor((rho N^2 - P N) / (N B)), 1, G) for every block; route = k largest
  block scores, ties to the lower group index, stored in ascending group order;
* block score = mean over the block's members of u_i[g];
* weights w_p = 1 / max(|d_p|^2, 1e-30) normalised to sum P, so the weighted
  least-squares objective is the summed squared relative error on the probes;
* subspace = top-r eigenvectors of the uncentred weighted residual second moment;
* ridge: lambda * I added to the centred weighted Gram, bias unpenalised;
* the other split of the pair budget (``route_global``): every block keeps its best
  group, the other (block, group) pairs follow in descending score (ties to the lower
  block, then group) while the cumulative n_b n_g fits the head's budget.

Parity pins live in tests/test_oracle_pins.py (density-100% identity, brute-force
masked attention, library dense attention, normal-equation ridge, eigh projectors,
planted affine residual, brute-force metric, fill invariants and brute force,
planted clusters, route invariants, the global allocation's hand-worked fixture,
invariants and single-block reduction).  The absolute error level at 22 % density on
synthetic inputs has no pin on the pages: parity unpinned for that number.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np


class NonFiniteError(ValueError):
    """A NaN reached a decision (fill or route); the call rejects it."""


# ----------------------------------------------------------------------------- counts

def n_groups(n: int, block: int) -> int:
    """G = Gq = ceil(N / B): groups of capacity B cover all N tokens (reading)."""
    return -(-n // block)


def midpoint_stride(n: int, count: int) -> np.ndarray:
    """Indices floor((2m+1) n / (2 count)), m < count (reading of 'sampled queries')."""
    if count < 1 or count > n:
        raise ValueError(f"need 1 <= count <= n, got count={count} n={n}")
    m = np.arange(count, dtype=np.int64)
    return ((2 * m + 1) * n) // (2 * count)


def route_k(n: int, block: int, density: float, n_probe: int) -> int:
    """Uniform number of routed key groups per query block.

    The executed-pair budget counts probe rows ([abs]: the density includes the
    exact probes): k*N*B + P*N <= rho*N^2, so k = floor((rho N^2 - P N) / (N B)),
    clamped to [1, G].  Evaluated in IEEE double in this exact order.
    """
    g = n_groups(n, block)
    num = density * n * n - float(n_probe * n)
    k = math.floor(num / float(n * block))
    return int(min(max(k, 1), g))


# ------------------------------------------------------------------ step 1: profiles

def key_response_profiles(q: np.ndarray, k: np.ndarray, sample_idx: np.ndarray,
                          tau: float) -> np.ndarray:
    """[N, S] profile of every key: its scaled logit against each sampled query.

    [abs]: keys are grouped by how they respond to sampled queries.
    """
    return tau * (k @ q[sample_idx].T)


# ------------------------------------------------------------- step 2/4: clustering

def fill(dist: np.ndarray, cap: int) -> np.ndarray:
    """Capacity-constrained assignment of n items to G groups (capacity ``cap``).

    Rounds until every item is placed: every unplaced item proposes to its nearest
    group that still has room (ties -> lowest group index); every group takes its
    proposers in ascending (distance, item index) order while it has room.  Values
    are compared as float32 with plain '<'.  Accepted items never move again.
    """
    dist = np.asarray(dist, dtype=np.float32)
    n, g_count = dist.shape
    if np.isnan(dist).any():
        raise NonFiniteError("NaN distance")
    if g_count * cap < n:
        raise ValueError("groups * capacity < items")
    room = np.full(g_count, cap, dtype=np.int64)
    labels = np.full(n, -1, dtype=np.int64)
    while True:
        unplaced = np.flatnonzero(labels < 0)
        if unplaced.size == 0:
            return labels
        open_groups = np.flatnonzero(room > 0)
        choice = open_groups[np.argmin(dist[np.ix_(unplaced, open_groups)], axis=1)]
        for g in np.unique(choice):
            proposers = unplaced[choice == g]
            order = np.lexsort((proposers, dist[proposers, g]))
            taken = proposers[order[: room[g]]]
            labels[taken] = g
            room[g] -= taken.size


def chunk_labels(n: int, cap: int) -> np.ndarray:
    """Contiguous chunks of ``cap`` items in token order (the k-means start)."""
    return np.arange(n, dtype=np.int64) // cap


def group_means(x: np.ndarray, labels: np.ndarray, g_count: int,
                previous: Optional[np.ndarray] = None) -> np.ndarray:
    """fp64 mean of each group's members; an empty group keeps ``previous``."""
    out = np.zeros((g_count, x.shape[1])) if previous is None else previous.copy()
    for g in range(g_count):
        members = x[labels == g]
        if members.shape[0]:
            out[g] = members.mean(axis=0)
    return out


def squared_distances(x: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """D[i][g] = sum_e (x_i[e] - c_g[e])^2 in fp64, straight from the definition."""
    d = np.empty((x.shape[0], centroids.shape[0]))
    for g in range(centroids.shape[0]):
        diff = x - centroids[g]
        d[:, g] = np.einsum("ie,ie->i", diff, diff)
    return d


def balanced_kmeans(x: np.ndarray, g_count: int, cap: int, iters: int,
                    dump: Optional[list] = None):
    """Balanced k-means: chunk-mean start, then ``iters`` rounds of (distances,
    ``fill``, member means).  Returns (labels, centroids).  ``dump`` collects every
    float32 distance matrix handed to ``fill``."""
    n = x.shape[0]
    labels = chunk_labels(n, cap)
    cent = group_means(x, labels, g_count)
    for _ in range(iters):
        d32 = squared_distances(x, cent).astype(np.float32)
        if dump is not None:
            dump.append(d32)
        labels = fill(d32, cap)
        cent = group_means(x, labels, g_count, previous=cent)
    return labels, cent


def labels_to_perm(labels: np.ndarray, g_count: int, cap: int):
    """perm[g*cap + j] = j-th member of group g in token order (-1 pads), sizes[g]."""
    perm = np.full(g_count * cap, -1, dtype=np.int64)
    sizes = np.zeros(g_count, dtype=np.int64)
    for g in range(g_count):
        members = np.flatnonzero(labels == g)
        if members.size > cap:
            raise ValueError("group over capacity")
        perm[g * cap: g * cap + members.size] = members
        sizes[g] = members.size
    return perm, sizes


def partition(q: np.ndarray, k: np.ndarray, tau: float, block: int, n_sampled: int,
              iters: int, sample_idx: Optional[np.ndarray] = None,
              dump: Optional[dict] = None) -> dict:
    """Response-Coupled Partitioning, one asymmetric pass ([abs], [news]).

    Keys are clustered by their response profiles; the key-group mean keys mu_g
    give every query the coordinates u_i[g] = tau q_i . mu_g (the response-space
    centroid of group g is tau Q_S mu_g, linear in the key); queries are then
    clustered in those coordinates.  Keys are never re-clustered afterwards.
    Returns key/query labels, mu, the coordinates and the block scores (fp32; the
    "centroid" reading of ``routing_scores``).
    """
    n = q.shape[0]
    g_count = n_groups(n, block)
    s_idx = midpoint_stride(n, n_sampled) if sample_idx is None else np.asarray(sample_idx)
    prof = key_response_profiles(q, k, s_idx, tau)
    kd = [] if dump is not None else None
    key_labels, _ = balanced_kmeans(prof, g_count, block, iters, kd)
    mu = group_means(k, key_labels, g_count)
    coords = tau * (q @ mu.T)
    qd = [] if dump is not None else None
    query_labels, _ = balanced_kmeans(coords, g_count, block, iters, qd)
    block_scores = group_means(coords, query_labels, g_count).astype(np.float32)
    if dump is not None:
        dump["key_dist"] = kd
        dump["query_dist"] = qd
    return {"sample_idx": s_idx, "key_labels": key_labels, "mu": mu, "coords": coords,
            "query_labels": query_labels, "block_scores": block_scores}


def partition_semantic(q: np.ndarray, k: np.ndarray, tau: float, block: int, iters: int,
                       dump: Optional[dict] = None) -> dict:
    """The semantic block partition the method is compared against ([abs]: "semantic
    block-sparse attention without residual correction"; [news], ablations paragraph).
    The pages do not state its rule; the reading taken is balanced k-means on the raw
    keys and, independently, on the raw queries (squared Euclidean distance, the same
    chunk start, fill and iteration count), with the routing scores of the response-
    coupled partition (mean over a block's queries of tau q_i . mu_g)."""
    n = q.shape[0]
    g_count = n_groups(n, block)
    kd = [] if dump is not None else None
    key_labels, _ = balanced_kmeans(k, g_count, block, iters, kd)
    mu = group_means(k, key_labels, g_count)
    qd = [] if dump is not None else None
    query_labels, _ = balanced_kmeans(q, g_count, block, iters, qd)
    coords = tau * (q @ mu.T)
    block_scores = group_means(coords, query_labels, g_count).astype(np.float32)
    if dump is not None:
        dump["key_dist"] = kd
        dump["query_dist"] = qd
    return {"key_labels": key_labels, "mu": mu, "coords": coords, "query_labels": query_labels,
            "block_scores": block_scores}


def routing_scores(q: np.ndarray, k: np.ndarray, tau: float, key_labels: np.ndarray, query_labels: np.ndarray,
                   g_count: int, mode: str = "centroid") -> np.ndarray:
    """Block-routing scores Sc[b][g] (fp32) under the three readings of "routing up to
    a target density" the comparison covers ([abs]; [news], components paragraph):

    * "centroid": tau qbar_b . mu_g, the mean over block b of the query coordinates
      (the method's reading; equals ``partition()["block_scores"]``);
    * "size_corrected": tau qbar_b . mu_g + log n_g, the first-order log of the
      attention mass the block's mean query puts on group g (n_g members);
    * "lse": log sum_{j in g} exp(tau qbar_b . k_j), that mass itself.
    qbar_b and mu_g are the member means of block b and group g (fp64)."""
    qbar = group_means(q, query_labels, g_count)
    mu = group_means(k, key_labels, g_count)
    if mode == "centroid":
        return (tau * (qbar @ mu.T)).astype(np.float32)
    sizes = np.bincount(key_labels, minlength=g_count)
    if mode == "size_corrected":
        return (tau * (qbar @ mu.T) + np.log(np.maximum(sizes, 1))[None, :]).astype(np.float32)
    if mode == "lse":
        out = np.empty((qbar.shape[0], g_count))
        logits = tau * (qbar @ k.T)                       # [Gq, N]
        for g in range(g_count):
            x = logits[:, key_labels == g]
            m = x.max(axis=1, keepdims=True)
            out[:, g] = (m + np.log(np.exp(x - m).sum(axis=1, keepdims=True)))[:, 0]
        return out.astype(np.float32)
    raise ValueError(f"unknown routing score mode {mode}")


# ------------------------------------------------------------------ step 5: routing

def route(block_scores: np.ndarray, k: int) -> np.ndarray:
    """For every query block, the k key groups with the largest fp32 score
    (ties -> lower group index), listed in ascending group order."""
    sc = np.asarray(block_scores, dtype=np.float32)
    if np.isnan(sc).any():
        raise NonFiniteError("NaN block score")
    gq, g_count = sc.shape
    if not 1 <= k <= g_count:
        raise ValueError("k out of range")
    idx = np.arange(g_count)
    out = np.empty((gq, k), dtype=np.int64)
    for b in range(gq):
        order = np.lexsort((idx, -sc[b]))
        out[b] = np.sort(order[:k])
    return out


def route_global(block_scores: np.ndarray, key_sizes: np.ndarray, block_sizes: np.ndarray,
                 n: int, n_probe: int, density: float) -> list:
    """Global budget allocation, the other reading of "routing up to a target density"
    ([abs]): the executed-pair budget floor(rho N^2 - P N) (real sizes, probes counted)
    is shared by all blocks of the head instead of a uniform k.  Every block keeps its
    best group (largest fp32 score, ties -> lower group); the other (block, group) pairs
    follow in descending score order (ties -> lower block, then lower group) and are
    taken while the cumulative pair count n_b n_g stays within the budget (the longest
    prefix of that order that fits).  Returns, per block, its groups in ascending order.
    """
    sc = np.asarray(block_scores, dtype=np.float32)
    if np.isnan(sc).any():
        raise NonFiniteError("NaN block score")
    gq, g_count = sc.shape
    budget = math.floor(density * n * n - float(n_probe * n))
    idx = np.arange(g_count)
    chosen = [set() for _ in range(gq)]
    spent = 0
    best = np.empty(gq, dtype=np.int64)
    for b in range(gq):
        best[b] = np.lexsort((idx, -sc[b]))[0]
        chosen[b].add(int(best[b]))
        spent += int(block_sizes[b]) * int(key_sizes[best[b]])
    # candidates: descending score, then block, then group (np.lexsort: last key primary)
    bb, gg = np.meshgrid(np.arange(gq), idx, indexing="ij")
    mask = gg != best[:, None]
    cb, cg = bb[mask], gg[mask]
    order = np.lexsort((cg, cb, -sc[cb, cg]))
    for t in order:
        b, g = int(cb[t]), int(cg[t])
        cost = int(block_sizes[b]) * int(key_sizes[g])
        if spent + cost > budget:
            break
        spent += cost
        chosen[b].add(g)
    return [np.array(sorted(c), dtype=np.int64) for c in chosen]


def executed_pairs(routes: np.ndarray, key_sizes: np.ndarray, block_sizes: np.ndarray,
                   n_probe: int, n: int) -> int:
    """Pairs the call evaluates: routed (block, group) tiles at their real sizes plus
    every probe row against all N keys ([abs]: probes are counted)."""
    total = 0
    for b in range(len(routes)):
        total += int(block_sizes[b]) * int(sum(int(key_sizes[g]) for g in routes[b]))
    return total + int(n_probe) * int(n)


# ----------------------------------------------------------- steps 6/7: attention

def _softmax_rows_times_v(logits: np.ndarray, v: np.ndarray) -> np.ndarray:
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    return (p @ v) / p.sum(axis=1, keepdims=True)


def sparse_attention(q, k, v, tau, key_labels, query_labels, routes) -> np.ndarray:
    """s_i = softmax over the union of the routed groups' keys of block(i) ([abs])."""
    n, d = q.shape
    out = np.zeros((n, v.shape[1]))
    for b in range(len(routes)):
        rows = np.flatnonzero(query_labels == b)
        if rows.size == 0:
            continue
        cols = np.flatnonzero(np.isin(key_labels, routes[b]))
        out[rows] = _softmax_rows_times_v(tau * (q[rows] @ k[cols].T), v[cols])
    return out


def dense_attention_rows(q, k, v, tau, rows, chunk: int = 1024) -> np.ndarray:
    """Exact softmax attention of the given query rows against all N keys."""
    rows = np.asarray(rows)
    out = np.zeros((rows.size, v.shape[1]))
    for s in range(0, rows.size, chunk):
        r = rows[s:s + chunk]
        out[s:s + r.size] = _softmax_rows_times_v(tau * (q[r] @ k.T), v)
    return out


# ----------------------------------------------------------------- step 8: the fit

def jacobi_eigh(c: np.ndarray, max_sweeps: int = 60):
    """Cyclic two-sided Jacobi for a symmetric matrix.  Returns eigenvalues in
    descending order (stable on ties) and the matching orthonormal eigenvectors."""
    a = np.array(c, dtype=np.float64, copy=True)
    n = a.shape[0]
    vec = np.eye(n)
    scale = np.linalg.norm(a)
    for _ in range(max_sweeps):
        off = math.sqrt(max(float(np.sum(a * a) - np.sum(np.diag(a) ** 2)), 0.0))
        if off <= 1e-14 * scale or scale == 0.0:
            break
        for p in range(n - 1):
            for r in range(p + 1, n):
                apr = a[p, r]
                if abs(apr) <= 1e-18 * scale:
                    a[p, r] = a[r, p] = 0.0
                    continue
                theta = (a[r, r] - a[p, p]) / (2.0 * apr)
                t = (1.0 if theta >= 0 else -1.0) / (abs(theta) + math.sqrt(theta * theta + 1.0))
                cs = 1.0 / math.sqrt(t * t + 1.0)
                sn = t * cs
                colp, colr = a[:, p].copy(), a[:, r].copy()
                a[:, p] = cs * colp - sn * colr
                a[:, r] = sn * colp + cs * colr
                rowp, rowr = a[p, :].copy(), a[r, :].copy()
                a[p, :] = cs * rowp - sn * rowr
                a[r, :] = sn * rowp + cs * rowr
                a[p, r] = a[r, p] = 0.0
                vp, vr = vec[:, p].copy(), vec[:, r].copy()
                vec[:, p] = cs * vp - sn * vr
                vec[:, r] = sn * vp + cs * vr
    evals = np.diag(a).copy()
    order = np.argsort(-evals, kind="stable")
    return evals[order], vec[:, order]


def cholesky(a: np.ndarray) -> np.ndarray:
    """Lower-triangular L with L L^T = a (a symmetric positive definite)."""
    n = a.shape[0]
    low = np.zeros_like(a, dtype=np.float64)
    for j in range(n):
        s = a[j, j] - low[j, :j] @ low[j, :j]
        if not s > 0.0:
            raise np.linalg.LinAlgError("matrix not positive definite")
        low[j, j] = math.sqrt(s)
        low[j + 1:, j] = (a[j + 1:, j] - low[j + 1:, :j] @ low[j, :j]) / low[j, j]
    return low


def cholesky_solve(low: np.ndarray, rhs: np.ndarray) -> np.ndarray:
    """Solve (L L^T) x = rhs by forward then backward substitution (rhs [n] or [n, m])."""
    n = low.shape[0]
    y = np.array(rhs, dtype=np.float64, copy=True)
    for i in range(n):
        y[i] = (y[i] - low[i, :i] @ y[:i]) / low[i, i]
    for i in range(n - 1, -1, -1):
        y[i] = (y[i] - low[i + 1:, i] @ y[i + 1:]) / low[i, i]
    return y


def probe_weights(d_probe: np.ndarray, mode: str = "inv_norm",
                  weights: Optional[np.ndarray] = None) -> np.ndarray:
    """Per-probe weights normalised to sum P.  'inv_norm' (default reading):
    1/max(|d_p|^2, 1e-30), so the weighted squared error is the squared relative
    error the pages measure; 'uniform': all ones; or caller-supplied weights."""
    p = d_probe.shape[0]
    if weights is not None:
        w = np.asarray(weights, dtype=np.float64).copy()
    elif mode == "uniform":
        w = np.ones(p)
    else:
        w = 1.0 / np.maximum(np.einsum("pe,pe->p", d_probe, d_probe), 1e-30)
    total = w.sum()
    if not total > 0.0:
        raise ValueError("weights must have a positive sum")
    return w * (p / total)


def ridge_affine(x: np.ndarray, z: np.ndarray, w: np.ndarray, ridge_lambda: float,
                 ridge_mode: str = "absolute"):
    """Weighted ridge regression z ~ A x + b with an unpenalised bias ([abs]: the
    affine correction is fitted by weighted ridge regression).  Centring at the
    weighted means removes the bias from the penalised system:
    A = (Z_c^T W X_c)(X_c^T W X_c + lambda I)^-1, b = zbar - A xbar (Cholesky).
    ``ridge_mode`` "relative" (the other reading of the unstated lambda scale) uses
    lambda * tr(X_c^T W X_c) / d in place of lambda."""
    wsum = w.sum()
    xbar = (w @ x) / wsum
    zbar = (w @ z) / wsum
    xc, zc = x - xbar, z - zbar
    gram = xc.T @ (w[:, None] * xc)
    lam = ridge_lambda * np.trace(gram) / x.shape[1] if ridge_mode == "relative" else ridge_lambda
    gram = gram + lam * np.eye(x.shape[1])
    cross = zc.T @ (w[:, None] * xc)                 # [r, d]
    a = cholesky_solve(cholesky(gram), cross.T).T    # gram is symmetric
    return a, zbar - a @ xbar


def fit_residual(s_probe: np.ndarray, d_probe: np.ndarray, ridge_lambda: float,
                 rank: int, weight_mode: str = "inv_norm",
                 weights: Optional[np.ndarray] = None, ridge_mode: str = "absolute") -> dict:
    """Probe-Fitted Residual Reconstruction, the fit ([abs], [news]).

    Residual y_p = d_p - s_p of every probe; U_r = top-r eigenvectors of
    C = sum_p w_p y_p y_p^T; targets z_p = U_r^T y_p; weighted ridge of z on s with
    an unpenalised bias:  A = (Z_c^T W X_c)(X_c^T W X_c + lambda I)^-1,
    b = zbar - A xbar.  Exported as M = U_r A (d x d) and beta = U_r b (d).
    """
    x = np.asarray(s_probe, dtype=np.float64)
    y = np.asarray(d_probe, dtype=np.float64) - x
    p, d = x.shape
    w = probe_weights(d_probe, weight_mode, weights)
    c = (y * w[:, None]).T @ y
    evals, evecs = jacobi_eigh(c)
    r = min(rank, d)
    u = evecs[:, :r]
    z = y @ u
    a, b = ridge_affine(x, z, w, ridge_lambda, ridge_mode)
    gap = (evals[r - 1] - evals[r]) / evals[0] if r < d and evals[0] > 0 else np.inf
    return {"M": u @ a, "beta": u @ b, "U": u, "A": a, "b": b, "evals": evals,
            "weights": w, "eigengap": gap}


# ---------------------------------------------------------------- step 9: apply

def apply_residual(s: np.ndarray, m: np.ndarray, beta: np.ndarray,
                   probe_idx: np.ndarray, d_probe: np.ndarray) -> np.ndarray:
    """o_i = s_i + M s_i + beta for unprobed rows; probe rows take their exact
    dense output ([abs]: the predicted residual is added to unprobed queries)."""
    out = s + s @ m.T + beta
    out[np.asarray(probe_idx)] = d_probe
    return out


# --------------------------------------------------------------- step 10: metric

def rel_l2_errors(o: np.ndarray, o_dense: np.ndarray, probe_idx: np.ndarray) -> dict:
    """e_i = |o_i - o*_i| / |o*_i| over the unprobed rows; mean and nearest-rank p99."""
    keep = np.ones(o.shape[0], dtype=bool)
    keep[np.asarray(probe_idx)] = False
    diff = o[keep] - o_dense[keep]
    e = np.sqrt(np.einsum("ie,ie->i", diff, diff)) / np.sqrt(
        np.einsum("ie,ie->i", o_dense[keep], o_dense[keep]))
    es = np.sort(e)
    p99 = float(es[max(int(math.ceil(0.99 * es.size)) - 1, 0)]) if es.size else float("nan")
    return {"errors": e, "mean": float(e.mean()) if e.size else float("nan"), "p99": p99}


# ---------------------------------------------------------------- the whole call

def sparsepr_head(q, k, v, *, block, n_sampled, n_probe, density, ridge_lambda, rank,
                  kmeans_iters=4, scale=None, weight_mode="inv_norm", inject=None,
                  dump=None, partition_mode="response", route_scores="centroid",
                  route_budget="uniform") -> dict:
    """One SparsePR call on one (batch, head).  ``inject`` may hold any of
    sample_idx, probe_idx, key_labels, query_labels, routes (e.g. the CUDA path's
    decisions) to run the later steps on them.  ``partition_mode`` "semantic" swaps
    Response-Coupled Partitioning for the semantic baseline partition (the ablation);
    the result's "S" is then the uncorrected semantic block-sparse output.
    ``route_budget`` "global" shares the pair budget across the blocks (route_global)
    instead of a uniform k; routes are then per-block arrays of different lengths."""
    inject = inject or {}
    n, d = q.shape
    tau = 1.0 / math.sqrt(d) if scale is None or scale <= 0 else float(scale)
    g_count = n_groups(n, block)
    if "key_labels" in inject and "query_labels" in inject:
        part = {"key_labels": np.asarray(inject["key_labels"]),
                "query_labels": np.asarray(inject["query_labels"])}
    elif partition_mode == "semantic":
        part = partition_semantic(q, k, tau, block, kmeans_iters, dump)
    else:
        part = partition(q, k, tau, block, n_sampled, kmeans_iters,
                         inject.get("sample_idx"), dump)
    kl, ql = part["key_labels"], part["query_labels"]
    key_sizes = np.bincount(kl, minlength=g_count)
    block_sizes = np.bincount(ql, minlength=g_count)
    kk = route_k(n, block, density, n_probe)
    if "routes" in inject:
        routes = inject["routes"]
        routes = [np.asarray(r)[np.asarray(r) >= 0] for r in routes] if route_budget == "global" else np.asarray(routes)
    else:
        scores = part["block_scores"] if route_scores == "centroid" else routing_scores(
            q, k, tau, kl, ql, g_count, route_scores)
        routes = (route_global(scores, key_sizes, block_sizes, n, n_probe, density) if route_budget == "global"
                  else route(scores, kk))
    probe_idx = np.asarray(inject["probe_idx"]) if "probe_idx" in inject else midpoint_stride(n, n_probe)
    pairs = executed_pairs(routes, key_sizes, block_sizes, probe_idx.size, n)
    s = sparse_attention(q, k, v, tau, kl, ql, routes)
    d_probe = dense_attention_rows(q, k, v, tau, probe_idx)
    fit = fit_residual(s[probe_idx], d_probe, ridge_lambda, rank, weight_mode)
    o = apply_residual(s, fit["M"], fit["beta"], probe_idx, d_probe)
    return {**part, "k": kk, "routes": routes, "probe_idx": probe_idx,
            "executed_pairs": pairs, "density": pairs / float(n * n), "S": s,
            "probe_out": d_probe, "fit": fit, "O": o, "tau": tau}
