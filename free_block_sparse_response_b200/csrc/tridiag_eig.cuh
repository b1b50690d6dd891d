// Top-r eigenvectors of a symmetric matrix in fp64, one CTA (included by fit.cu).
//
//   1. Householder tridiagonalisation, C -> Q^T C Q = tridiag(d, e), the reflectors
//      I - tau v v^T kept (v_0 = 1);
//   2. the r largest eigenvalues of the tridiagonal matrix by bisection on Sturm counts,
//      16 evaluation points per step (each step narrows the interval 17-fold), 16 threads
//      per eigenvalue;
//   3. each eigenvector of the tridiagonal matrix by 3 steps of inverse iteration
//      (Gaussian elimination with partial pivoting on T - lambda I), one thread per
//      eigenvalue, a different start vector per eigenvalue;
//   4. back-transformation by the reflectors (16 threads per vector), then modified
//      Gram-Schmidt among eigenvectors whose eigenvalues lie within 1e-3 ||T|| of each
//      other (what the fit uses of a cluster is its span).
// About 4/3 D^3 flops for step 1 instead of the ~4 D^3 per sweep of cyclic Jacobi.
#pragma once

#include "common.cuh"

namespace spr {

constexpr int kTriMaxR = 32;
constexpr int kTriThreads = 512;

// 1/x for |x| in [1e-30, 1e30]: the fp32 estimate refined by two Newton-Raphson steps
// (y <- y (2 - x y), each squaring the relative error) to fp64 rounding level.
__device__ __forceinline__ double tri_rcp(double x) {
  double y = static_cast<double>(__frcp_rn(static_cast<float>(x)));
  y = y * fma(-x, y, 2.0);
  y = y * fma(-x, y, 2.0);
  return y;
}

// Number of eigenvalues of tridiag(d, e) below x (Sturm sequence of the LDL^T pivots;
// a pivot smaller than pivmin in magnitude is replaced by -pivmin).
template <int D>
__device__ __forceinline__ int tri_sturm_count(const double* dd, const double* e2, double x, double pivmin) {
  double q = dd[0] - x;
  if (fabs(q) < pivmin) q = -pivmin;
  int c = q < 0.0;
  for (int i = 1; i < D; ++i) {
    const double r = tri_rcp(fmin(fabs(q), 1e30));
    q = (dd[i] - x) - e2[i - 1] * (q < 0.0 ? -r : r);
    if (fabs(q) < pivmin) q = -pivmin;
    c += q < 0.0;
  }
  return c;
}

// C [D x (D + 1)] is destroyed.  On return U (fp32, R x D, row a = eigenvector of the
// a-th largest eigenvalue) holds the vectors and evals[a] the eigenvalues.  Scratch:
// pack (>= D (D - 1) / 2 doubles), stage (>= D + kTriThreads doubles and >= R D floats); C holds the
// inverse-iteration factors.  All kTriThreads threads of the CTA call it.
template <int D>
__device__ void top_eigvecs_tridiagonal(double* C, double* pack, double* stage, float* U, int R, double* dd,
                                        double* ee, double* e2, double* tauh, double* evals, double* sh) {
  constexpr int LD = D + 1;
  constexpr int kWarps = kTriThreads / 32;
  constexpr int kBatch = (D + 1) / 4 < 32 ? (D + 1) / 4 : 32;  // inverse iterations whose factors fit in C
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double* vbuf = stage;
  double* pbuf = stage + D;

  // ---- 1. tridiagonalisation (reflector k annihilates column k below the subdiagonal)
  for (int k = 0; k < D - 2; ++k) {
    const int m = D - k - 1, r0 = k + 1;
    double* shk = sh + 2 * (k & 1);  // alternate slots: readers of step k - 1 may still run
    if (warp == 0) {
      double s2 = 0.0;
      for (int i = 1 + lane; i < m; i += 32) {
        const double v = C[(r0 + i) * LD + k];
        s2 += v * v;
      }
      s2 = warp_sum_d(s2);
      if (lane == 0) {
        const double alpha = C[r0 * LD + k];
        double tau = 0.0, beta = alpha, scale = 0.0;
        if (s2 > 0.0) {
          const double mu = sqrt(alpha * alpha + s2);
          beta = alpha >= 0.0 ? -mu : mu;
          tau = (beta - alpha) / beta;
          scale = 1.0 / (alpha - beta);
        }
        shk[0] = tau;
        shk[1] = scale;
        tauh[k] = tau;
        ee[k] = beta;
        dd[k] = C[k * LD + k];
      }
    }
    __syncthreads();
    const double tau = shk[0], scale = shk[1];
    if (tau == 0.0) continue;  // nothing to annihilate (the same branch for every thread)
    // p = tau A v in kParts column ranges: thread (part, i) sums rows j of its range of
    // column i (A is symmetric), v_j read straight from column k (v_0 = 1)
    {
      constexpr int kParts = kTriThreads / D, kSpan = D / kParts;
      const int i = tid % D, part = tid / D;
      double acc = 0.0;
      if (i < m) {
        const int j1 = min(m, (part + 1) * kSpan);
        for (int j = part * kSpan; j < j1; ++j) {
          const double vj = j == 0 ? 1.0 : C[(r0 + j) * LD + k] * scale;
          acc = fma(C[(r0 + j) * LD + r0 + i], vj, acc);
        }
        if (part == 0) vbuf[i] = i == 0 ? 1.0 : C[(r0 + i) * LD + k] * scale;
      }
      pbuf[part * D + i] = acc;
    }
    __syncthreads();
    {
      constexpr int kParts = kTriThreads / D, kT = D / 32;
      // every warp: its lanes' p_j and v_j (j = lane + 32 t), p . v, then its rows' update
      double pj[kT], vj[kT];
      double pv = 0.0;
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const int j = lane + 32 * t;
        double sp = 0.0;
#pragma unroll
        for (int q = 0; q < kParts; ++q) sp += pbuf[q * D + j];
        pj[t] = j < m ? tau * sp : 0.0;
        vj[t] = j < m ? vbuf[j] : 0.0;
        pv = fma(pj[t], vj[t], pv);
      }
      pv = warp_sum_d(pv);
      const double kc = -0.5 * tau * pv;  // w = p + kc v;  A <- A - v w^T - w v^T
      for (int i = warp; i < m; i += kWarps) {
        double pi = 0.0;
#pragma unroll
        for (int q = 0; q < kParts; ++q) pi += pbuf[q * D + i];
        const double vi = vbuf[i], wi = tau * pi + kc * vi;
        double* row = C + (r0 + i) * LD + r0;
#pragma unroll
        for (int t = 0; t < kT; ++t) {
          const int j = lane + 32 * t;
          if (j < m) row[j] -= vi * (pj[t] + kc * vj[t]) + wi * vj[t];
        }
      }
      if (warp == 0)  // the reflector, kept in column k for the back-transformation
        for (int i = lane; i < m; i += 32) C[(r0 + i) * LD + k] = vbuf[i];
    }
    __syncthreads();
  }
  if (tid == 0) {
    dd[D - 2] = C[(D - 2) * LD + D - 2];
    dd[D - 1] = C[(D - 1) * LD + D - 1];
    ee[D - 2] = C[(D - 1) * LD + D - 2];
    tauh[D - 2] = 0.0;
  }
  __syncthreads();
  // reflectors, packed: v_k (rows k + 1 .. D - 1) at pack + k (D - 1) - k (k - 1) / 2
  for (int k = 0; k < D - 2; ++k) {
    const int off = k * (D - 1) - k * (k - 1) / 2, m = D - 1 - k;
    for (int i = tid; i < m; i += kTriThreads) pack[off + i] = C[(k + 1 + i) * LD + k];
  }
  for (int i = tid; i < D - 1; i += kTriThreads) e2[i] = ee[i] * ee[i];
  if (warp == 0) {  // Gershgorin interval of T
    double lo = 1e300, hi = -1e300;
    for (int i = lane; i < D; i += 32) {
      const double rad = (i > 0 ? fabs(ee[i - 1]) : 0.0) + (i < D - 1 ? fabs(ee[i]) : 0.0);
      lo = fmin(lo, dd[i] - rad);
      hi = fmax(hi, dd[i] + rad);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      const double tn = fmax(fmax(fabs(lo), fabs(hi)), 1e-300);
      sh[4] = lo - 1e-14 * tn;
      sh[5] = hi + 1e-14 * tn;
      sh[6] = tn;
    }
  }
  __syncthreads();
  const double tnorm = sh[6];
  if (tnorm < 1e-250) {  // (numerically) zero matrix: every basis is an eigenbasis
    for (int x = tid; x < R * D; x += kTriThreads) U[x] = (x % D == x / D) ? 1.f : 0.f;
    for (int a = tid; a < R; a += kTriThreads) evals[a] = 0.0;
    __syncthreads();
    return;
  }
  const double pivmin = fmax(1e-30, 1e-290 * tnorm);

  // ---- 2. the R largest eigenvalues: group of 16 threads per eigenvalue, 16 points per step
  {
    const int sub = tid & 15;
    const unsigned int hmask = (tid & 16) ? 0xffff0000u : 0x0000ffffu;
    for (int a0 = 0; a0 < R; a0 += kTriThreads / 16) {
      const int a = a0 + (tid >> 4);
      const bool act = a < R;
      const int j = D - 1 - a;  // ascending index of the eigenvalue
      double l = sh[4], h = sh[5];
      for (int it = 0; it < 64; ++it) {
        const double x = l + (h - l) * static_cast<double>(sub + 1) * (1.0 / 17.0);
        const int cnt = act ? tri_sturm_count<D>(dd, e2, x, pivmin) : 0;
        const unsigned int bal = __ballot_sync(0xffffffffu, cnt > j) & hmask;
        const int t = bal != 0u ? ((__ffs(bal) - 1) & 15) : 16;  // first point above eigenvalue j
        const double nl = t == 0 ? l : l + (h - l) * static_cast<double>(t) * (1.0 / 17.0);
        const double nh = t == 16 ? h : l + (h - l) * static_cast<double>(t + 1) * (1.0 / 17.0);
        l = nl;
        h = nh;
        const bool done = !act || h - l <= 4.0e-16 * fmax(fabs(l), fabs(h)) + pivmin;
        if (__all_sync(0xffffffffu, done)) break;
      }
      if (act && sub == 0) evals[a] = 0.5 * (l + h);
    }
  }
  __syncthreads();

  // ---- 3 + 4. eigenvectors, kBatch at a time.  Factors of thread s in C at
  // [(i * 4 + f) * kBatch + s] (f: pivot, first and second superdiagonal, right side /
  // solution), so that a warp's accesses at one i are consecutive.
  float* Us = reinterpret_cast<float*>(stage);
  const double epsn = 2.3e-16 * tnorm;
  for (int b0 = 0; b0 < R; b0 += kBatch) {
    const int nb = R - b0 < kBatch ? R - b0 : kBatch;
    if (tid < nb) {
      const int a = b0 + tid;
      const double lam = evals[a];
      auto S = [&](int i, int f) -> double& { return C[(i * 4 + f) * kBatch + tid]; };
      for (int i = 0; i < D; ++i) {  // start vector: a fixed hash of (eigenvalue, row)
        const unsigned int hv = static_cast<unsigned int>(i) * 2654435761u + static_cast<unsigned int>(a) * 40503u;
        S(i, 3) = static_cast<double>(hv % 1000003u) * (1.0 / 1000003.0) - 0.5;
      }
      for (int itn = 0; itn < 3; ++itn) {
        // (T - lam I) x = z: elimination with row interchanges, streamed over the rows
        double cur0 = dd[0] - lam, cur1 = ee[0], yi = S(0, 3);
        for (int i = 0; i < D - 1; ++i) {
          const double c = ee[i], an = dd[i + 1] - lam, bn = i + 1 < D - 1 ? ee[i + 1] : 0.0;
          const double zn = S(i + 1, 3);
          if (fabs(cur0) >= fabs(c)) {
            const double piv = cur0 != 0.0 ? cur0 : epsn;
            const double lm = c / piv;
            S(i, 0) = piv;
            S(i, 1) = cur1;
            S(i, 2) = 0.0;
            S(i, 3) = yi;
            cur0 = an - lm * cur1;
            cur1 = bn;
            yi = zn - lm * yi;
          } else {
            const double lm = cur0 / c;
            S(i, 0) = c;
            S(i, 1) = an;
            S(i, 2) = bn;
            S(i, 3) = zn;
            cur0 = cur1 - lm * an;
            cur1 = -lm * bn;
            yi = yi - lm * zn;
          }
        }
        S(D - 1, 0) = cur0 != 0.0 ? cur0 : epsn;
        S(D - 1, 1) = 0.0;
        S(D - 1, 2) = 0.0;
        S(D - 1, 3) = yi;
        double x1 = 0.0, x2 = 0.0, mx = 0.0;
        for (int i = D - 1; i >= 0; --i) {
          const double xi = (S(i, 3) - S(i, 1) * x1 - S(i, 2) * x2) / S(i, 0);
          S(i, 3) = xi;
          x2 = x1;
          x1 = xi;
          mx = fmax(mx, fabs(xi));
        }
        if (!(mx > 0.0) || !isfinite(mx)) {  // no usable solution: fall back to a unit vector
          for (int i = 0; i < D; ++i) S(i, 3) = i == a % D ? 1.0 : 0.0;
          continue;
        }
        const double imx = 1.0 / mx;
        double n2 = 0.0;
        for (int i = 0; i < D; ++i) {
          const double t = S(i, 3) * imx;
          n2 += t * t;
        }
        const double inv = imx / sqrt(n2);
        for (int i = 0; i < D; ++i) S(i, 3) *= inv;
      }
    }
    __syncthreads();
    // back-transformation u = H_0 H_1 ... H_{D-3} z: 16 threads (half a warp) per vector,
    // thread sub holding entries sub, sub + 16, ...
    {
      constexpr int kE = D / 16;
      const int g = tid >> 4, sub = tid & 15;
      const bool act = g < nb;
      double z[kE];
#pragma unroll
      for (int q = 0; q < kE; ++q) z[q] = act ? C[((sub + 16 * q) * 4 + 3) * kBatch + g] : 0.0;
      for (int k = D - 3; k >= 0; --k) {
        const double tk = tauh[k];
        if (tk == 0.0) continue;
        const int off = k * (D - 1) - k * (k - 1) / 2 - (k + 1);  // pack index of entry i: off + i
        double part = 0.0;
#pragma unroll
        for (int q = 0; q < kE; ++q) {
          const int i = sub + 16 * q;
          if (i > k) part = fma(pack[off + i], z[q], part);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        const double sk = tk * part;
#pragma unroll
        for (int q = 0; q < kE; ++q) {
          const int i = sub + 16 * q;
          if (i > k) z[q] = fma(-sk, pack[off + i], z[q]);
        }
      }
      if (act) {
#pragma unroll
        for (int q = 0; q < kE; ++q) Us[(b0 + g) * D + sub + 16 * q] = static_cast<float>(z[q]);
      }
    }
    __syncthreads();
  }
  // ---- Gram-Schmidt among close eigenvalues (one warp; clusters are rare)
  if (warp == 0) {
    for (int a = 1; a < R; ++a) {
      float* ua = Us + a * D;
      bool touched = false;
      for (int b = 0; b < a; ++b) {
        if (fabs(evals[a] - evals[b]) >= 1e-3 * tnorm) continue;
        const float* ub = Us + b * D;
        double dot = 0.0;
        for (int i = lane; i < D; i += 32) dot += static_cast<double>(ua[i]) * ub[i];
        dot = warp_sum_d(dot);
        for (int i = lane; i < D; i += 32) ua[i] = static_cast<float>(static_cast<double>(ua[i]) - dot * ub[i]);
        __syncwarp();
        touched = true;
      }
      if (touched) {
        double n2 = 0.0;
        for (int i = lane; i < D; i += 32) n2 += static_cast<double>(ua[i]) * ua[i];
        n2 = warp_sum_d(n2);
        const double inv = n2 > 0.0 ? 1.0 / sqrt(n2) : 0.0;
        for (int i = lane; i < D; i += 32) ua[i] = static_cast<float>(ua[i] * inv);
        __syncwarp();
      }
    }
  }
  __syncthreads();
  for (int x = tid; x < R * D; x += kTriThreads) U[x] = Us[x];
  __syncthreads();
}

}  // namespace spr
