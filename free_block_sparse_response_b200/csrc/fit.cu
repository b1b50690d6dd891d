// Probe-Fitted Residual Reconstruction: the fit and the apply step (sm_100a).
//
// Source: SparsePR abstract (arXiv 2608.18484, arxivdaily.com English abstract): exact
// probe rows calibrate an affine correction from the sparse output to the dense-minus-
// sparse difference by weighted ridge regression, and the predicted residual is added
// to every unprobed row; the skillfed.io article's paragraph on the two components adds
// that the correction lives in the output subspace seen in the probe residuals.
//
// Fit, one CTA per (batch, head), fp64 throughout:
//   w_p (caller / 1/|d_p|^2 / uniform) scaled to sum P;  y_p = d_p - s_p;
//   C = sum_p w_p y_p y_p^T;  U_r = eigenvectors of the r largest eigenvalues (r <= 32:
//   Householder tridiagonalisation, bisection and inverse iteration; larger r: cyclic
//   Jacobi with the round-robin parallel ordering);  z_p = U_r^T y_p;
//   A = (Z_c^T W X_c)(X_c^T W X_c + lambda I)^-1 by Cholesky;  b = zbar - A xbar;
//   M = U_r A, beta = U_r b.
#include "common.cuh"
#include "fit.cuh"
#include "tridiag_eig.cuh"

namespace spr {

constexpr int kFitThreads = 512;
constexpr int kStageRows = 16;

__device__ double block_sum_d(double v, double* red) {
  v = warp_sum_d(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = 0.0;
  for (int w = 0; w < kFitThreads / 32; ++w) s += red[w];
  return s;
}

// Reciprocal and reciprocal square root in fp64 by Newton-Raphson refinement of the fp32
// hardware estimates (y <- y (2 - x y), and y <- y (3 - x y^2) / 2): each step squares
// the relative error, so two steps take the ~2^-22 seed to fp64 rounding level.  Used
// on the latency-critical path of the Jacobi rotations, for arguments well inside the
// fp32 range (the callers keep them there).
__device__ __forceinline__ double rcp_nr(double x) {
  double y = static_cast<double>(__frcp_rn(static_cast<float>(x)));
  y = y * fma(-x, y, 2.0);
  y = y * fma(-x, y, 2.0);
  return y;
}
__device__ __forceinline__ double rsqrt_nr(double x) {
  double y = static_cast<double>(rsqrtf(static_cast<float>(x)));
  const double hx = 0.5 * x;
  y = y * fma(-hx * y, y, 1.5);
  y = y * fma(-hx * y, y, 1.5);
  return y;
}

__host__ __device__ size_t fit_scratch_doubles(int P, int d) {
  return static_cast<size_t>(d) * d + static_cast<size_t>(P) * d + static_cast<size_t>(d) * d + 4ull * d;
}

template <int D>
__global__ void __launch_bounds__(kFitThreads)
    fit_kernel(const float* __restrict__ xs_all, const float* __restrict__ dp_all,
               const float* __restrict__ weights, int P, double lambda, int R, int weight_mode,
               double* __restrict__ scratch, float* __restrict__ M_out, float* __restrict__ beta_out,
               int* __restrict__ status) {
  constexpr int LD = D + 1;
  extern __shared__ __align__(16) double sm[];
  double* C = sm;                          // D x LD
  double* w = C + D * LD;                  // P
  double* stage = w + P;                   // kStageRows x D
  float* Vt = reinterpret_cast<float*>(stage + kStageRows * D);  // D x D eigenvectors (rows), fp32
  __shared__ double red[kFitThreads / 32];
  __shared__ double pc[D / 2], ps[D / 2];
  __shared__ int pp[D / 2], pq[D / 2], order[D];
  __shared__ double xbar[D], zbar[D], bvec[D];
  __shared__ int s_fail;
  __shared__ double t_dd[D], t_ee[D], t_e2[D], t_tau[D], t_evals[kTriMaxR], t_sh[8];
  static_assert(kTriThreads == kFitThreads, "the eigensolver runs on the fit's CTA");

  const int head = blockIdx.x, tid = threadIdx.x;
  const float* xs = xs_all + static_cast<size_t>(head) * P * D;
  const float* dp = dp_all + static_cast<size_t>(head) * P * D;
  double* Z = scratch + static_cast<size_t>(head) * fit_scratch_doubles(P, D) + D * D;  // P x R
  double* A = Z + static_cast<size_t>(P) * D;  // R x D
  if (tid == 0) s_fail = 0;

  // ---- weights
  for (int p = tid; p < P; p += kFitThreads) {
    double wp = 1.0;
    if (weights != nullptr) {
      wp = weights[static_cast<size_t>(head) * P + p];
    } else if ((weight_mode & kWeightModeMask) == 0) {
      double n2 = 0.0;
      for (int e = 0; e < D; ++e) {
        const double v = dp[static_cast<size_t>(p) * D + e];
        n2 += v * v;
      }
      wp = 1.0 / fmax(n2, 1e-30);
    }
    w[p] = wp;
  }
  __syncthreads();
  double wsum = 0.0;
  for (int p = tid; p < P; p += kFitThreads) wsum += w[p];
  wsum = block_sum_d(wsum, red);
  if (!(wsum > 0.0)) {
    if (tid == 0) record_error(status, kErrInvalidArg);
    wsum = P;
    for (int p = tid; p < P; p += kFitThreads) w[p] = 1.0;
  }
  __syncthreads();
  for (int p = tid; p < P; p += kFitThreads) w[p] *= static_cast<double>(P) / wsum;
  __syncthreads();

  // ---- C = sum_p w_p y_p y_p^T.  Thread (bi, bj) accumulates rows bi + kNrb k' x columns
  // bj + kNcb k (a kRb x kCb block, columns interleaved so that a warp's reads of a staged
  // row hit consecutive words); the rows are staged 16 at a time as y_p and w_p y_p.
  constexpr int kPer = D * D / kFitThreads;
  constexpr int kNcb = 16, kCb = D / kNcb, kNrb = kFitThreads / kNcb, kRb = D / kNrb;
  static_assert(kRb * kCb == kPer, "block shape");
  const int bj = tid % kNcb, bi = tid / kNcb;
  double acc[kRb][kCb];
  auto acc_zero = [&]() {
#pragma unroll
    for (int k1 = 0; k1 < kRb; ++k1)
#pragma unroll
      for (int k2 = 0; k2 < kCb; ++k2) acc[k1][k2] = 0.0;
  };
  // acc += (w_r y_r)[rows] (y_r)[cols] for the staged rows r
  auto acc_rows = [&](const double* wys, const double* ys, int nr) {
    for (int r = 0; r < nr; ++r) {
      double yi[kRb], yj[kCb];
#pragma unroll
      for (int k1 = 0; k1 < kRb; ++k1) yi[k1] = wys[r * D + bi + kNrb * k1];
#pragma unroll
      for (int k2 = 0; k2 < kCb; ++k2) yj[k2] = ys[r * D + bj + kNcb * k2];
#pragma unroll
      for (int k1 = 0; k1 < kRb; ++k1)
#pragma unroll
        for (int k2 = 0; k2 < kCb; ++k2) acc[k1][k2] = fma(yi[k1], yj[k2], acc[k1][k2]);
    }
  };
  acc_zero();
  {
    double* wst = C;  // staged w_p y_p (C is written after the loop)
    for (int p0 = 0; p0 < P; p0 += kStageRows) {
      __syncthreads();
      for (int x = tid; x < kStageRows * D; x += kFitThreads) {
        const int p = p0 + x / D, e = x % D;
        const double yv = p < P ? (static_cast<double>(dp[static_cast<size_t>(p) * D + e]) -
                                   static_cast<double>(xs[static_cast<size_t>(p) * D + e])) : 0.0;
        stage[x] = yv;
        wst[x] = p < P ? w[p] * yv : 0.0;
      }
      __syncthreads();
      acc_rows(wst, stage, min(kStageRows, P - p0));
    }
  }
  __syncthreads();
#pragma unroll
  for (int k1 = 0; k1 < kRb; ++k1)
#pragma unroll
    for (int k2 = 0; k2 < kCb; ++k2) C[(bi + kNrb * k1) * LD + bj + kNcb * k2] = acc[k1][k2];
  __syncthreads();

  // ---- eigenvectors of the R largest eigenvalues
  const bool tri = R <= kTriMaxR;
  if (tri) {
    top_eigvecs_tridiagonal<D>(C, reinterpret_cast<double*>(Vt), stage, Vt, R, t_dd, t_ee, t_e2, t_tau, t_evals,
                               t_sh);
  } else {
  for (int x = tid; x < D * D; x += kFitThreads) Vt[x] = (x / D == x % D) ? 1.f : 0.f;
  __syncthreads();
  // ---- Jacobi, round-robin parallel ordering
  double total = 0.0;
  for (int x = tid; x < D * D; x += kFitThreads) {
    const double v = C[(x / D) * LD + x % D];
    total += v * v;
  }
  total = block_sum_d(total, red);
  const double tol2 = 1e-20 * total;  // stop at off-diagonal norm <= 1e-10 |C|
  // this thread's 2x2 blocks (a, b), a <= b, of the pair slots (fixed for all rounds)
  constexpr int kBlocks = (D / 2) * (D / 2 + 1) / 2;
  constexpr int kBlocksPer = (kBlocks + kFitThreads - 1) / kFitThreads;
  int blk_a[kBlocksPer], blk_b[kBlocksPer];
#pragma unroll
  for (int i = 0; i < kBlocksPer; ++i) {
    const int x = tid + i * kFitThreads;
    blk_a[i] = -1;
    blk_b[i] = -1;
    if (x < kBlocks) {
      int a = 0, first = 0;  // first = index of block (a, a)
      while (first + (D / 2 - a) <= x) {
        first += D / 2 - a;
        ++a;
      }
      blk_a[i] = a;
      blk_b[i] = a + (x - first);
    }
  }
  for (int sweep = 0; sweep < 40; ++sweep) {
    double off = 0.0;
    for (int x = tid; x < D * D; x += kFitThreads) {
      const int i = x / D, j = x % D;
      if (i != j) {
        const double v = C[i * LD + j];
        off += v * v;
      }
    }
    off = block_sum_d(off, red);
    if (off <= tol2 || total == 0.0) break;
    for (int round = 0; round < D - 1; ++round) {
      if (tid < D / 2) {
        int p, q;
        if (tid == 0) {
          p = round;
          q = D - 1;
        } else {
          p = (round + tid) % (D - 1);
          q = (round - tid + (D - 1)) % (D - 1);
        }
        if (p > q) {
          const int t = p;
          p = q;
          q = t;
        }
        const double apq = C[p * LD + q];
        const double app = C[p * LD + p], aqq = C[q * LD + q];
        double c = 1.0, sn = 0.0;
        if (apq != 0.0 && apq * apq > 1e-30 * fabs(app * aqq) && apq * apq > 1e-36 * total) {
          // t = tan of the annihilating angle, the smaller root of t^2 + 2 theta t - 1 = 0
          const double den = 2.0 * apq;
          const double theta = fabs(den) > 1e-30 && fabs(den) < 1e30 ? (aqq - app) * rcp_nr(den) : (aqq - app) / den;
          const double at = fabs(theta);
          double t;
          if (at > 1e15) {
            t = 0.5 / theta;  // sqrt(theta^2 + 1) = |theta| to fp64 precision
          } else {
            const double h = theta * theta + 1.0;
            t = rcp_nr(at + h * rsqrt_nr(h));
            if (theta < 0.0) t = -t;
          }
          c = rsqrt_nr(t * t + 1.0);
          sn = t * c;
        }
        pp[tid] = p;
        pq[tid] = q;
        pc[tid] = c;
        ps[tid] = sn;
      }
      __syncthreads();
      // C <- R C R^T with R the product of this round's D/2 disjoint plane rotations
      // (rows p, q of R: (c, -s), (s, c)), one 2x2 block {p_a, q_a} x {p_b, q_b} at a
      // time: B <- R_a B R_b^T for a <= b, the mirror block written as its transpose;
      // the annihilated element of a rotated pair is stored as an exact zero.
#pragma unroll
      for (int i = 0; i < kBlocksPer; ++i) {
        const int a = blk_a[i], b = blk_b[i];
        if (a < 0) continue;
        const double sa = ps[a], sb = ps[b];
        if (sa == 0.0 && sb == 0.0) continue;
        const double ca = pc[a], cb = pc[b];
        const int pa = pp[a], qa = pq[a], pb = pp[b], qb = pq[b];
        const double b00 = C[pa * LD + pb], b01 = C[pa * LD + qb], b10 = C[qa * LD + pb], b11 = C[qa * LD + qb];
        const double t00 = b00 * cb - b01 * sb, t01 = b00 * sb + b01 * cb;
        const double t10 = b10 * cb - b11 * sb, t11 = b10 * sb + b11 * cb;
        const double n00 = ca * t00 - sa * t10, n01 = ca * t01 - sa * t11;
        const double n10 = sa * t00 + ca * t10, n11 = sa * t01 + ca * t11;
        if (a == b) {
          C[pa * LD + pa] = n00;
          C[qa * LD + qa] = n11;
          const double z = sa != 0.0 ? 0.0 : n01;
          C[pa * LD + qa] = z;
          C[qa * LD + pa] = z;
        } else {
          C[pa * LD + pb] = n00;
          C[pa * LD + qb] = n01;
          C[qa * LD + pb] = n10;
          C[qa * LD + qb] = n11;
          C[pb * LD + pa] = n00;
          C[qb * LD + pa] = n01;
          C[pb * LD + qa] = n10;
          C[qb * LD + qa] = n11;
        }
      }
      for (int x = tid; x < (D / 2) * D; x += kFitThreads) {  // eigenvector rows: V^T <- R V^T
        const int t = x / D, j = x % D;
        const double sn = ps[t];
        if (sn != 0.0) {
          const int p = pp[t], q = pq[t];
          const float cf = static_cast<float>(pc[t]), sf = static_cast<float>(sn);
          const float vp = Vt[p * D + j], vq = Vt[q * D + j];
          Vt[p * D + j] = cf * vp - sf * vq;
          Vt[q * D + j] = sf * vp + cf * vq;
        }
      }
      __syncthreads();
    }
  }
  // ---- eigenvalues descending (stable on ties)
  for (int i = tid; i < D; i += kFitThreads) {
    const double li = C[i * LD + i];
    int rank = 0;
    for (int j = 0; j < D; ++j) {
      const double lj = C[j * LD + j];
      rank += (lj > li) || (lj == li && j < i);
    }
    order[rank] = i;
  }
  __syncthreads();
  }
  // row a of U_r: the a-th largest eigenvalue's eigenvector (fp32)
  auto urow = [&](int a) -> const float* { return tri ? Vt + a * D : Vt + static_cast<size_t>(order[a]) * D; };

  // ---- pass A over the probes, 16 rows at a time: z_p = U_r^T y_p (to scratch) and the
  // per-thread parts of sum_p w_p x_p (thread tid always holds dim tid % D)
  double xpart = 0.0;
  for (int p0 = 0; p0 < P; p0 += kStageRows) {
    __syncthreads();
    for (int x = tid; x < kStageRows * D; x += kFitThreads) {
      const int p = p0 + x / D, e = x % D;
      double yv = 0.0;
      if (p < P) {
        const double xv = xs[static_cast<size_t>(p) * D + e];
        yv = static_cast<double>(dp[static_cast<size_t>(p) * D + e]) - xv;
        xpart += w[p] * xv;
      }
      stage[x] = yv;
    }
    __syncthreads();
    // output (r, a): lanes of a warp take consecutive a, and walk the dims from (e + a) % D,
    // so that the 32 eigenvector rows they read sit in 32 different banks
    for (int x = tid; x < kStageRows * R; x += kFitThreads) {
      const int r = x / R, a = x % R;
      if (p0 + r >= P) continue;
      const float* u = urow(a);
      const double* y = stage + r * D;
      double acc0 = 0.0, acc1 = 0.0;
      for (int e0 = 0; e0 < D; e0 += 2) {
        const int e = (e0 + a) & (D - 1), f = (e0 + 1 + a) & (D - 1);
        acc0 = fma(static_cast<double>(u[e]), y[e], acc0);
        acc1 = fma(static_cast<double>(u[f]), y[f], acc1);
      }
      Z[static_cast<size_t>(p0 + r) * R + a] = acc0 + acc1;
    }
  }
  __syncthreads();
  {
    double* part = C;  // free until the Gram is written
    part[tid] = xpart;
    __syncthreads();
    for (int e = tid; e < D; e += kFitThreads) {
      double sx = 0.0;
      for (int t = e; t < kFitThreads; t += D) sx += part[t];
      xbar[e] = sx / static_cast<double>(P);
    }
    __syncthreads();
    // zbar: 16 interleaved partial sums per a, then their total
    for (int x = tid; x < 16 * R; x += kFitThreads) {
      const int a = x % R, prt = x / R;
      double sz = 0.0;
      for (int p = prt; p < P; p += 16) sz += w[p] * Z[static_cast<size_t>(p) * R + a];
      part[x] = sz;
    }
    __syncthreads();
    for (int a = tid; a < R; a += kFitThreads) {
      double sz = 0.0;
      for (int prt = 0; prt < 16; ++prt) sz += part[prt * R + a];
      zbar[a] = sz / static_cast<double>(P);
    }
    __syncthreads();
  }

  // ---- pass B: Gram = X_c^T W X_c (register blocks as for C) and cross = Z_c^T W X_c
  // (registers when R <= kTriMaxR: thread tid holds dim tid % D of rows a = tid / D + k (512 / D))
  constexpr int kCross = kTriMaxR * D / kFitThreads;
  const bool cross_regs = R <= kTriMaxR;
  double cacc[kCross];
#pragma unroll
  for (int k = 0; k < kCross; ++k) cacc[k] = 0.0;
  acc_zero();
  double* wxs = C;                        // staged w_p x_c rows [16][D]
  double* zst = C + kStageRows * D;       // staged Z_c rows [16][R]
  for (int p0 = 0; p0 < P; p0 += kStageRows) {
    __syncthreads();
    for (int x = tid; x < kStageRows * D; x += kFitThreads) {
      const int p = p0 + x / D, e = x % D;
      const double xc = p < P ? static_cast<double>(xs[static_cast<size_t>(p) * D + e]) - xbar[e] : 0.0;
      stage[x] = xc;
      wxs[x] = p < P ? w[p] * xc : 0.0;
    }
    for (int x = tid; x < kStageRows * R; x += kFitThreads) {
      const int p = p0 + x / R, a = x % R;
      zst[x] = p < P ? Z[static_cast<size_t>(p) * R + a] - zbar[a] : 0.0;
    }
    __syncthreads();
    const int nr = min(kStageRows, P - p0);
    acc_rows(wxs, stage, nr);
    if (cross_regs) {
      for (int r = 0; r < nr; ++r) {
        const double wx = wxs[r * D + tid % D];
#pragma unroll
        for (int k = 0; k < kCross; ++k) {
          const int a = tid / D + k * (kFitThreads / D);
          if (a < R) cacc[k] = fma(zst[r * R + a], wx, cacc[k]);
        }
      }
    }
  }
  __syncthreads();
  // ridge: lambda itself, or lambda times the mean diagonal entry of X_c^T W X_c (the
  // scale-relative reading, weight_mode | kRidgeRelative)
  double lam = lambda;
  if (weight_mode & kRidgeRelative) {
    double diag = 0.0;
#pragma unroll
    for (int k1 = 0; k1 < kRb; ++k1)
#pragma unroll
      for (int k2 = 0; k2 < kCb; ++k2)
        if (bi + kNrb * k1 == bj + kNcb * k2) diag += acc[k1][k2];
    lam = lambda * block_sum_d(diag, red) / static_cast<double>(D);
  }
#pragma unroll
  for (int k1 = 0; k1 < kRb; ++k1)
#pragma unroll
    for (int k2 = 0; k2 < kCb; ++k2) {
      const int i = bi + kNrb * k1, j = bj + kNcb * k2;
      C[i * LD + j] = acc[k1][k2] + (i == j ? lam : 0.0);
    }
  if (cross_regs) {
#pragma unroll
    for (int k = 0; k < kCross; ++k) {
      const int a = tid / D + k * (kFitThreads / D);
      if (a < R) A[static_cast<size_t>(a) * D + tid % D] = cacc[k];
    }
  } else {
    for (int x = tid; x < R * D; x += kFitThreads) {
      const int a = x / D, e = x % D;
      double sc = 0.0;
      for (int p = 0; p < P; ++p)
        sc += w[p] * (Z[static_cast<size_t>(p) * R + a] - zbar[a]) *
              (static_cast<double>(xs[static_cast<size_t>(p) * D + e]) - xbar[e]);
      A[x] = sc;
    }
  }
  __syncthreads();

  // ---- Cholesky (lower, in C), right-looking: column j scaled, then the trailing lower
  // triangle updated by all threads; the thread that finishes entry (j + 1, j + 1) takes
  // its square root at once (lane 0 of warp 0)
  const int lane = tid & 31, warp = tid >> 5;
  double* dinv = t_dd;  // 1 / L_jj (the eigensolver's scratch is free)
  auto take_root = [&](int j) {
    const double dj = C[j * LD + j];
    if (!(dj > 0.0)) {
      s_fail = 1;
      C[j * LD + j] = 1.0;
      dinv[j] = 1.0;
    } else {
      const double l = sqrt(dj);
      C[j * LD + j] = l;
      dinv[j] = 1.0 / l;
    }
  };
  if (tid == 0) take_root(0);
  __syncthreads();
  for (int j = 0; j < D; ++j) {
    for (int i = j + 1 + tid; i < D; i += kFitThreads) C[i * LD + j] *= dinv[j];
    __syncthreads();
    for (int i = j + 1 + warp; i < D; i += kFitThreads / 32) {
      const double lij = C[i * LD + j];
      for (int k = j + 1 + lane; k <= i; k += 32) C[i * LD + k] = fma(-lij, C[k * LD + j], C[i * LD + k]);
    }
    if (tid == 0 && j + 1 < D) take_root(j + 1);  // row j + 1 is warp 0's, entry j + 1 lane 0's
    __syncthreads();
  }
  // ---- solve (L L^T) a_row = cross_row: warp w takes right-hand sides 2 w, 2 w + 1, ...,
  // lane l holding entries l, l + 32, ...; column-oriented substitution (the owner lane
  // finishes entry j and broadcasts it, every lane updates its later entries)
  constexpr int kRow = D / 32;
  for (int a0 = 2 * warp; a0 < R; a0 += kFitThreads / 16) {
    const bool two = a0 + 1 < R;
    double* xg0 = A + static_cast<size_t>(a0) * D;
    double* xg1 = A + static_cast<size_t>(two ? a0 + 1 : a0) * D;
    double x0[kRow], x1[kRow];
#pragma unroll
    for (int q = 0; q < kRow; ++q) {
      x0[q] = xg0[lane + 32 * q];
      x1[q] = xg1[lane + 32 * q];
    }
#pragma unroll
    for (int q = 0; q < kRow; ++q) {
      for (int jl = 0; jl < 32; ++jl) {
        const int j = 32 * q + jl;
        if (lane == jl) {
          x0[q] *= dinv[j];
          x1[q] *= dinv[j];
        }
        const double v0 = __shfl_sync(0xffffffffu, x0[q], jl), v1 = __shfl_sync(0xffffffffu, x1[q], jl);
#pragma unroll
        for (int q2 = q; q2 < kRow; ++q2) {
          const int i = lane + 32 * q2;
          if (i > j) {
            const double l = C[i * LD + j];
            x0[q2] = fma(-l, v0, x0[q2]);
            x1[q2] = fma(-l, v1, x1[q2]);
          }
        }
      }
    }
#pragma unroll
    for (int q = kRow - 1; q >= 0; --q) {
      for (int jl = 31; jl >= 0; --jl) {
        const int j = 32 * q + jl;
        if (lane == jl) {
          x0[q] *= dinv[j];
          x1[q] *= dinv[j];
        }
        const double v0 = __shfl_sync(0xffffffffu, x0[q], jl), v1 = __shfl_sync(0xffffffffu, x1[q], jl);
#pragma unroll
        for (int q2 = 0; q2 <= q; ++q2) {
          const int i = lane + 32 * q2;
          if (i < j) {
            const double l = C[j * LD + i];
            x0[q2] = fma(-l, v0, x0[q2]);
            x1[q2] = fma(-l, v1, x1[q2]);
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kRow; ++q) {
      xg0[lane + 32 * q] = x0[q];
      if (two) xg1[lane + 32 * q] = x1[q];
    }
  }
  __syncthreads();
  // A (R x D) into shared memory (C is free now) for b and M
  double* As = C;
  for (int x = tid; x < R * D; x += kFitThreads) As[x] = A[x];
  __syncthreads();
  for (int a = tid; a < R; a += kFitThreads) {
    double sb = 0.0;
    for (int e = 0; e < D; ++e) sb += As[static_cast<size_t>(a) * D + e] * xbar[e];
    bvec[a] = zbar[a] - sb;
  }
  __syncthreads();
  // ---- M = U_r A, beta = U_r b
  const bool failed = s_fail != 0;
  for (int x = tid; x < D * D; x += kFitThreads) {
    const int i = x / D, j = x % D;
    double sm_ = 0.0;
    for (int a = 0; a < R; ++a)
      sm_ += static_cast<double>(urow(a)[i]) * As[static_cast<size_t>(a) * D + j];
    M_out[static_cast<size_t>(head) * D * D + x] = failed ? 0.f : static_cast<float>(sm_);
  }
  for (int i = tid; i < D; i += kFitThreads) {
    double s = 0.0;
    for (int a = 0; a < R; ++a) s += static_cast<double>(urow(a)[i]) * bvec[a];
    beta_out[static_cast<size_t>(head) * D + i] = failed ? 0.f : static_cast<float>(s);
  }
  if (failed && tid == 0) record_error(status, kErrInvalidArg);
}

// O = S + S M^T + beta.  CTA: 8 tiles of 64 rows (M^T staged once), 256 threads; thread
// (ty, tx) computes rows 4 ty .. 4 ty + 3 and columns (D / 16) tx .. + D / 16 of a tile
// (register tiling: 4 + D/16 shared loads per 4 D/16 FMAs).  M^T rows are padded by 4
// floats so the staging transpose and the vector reads avoid most bank conflicts.
constexpr int kApplyTile = 64;
constexpr int kApplyTiles = 8;

template <int D, typename TO>
__global__ void __launch_bounds__(256)
    apply_kernel(const float* __restrict__ S, const float* __restrict__ M, const float* __restrict__ beta, int N,
                 TO* __restrict__ O) {
  constexpr int kCols = D / 16;  // columns per thread: 8 (D = 128) or 4 (D = 64)
  constexpr int LDM = D + 4;
  extern __shared__ __align__(16) float fsm[];
  float* Mt = fsm;                // [e][j] = M[j][e], row stride LDM
  float* rows = Mt + D * LDM;     // kApplyTile x D
  const int head = blockIdx.y, tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const float* m = M + static_cast<size_t>(head) * D * D;
  for (int x = tid; x < D * D; x += 256) Mt[(x % D) * LDM + x / D] = m[x];
  const float* s = S + static_cast<size_t>(head) * N * D;
  float bt[kCols];
#pragma unroll
  for (int c = 0; c < kCols; ++c) bt[c] = beta[static_cast<size_t>(head) * D + tx * kCols + c];
  for (int tile = 0; tile < kApplyTiles; ++tile) {
    const int row0 = (blockIdx.x * kApplyTiles + tile) * kApplyTile;
    if (row0 >= N) break;
    __syncthreads();  // previous tile's reads of `rows` are done (and Mt is staged)
    for (int x = tid * 4; x < kApplyTile * D; x += 256 * 4) {
      const int r = row0 + x / D;
      const float4 v = r < N ? *reinterpret_cast<const float4*>(s + static_cast<size_t>(r) * D + x % D)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(rows + x) = v;
    }
    __syncthreads();
    float acc[4][kCols];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int c = 0; c < kCols; ++c) acc[i][c] = rows[(ty * 4 + i) * D + tx * kCols + c] + bt[c];
    }
#pragma unroll 4
    for (int e = 0; e < D; ++e) {
      float sv[4], mv[kCols];
#pragma unroll
      for (int i = 0; i < 4; ++i) sv[i] = rows[(ty * 4 + i) * D + e];
#pragma unroll
      for (int c = 0; c < kCols; c += 4) {
        const float4 q = *reinterpret_cast<const float4*>(Mt + e * LDM + tx * kCols + c);
        mv[c] = q.x;
        mv[c + 1] = q.y;
        mv[c + 2] = q.z;
        mv[c + 3] = q.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int c = 0; c < kCols; ++c) acc[i][c] = fmaf(sv[i], mv[c], acc[i][c]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = row0 + ty * 4 + i;
      if (r >= N) break;
      TO* dst = O + (static_cast<size_t>(head) * N + r) * D + tx * kCols;
#pragma unroll
      for (int c = 0; c < kCols; ++c) dst[c] = from_f32<TO>(acc[i][c]);
    }
  }
}

template <int D, typename TO>
__global__ void probe_overwrite_kernel(const int* __restrict__ probe_idx, const float* __restrict__ probe_out,
                                       int N, int P, TO* __restrict__ O) {
  const int p = blockIdx.x, head = blockIdx.y, e = threadIdx.x;
  const int tok = probe_idx[static_cast<size_t>(head) * P + p];
  O[(static_cast<size_t>(head) * N + tok) * D + e] =
      from_f32<TO>(probe_out[(static_cast<size_t>(head) * P + p) * D + e]);
}

// e_i = |o_i - o*_i| / |o*_i| per row (one warp per row); probe rows get NaN so that
// the mean over unprobed rows the pages report can skip them.
template <typename TO>
__global__ void row_errors_kernel(const TO* __restrict__ O, const float* __restrict__ ref, int N, int d,
                                  const int* __restrict__ probe_idx, int P, float* __restrict__ err) {
  const int head = blockIdx.y;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const size_t off = (static_cast<size_t>(head) * N + row) * d;
  float num = 0.f, den = 0.f;
  for (int e = lane; e < d; e += 32) {
    const float r = ref[off + e];
    const float diff = to_f32(O[off + e]) - r;
    num += diff * diff;
    den += r * r;
  }
  num = warp_sum(num);
  den = warp_sum(den);
  if (lane == 0) err[static_cast<size_t>(head) * N + row] = sqrtf(num) / sqrtf(den);
}

__global__ void mark_probe_rows_kernel(const int* __restrict__ probe_idx, int N, int P, float* __restrict__ err) {
  const int head = blockIdx.y;
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p < P) err[static_cast<size_t>(head) * N + probe_idx[static_cast<size_t>(head) * P + p]] = __int_as_float(0x7fc00000);
}

cudaError_t launch_row_errors(const void* O, bool o_f32, const float* ref, int heads, int N, int d,
                              const int* probe_idx, int P, float* err, cudaStream_t st) {
  dim3 grid(ceil_div(N, 8), heads);
  if (o_f32) row_errors_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(O), ref, N, d, probe_idx, P, err);
  else row_errors_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(O), ref, N, d, probe_idx, P, err);
  cudaError_t e = counted(cudaGetLastError(), 1);
  if (e != cudaSuccess || P == 0 || probe_idx == nullptr) return e;
  mark_probe_rows_kernel<<<dim3(ceil_div(P, 256), heads), 256, 0, st>>>(probe_idx, N, P, err);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_fit(const float* xs, const float* dp, const float* weights, int heads, int d, int P,
                       double lambda, int rank, int weight_mode, double* scratch, float* M, float* beta,
                       int* status, cudaStream_t st) {
  const int R = rank < d ? rank : d;
  const size_t smem = fit_smem_bytes(d, P);
  if (d == 64) {
    cudaError_t e = cudaFuncSetAttribute(fit_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    fit_kernel<64><<<heads, kFitThreads, smem, st>>>(xs, dp, weights, P, lambda, R, weight_mode, scratch, M, beta, status);
  } else {
    cudaError_t e = cudaFuncSetAttribute(fit_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    fit_kernel<128><<<heads, kFitThreads, smem, st>>>(xs, dp, weights, P, lambda, R, weight_mode, scratch, M, beta, status);
  }
  return counted(cudaGetLastError(), 1);
}

size_t fit_smem_bytes(int d, int P) {
  return (static_cast<size_t>(d) * (d + 1) + P + kStageRows * d) * sizeof(double) +
         static_cast<size_t>(d) * d * sizeof(float);
}

int fit_max_probes(int d) {
  const size_t base = fit_smem_bytes(d, 0), cap = 220 * 1024;
  return base >= cap ? 0 : static_cast<int>((cap - base) / sizeof(double));
}

template <int D, typename TO>
static cudaError_t launch_apply_t(const float* S, const float* M, const float* beta, const int* probe_idx,
                                  const float* probe_out, int heads, int N, int P, TO* O, cudaStream_t st) {
  const size_t smem = (static_cast<size_t>(D) * (D + 4) + kApplyTile * D) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(apply_kernel<D, TO>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  apply_kernel<D, TO><<<dim3(ceil_div(N, kApplyTile * kApplyTiles), heads), 256, smem, st>>>(S, M, beta, N, O);
  e = counted(cudaGetLastError(), 1);
  if (e != cudaSuccess || P == 0) return e;
  probe_overwrite_kernel<D, TO><<<dim3(P, heads), D, 0, st>>>(probe_idx, probe_out, N, P, O);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_probe_overwrite_bf16(const int* probe_idx, const float* probe_out, int heads, int N, int P,
                                       __nv_bfloat16* O, cudaStream_t st) {
  if (P == 0) return cudaSuccess;
  probe_overwrite_kernel<128, __nv_bfloat16><<<dim3(P, heads), 128, 0, st>>>(probe_idx, probe_out, N, P, O);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_apply(const float* S, const float* M, const float* beta, const int* probe_idx,
                         const float* probe_out, int heads, int N, int d, int P, void* O, bool out_f32,
                         cudaStream_t st) {
  if (d == 64) {
    if (out_f32) return launch_apply_t<64, float>(S, M, beta, probe_idx, probe_out, heads, N, P, static_cast<float*>(O), st);
    return launch_apply_t<64, __nv_bfloat16>(S, M, beta, probe_idx, probe_out, heads, N, P, static_cast<__nv_bfloat16*>(O), st);
  }
  if (out_f32) return launch_apply_t<128, float>(S, M, beta, probe_idx, probe_out, heads, N, P, static_cast<float*>(O), st);
  return launch_apply_t<128, __nv_bfloat16>(S, M, beta, probe_idx, probe_out, heads, N, P, static_cast<__nv_bfloat16*>(O), st);
}

}  // namespace spr
