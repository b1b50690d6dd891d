// Response-Coupled Partitioning kernels (sm_100a).
//
// Source: SparsePR abstract (arXiv 2608.18484, arxivdaily.com English abstract): keys
// with their paired values are grouped by how they respond to sampled queries; queries
// are grouped by their responses to the resulting key-group centroids (one asymmetric
// pass, per the skillfed.io article's paragraph on the two components).
//
// Both clusterings are balanced k-means with capacity B.  Distances are evaluated in
// the exactly equivalent head-dim form
//     D[i][g] = tau^2 (x_i - c_g)^T Gamma (x_i - c_g)
//             = tau^2 (x_i^T Gamma x_i - 2 x_i . (Gamma c_g) + c_g^T Gamma c_g)
// with Gamma = Q_S^T Q_S for keys (profiles r_j = tau Q_S k_j) and Gamma = mu^T mu for
// queries (coordinates u_i = tau mu q_i); c_g is the member mean in head-dim space,
// whose image is the profile-space centroid because both maps are linear.
#include "common.cuh"
#include "fill_select.cuh"
#include "partition.cuh"
#include "warp_mma.cuh"

namespace spr {

// ----------------------------------------------------------------------- small kernels

__global__ void midpoint_stride_kernel(int* idx, int n, int count) {
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m < count) idx[m] = static_cast<int>(((2ll * m + 1) * n) / (2ll * count));
}

// Gamma[h] = sum_r x_r x_r^T over the listed rows (rows == nullptr: rows 0..nrows-1).
template <typename T, int D>
__global__ void __launch_bounds__(256) gram_kernel(const T* __restrict__ X, size_t head_stride,
                                                   const int* __restrict__ rows, int nrows,
                                                   float* __restrict__ gamma) {
  constexpr int kRowsPerThread = 16 * D / 256;
  __shared__ float sx[32][D];
  const int head = blockIdx.y;
  const int r0 = blockIdx.x * 16;
  const int col = threadIdx.x % D;
  const int rsub = (threadIdx.x / D) * kRowsPerThread;
  X += head * head_stride;
  float acc[kRowsPerThread];
#pragma unroll
  for (int i = 0; i < kRowsPerThread; ++i) acc[i] = 0.f;
  for (int s0 = 0; s0 < nrows; s0 += 32) {
    __syncthreads();
    for (int x = threadIdx.x; x < 32 * D; x += 256) {
      const int s = s0 + x / D;
      float v = 0.f;
      if (s < nrows) {
        const int r = rows ? rows[s] : s;
        v = to_f32(X[static_cast<size_t>(r) * D + x % D]);
      }
      sx[x / D][x % D] = v;
    }
    __syncthreads();
    for (int s = 0; s < 32; ++s) {
      const float xc = sx[s][col];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) acc[i] += sx[s][r0 + rsub + i] * xc;
    }
  }
#pragma unroll
  for (int i = 0; i < kRowsPerThread; ++i)
    gamma[(static_cast<size_t>(head) * D + r0 + rsub + i) * D + col] = acc[i];
}

__global__ void split_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo, size_t count) {
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < count;
       x += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float v = src[x];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[x] = h;
    if (lo) lo[x] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// perm = contiguous chunks of `cap` tokens (the k-means start), sizes accordingly.
__global__ void chunk_perm_kernel(int* __restrict__ perm, int* __restrict__ sizes, int n, int G, int cap) {
  const int head = blockIdx.y;
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < G * cap; s += gridDim.x * blockDim.x) {
    perm[static_cast<size_t>(head) * G * cap + s] = s < n ? s : -1;
    if (s % cap == 0) sizes[static_cast<size_t>(head) * G + s / cap] = min(cap, n - s);
  }
}

// c_g = fp32 mean of the members listed in perm; empty groups keep c_g.  128 threads:
// warp w sums the members j = w, w + 4, ... in list order, lane l holding dims
// [l D/32, (l + 1) D/32) (one vector load per member), and the four partial sums are
// added in warp order at the end.
template <typename T, int D>
__device__ __forceinline__ void load_dims(const T* p, float (&v)[D / 32]);
template <>
__device__ __forceinline__ void load_dims<__nv_bfloat16, 128>(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
  v[0] = a.x, v[1] = a.y, v[2] = b.x, v[3] = b.y;
}
template <>
__device__ __forceinline__ void load_dims<__nv_bfloat16, 64>(const __nv_bfloat16* p, float (&v)[2]) {
  const uint32_t r = __ldg(reinterpret_cast<const unsigned int*>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r));
  v[0] = a.x, v[1] = a.y;
}
template <>
__device__ __forceinline__ void load_dims<float, 128>(const float* p, float (&v)[4]) {
  const float4 r = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = r.x, v[1] = r.y, v[2] = r.z, v[3] = r.w;
}
template <>
__device__ __forceinline__ void load_dims<float, 64>(const float* p, float (&v)[2]) {
  const float2 r = __ldg(reinterpret_cast<const float2*>(p));
  v[0] = r.x, v[1] = r.y;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) centroid_kernel(const T* __restrict__ X, int n, const int* __restrict__ perm,
                                                       const int* __restrict__ sizes, int G, int cap,
                                                       float* __restrict__ cent) {
  constexpr int kPer = D / 32;
  __shared__ float part[4][D];
  const int g = blockIdx.x, head = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t goff = static_cast<size_t>(head) * G + g;
  const int size = sizes[goff];
  if (size <= 0) return;
  const T* x = X + static_cast<size_t>(head) * n * D + lane * kPer;
  const int* pm = perm + goff * cap;
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
#pragma unroll 4
  for (int j = warp; j < size; j += 4) {
    float v[kPer];
    load_dims<T, D>(x + static_cast<size_t>(__ldg(pm + j)) * D, v);
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] += v[i];
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) part[warp][lane * kPer + i] = acc[i];
  __syncthreads();
  for (int e = threadIdx.x; e < D; e += 128)
    cent[goff * D + e] = (((part[0][e] + part[1][e]) + part[2][e]) + part[3][e]) / static_cast<float>(size);
}

// W = C Gamma (fp32 + bf16 hi/lo) and e_g = c_g . w_g; 8 groups per CTA, thread per dim.
template <int D>
__global__ void wmat_kernel(const float* __restrict__ cent, const float* __restrict__ gamma, int G,
                            float* __restrict__ wf, __nv_bfloat16* __restrict__ whi,
                            __nv_bfloat16* __restrict__ wlo, float* __restrict__ eg) {
  __shared__ float sc[8][D];
  __shared__ float red[8][D / 32];
  const int head = blockIdx.y, g0 = blockIdx.x * 8, e = threadIdx.x;
  const float* gm = gamma + static_cast<size_t>(head) * D * D;
  for (int j = 0; j < 8; ++j)
    sc[j][e] = g0 + j < G ? cent[(static_cast<size_t>(head) * G + g0 + j) * D + e] : 0.f;
  __syncthreads();
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int f = 0; f < D; ++f) {
    const float gv = gm[f * D + e];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += sc[j][f] * gv;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float part = warp_sum(acc[j] * sc[j][e]);
    if ((e & 31) == 0) red[j][e >> 5] = part;
  }
  __syncthreads();
  for (int j = 0; j < 8; ++j) {
    const int g = g0 + j;
    if (g >= G) break;
    const size_t o = (static_cast<size_t>(head) * G + g) * D + e;
    wf[o] = acc[j];
    const __nv_bfloat16 h = __float2bfloat16_rn(acc[j]);
    whi[o] = h;
    wlo[o] = __float2bfloat16_rn(acc[j] - __bfloat162float(h));
    if (e == 0) {
      float s = 0.f;
      for (int w = 0; w < D / 32; ++w) s += red[j][w];
      eg[static_cast<size_t>(head) * G + g] = s;
    }
  }
}

// One k-means iteration's group update, 8 groups of one head per CTA (256 threads): warp
// j sorts group g0 + j's members (the unsorted lists tmp[g * cap + slot], cursor[g] of
// them) into ascending token order by a shared-memory bitonic sort, writes perm and
// sizes, and sums the member rows in that order for the fp32 mean c_g (an empty group
// keeps its c_g); then W = C Gamma (fp32 and bf16 hi/lo) and e_g = c_g . w_g with the
// arithmetic of wmat_kernel.
template <typename T, int D>
__global__ void __launch_bounds__(256) group_update_kernel(const T* __restrict__ X, int n,
                                                           const int* __restrict__ cursor,
                                                           const int* __restrict__ tmp, int G, int cap,
                                                           const float* __restrict__ gamma, int* __restrict__ perm,
                                                           int* __restrict__ sizes, float* __restrict__ cent,
                                                           float* __restrict__ wf, __nv_bfloat16* __restrict__ whi,
                                                           __nv_bfloat16* __restrict__ wlo, float* __restrict__ eg) {
  constexpr int kPer = D / 32, kSets = 256 / D, kPerSet = 8 / kSets;
  constexpr int kGRows = 32;  // rows of Gamma staged at a time
  __shared__ int sv[8][128];
  __shared__ float sg[kGRows][D];
  __shared__ float sc[8][D];
  __shared__ float red[8][D / 32];
  const int head = blockIdx.y, g0 = blockIdx.x * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    // ---- members of group g0 + warp, sorted
    const int g = g0 + warp;
    const size_t gi = static_cast<size_t>(head) * G + g;
    const int size = g < G ? min(cursor[gi], cap) : 0;
    for (int t = lane; t < cap; t += 32) sv[warp][t] = t < size ? tmp[gi * cap + t] : 0x7fffffff;
    __syncwarp();
    for (int k = 2; k <= cap; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int t = lane; t < cap; t += 32) {
          const int p = t ^ j;
          if (p > t) {
            const int a = sv[warp][t], b = sv[warp][p];
            const bool up = (t & k) == 0;
            if ((a > b) == up) {
              sv[warp][t] = b;
              sv[warp][p] = a;
            }
          }
        }
        __syncwarp();
      }
    }
    if (g < G) {
      for (int t = lane; t < cap; t += 32) perm[gi * cap + t] = t < size ? sv[warp][t] : -1;
      if (lane == 0) sizes[gi] = size;
    }
    // ---- c_g: lane l sums dims [l kPer, (l + 1) kPer) over the members in token order
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
    const T* x = X + static_cast<size_t>(head) * n * D + lane * kPer;
#pragma unroll 8
    for (int j = 0; j < size; ++j) {
      float v[kPer];
      load_dims<T, D>(x + static_cast<size_t>(sv[warp][j]) * D, v);
#pragma unroll
      for (int i = 0; i < kPer; ++i) acc[i] += v[i];
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane * kPer + i;
      float c = 0.f;
      if (g < G) {
        c = size > 0 ? acc[i] / static_cast<float>(size) : cent[gi * D + e];
        if (size > 0) cent[gi * D + e] = c;
      }
      sc[warp][e] = c;
    }
  }
  __syncthreads();
  // ---- W = C Gamma and e_g, thread (set, e): groups set * kPerSet + j
  const int e = threadIdx.x % D, set = threadIdx.x / D;
  const float* gm = gamma + static_cast<size_t>(head) * D * D;
  float acc[kPerSet];
#pragma unroll
  for (int j = 0; j < kPerSet; ++j) acc[j] = 0.f;
  for (int f0 = 0; f0 < D; f0 += kGRows) {
    for (int x = threadIdx.x; x < kGRows * D; x += 256) sg[x / D][x % D] = __ldg(gm + f0 * D + x);
    __syncthreads();
#pragma unroll 8
    for (int f = 0; f < kGRows; ++f) {
      const float gv = sg[f][e];
#pragma unroll
      for (int j = 0; j < kPerSet; ++j) acc[j] += sc[set * kPerSet + j][f0 + f] * gv;
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < kPerSet; ++j) {
    const float part = warp_sum(acc[j] * sc[set * kPerSet + j][e]);
    if ((e & 31) == 0) red[set * kPerSet + j][e >> 5] = part;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPerSet; ++j) {
    const int gl = set * kPerSet + j, g = g0 + gl;
    if (g >= G) break;
    const size_t o = (static_cast<size_t>(head) * G + g) * D + e;
    wf[o] = acc[j];
    const __nv_bfloat16 h = __float2bfloat16_rn(acc[j]);
    whi[o] = h;
    wlo[o] = __float2bfloat16_rn(acc[j] - __bfloat162float(h));
    if (e == 0) {
      float s = 0.f;
      for (int w = 0; w < D / 32; ++w) s += red[gl][w];
      eg[static_cast<size_t>(head) * G + g] = s;
    }
  }
}

// ---------------------------------------------------------------- row GEMM (tensor core)
// acc[i][c] = x_i . B_c over a 128-row tile; all columns streamed in chunks of 64.
//   NORM: out[i] = sum_c acc[i][c] * x_i[c]        (x_i^T Gamma x_i, B = Gamma)
//   DIST: D[i][c] = tau2 (nrm_i - 2 acc + e_c), written in full, plus the row argmin
//         (ties to the lower column) as the first proposal of the capacity fill.
constexpr int kGemmRows = 128;
constexpr int kGemmCols = 64;

template <int D, bool DIST, bool SPLIT>
__global__ void __launch_bounds__(256)
    rowgemm_mma_kernel(const __nv_bfloat16* __restrict__ X, int n, const __nv_bfloat16* __restrict__ Bhi,
                       const __nv_bfloat16* __restrict__ Blo, int ncols, const float* __restrict__ nrm,
                       const float* __restrict__ ecol, float tau2, float* __restrict__ Dout, int ldd,
                       int* __restrict__ prop_g, float* __restrict__ prop_v, float* __restrict__ nrm_out,
                       int* __restrict__ status) {
  constexpr int kCh = D / 8;
  constexpr int kBStage = kGemmCols * D * 2;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sX = smem;
  uint8_t* sB = sX + kGemmRows * D * 2;  // [2 stages][hi, lo]
  const int head = blockIdx.y;
  const int row0 = blockIdx.x * kGemmRows;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  X += static_cast<size_t>(head) * n * D;
  Bhi += static_cast<size_t>(head) * ncols * D;
  if (SPLIT) Blo += static_cast<size_t>(head) * ncols * D;

  for (int x = tid; x < kGemmRows * kCh; x += 256) {
    const int r = x / kCh, ch = x % kCh;
    const int row = row0 + r;
    cp_async_16(smem_u32(sX) + swz<D>(r, ch), row < n ? X + static_cast<size_t>(row) * D + ch * 8 : X,
                row < n ? 16 : 0);
  }
  cp_async_commit();
  const int n_chunks = ceil_div(ncols, kGemmCols);
  auto load_chunk = [&](int t) {
    const uint32_t base = smem_u32(sB) + (t & 1) * kBStage * (SPLIT ? 2 : 1);
    for (int x = tid; x < kGemmCols * kCh; x += 256) {
      const int c = x / kCh, ch = x % kCh;
      const int col = t * kGemmCols + c;
      const size_t off = col < ncols ? static_cast<size_t>(col) * D + ch * 8 : 0;
      cp_async_16(base + swz<D>(c, ch), Bhi + off, col < ncols ? 16 : 0);
      if (SPLIT) cp_async_16(base + kBStage + swz<D>(c, ch), Blo + off, col < ncols ? 16 : 0);
    }
  };
  load_chunk(0);
  cp_async_commit();

  const int g8 = lane >> 2, t4 = lane & 3;
  const int rloc[2] = {warp * 16 + g8, warp * 16 + g8 + 8};
  float nrm_row[2] = {0.f, 0.f};
  if (DIST) {
    const float* nr = nrm + static_cast<size_t>(head) * n;
    nrm_row[0] = row0 + rloc[0] < n ? nr[row0 + rloc[0]] : 0.f;
    nrm_row[1] = row0 + rloc[1] < n ? nr[row0 + rloc[1]] : 0.f;
  }
  unsigned long long best[2] = {~0ull, ~0ull};
  float part[2] = {0.f, 0.f};
  bool saw_nan = false;
  uint32_t af[D / 16][4];

  for (int t = 0; t < n_chunks; ++t) {
    if (t + 1 < n_chunks) load_chunk(t + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldmatrix_x4(af[kk], smem_u32(sX) + swz<D>(warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                                                   kk * 2 + (lane >> 4)));
    }
    const uint32_t base = smem_u32(sB) + (t & 1) * kBStage * (SPLIT ? 2 : 1);
    float acc[kGemmCols / 8][4];
#pragma unroll
    for (int i = 0; i < kGemmCols / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
    for (int part_i = 0; part_i < (SPLIT ? 2 : 1); ++part_i) {
      const uint32_t bb = base + part_i * kBStage;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int nt2 = 0; nt2 < kGemmCols / 16; ++nt2) {
          uint32_t bf[4];
          ldmatrix_x4(bf, bb + swz<D>(nt2 * 16 + (lane & 7) + (lane >> 4) * 8, kk * 2 + ((lane >> 3) & 1)));
          mma_bf16_16816(acc[2 * nt2], af[kk], &bf[0]);
          mma_bf16_16816(acc[2 * nt2 + 1], af[kk], &bf[2]);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < kGemmCols / 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int h = c >> 1;
        const int cl = nt * 8 + 2 * t4 + (c & 1);
        const int col = t * kGemmCols + cl;
        const int row = row0 + rloc[h];
        if (DIST) {
          const float v = tau2 * (nrm_row[h] - 2.f * acc[nt][c] + __ldg(ecol + static_cast<size_t>(head) * ncols + min(col, ncols - 1)));
          if (col < ncols && row < n) {
            saw_nan |= (v != v);
            const unsigned long long key = decision_key(v, col);
            best[h] = key < best[h] ? key : best[h];
            acc[nt][c] = v;
          }
        } else {
          if (col < ncols) {
            const int ch = col >> 3;
            const __nv_bfloat16* xr = reinterpret_cast<const __nv_bfloat16*>(sX + swz<D>(rloc[h], ch));
            part[h] += acc[nt][c] * __bfloat162float(xr[col & 7]);
          }
        }
      }
    }
    if (DIST) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = row0 + rloc[h];
        if (row >= n) continue;
        float* drow = Dout + (static_cast<size_t>(head) * n + row) * ldd;
#pragma unroll
        for (int nt = 0; nt < kGemmCols / 8; ++nt) {
          const int col = t * kGemmCols + nt * 8 + 2 * t4;
          if (col + 1 < ncols && (ldd % 2 == 0)) {
            *reinterpret_cast<float2*>(drow + col) = make_float2(acc[nt][2 * h], acc[nt][2 * h + 1]);
          } else {
            if (col < ncols) drow[col] = acc[nt][2 * h];
            if (col + 1 < ncols) drow[col + 1] = acc[nt][2 * h + 1];
          }
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = row0 + rloc[h];
    if (DIST) {
      unsigned long long b = best[h];
      const unsigned long long b1 = __shfl_xor_sync(0xffffffffu, b, 1);
      b = b1 < b ? b1 : b;
      const unsigned long long b2 = __shfl_xor_sync(0xffffffffu, b, 2);
      b = b2 < b ? b2 : b;
      if (t4 == 0 && row < n) {
        const size_t o = static_cast<size_t>(head) * n + row;
        const int col = static_cast<int>(b & 0xffffffffu);
        prop_g[o] = col;
        prop_v[o] = Dout[o * ldd + col];
      }
    } else {
      float p = part[h];
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      if (t4 == 0 && row < n) nrm_out[static_cast<size_t>(head) * n + row] = p;
    }
  }
  if (DIST && saw_nan) record_error(status, kErrNonFinite);
}

// fp32 inputs: the same row GEMM in exact fp32 (SIMT), one warp per row.
template <int D, bool DIST>
__global__ void __launch_bounds__(256)
    rowgemm_f32_kernel(const float* __restrict__ X, int n, const float* __restrict__ B, int ncols,
                       const float* __restrict__ nrm, const float* __restrict__ ecol, float tau2,
                       float* __restrict__ Dout, int ldd, int* __restrict__ prop_g, float* __restrict__ prop_v,
                       float* __restrict__ nrm_out, int* __restrict__ status) {
  const int head = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= n) return;
  const float* x = X + (static_cast<size_t>(head) * n + row) * D;
  const float* b = B + static_cast<size_t>(head) * ncols * D;
  float xr[D / 32];
#pragma unroll
  for (int i = 0; i < D / 32; ++i) xr[i] = x[lane + 32 * i];
  unsigned long long best = ~0ull;
  float nsum = 0.f;
  bool saw_nan = false;
  for (int c = 0; c < ncols; ++c) {
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) dot += xr[i] * b[static_cast<size_t>(c) * D + lane + 32 * i];
    dot = warp_sum(dot);
    if (DIST) {
      const float v = tau2 * (nrm[static_cast<size_t>(head) * n + row] - 2.f * dot + ecol[static_cast<size_t>(head) * ncols + c]);
      if (lane == 0) Dout[(static_cast<size_t>(head) * n + row) * ldd + c] = v;
      saw_nan |= (v != v);
      const unsigned long long key = decision_key(v, c);
      best = key < best ? key : best;
    } else {
      nsum += dot * x[c];
    }
  }
  if (lane == 0) {
    const size_t o = static_cast<size_t>(head) * n + row;
    if (DIST) {
      const int col = static_cast<int>(best & 0xffffffffu);
      prop_g[o] = col;
      prop_v[o] = Dout[o * ldd + col];
      if (saw_nan) record_error(status, kErrNonFinite);
    } else {
      nrm_out[o] = nsum;
    }
  }
}

// --------------------------------------------------------------- capacity-constrained fill
// Rounds: every unplaced item proposes to its nearest group with room (ties -> lower
// group); each group accepts its proposers in ascending (distance, token) order while
// it has room.  One cooperative launch runs every round for every head.  Full groups
// are tracked in a per-head bitmap so a proposal reads only its distance row.

__global__ void fill_init_kernel(FillArgs a) {
  const size_t items = static_cast<size_t>(a.heads) * a.n;
  const size_t groups = static_cast<size_t>(a.heads) * a.G;
  const size_t words = static_cast<size_t>(a.heads) * ((a.G + 31) / 32);
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < items;
       x += static_cast<size_t>(gridDim.x) * blockDim.x) {
    a.labels[x] = -1;
    a.list0[x] = static_cast<int>(x);
  }
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < groups;
       x += static_cast<size_t>(gridDim.x) * blockDim.x) {
    a.room[x] = a.cap;
    a.cnt[x] = 0;
    a.cursor[x] = 0;
  }
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < words;
       x += static_cast<size_t>(gridDim.x) * blockDim.x)
    a.closed[x] = 0u;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    a.list_len[0] = static_cast<int>(items);
    a.list_len[1] = 0;
  }
}

constexpr int kFillThreads = 256;
constexpr size_t kFillStageLimit = 64 * 1024;  // bytes of full-group bitmaps staged per block

// MAXW = 32-group words of a distance row held per lane (G <= 32 MAXW).
template <int MAXW>
__global__ void __launch_bounds__(kFillThreads, 3) fill_coop_kernel(FillArgs a) {
  __shared__ unsigned int hist[kFillThreads / 32][256];
  __shared__ int scan_tmp[kFillThreads];
  extern __shared__ unsigned int s_closed[];  // [heads * words] when a.stage_closed
  const unsigned int nblocks = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gthread = blockIdx.x * kFillThreads + tid;
  const int nthreads = nblocks * kFillThreads;
  const int gwarp = gthread >> 5;
  const int nwarps = nthreads >> 5;
  const int n = a.n, G = a.G;
  const int words = (G + 31) / 32;
  int* lists[2] = {a.list0, a.list1};
  int cur = 0;
  const int max_rounds = n + 2;
  for (int round = 0;; ++round) {
    const int ncur = __ldcg(a.list_len + cur);
    const int* L = lists[cur];
    // ---- propose
    if (round == 0 && a.prop_g0 != nullptr) {
      // first proposals: the row argmins the distance kernel found
      for (int x = gthread; x < ncur; x += nthreads) {
        const int item = __ldcg(L + x);
        const int h = item / n;
        const int g = a.prop_g0[item];
        a.prop_g[item] = g;
        a.prop_v[item] = a.prop_v0[item];
        atomicAdd(a.cnt + static_cast<size_t>(h) * G + g, 1);
      }
    } else {
      // The full-group bitmaps of all heads are staged in shared memory once per round
      // (when they fit), so a proposal waits only for its own distance row.
      const unsigned int* closed_all = a.closed;
      if (a.stage_closed) {
        for (int x = tid; x < a.heads * words; x += kFillThreads) s_closed[x] = __ldcg(a.closed + x);
        __syncthreads();
        closed_all = s_closed;
      }
      // One item per warp, with the item's whole distance row (up to MAXW values per
      // lane) requested before any is used; full-group bitmap words are warp-uniform.
      for (int x = gwarp; x < ncur; x += nwarps) {
        const int item = __ldcg(L + x);
        const int h = item / n;
        const float* drow = a.D + static_cast<size_t>(item) * a.ldd;
        const unsigned int* closed = closed_all + static_cast<size_t>(h) * words;
        float v[MAXW];
#pragma unroll
        for (int u = 0; u < MAXW; ++u) {
          const int g = u * 32 + lane;
          v[u] = g < G ? __ldcg(drow + g) : 0.f;
        }
        unsigned long long best = ~0ull;
        bool saw_nan = false;
#pragma unroll
        for (int u = 0; u < MAXW; ++u) {
          const int g = u * 32 + lane;
          if (u < words && g < G && !(((a.stage_closed ? closed[u] : __ldcg(closed + u)) >> lane) & 1u)) {
            saw_nan |= (v[u] != v[u]);
            const unsigned long long key = decision_key(v[u], g);
            best = key < best ? key : best;
          }
        }
        best = warp_min_u64(best);
        saw_nan = __any_sync(0xffffffffu, saw_nan);
        if (lane == 0) {
          if (saw_nan) record_error(&a.hdr->status, kErrNonFinite);
          if (best == ~0ull) {
            record_error(&a.hdr->status, kErrInvalidArg);
          } else {
            const int g = static_cast<int>(best & 0xffffffffu);
            a.prop_g[item] = g;
            a.prop_v[item] = __ldcg(drow + g);
            atomicAdd(a.cnt + static_cast<size_t>(h) * G + g, 1);
          }
        }
      }
    }
    if (!grid_barrier(a.hdr, nblocks)) return;
    // ---- bucket offsets (exclusive scan of counts, per head)
    for (int h = blockIdx.x; h < a.heads; h += nblocks) {
      const int* cnt = a.cnt + static_cast<size_t>(h) * G;
      int* offs = a.offs + static_cast<size_t>(h) * G;
      const int per = ceil_div(G, kFillThreads);
      const int g0 = tid * per;
      int local = 0;
      for (int g = g0; g < min(G, g0 + per); ++g) local += __ldcg(cnt + g);
      scan_tmp[tid] = local;
      __syncthreads();
      for (int o = 1; o < kFillThreads; o <<= 1) {
        const int y = tid >= o ? scan_tmp[tid - o] : 0;
        __syncthreads();
        scan_tmp[tid] += y;
        __syncthreads();
      }
      int run = scan_tmp[tid] - local;
      for (int g = g0; g < min(G, g0 + per); ++g) {
        offs[g] = run;
        run += __ldcg(cnt + g);
      }
      __syncthreads();
    }
    if (!grid_barrier(a.hdr, nblocks)) return;
    // ---- scatter proposals into per-group buckets
    for (int x = gthread; x < ncur; x += nthreads) {
      const int item = __ldcg(L + x);
      const int h = item / n;
      const int i = item - h * n;
      const int g = __ldcg(a.prop_g + item);
      const size_t gi = static_cast<size_t>(h) * G + g;
      const int slot = atomicAdd(a.cursor + gi, 1);
      a.bucket[static_cast<size_t>(h) * n + __ldcg(a.offs + gi) + slot] = decision_key(__ldcg(a.prop_v + item), i);
    }
    if (!grid_barrier(a.hdr, nblocks)) return;
    // ---- each group accepts its best proposers while it has room
    const int next = cur ^ 1;
    for (int x = gwarp; x < a.heads * G; x += nwarps) {
      const int c = __ldcg(a.cnt + x);
      if (c == 0) continue;
      const int h = x / G, g = x - h * G;
      const int r = __ldcg(a.room + x);
      const unsigned long long* bk = a.bucket + static_cast<size_t>(h) * n + __ldcg(a.offs + x);
      int* lab = a.labels + static_cast<size_t>(h) * n;
      const unsigned long long thr = c <= r ? ~0ull : warp_select_kth(bk, c, r, hist[warp]);
      for (int e0 = 0; e0 < c; e0 += 256) {
        unsigned long long kb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = e0 + u * 32 + lane;
          kb[u] = e < c ? __ldcg(bk + e) : ~0ull;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (e0 + u * 32 + lane >= c) continue;
          const int i = static_cast<int>(kb[u] & 0xffffffffu);
          if (kb[u] <= thr) {
            lab[i] = g;
          } else {
            const int pos = atomicAdd(a.list_len + next, 1);
            lists[next][pos] = h * n + i;
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        const int left = r - min(c, r);
        a.room[x] = left;
        a.cnt[x] = 0;
        a.cursor[x] = 0;
        if (left == 0) atomicOr(a.closed + static_cast<size_t>(h) * words + g / 32, 1u << (g % 32));
      }
    }
    if (!grid_barrier(a.hdr, nblocks)) return;
    if (__ldcg(a.list_len + next) == 0) break;
    if (round >= max_rounds) {
      if (gthread == 0) record_error(&a.hdr->status, kErrTimeout);
      return;
    }
    if (gthread == 0) a.list_len[cur] = 0;
    cur = next;
  }
}

// ----------------------------------------------------------------- labels -> permutation
__global__ void perm_scatter_kernel(const int* __restrict__ labels, int n, int G, int cap,
                                    int* __restrict__ cursor, int* __restrict__ tmp, int heads,
                                    int* __restrict__ status) {
  const size_t items = static_cast<size_t>(heads) * n;
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < items;
       x += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int h = static_cast<int>(x / n);
    const int i = static_cast<int>(x - static_cast<size_t>(h) * n);
    const int g = labels[x];
    if (g < 0 || g >= G) {
      record_error(status, kErrInvalidArg);
      continue;
    }
    const size_t gi = static_cast<size_t>(h) * G + g;
    const int slot = atomicAdd(cursor + gi, 1);
    if (slot < cap) tmp[gi * cap + slot] = i;
    else record_error(status, kErrInvalidArg);
  }
}

// Sort each group's members by token (bitonic, cap = power of two <= 1024).
__global__ void perm_sort_kernel(const int* __restrict__ cursor, const int* __restrict__ tmp, int G,
                                 int cap, int* __restrict__ perm, int* __restrict__ sizes) {
  extern __shared__ int sv[];
  const int g = blockIdx.x, head = blockIdx.y, t = threadIdx.x;
  const size_t gi = static_cast<size_t>(head) * G + g;
  const int size = min(cursor[gi], cap);
  sv[t] = t < size ? tmp[gi * cap + t] : 0x7fffffff;
  __syncthreads();
  for (int k = 2; k <= cap; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int p = t ^ j;
      if (p > t) {
        const int a = sv[t], b = sv[p];
        const bool up = (t & k) == 0;
        if ((a > b) == up) {
          sv[t] = b;
          sv[p] = a;
        }
      }
      __syncthreads();
    }
  }
  perm[gi * cap + t] = t < size ? sv[t] : -1;
  if (t == 0) sizes[gi] = size;
}

// Sc[b][g] = tau * qbar_b . mu_g: a 64 x 64 output tile per CTA, 4 x 4 per thread, the
// dimension staged 32 at a time; every dot product is summed in ascending dimension order
// by fused multiply-adds.
template <int D>
__global__ void __launch_bounds__(256) block_score_kernel(const float* __restrict__ qbar, const float* __restrict__ mu,
                                                          int G, float tau, float* __restrict__ sc) {
  __shared__ float sa[32][65], sb[32][65];  // [dimension][row]
  const int head = blockIdx.z;
  const int b0 = blockIdx.y * 64, g0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int e0 = 0; e0 < D; e0 += 32) {
    for (int x = threadIdx.x; x < 64 * 32; x += 256) {
      const int r = x >> 5, e = x & 31;
      sa[e][r] = b0 + r < G ? qbar[(static_cast<size_t>(head) * G + b0 + r) * D + e0 + e] : 0.f;
      sb[e][r] = g0 + r < G ? mu[(static_cast<size_t>(head) * G + g0 + r) * D + e0 + e] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int e = 0; e < 32; ++e) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = sa[e][ty + 16 * i];
        bv[i] = sb[e][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = b0 + ty + 16 * i;
    if (b >= G) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int g = g0 + tx + 16 * j;
      if (g < G) sc[(static_cast<size_t>(head) * G + b) * G + g] = tau * acc[i][j];
    }
  }
}

// ----------------------------------------------------------------------------- launchers


__global__ void identity_kernel(float* __restrict__ gamma, int heads, int d) {
  const size_t total = static_cast<size_t>(heads) * d * d;
  for (size_t x = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; x < total;
       x += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t e = x % (static_cast<size_t>(d) * d);
    gamma[x] = (e / d == e % d) ? 1.0f : 0.0f;
  }
}

cudaError_t launch_identity(float* gamma, int heads, int d, cudaStream_t st) {
  identity_kernel<<<ceil_div(heads * d * d, 256), 256, 0, st>>>(gamma, heads, d);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_midpoint_stride(int* idx, int n, int count, cudaStream_t st) {
  midpoint_stride_kernel<<<ceil_div(count, 256), 256, 0, st>>>(idx, n, count);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_gram(const void* X, bool f32, size_t head_stride, const int* rows, int nrows, int heads,
                        int d, float* gamma, cudaStream_t st) {
  dim3 grid(d / 16, heads);
  if (f32) {
    if (d == 64) gram_kernel<float, 64><<<grid, 256, 0, st>>>(static_cast<const float*>(X), head_stride, rows, nrows, gamma);
    else gram_kernel<float, 128><<<grid, 256, 0, st>>>(static_cast<const float*>(X), head_stride, rows, nrows, gamma);
  } else {
    if (d == 64) gram_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), head_stride, rows, nrows, gamma);
    else gram_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), head_stride, rows, nrows, gamma);
  }
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_split_bf16(const float* src, __nv_bfloat16* hi, __nv_bfloat16* lo, size_t count, cudaStream_t st) {
  const int blocks = static_cast<int>(std::min<size_t>(4096, (count + 255) / 256));
  split_bf16_kernel<<<blocks, 256, 0, st>>>(src, hi, lo, count);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_chunk_perm(int* perm, int* sizes, int n, int G, int cap, int heads, cudaStream_t st) {
  chunk_perm_kernel<<<dim3(ceil_div(G * cap, 256), heads), 256, 0, st>>>(perm, sizes, n, G, cap);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_centroid(const void* X, bool f32, int n, const int* perm, const int* sizes, int G, int cap,
                            int heads, int d, float* cent, cudaStream_t st) {
  dim3 grid(G, heads);
  if (f32) {
    if (d == 64) centroid_kernel<float, 64><<<grid, 128, 0, st>>>(static_cast<const float*>(X), n, perm, sizes, G, cap, cent);
    else centroid_kernel<float, 128><<<grid, 128, 0, st>>>(static_cast<const float*>(X), n, perm, sizes, G, cap, cent);
  } else {
    if (d == 64) centroid_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(X), n, perm, sizes, G, cap, cent);
    else centroid_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(X), n, perm, sizes, G, cap, cent);
  }
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_wmat(const float* cent, const float* gamma, int G, int heads, int d, float* wf,
                        __nv_bfloat16* whi, __nv_bfloat16* wlo, float* eg, cudaStream_t st) {
  dim3 grid(ceil_div(G, 8), heads);
  if (d == 64) wmat_kernel<64><<<grid, 64, 0, st>>>(cent, gamma, G, wf, whi, wlo, eg);
  else wmat_kernel<128><<<grid, 128, 0, st>>>(cent, gamma, G, wf, whi, wlo, eg);
  return counted(cudaGetLastError(), 1);
}

template <int D, bool DIST, bool SPLIT>
static cudaError_t launch_rowgemm_mma_t(const RowGemmArgs& a, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(kGemmRows) * D * 2 + 2ull * kGemmCols * D * 2 * (SPLIT ? 2 : 1);
  auto kern = rowgemm_mma_kernel<D, DIST, SPLIT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(ceil_div(a.n, kGemmRows), a.heads), 256, smem, st>>>(
      static_cast<const __nv_bfloat16*>(a.X), a.n, a.Bhi, a.Blo, a.ncols, a.nrm, a.ecol, a.tau2, a.Dout, a.ldd,
      a.prop_g, a.prop_v, a.nrm_out, a.status);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_rowgemm(const RowGemmArgs& a, bool dist, cudaStream_t st) {
  if (a.f32) {
    dim3 grid(ceil_div(a.n, 8), a.heads);
    const float* X = static_cast<const float*>(a.X);
    if (a.d == 64) {
      if (dist) rowgemm_f32_kernel<64, true><<<grid, 256, 0, st>>>(X, a.n, a.Bf32, a.ncols, a.nrm, a.ecol, a.tau2, a.Dout, a.ldd, a.prop_g, a.prop_v, a.nrm_out, a.status);
      else rowgemm_f32_kernel<64, false><<<grid, 256, 0, st>>>(X, a.n, a.Bf32, a.ncols, a.nrm, a.ecol, a.tau2, a.Dout, a.ldd, a.prop_g, a.prop_v, a.nrm_out, a.status);
    } else {
      if (dist) rowgemm_f32_kernel<128, true><<<grid, 256, 0, st>>>(X, a.n, a.Bf32, a.ncols, a.nrm, a.ecol, a.tau2, a.Dout, a.ldd, a.prop_g, a.prop_v, a.nrm_out, a.status);
      else rowgemm_f32_kernel<128, false><<<grid, 256, 0, st>>>(X, a.n, a.Bf32, a.ncols, a.nrm, a.ecol, a.tau2, a.Dout, a.ldd, a.prop_g, a.prop_v, a.nrm_out, a.status);
    }
    return counted(cudaGetLastError(), 1);
  }
  const bool split = a.Blo != nullptr;
  if (a.d == 64) {
    if (dist) return split ? launch_rowgemm_mma_t<64, true, true>(a, st) : launch_rowgemm_mma_t<64, true, false>(a, st);
    return split ? launch_rowgemm_mma_t<64, false, true>(a, st) : launch_rowgemm_mma_t<64, false, false>(a, st);
  }
  if (dist) return split ? launch_rowgemm_mma_t<128, true, true>(a, st) : launch_rowgemm_mma_t<128, true, false>(a, st);
  return split ? launch_rowgemm_mma_t<128, false, true>(a, st) : launch_rowgemm_mma_t<128, false, false>(a, st);
}

cudaError_t launch_fill(const FillArgs& a, cudaStream_t st) {
  fill_init_kernel<<<1024, 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(&a.hdr->barrier_count, 0, 2 * sizeof(unsigned int), st);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int words = ceil_div(a.G, 32);
  if (words > 32) return cudaErrorInvalidValue;
  void* kern = words <= 8 ? reinterpret_cast<void*>(fill_coop_kernel<8>)
               : words <= 20 ? reinterpret_cast<void*>(fill_coop_kernel<20>)
                             : reinterpret_cast<void*>(fill_coop_kernel<32>);
  FillArgs args = a;
  const size_t closed_bytes = sizeof(unsigned int) * static_cast<size_t>(a.heads) * words;
  args.stage_closed = closed_bytes <= kFillStageLimit ? 1 : 0;
  args.d_vec4 = (a.ldd % 4 == 0 && (reinterpret_cast<uintptr_t>(a.D) & 15u) == 0) ? 1 : 0;
  const size_t smem = args.stage_closed ? closed_bytes : 0;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFillThreads, smem);
  if (e != cudaSuccess) return e;
  const int blocks = sms * std::min(per_sm, 4);
  void* params[] = {&args};
  e = cudaLaunchCooperativeKernel(kern, dim3(blocks), dim3(kFillThreads), params, smem, st);
  return counted(e, 2);
}

cudaError_t launch_build_perm(const int* labels, int n, int G, int cap, int heads, int* cursor, int* tmp,
                              int* perm, int* sizes, int* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(cursor, 0, static_cast<size_t>(heads) * G * sizeof(int), st);
  if (e != cudaSuccess) return e;
  perm_scatter_kernel<<<1024, 256, 0, st>>>(labels, n, G, cap, cursor, tmp, heads, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  perm_sort_kernel<<<dim3(G, heads), cap, cap * sizeof(int), st>>>(cursor, tmp, G, cap, perm, sizes);
  return counted(cudaGetLastError(), 2);
}

cudaError_t launch_group_update(const void* X, bool f32, int n, const int* cursor, const int* tmp, int G, int cap,
                                int heads, int d, const float* gamma, int* perm, int* sizes, float* cent, float* wf,
                                __nv_bfloat16* whi, __nv_bfloat16* wlo, float* eg, cudaStream_t st) {
  if (cap > 128 || (cap & (cap - 1)) != 0) return cudaErrorInvalidValue;
  dim3 grid(ceil_div(G, 8), heads);
  if (f32) {
    if (d == 64)
      group_update_kernel<float, 64><<<grid, 256, 0, st>>>(static_cast<const float*>(X), n, cursor, tmp, G, cap, gamma,
                                                           perm, sizes, cent, wf, whi, wlo, eg);
    else
      group_update_kernel<float, 128><<<grid, 256, 0, st>>>(static_cast<const float*>(X), n, cursor, tmp, G, cap,
                                                            gamma, perm, sizes, cent, wf, whi, wlo, eg);
  } else {
    if (d == 64)
      group_update_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), n, cursor,
                                                                   tmp, G, cap, gamma, perm, sizes, cent, wf, whi,
                                                                   wlo, eg);
    else
      group_update_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), n, cursor,
                                                                    tmp, G, cap, gamma, perm, sizes, cent, wf, whi,
                                                                    wlo, eg);
  }
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_perm_scatter(const int* labels, int n, int G, int cap, int heads, int* cursor, int* tmp,
                                int* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(cursor, 0, static_cast<size_t>(heads) * G * sizeof(int), st);
  if (e != cudaSuccess) return e;
  perm_scatter_kernel<<<1024, 256, 0, st>>>(labels, n, G, cap, cursor, tmp, heads, status);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_block_scores(const float* qbar, const float* mu, int G, int heads, int d, float tau,
                                float* sc, cudaStream_t st) {
  dim3 grid(ceil_div(G, 64), ceil_div(G, 64), heads);
  if (d == 64) block_score_kernel<64><<<grid, 256, 0, st>>>(qbar, mu, G, tau, sc);
  else block_score_kernel<128><<<grid, 256, 0, st>>>(qbar, mu, G, tau, sc);
  return counted(cudaGetLastError(), 1);
}

}  // namespace spr
