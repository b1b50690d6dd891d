// Centroid-based block routing (sm_100a).
//
// Source: SparsePR abstract (arXiv 2608.18484, arxivdaily.com English abstract): query
// groups share one sparse route chosen from their responses to the key-group centroids,
// and the executed-pair density counts the exact probe rows.  Each query block keeps the
// k key groups with the largest score (ties to the lower group), listed in ascending
// group order; one warp per block row selects them by radix select on 64-bit keys.
#include <cuda_bf16.h>

#include "common.cuh"
#include "route.cuh"

namespace spr {

// Smaller key = preferred: high word = inverted order key of the score (largest score
// first; NaN ranks last), low word = group index (lower group first on ties).
__device__ __forceinline__ unsigned long long route_key(float v, int g) {
  const uint32_t hi = (v != v) ? 0xffffffffu : ~float_order_key(v);
  return (static_cast<unsigned long long>(hi) << 32) | static_cast<uint32_t>(g);
}

__global__ void __launch_bounds__(256)
    route_topk_kernel(const float* __restrict__ sc, int Gq, int G, int k, int* __restrict__ route,
                      const int* __restrict__ key_gsize, const int* __restrict__ qblock_size,
                      unsigned long long* __restrict__ pairs, int* __restrict__ status) {
  __shared__ unsigned int hist[8][256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int head = blockIdx.y;
  const int b = blockIdx.x * 8 + warp;
  if (b >= Gq) return;
  const float* row = sc + (static_cast<size_t>(head) * Gq + b) * G;
  unsigned int* h = hist[warp];
  // radix select the k-th smallest key
  unsigned long long prefix = 0;
  int kth = k;
  bool saw_nan = false;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int x = lane; x < 256; x += 32) h[x] = 0;
    __syncwarp();
    const unsigned long long hmask = shift == 56 ? 0ull : (~0ull << (shift + 8));
    for (int g = lane; g < G; g += 32) {
      const float v = row[g];
      saw_nan |= (v != v);
      const unsigned long long key = route_key(v, g);
      if ((key & hmask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    unsigned int local[8], tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      local[j] = h[8 * lane + j];
      tot += local[j];
    }
    unsigned int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned int excl = incl - tot;
    const bool mine = excl < static_cast<unsigned int>(kth) && static_cast<unsigned int>(kth) <= incl;
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    int digit = 0;
    unsigned int before = 0;
    if (mine) {
      unsigned int acc = excl;
      for (int j = 0; j < 8; ++j) {
        if (acc + local[j] >= static_cast<unsigned int>(kth)) {
          digit = 8 * lane + j;
          before = acc;
          break;
        }
        acc += local[j];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    before = __shfl_sync(0xffffffffu, before, src);
    kth -= static_cast<int>(before);
    prefix |= static_cast<unsigned long long>(digit) << shift;
    __syncwarp();
  }
  // emit the selected groups in ascending order and count the executed pairs
  int* out = route + (static_cast<size_t>(head) * Gq + b) * k;
  int written = 0;
  long long member_sum = 0;
  for (int g0 = 0; g0 < G; g0 += 32) {
    const int g = g0 + lane;
    const bool sel = g < G && route_key(row[g], g) <= prefix;
    const unsigned int ball = __ballot_sync(0xffffffffu, sel);
    const int slot = written + __popc(ball & ((1u << lane) - 1u));
    if (sel && slot < k) {
      out[slot] = g;
      if (key_gsize != nullptr) member_sum += key_gsize[static_cast<size_t>(head) * G + g];
    }
    written += __popc(ball);
  }
  saw_nan = __any_sync(0xffffffffu, saw_nan);
  if (lane == 0 && (saw_nan || written != k)) record_error(status, written != k ? kErrInvalidArg : kErrNonFinite);
  if (pairs != nullptr) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) member_sum += __shfl_xor_sync(0xffffffffu, member_sum, o);
    if (lane == 0) {
      const long long nb = qblock_size[static_cast<size_t>(head) * Gq + b];
      atomicAdd(pairs + head, static_cast<unsigned long long>(nb * member_sum));
    }
  }
}

// Global budget allocation (the other reading of routing up to a target density): the
// pair budget of a head is shared by its blocks.  Every block keeps its best group; the
// other (block, group) pairs, ordered by descending score, then block, then group, are
// taken while the cumulative pairs n_b n_g stay within the budget.  One CTA per head:
//   pass 0   best group of every block (warp per block row), and the cost histogram of
//            the top 8 bits of every pair's score key (the best pairs taken out again);
//   pass 1-3 the next 8 bits among the pairs whose higher bits match the crossing bin:
//            after them the score key T of the first pair that no longer fits is known;
//   tie pass the pairs with score key T in (block, group) order, a block-wide prefix sum
//            of their costs: the crossing pair itself;
//   emit     every block's best group and the pairs before the crossing one, ascending,
//            then -1, and the executed pairs.
// Histograms are per warp (no atomics across warps; lanes with the same digit add their
// costs once, through a warp match and reduction), summed per bin between passes.
constexpr int kRgThreads = 1024;
constexpr int kRgWarps = kRgThreads / 32;

__device__ __forceinline__ uint32_t score_hi(float v) { return (v != v) ? 0xffffffffu : ~float_order_key(v); }

constexpr int kRgU = 8;  // independent loads per lane in flight

// Scores and key-group sizes of groups g0 + 32 u + lane, u < kRgU, of one block row.
__device__ __forceinline__ void load_row_chunk(const float* __restrict__ row, const int* __restrict__ ks, int G,
                                               int g0, int lane, float (&v)[kRgU], int (&kz)[kRgU]) {
#pragma unroll
  for (int u = 0; u < kRgU; ++u) {
    const int g = g0 + 32 * u + lane;
    v[u] = g < G ? __ldg(row + g) : 0.f;
    kz[u] = g < G ? __ldg(ks + g) : 0;
  }
}

__device__ __forceinline__ void warp_hist_add(unsigned long long* hw, int digit, int cost) {
  const unsigned int peers = __match_any_sync(0xffffffffu, digit);
  const int sum = __reduce_add_sync(peers, cost);
  if (digit >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1) hw[digit] += static_cast<unsigned long long>(sum);
  __syncwarp();  // the next leader of this digit may be another lane
}

__global__ void __launch_bounds__(kRgThreads)
    route_global_kernel(const float* __restrict__ sc, int Gq, int G, long long budget, int* __restrict__ route,
                        const int* __restrict__ key_gsize, const int* __restrict__ qblock_size,
                        unsigned long long* __restrict__ pairs, int* __restrict__ status) {
  // dynamic: per-warp histograms [kRgWarps][256] u64, then the best group of every block
  extern __shared__ unsigned long long s_hist[];
  int* s_best = reinterpret_cast<int*>(s_hist + kRgWarps * 256);
  __shared__ unsigned long long s_tot[256];
  __shared__ long long s_wsum[kRgWarps];
  __shared__ long long s_spent, s_below;
  __shared__ uint32_t s_prefix;
  __shared__ int s_cross, s_found;
  __shared__ unsigned long long s_kstar;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int head = blockIdx.x;
  const float* scs = sc + static_cast<size_t>(head) * Gq * G;
  const int* ks = key_gsize + static_cast<size_t>(head) * G;
  const int* bs = qblock_size + static_cast<size_t>(head) * Gq;
  unsigned long long* hw = s_hist + warp * 256;
  if (tid == 0) {
    s_spent = 0;
    s_below = 0;
    s_prefix = 0;
    s_cross = 0;
    s_found = 0;
    s_kstar = 0;
  }
  for (int x = lane; x < 256; x += 32) hw[x] = 0;
  __syncthreads();
  // pass 0 (group and block sizes are at most B = 128: a pair costs <= 2^14, a warp's sum fits an int)
  bool saw_nan = false;
  for (int b = warp; b < Gq; b += kRgWarps) {
    const float* row = scs + static_cast<size_t>(b) * G;
    const int nb = bs[b];
    unsigned long long best = ~0ull;
    for (int g0 = 0; g0 < G; g0 += 32 * kRgU) {
      float v[kRgU];
      int kz[kRgU];
      load_row_chunk(row, ks, G, g0, lane, v, kz);
#pragma unroll
      for (int u = 0; u < kRgU; ++u) {
        if (g0 + 32 * u >= G) break;
        const int g = g0 + 32 * u + lane;
        int digit = -1, cost = 0;
        if (g < G) {
          saw_nan |= (v[u] != v[u]);
          const uint32_t hi = score_hi(v[u]);
          const unsigned long long key = (static_cast<unsigned long long>(hi) << 32) | static_cast<uint32_t>(g);
          best = key < best ? key : best;
          digit = static_cast<int>(hi >> 24);
          cost = nb * kz[u];
        }
        warp_hist_add(hw, digit, cost);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
      best = y < best ? y : best;
    }
    __syncwarp();
    if (lane == 0) {
      const int g = static_cast<int>(best & 0xffffffffu);
      const unsigned long long c = static_cast<unsigned long long>(nb) * ks[g];
      s_best[b] = g;
      hw[static_cast<uint32_t>(best >> 32) >> 24] -= c;  // the best pair is no candidate
      atomicAdd(reinterpret_cast<unsigned long long*>(&s_spent), c);
    }
    __syncwarp();
  }
  __syncthreads();
  const long long rem = budget - s_spent;  // pairs left for the candidates
  if (rem >= 0) {
    // passes 0-3: the crossing score key, 8 bits at a time
    for (int level = 0; level < 4; ++level) {
      const int shift = 24 - 8 * level;
      if (level > 0) {
        const uint32_t mask = ~0u << (shift + 8), prefix = s_prefix;
        for (int x = lane; x < 256; x += 32) hw[x] = 0;
        __syncwarp();
        for (int b = warp; b < Gq; b += kRgWarps) {
          const float* row = scs + static_cast<size_t>(b) * G;
          const int nb = bs[b], bg = s_best[b];
          for (int g0 = 0; g0 < G; g0 += 32 * kRgU) {
            float v[kRgU];
            int kz[kRgU];
            load_row_chunk(row, ks, G, g0, lane, v, kz);
#pragma unroll
            for (int u = 0; u < kRgU; ++u) {
              if (g0 + 32 * u >= G) break;
              const int g = g0 + 32 * u + lane;
              int digit = -1, cost = 0;
              if (g < G && g != bg) {
                const uint32_t hi = score_hi(v[u]);
                if ((hi & mask) == prefix) {
                  digit = static_cast<int>((hi >> shift) & 255u);
                  cost = nb * kz[u];
                }
              }
              if (__any_sync(0xffffffffu, digit >= 0)) warp_hist_add(hw, digit, cost);
            }
          }
        }
      }
      __syncthreads();
      if (tid < 256) {
        unsigned long long t = 0;
        for (int w = 0; w < kRgWarps; ++w) t += s_hist[w * 256 + tid];
        s_tot[tid] = t;
      }
      __syncthreads();
      if (tid == 0) {
        long long below = s_below;
        int d = 0;
        for (; d < 256; ++d) {
          const long long c = static_cast<long long>(s_tot[d]);
          if (below + c > rem) break;
          below += c;
        }
        if (d < 256) {
          s_cross = 1;
          s_below = below;
          s_prefix |= static_cast<uint32_t>(d) << shift;
        }
        // d == 256 only at level 0 (every candidate fits); below it the chosen bin crosses
      }
      __syncthreads();
      if (!s_cross) break;
    }
    if (s_cross) {
      // tie pass: the pairs with score key T in ascending b G + g order; thread t takes
      // kRgU consecutive pairs of each chunk, so chunk order = thread order = pair order
      const uint32_t T = s_prefix;
      const long long cand = static_cast<long long>(Gq) * G;
      for (long long x0 = 0; x0 < cand; x0 += static_cast<long long>(kRgThreads) * kRgU) {
        const long long xt = x0 + static_cast<long long>(tid) * kRgU;
        int cost[kRgU];  // tie costs (0: no tie; a zero-cost tie adds nothing and never crosses)
        int tsum = 0;
#pragma unroll
        for (int u = 0; u < kRgU; ++u) {
          cost[u] = 0;
          const long long x = xt + u;
          if (x < cand) {
            const int b = static_cast<int>(x / G), g = static_cast<int>(x - static_cast<long long>(b) * G);
            if (g != s_best[b] && score_hi(__ldg(scs + x)) == T) cost[u] = bs[b] * ks[g];
          }
          tsum += cost[u];
        }
        if (!__syncthreads_or(tsum > 0)) continue;
        int incl = tsum;  // warp-inclusive prefix of the threads' tie costs
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        long long run = s_below;
        for (int w = 0; w < warp; ++w) run += s_wsum[w];
        run += incl - tsum;  // cost of the ties before this thread's first pair
        if (tsum > 0 && run + tsum > rem) {
#pragma unroll
          for (int u = 0; u < kRgU; ++u) {
            if (cost[u] > 0 && run <= rem && run + cost[u] > rem) {
              s_kstar = (static_cast<unsigned long long>(T) << 32) | static_cast<uint32_t>(xt + u);
              s_found = 1;
            }
            run += cost[u];
          }
        }
        __syncthreads();
        if (s_found) break;
        if (tid == 0) {
          long long t = 0;
          for (int w = 0; w < kRgWarps; ++w) t += s_wsum[w];
          s_below += t;
        }
        __syncthreads();
      }
    }
  }
  const bool cross = s_cross != 0;
  const unsigned long long kstar = s_kstar;  // the first candidate that does not fit
  // emit: every block's best group and the candidates before kstar
  for (int b = warp; b < Gq; b += kRgWarps) {
    const float* row = scs + static_cast<size_t>(b) * G;
    int* out = route + (static_cast<size_t>(head) * Gq + b) * G;
    const int bg = s_best[b];
    int written = 0;
    long long member_sum = 0;
    for (int g0 = 0; g0 < G; g0 += 32 * kRgU) {
      float v[kRgU];
      int kz[kRgU];
      load_row_chunk(row, ks, G, g0, lane, v, kz);
#pragma unroll
      for (int u = 0; u < kRgU; ++u) {
        if (g0 + 32 * u >= G) break;
        const int g = g0 + 32 * u + lane;
        bool sel = false;
        if (g < G) {
          if (g == bg) {
            sel = true;
          } else if (rem >= 0) {
            const unsigned long long key =
                (static_cast<unsigned long long>(score_hi(v[u])) << 32) | static_cast<uint32_t>(b * G + g);
            sel = !cross || key < kstar;
          }
        }
        const unsigned int ball = __ballot_sync(0xffffffffu, sel);
        const int slot = written + __popc(ball & ((1u << lane) - 1u));
        if (sel) {
          out[slot] = g;
          member_sum += kz[u];
        }
        written += __popc(ball);
      }
    }
    for (int sidx = written + lane; sidx < G; sidx += 32) out[sidx] = -1;
    if (pairs != nullptr) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) member_sum += __shfl_xor_sync(0xffffffffu, member_sum, o);
      if (lane == 0)
        atomicAdd(pairs + head, static_cast<unsigned long long>(static_cast<long long>(bs[b]) * member_sum));
    }
  }
  saw_nan = __syncthreads_or(saw_nan);
  if (tid == 0 && saw_nan) record_error(status, kErrNonFinite);
}

// Sc[b][g] += log n_g (size-corrected scores).
__global__ void size_correct_kernel(float* __restrict__ sc, const int* __restrict__ key_gsize, int Gq, int G) {
  const int head = blockIdx.y;
  const size_t base = static_cast<size_t>(head) * Gq * G;
  for (int x = blockIdx.x * blockDim.x + threadIdx.x; x < Gq * G; x += gridDim.x * blockDim.x) {
    const int g = x % G;
    sc[base + x] += logf(static_cast<float>(max(key_gsize[static_cast<size_t>(head) * G + g], 1)));
  }
}

// Sc[b][g] = log sum_{j in g} exp(tau qbar_b . k_j): one CTA per (group, head, 256
// blocks); the group's keys in shared memory, read by every thread at once;
// thread = block b, its qbar_b in registers, online max / sum over the members.
__global__ void __launch_bounds__(256) lse_scores_kernel(const __nv_bfloat16* __restrict__ K, int N, int Gq, int G,
                                                         const int* __restrict__ key_perm,
                                                         const int* __restrict__ key_gsize,
                                                         const float* __restrict__ qbar, float tau,
                                                         float* __restrict__ sc) {
  __shared__ __nv_bfloat16 sk[128][128];  // every thread reads the same element: broadcast
  const int g = blockIdx.x, head = blockIdx.y, b = blockIdx.z * 256 + threadIdx.x;
  const size_t grp = static_cast<size_t>(head) * G + g;
  const int gs = min(__ldg(key_gsize + grp), 128);
  for (int x = threadIdx.x; x < gs * 128; x += 256) {
    const int j = x >> 7, e = x & 127;
    const int tok = __ldg(key_perm + grp * 128 + j);
    sk[j][e] = K[(static_cast<size_t>(head) * N + tok) * 128 + e];
  }
  __syncthreads();
  if (b >= Gq) return;
  float qv[128];
  const float* qb = qbar + (static_cast<size_t>(head) * Gq + b) * 128;
#pragma unroll
  for (int e = 0; e < 128; ++e) qv[e] = qb[e] * tau;
  float m = -__builtin_huge_valf(), s = 0.f;
  for (int j = 0; j < gs; ++j) {
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 128; ++e) acc = fmaf(qv[e], __bfloat162float(sk[j][e]), acc);
    if (acc > m) {
      s = s * expf(m - acc) + 1.f;
      m = acc;
    } else {
      s += expf(acc - m);
    }
  }
  sc[(static_cast<size_t>(head) * Gq + b) * G + g] = gs > 0 ? m + logf(s) : -__builtin_huge_valf();
}

__global__ void pairs_init_kernel(unsigned long long* pairs, int heads, long long probe_pairs) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < heads) pairs[h] = static_cast<unsigned long long>(probe_pairs);
}

cudaError_t launch_route(const float* sc, int heads, int Gq, int G, int k, int* route, const int* key_gsize,
                         const int* qblock_size, long long* pairs, long long probe_pairs, int* status,
                         cudaStream_t st) {
  unsigned long long* up = reinterpret_cast<unsigned long long*>(pairs);
  if (up != nullptr) {
    pairs_init_kernel<<<ceil_div(heads, 256), 256, 0, st>>>(up, heads, probe_pairs);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  route_topk_kernel<<<dim3(ceil_div(Gq, 8), heads), 256, 0, st>>>(sc, Gq, G, k, route, key_gsize, qblock_size,
                                                                   up, status);
  return counted(cudaGetLastError(), up != nullptr ? 2 : 1);
}

cudaError_t launch_route_global(const float* sc, int heads, int Gq, int G, long long budget, int* route,
                                const int* key_gsize, const int* qblock_size, long long* pairs, long long probe_pairs,
                                int* status, cudaStream_t st) {
  unsigned long long* up = reinterpret_cast<unsigned long long*>(pairs);
  if (up != nullptr) {
    pairs_init_kernel<<<ceil_div(heads, 256), 256, 0, st>>>(up, heads, probe_pairs);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t smem = sizeof(unsigned long long) * kRgWarps * 256 + sizeof(int) * Gq;
  cudaError_t e = cudaFuncSetAttribute(route_global_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  route_global_kernel<<<heads, kRgThreads, smem, st>>>(sc, Gq, G, budget, route, key_gsize, qblock_size, up,
                                                       status);
  return counted(cudaGetLastError(), up != nullptr ? 2 : 1);
}

cudaError_t launch_route_scores(int mode, float* sc, const void* K, int N, int heads, int Gq, int G,
                                const int* key_perm, const int* key_gsize, const float* qbar, float tau,
                                cudaStream_t st) {
  if (mode == 1) {
    size_correct_kernel<<<dim3(ceil_div(Gq * G, 256), heads), 256, 0, st>>>(sc, key_gsize, Gq, G);
  } else if (mode == 2) {
    lse_scores_kernel<<<dim3(G, heads, ceil_div(Gq, 256)), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(K), N, Gq, G, key_perm, key_gsize, qbar, tau, sc);
  } else {
    return cudaSuccess;
  }
  return counted(cudaGetLastError(), 1);
}

}  // namespace spr
