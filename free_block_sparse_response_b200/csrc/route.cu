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
// (1) the best group of every block; (2) a radix select, weighted by the pair cost, of
// the first candidate that no longer fits (64-bit keys: inverted score order key, then
// b G + g); (3) every block's groups in ascending order, -1 after them, and the pairs.
constexpr int kRgThreads = 1024;

__global__ void __launch_bounds__(kRgThreads)
    route_global_kernel(const float* __restrict__ sc, int Gq, int G, long long budget, int* __restrict__ route,
                        const int* __restrict__ key_gsize, const int* __restrict__ qblock_size,
                        unsigned long long* __restrict__ pairs, int* __restrict__ status) {
  extern __shared__ int s_best[];  // [Gq] best group per block
  __shared__ unsigned long long hist[256];
  __shared__ long long s_spent, s_below;
  __shared__ unsigned long long s_prefix;
  __shared__ int s_cross, s_digit;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = kRgThreads / 32;
  const int head = blockIdx.x;
  const float* scs = sc + static_cast<size_t>(head) * Gq * G;
  const int* ks = key_gsize + static_cast<size_t>(head) * G;
  const int* bs = qblock_size + static_cast<size_t>(head) * Gq;
  if (tid == 0) {
    s_spent = 0;
    s_below = 0;
    s_prefix = 0;
    s_cross = 0;
  }
  __syncthreads();
  // (1) best group of every block (smallest route key), its pairs
  bool saw_nan = false;
  for (int b = warp; b < Gq; b += nwarps) {
    unsigned long long best = ~0ull;
    for (int g = lane; g < G; g += 32) {
      const float v = scs[static_cast<size_t>(b) * G + g];
      saw_nan |= (v != v);
      const unsigned long long key = route_key(v, g);
      best = key < best ? key : best;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, best, o);
      best = y < best ? y : best;
    }
    if (lane == 0) {
      const int g = static_cast<int>(best & 0xffffffffu);
      s_best[b] = g;
      atomicAdd(reinterpret_cast<unsigned long long*>(&s_spent),
                static_cast<unsigned long long>(static_cast<long long>(bs[b]) * ks[g]));
    }
  }
  __syncthreads();
  const long long rem = budget - s_spent;  // pairs left for the other candidates
  // (2) weighted radix select: the first candidate (ascending key) whose cumulative cost
  // exceeds rem; every candidate before it is taken.  s_cross = 0: all candidates fit.
  auto ckey = [&](int b, int g, float v) {
    const uint32_t hi = (v != v) ? 0xffffffffu : ~float_order_key(v);
    return (static_cast<unsigned long long>(hi) << 32) | static_cast<uint32_t>(b * G + g);
  };
  const long long cand = static_cast<long long>(Gq) * G;
  if (rem >= 0) {
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int x = tid; x < 256; x += kRgThreads) hist[x] = 0;
      __syncthreads();
      const unsigned long long hmask = shift == 56 ? 0ull : (~0ull << (shift + 8));
      const unsigned long long prefix = s_prefix;
      for (long long x0 = 0; x0 < cand; x0 += kRgThreads) {
        const long long x = x0 + tid;
        int digit = -1, cost = 0;
        if (x < cand) {
          const int b = static_cast<int>(x / G), g = static_cast<int>(x - static_cast<long long>(b) * G);
          if (g != s_best[b]) {
            const unsigned long long key = ckey(b, g, scs[x]);
            if ((key & hmask) == prefix) {
              digit = static_cast<int>((key >> shift) & 255u);
              cost = bs[b] * ks[g];
            }
          }
        }
        // lanes with the same digit add their costs once (a leader per digit)
        const unsigned int peers = __match_any_sync(0xffffffffu, digit);
        const int sum = __reduce_add_sync(peers, cost);
        if (digit >= 0 && lane == __ffs(peers) - 1 && sum > 0)
          atomicAdd(&hist[digit], static_cast<unsigned long long>(sum));
      }
      __syncthreads();
      if (tid == 0) {
        long long below = s_below;
        int d = 0;
        for (; d < 256; ++d) {
          const long long hcost = static_cast<long long>(hist[d]);
          if (below + hcost > rem) break;
          below += hcost;
        }
        if (d == 256) {
          // everything under this prefix fits (only possible at the top level: below it,
          // the prefix was chosen because its bin crosses)
          s_digit = -1;
        } else {
          s_digit = d;
          s_below = below;
          s_prefix = prefix | (static_cast<unsigned long long>(d) << shift);
          s_cross = 1;
        }
      }
      __syncthreads();
      if (s_digit < 0) break;
    }
  }
  const bool cross = s_cross != 0;
  const unsigned long long kstar = s_prefix;  // the first candidate that does not fit
  // (3) routes: every block's kept best group and the candidates before kstar
  for (int b = warp; b < Gq; b += nwarps) {
    int* out = route + (static_cast<size_t>(head) * Gq + b) * G;
    int written = 0;
    long long member_sum = 0;
    for (int g0 = 0; g0 < G; g0 += 32) {
      const int g = g0 + lane;
      bool sel = false;
      if (g < G) {
        if (g == s_best[b]) {
          sel = true;
        } else if (rem >= 0) {
          sel = !cross || ckey(b, g, scs[static_cast<size_t>(b) * G + g]) < kstar;
        }
      }
      const unsigned int ball = __ballot_sync(0xffffffffu, sel);
      const int slot = written + __popc(ball & ((1u << lane) - 1u));
      if (sel) {
        out[slot] = g;
        member_sum += ks[g];
      }
      written += __popc(ball);
    }
    for (int sidx = written + lane; sidx < G; sidx += 32) out[sidx] = -1;
    if (pairs != nullptr) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) member_sum += __shfl_xor_sync(0xffffffffu, member_sum, o);
      if (lane == 0) atomicAdd(pairs + head, static_cast<unsigned long long>(static_cast<long long>(bs[b]) * member_sum));
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
  route_global_kernel<<<heads, kRgThreads, sizeof(int) * Gq, st>>>(sc, Gq, G, budget, route, key_gsize,
                                                                     qblock_size, up, status);
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
