// Decision helpers of the capacity-constrained fill (internal to the library), shared
// by the fill kernels and the fused tensor-core assignment kernel so that every path
// takes its decisions with the same code.
#pragma once

#include "common.cuh"

namespace spr {

// Total order of (value, index) for the fill's decisions: fp32 values compared as with
// plain '<' (+-0 equal), NaN after everything, ties to the lower index.
__device__ __forceinline__ unsigned long long decision_key(float v, int idx) {
  const uint32_t ok = (v != v) ? 0xffffffffu : float_order_key(v);
  return (static_cast<unsigned long long>(ok) << 32) | static_cast<uint32_t>(idx);
}

__device__ __forceinline__ unsigned long long warp_min_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, v, o);
    v = y < v ? y : v;
  }
  return v;
}

// One digit of the radix select: from the warp's 256-bin histogram of the keys that share
// the prefix so far, the bin holding the kth key (1-based), the count before it and the
// count in it.
__device__ __forceinline__ void select_digit(const unsigned int* hist, int kth, int& digit, unsigned int& before,
                                             unsigned int& in_bin) {
  const int lane = threadIdx.x & 31;
  unsigned int local[8];
  unsigned int tot = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    local[j] = hist[8 * lane + j];
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
  digit = 0;
  before = 0;
  in_bin = 0;
  if (mine) {
    unsigned int acc = excl;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (acc + local[j] >= static_cast<unsigned int>(kth)) {
        digit = 8 * lane + j;
        before = acc;
        in_bin = local[j];
        break;
      }
      acc += local[j];
    }
  }
  digit = __shfl_sync(0xffffffffu, digit, src);
  before = __shfl_sync(0xffffffffu, before, src);
  in_bin = __shfl_sync(0xffffffffu, in_bin, src);
}

// Key of the kth smallest (1-based) of `count` distinct 64-bit keys, by a warp: radix
// select on 8-bit digits, starting below the bits all keys share and stopping as soon
// as the selected digit bin holds a single key.  `key(e)` returns key e (< count); with
// keys held in registers no pass reads memory.
template <class KeyAt>
__device__ inline unsigned long long warp_select_kth_by(KeyAt key_at, int count, int kth, unsigned int* hist) {
  const int lane = threadIdx.x & 31;
  unsigned long long kmin = ~0ull, kmax = 0ull;
  key_at.for_each(count, [&](unsigned long long k) {
    kmin = k < kmin ? k : kmin;
    kmax = k > kmax ? k : kmax;
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, kmin, o);
    const unsigned long long b = __shfl_xor_sync(0xffffffffu, kmax, o);
    kmin = a < kmin ? a : kmin;
    kmax = b > kmax ? b : kmax;
  }
  if (kmin == kmax) return kmin;
  const int top = 63 - __clzll(static_cast<long long>(kmin ^ kmax));  // highest differing bit
  int shift = (top / 8) * 8;
  unsigned long long prefix = shift + 8 >= 64 ? 0ull : (kmin & (~0ull << (shift + 8)));
  for (; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    const unsigned long long hmask = shift + 8 >= 64 ? 0ull : (~0ull << (shift + 8));
    key_at.for_each(count, [&](unsigned long long k) {
      if ((k & hmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    });
    __syncwarp();
    int digit;
    unsigned int before, in_bin;
    select_digit(hist, kth, digit, before, in_bin);
    kth -= static_cast<int>(before);
    prefix |= static_cast<unsigned long long>(digit) << shift;
    __syncwarp();
    if (in_bin == 1 || shift == 0) {
      // the kth key is the only key with this prefix: fetch it
      const unsigned long long pmask = ~0ull << shift;
      unsigned long long found = ~0ull;
      key_at.for_each(count, [&](unsigned long long k) {
        if ((k & pmask) == prefix) found = k;
      });
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, found, o);
        found = y < found ? y : found;
      }
      return found;
    }
  }
  return prefix;
}

// Keys in memory, read by the warp 256 at a time (8 per lane in flight).
struct KeysInMemory {
  const unsigned long long* keys;
  template <class F>
  __device__ __forceinline__ void for_each(int count, F f) const {
    const int lane = threadIdx.x & 31;
    for (int e0 = 0; e0 < count; e0 += 256) {
      unsigned long long kb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = e0 + u * 32 + lane;
        kb[u] = e < count ? __ldcg(keys + e) : ~0ull;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (e0 + u * 32 + lane < count) f(kb[u]);
    }
  }
};

// At most 256 keys held by the warp, key u * 32 + lane in kb[u] of that lane.
struct KeysInRegisters {
  const unsigned long long (&kb)[8];
  template <class F>
  __device__ __forceinline__ void for_each(int count, F f) const {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (u * 32 + lane < count) f(kb[u]);
  }
};

__device__ inline unsigned long long warp_select_kth(const unsigned long long* keys, int count, int kth,
                                                     unsigned int* hist) {
  return warp_select_kth_by(KeysInMemory{keys}, count, kth, hist);
}

}  // namespace spr
