// Shared device helpers of the SparsePR CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spr {

enum : int {
  kOk = 0,
  kErrInvalidArg = 1,
  kErrUnsupported = 2,
  kErrCuda = 3,
  kErrTimeout = 4,
  kErrNonFinite = 5
};

// Every bounded wait gives up after this long and records kErrTimeout.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Bound of the cooperative fill's grid barrier.  A build can shorten it (e.g.
// -DSPR_GRID_WAIT_LIMIT_NS=0) so that an ordinary call's barrier waits run out and take
// their error path: the barrier guards no asynchronous copy or tensor-core operation,
// so giving up early leaves nothing in flight.
#ifndef SPR_GRID_WAIT_LIMIT_NS
#define SPR_GRID_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr uint64_t kGridWaitLimitNs = SPR_GRID_WAIT_LIMIT_NS;

// The workspace starts with this block; the rest is carved per stage.
struct WorkspaceHeader {
  int status;    // first device-side error since the last partition call, else 0
  int grid_abort;  // set by a CTA of a cooperative kernel whose bounded wait gave up
  unsigned int barrier_count;  // grid barrier of the cooperative fill kernel
  unsigned int barrier_gen;
  // Source of the group-ordered K / V copy in the workspace: K, V, key_perm, key_gsize
  // pointers, N << 32 | G, heads (all zero: no copy).  Cleared with the header.
  unsigned long long kv_tag[6];
  int pad[48];
};
static_assert(sizeof(WorkspaceHeader) == 256, "header must keep 256-byte alignment");

__device__ __forceinline__ void record_error(int* status, int code) {
  atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier for a cooperative launch (all blocks co-resident).  The wait is
// bounded: on timeout it records kErrTimeout and every caller sees `false`.
__device__ __forceinline__ bool grid_barrier(WorkspaceHeader* hdr, unsigned int nblocks) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    s_ok = 1;
    unsigned int gen = ld_acquire_u32(&hdr->barrier_gen);
    __threadfence();
    unsigned int arrived = atomicAdd(&hdr->barrier_count, 1u);
    if (arrived == nblocks - 1) {
      atomicExch(&hdr->barrier_count, 0u);
      __threadfence();
      atomicAdd(&hdr->barrier_gen, 1u);
    } else {
      uint64_t t0 = globaltimer_ns();
      while (ld_acquire_u32(&hdr->barrier_gen) == gen) {
        if (globaltimer_ns() - t0 > kGridWaitLimitNs) {
          record_error(&hdr->status, kErrTimeout);
          s_ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    if (*(volatile int*)&hdr->status == kErrTimeout) s_ok = 0;
  }
  __syncthreads();
  return s_ok != 0;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Order-preserving map of a float to uint32 (a < b  <=>  key(a) < key(b)); -0.0 is
// folded onto +0.0 first so that the two compare equal, as with plain '<'.  NaN
// must be handled by the caller.
__device__ __forceinline__ uint32_t float_order_key(float f) {
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float float_from_order_key(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Number of routed groups in a route row of capacity k: rows hold ascending key groups,
// then -1 padding when the pair budget is allocated per head rather than per block.
__device__ __forceinline__ int routed_len(const int* __restrict__ row, int k) {
  if (k <= 0 || __ldg(row + k - 1) >= 0) return k;
  int lo = 0, hi = k - 1;  // row[hi] < 0; the first negative entry lies in [lo, hi]
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(row + mid) < 0)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo;
}

// Host-side count of kernels this library has enqueued (all devices, all threads).
void note_launches(int n);
inline cudaError_t counted(cudaError_t e, int n) {
  if (e == cudaSuccess) note_launches(n);
  return e;
}

}  // namespace spr
