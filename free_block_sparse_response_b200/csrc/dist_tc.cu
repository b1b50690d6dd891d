// Balanced k-means distances on 5th-generation tensor cores (sm_100a).
//
// For every item i (a key or a query row, bf16, head dim 128) and group g:
//     D[i][g] = tau^2 (n_i - 2 x_i . w_g + e_g),   w_g = Gamma c_g,  e_g = c_g . w_g,
// the head-dim form of the squared response-space distance used by Response-Coupled
// Partitioning (SparsePR abstract, arXiv 2608.18484).  w_g enters as bf16 hi + lo, so
// the cross term carries ~16-bit precision.  The full fp32 row is written (row stride
// ldd, a multiple of 4) and its argmin (ties to the lower group) is the first proposal
// of the capacity fill.
//
// One CTA per 128 items; groups streamed in chunks of 128 (W double-buffered, cp.async
// into 128B-swizzled tiles); the accumulator chunk lives in TMEM (two buffers, so the
// MMA of chunk c+1 overlaps the epilogue of chunk c).  Warps 0-1 load, warp 2 issues the
// MMAs, warps 4-11 run the epilogue: each row is owned by two threads (columns 0-63 and
// 64-127 of every chunk), which stage their half-row in shared memory and write it with
// one bulk copy, so HBM sees full lines.  The row argmin is a strict '<' scan in
// ascending column order (first minimum wins, +-0 compare equal), merged across the two
// halves at the end.  Every wait is bounded.
#include "common.cuh"
#include "partition.cuh"
#include "tcgen05.cuh"
#include "warp_mma.cuh"

namespace spr {
namespace {

constexpr int kDtThreads = 384;
constexpr int kDtProducers = 64;
constexpr uint32_t kDtTile = 128 * 128 * 2;
constexpr uint32_t kDtTmemCols = 256;
constexpr float kDtInf = __builtin_huge_valf();
constexpr uint32_t kStageStride = 32 * 4 + 16;   // one staged 32-column row segment + pad

enum : int { kXFull = 0, kWFull0 = 1, kWEmpty0 = 3, kAccFull0 = 5, kAccEmpty0 = 7, kDtDrain = 9, kDtBars = 10 };

__device__ __forceinline__ unsigned long long dist_key(float v, int idx) {
  const uint32_t ok = (v != v) ? 0xffffffffu : float_order_key(v);
  return (static_cast<unsigned long long>(ok) << 32) | static_cast<uint32_t>(idx);
}

template <bool SPLIT>
__global__ void __launch_bounds__(kDtThreads, 1)
    dist_tc_kernel(const __nv_bfloat16* __restrict__ X, int n, const __nv_bfloat16* __restrict__ Whi,
                   const __nv_bfloat16* __restrict__ Wlo, int ncols, int ldd, const float* __restrict__ nrm,
                   const float* __restrict__ ecol, float tau2, float* __restrict__ Dout, int* __restrict__ prop_g,
                   float* __restrict__ prop_v, int* __restrict__ status) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bars[kDtBars];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ float s_best_v[128];
  __shared__ int s_best_c[128];
  constexpr int kWStage = kDtTile * (SPLIT ? 2 : 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int head = blockIdx.y;
  const int row0 = blockIdx.x * 128;
  const uint32_t sbase = (tc::saddr(dsmem) + 1023u) & ~1023u;
  const uint32_t sX = sbase;
  const uint32_t sW[2] = {sbase + kDtTile, sbase + kDtTile + kWStage};
  const uint32_t sStage = sbase + kDtTile + 2 * kWStage;  // 256 staged row segments
  float* s_e = reinterpret_cast<float*>(dsmem + (sbase - tc::saddr(dsmem)) + kDtTile + 2 * kWStage +
                                        256 * kStageStride);
  auto bar = [&](int i) { return tc::saddr(&bars[i]); };
  const int n_chunks = ceil_div(ncols, 128);

  X += static_cast<size_t>(head) * n * 128;
  Whi += static_cast<size_t>(head) * ncols * 128;
  if (SPLIT) Wlo += static_cast<size_t>(head) * ncols * 128;

  if (tid == 0) {
    tc::mbar_init(bar(kXFull), kDtProducers);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(kWFull0 + s), kDtProducers);
      tc::mbar_init(bar(kWEmpty0 + s), 1);
      tc::mbar_init(bar(kAccFull0 + s), 1);
      tc::mbar_init(bar(kAccEmpty0 + s), 256);
    }
    tc::mbar_init(bar(kDtDrain), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // tau^2 e_g, padded with +inf to whole chunks
  for (int c = tid; c < n_chunks * 128; c += kDtThreads)
    s_e[c] = c < ncols ? tau2 * ecol[static_cast<size_t>(head) * ncols + c] : kDtInf;
  if (warp == 2) {
    tc::tmem_alloc(tc::saddr(&tmem_slot), kDtTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = tmem_slot;
  volatile int* abort_v = &abort_flag;

  if (warp < 2) {
    // ------------------------------------------------------------------ producers
    const int pt = tid, ch = pt & 15, r0 = pt >> 4;
#pragma unroll 4
    for (int i = 0; i < 32; ++i) {
      const int r = r0 + 4 * i;
      const int row = row0 + r;
      cp_async_16(sX + tc::sw128_offset(r, ch), row < n ? X + static_cast<size_t>(row) * 128 + ch * 8 : X,
                  row < n ? 16 : 0);
    }
    tc::cp_async_arrive_noinc(bar(kXFull));
    for (int c = 0; c < n_chunks; ++c) {
      const int s = c & 1;
      if (c >= 2 && !tc::mbar_wait(bar(kWEmpty0 + s), ((c >> 1) - 1) & 1, abort_v, status)) break;
#pragma unroll 4
      for (int i = 0; i < 32; ++i) {
        const int r = r0 + 4 * i;
        const int col = c * 128 + r;
        const size_t off = col < ncols ? static_cast<size_t>(col) * 128 + ch * 8 : 0;
        cp_async_16(sW[s] + tc::sw128_offset(r, ch), Whi + off, col < ncols ? 16 : 0);
        if (SPLIT) cp_async_16(sW[s] + kDtTile + tc::sw128_offset(r, ch), Wlo + off, col < ncols ? 16 : 0);
      }
      tc::cp_async_arrive_noinc(bar(kWFull0 + s));
    }
    cp_async_wait<0>();
  } else if (warp == 2) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kId = tc::idesc_bf16(128, 128, false, false);
      bool ok = tc::mbar_wait(bar(kXFull), 0, abort_v, status);
      tc::fence_proxy_async();
      for (int c = 0; ok && c < n_chunks; ++c) {
        const int s = c & 1;
        if (!tc::mbar_wait(bar(kWFull0 + s), (c >> 1) & 1, abort_v, status)) break;
        tc::fence_proxy_async();
        if (c >= 2 && !tc::mbar_wait(bar(kAccEmpty0 + s), ((c >> 1) - 1) & 1, abort_v, status)) break;
        tc::fence_after_sync();
        const uint32_t acc = tbase + s * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          const uint64_t adesc = tc::sdesc_sw128(sX + koff, 16, 1024);
          tc::mma_ss(acc, adesc, tc::sdesc_sw128(sW[s] + koff, 16, 1024), kId, kk > 0 ? 1u : 0u);
          if (SPLIT) tc::mma_ss(acc, adesc, tc::sdesc_sw128(sW[s] + kDtTile + koff, 16, 1024), kId, 1u);
        }
        tc::mma_commit(bar(kWEmpty0 + s));
        tc::mma_commit(bar(kAccFull0 + s));
      }
      tc::mma_commit(bar(kDtDrain));
      const uint64_t t0 = globaltimer_ns();
      while (!tc::mbar_try_wait(bar(kDtDrain), 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    const int r = (warp & 3) * 32 + lane;     // row within the tile == TMEM lane
    const int half = (warp - 4) >> 2;         // columns [64 half, 64 half + 64) of each chunk
    const int row = row0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float tnr = row < n ? tau2 * nrm[static_cast<size_t>(head) * n + row] : 0.f;
    const float m2t = -2.f * tau2;
    float* drow = Dout + (static_cast<size_t>(head) * n + (row < n ? row : 0)) * ldd;
    const uint32_t my_stage = sStage + (half * 128 + r) * kStageStride;
    float best_v = kDtInf;
    int best_c = -1;
    float nan_probe = 0.f;
    for (int c = 0; c < n_chunks; ++c) {
      const int s = c & 1;
      const bool ok = tc::mbar_wait(bar(kAccFull0 + s), (c >> 1) & 1, abort_v, status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::fence_after_sync();
      uint32_t u[64];
      const uint32_t buf = tbase + lane_off + s * 128 + half * 64;
      tc::tmem_ld32(buf, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
      tc::tmem_ld32(buf + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      tc::mbar_arrive(bar(kAccEmpty0 + s));
      const int c0 = c * 128 + half * 64;
      const float4* e4 = reinterpret_cast<const float4*>(s_e + c0);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 e = e4[q];
        const float ev[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int j = 4 * q + t;
          const float v = fmaf(m2t, __uint_as_float(u[j]), tnr) + ev[t];
          u[j] = __float_as_uint(v);
          nan_probe += v;
          if (v < best_v) {
            best_v = v;
            best_c = c0 + j;
          }
        }
      }
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        tc::bulk_wait_read();  // the previous copy out of this staging row has been read
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = sub * 32 + 4 * q;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(my_stage + 16 * q), "r"(u[j]),
                       "r"(u[j + 1]), "r"(u[j + 2]), "r"(u[j + 3])
                       : "memory");
        }
        tc::fence_proxy_async();
        const int cols = min(32, ldd - (c0 + sub * 32));
        if (row < n && cols > 0) {
          tc::bulk_store(drow + c0 + sub * 32, my_stage, static_cast<uint32_t>(cols) * 4u);
          tc::bulk_commit();
        }
      }
    }
    tc::bulk_wait_all();
    if (half == 1) {
      s_best_v[r] = best_v;
      s_best_c[r] = best_c;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight epilogue warps only
    if (half == 0 && row < n) {
      const float v1 = s_best_v[r];
      const int c1 = s_best_c[r];
      // half 0 holds the lower columns of every chunk: take half 1 only if strictly smaller,
      // or equal with a lower column (a later chunk's half 0 can exceed an earlier half 1)
      if (c1 >= 0 && (best_c < 0 || v1 < best_v || (v1 == best_v && c1 < best_c))) {
        best_v = v1;
        best_c = c1;
      }
      if (best_c < 0) best_c = 0;
      const size_t o = static_cast<size_t>(head) * n + row;
      prop_g[o] = best_c;
      prop_v[o] = best_v;
    }
    if (__any_sync(0xffffffffu, nan_probe != nan_probe) && lane == 0) record_error(status, kErrNonFinite);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, kDtTmemCols);
  }
}

}  // namespace

cudaError_t launch_dist_tc(const RowGemmArgs& a, int ldd, cudaStream_t st) {
  const bool split = a.Blo != nullptr;
  const size_t smem = kDtTile + 2ull * kDtTile * (split ? 2 : 1) + 256ull * kStageStride + 1024 +
                      sizeof(float) * ceil_div(a.ncols, 128) * 128;
  if (smem > 227 * 1024 || ldd % 4 != 0 || ldd < a.ncols) return cudaErrorInvalidValue;
  auto kern = split ? dist_tc_kernel<true> : dist_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(ceil_div(a.n, 128), a.heads), kDtThreads, smem, st>>>(
      static_cast<const __nv_bfloat16*>(a.X), a.n, a.Bhi, a.Blo, a.ncols, ldd, a.nrm, a.ecol, a.tau2, a.Dout,
      a.prop_g, a.prop_v, a.status);
  return counted(cudaGetLastError(), 1);
}

}  // namespace spr
