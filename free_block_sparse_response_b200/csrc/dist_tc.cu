// Balanced k-means distances on 5th-generation tensor cores (sm_100a).
//
// For every item i (a key or a query row, bf16, head dim 128) and group g:
//     D[i][g] = tau^2 (n_i - 2 x_i . w_g + e_g),   w_g = Gamma c_g,  e_g = c_g . w_g,
// the head-dim form of the squared response-space distance used by Response-Coupled
// Partitioning (SparsePR abstract, arXiv 2608.18484).  w_g enters as bf16 hi + lo, so
// the cross term carries ~16-bit precision.  The full fp32 row is written (row stride
// ldd, a multiple of 4), its argmin (ties to the lower group) is the first proposal of
// the capacity fill, and the minimum of each 64-column segment is kept for the later
// proposals.
//
// Persistent: one CTA per SM loops over (head, 128-item tile) work items; groups are
// streamed in chunks of 128 (W double-buffered, TMA into 128B-swizzled tiles); the
// accumulator chunk lives in TMEM (two buffers, so the MMA of chunk c+1 -- also of the
// next item -- overlaps the epilogue of chunk c).  Warp 0 loads, warp 2 issues the
// MMAs, warps 4-11 run the epilogue: each row is owned by two threads (columns 0-63 and
// 64-127 of every chunk); a warp transposes its 32 rows x 32 columns through shared
// memory so that each 16-byte-per-lane store instruction writes 128 contiguous bytes of
// each of 4 rows.  The row argmin is a strict '<' scan in
// ascending column order (first minimum wins, +-0 compare equal), merged across the two
// halves at the end.  Every wait is bounded.
#include <cuda.h>

#include "attention.cuh"
#include "common.cuh"
#include "partition.cuh"
#include "tcgen05.cuh"
#include "warp_mma.cuh"

namespace spr {
namespace {

constexpr int kDtThreads = 384;
constexpr uint32_t kDtTile = 128 * 128 * 2;
constexpr uint32_t kDtTmemCols = 256;
constexpr float kDtInf = __builtin_huge_valf();
constexpr uint32_t kWarpStage = 32 * 32 * 4;  // one warp's 32 x 32 fp32 transpose block

enum : int {
  kXFull0 = 0, kXEmpty0 = 2, kWFull0 = 4, kWEmpty0 = 6, kAccFull0 = 8, kAccEmpty0 = 10, kDtDrain = 12, kDtBars = 13
};

// Packed pairs of fp32: one f32x2 instruction, each lane rounded exactly as the scalar op.
__device__ __forceinline__ uint64_t dt_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void dt_f32x2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t dt_ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t dt_fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ unsigned long long dist_key(float v, int idx) {
  const uint32_t ok = (v != v) ? 0xffffffffu : float_order_key(v);
  return (static_cast<unsigned long long>(ok) << 32) | static_cast<uint32_t>(idx);
}

template <bool SPLIT>
__global__ void __launch_bounds__(kDtThreads, 1)
    dist_tc_kernel(const __grid_constant__ CUtensorMap tmX, int n, const __grid_constant__ CUtensorMap tmWhi,
                   const __grid_constant__ CUtensorMap tmWlo, int ncols, int ldd, const float* __restrict__ nrm,
                   const float* __restrict__ ecol, float tau2, float* __restrict__ Dout, int* __restrict__ prop_g,
                   float* __restrict__ prop_v, unsigned long long* __restrict__ seg_min, int nseg,
                   int* __restrict__ status, int heads) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bars[kDtBars];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ float s_best_v[128];
  __shared__ int s_best_c[128];
  constexpr int kWStage = kDtTile * (SPLIT ? 2 : 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = (tc::saddr(dsmem) + 1023u) & ~1023u;
  const uint32_t sX = sbase;
  const uint32_t sW[2] = {sbase + kDtTile, sbase + kDtTile + kWStage};
  const uint32_t sStage = sbase + kDtTile + 2 * kWStage;  // 8 warps x 4 KB transpose blocks
  float* s_e = reinterpret_cast<float*>(dsmem + (sbase - tc::saddr(dsmem)) + kDtTile + 2 * kWStage +
                                        8 * kWarpStage);
  auto bar = [&](int i) { return tc::saddr(&bars[i]); };
  const int n_chunks = ceil_div(ncols, 128);
  const int tiles = ceil_div(n, 128);
  const int total = heads * tiles;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      if (s == 0) {
        tc::mbar_init(bar(kXFull0), 1);
        tc::mbar_init(bar(kXEmpty0), 1);
      }
      tc::mbar_init(bar(kWFull0 + s), 1);
      tc::mbar_init(bar(kWEmpty0 + s), 1);
      tc::mbar_init(bar(kAccFull0 + s), 1);
      tc::mbar_init(bar(kAccEmpty0 + s), 256);
    }
    tc::mbar_init(bar(kDtDrain), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    tc::tmem_alloc(tc::saddr(&tmem_slot), kDtTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = tmem_slot;
  volatile int* abort_v = &abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // One lane: the item tile of X (two TMA boxes of 64 columns x 128 rows), then per
    // chunk the 128 rows of W (hi, and lo when split).  Rows past a head's n items or
    // ncols groups come from the next head (or are zero past the tensor): they only feed
    // rows that are never stored and columns whose e term is +inf.
    if (lane == 0) {
      bool ok = true;
      int last_it = -1, last_q = -1;
      for (int w = blockIdx.x, it = 0; ok && w < total; w += gridDim.x, ++it) {
        const int head = w / tiles, row0 = (w - head * tiles) * 128;
        if (it >= 1 && !tc::mbar_wait(bar(kXEmpty0), (it - 1) & 1, abort_v, status)) break;
        tc::mbar_arrive_expect_tx(bar(kXFull0), kDtTile);
        tc::tma_load_2d(sX, &tmX, 0, head * n + row0, bar(kXFull0));
        tc::tma_load_2d(sX + 128 * 128, &tmX, 64, head * n + row0, bar(kXFull0));
        last_it = it;
        for (int c = 0; c < n_chunks; ++c) {
          const int q = it * n_chunks + c, s = q & 1;
          if (q >= 2 && !tc::mbar_wait(bar(kWEmpty0 + s), ((q >> 1) - 1) & 1, abort_v, status)) {
            ok = false;
            break;
          }
          const int wrow = head * ncols + c * 128;
          tc::mbar_arrive_expect_tx(bar(kWFull0 + s), kWStage);
          tc::tma_load_2d(sW[s], &tmWhi, 0, wrow, bar(kWFull0 + s));
          tc::tma_load_2d(sW[s] + 128 * 128, &tmWhi, 64, wrow, bar(kWFull0 + s));
          if (SPLIT) {
            tc::tma_load_2d(sW[s] + kDtTile, &tmWlo, 0, wrow, bar(kWFull0 + s));
            tc::tma_load_2d(sW[s] + kDtTile + 128 * 128, &tmWlo, 64, wrow, bar(kWFull0 + s));
          }
          last_q = q;
        }
      }
      // copies still in flight after an abort land before the CTA exits (bounded waits)
      auto drain = [&](uint32_t b, uint32_t parity) {
        const uint64_t t0 = globaltimer_ns();
        while (!tc::mbar_try_wait(b, parity)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
      };
      for (int q = last_q - 1; q <= last_q; ++q)
        if (q >= 0) drain(bar(kWFull0 + (q & 1)), (q >> 1) & 1);
      if (last_it >= 0) drain(bar(kXFull0), last_it & 1);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kId = tc::idesc_bf16(128, 128, false, false);
      bool ok = true;
      for (int w = blockIdx.x, it = 0; ok && w < total; w += gridDim.x, ++it) {
        if (!tc::mbar_wait(bar(kXFull0), it & 1, abort_v, status)) break;
        tc::fence_proxy_async();
        for (int c = 0; c < n_chunks; ++c) {
          const int q = it * n_chunks + c, s = q & 1;
          if (!tc::mbar_wait(bar(kWFull0 + s), (q >> 1) & 1, abort_v, status) ||
              (q >= 2 && !tc::mbar_wait(bar(kAccEmpty0 + s), ((q >> 1) - 1) & 1, abort_v, status))) {
            ok = false;
            break;
          }
          tc::fence_proxy_async();
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
        if (ok) tc::mma_commit(bar(kXEmpty0));
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
    const int etid = tid - 128;               // 0..255 among the epilogue warps
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float m2t = -2.f * tau2;
    const uint32_t wstage = sStage + static_cast<uint32_t>(warp - 4) * kWarpStage;
    int loaded_head = -1;
    bool aborted = false;  // after a failed wait: keep passing the named barriers, skip the work
    for (int w = blockIdx.x, it = 0; w < total; w += gridDim.x, ++it) {
      const int head = w / tiles, row0 = (w - head * tiles) * 128;
      if (head != loaded_head) {  // tau^2 e_g of this head, padded with +inf to whole chunks
        asm volatile("bar.sync 1, 256;" ::: "memory");
        for (int c = etid; c < n_chunks * 128; c += 256)
          s_e[c] = c < ncols ? tau2 * ecol[static_cast<size_t>(head) * ncols + c] : kDtInf;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        loaded_head = head;
      }
      const int row = row0 + r;
      const float tnr = row < n ? tau2 * nrm[static_cast<size_t>(head) * n + row] : 0.f;
      // a distance is non-finite only if its row term or its column term is
      bool nonfinite = !isfinite(tnr);
      for (int c = etid; c < ncols; c += 256) nonfinite |= !isfinite(s_e[c]);
      float best_v = kDtInf;
      int best_c = -1;
      const int wrow0 = row0 + (warp & 3) * 32;
      const bool full_rows = wrow0 + 32 <= n;
      for (int c = 0; c < n_chunks && !aborted; ++c) {
        const int q = it * n_chunks + c, s = q & 1;
        const bool got = tc::mbar_wait(bar(kAccFull0 + s), (q >> 1) & 1, abort_v, status);
        if (!__all_sync(0xffffffffu, got)) {
          aborted = true;
          break;
        }
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
        // this 64-column segment's first minimum: four independent strict '<' scans over
        // the columns j = t (mod 4), each in ascending order, then merged (smaller value
        // wins, equal values -- +-0 included -- go to the lower column), which is the
        // first minimum of the whole segment
        float cv[4] = {kDtInf, kDtInf, kDtInf, kDtInf};
        int cc[4] = {-1, -1, -1, -1};
        const uint64_t m2 = dt_f32x2(m2t, m2t), tn2 = dt_f32x2(tnr, tnr);
#pragma unroll
        for (int qq = 0; qq < 16; ++qq) {
          const float4 e = e4[qq];
          float v[4];
          dt_f32x2_split(dt_fadd2(dt_ffma2(dt_f32x2(__uint_as_float(u[4 * qq]), __uint_as_float(u[4 * qq + 1])), m2, tn2),
                                  dt_f32x2(e.x, e.y)),
                         v[0], v[1]);
          dt_f32x2_split(dt_fadd2(dt_ffma2(dt_f32x2(__uint_as_float(u[4 * qq + 2]), __uint_as_float(u[4 * qq + 3])), m2,
                                           tn2),
                                  dt_f32x2(e.z, e.w)),
                         v[2], v[3]);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            u[4 * qq + t] = __float_as_uint(v[t]);
            if (v[t] < cv[t]) {
              cv[t] = v[t];
              cc[t] = 4 * qq + t;
            }
          }
        }
        float seg_v = cv[0];
        int seg_c = cc[0];
#pragma unroll
        for (int t = 1; t < 4; ++t) {
          if (cc[t] >= 0 && (seg_c < 0 || cv[t] < seg_v || (cv[t] == seg_v && cc[t] < seg_c))) {
            seg_v = cv[t];
            seg_c = cc[t];
          }
        }
        // segments in ascending column order: a strictly smaller minimum wins
        if (seg_c >= 0 && seg_v < best_v) {
          best_v = seg_v;
          best_c = c0 + seg_c;
        }
        if (seg_min != nullptr && row < n)
          seg_min[(static_cast<size_t>(head) * n + row) * nseg + 2 * c + half] =
              seg_c >= 0 ? dist_key(seg_v, c0 + seg_c) : ~0ull;
        // transpose 32 rows x 32 columns at a time through shared memory: lane l writes its
        // row's chunk k at chunk position k ^ (l & 7) (conflict-free), then reads column l
        // of every row, so each global store covers 128 contiguous bytes of one row
        const size_t rowbase = static_cast<size_t>(head) * n + wrow0;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int j = blk * 32 + 4 * k;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(wstage + lane * 128 + ((k ^ (lane & 7)) << 4)),
                         "r"(u[j]), "r"(u[j + 1]), "r"(u[j + 2]), "r"(u[j + 3])
                         : "memory");
          }
          __syncwarp();
          // lane l stores 4 consecutive columns (16 B) of row rr + (l >> 3): every store
          // instruction writes 128 contiguous bytes of each of 4 rows
          const int col = c0 + blk * 32 + 4 * (lane & 7);
          if (col < ldd) {
            const int rsub = lane >> 3;
            float* dst = Dout + (rowbase + rsub) * ldd + col;
#pragma unroll
            for (int rr = 0; rr < 32; rr += 4) {
              const int row_l = rr + rsub;
              if (full_rows || wrow0 + row_l < n) {
                float4 v;
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                             : "r"(wstage + row_l * 128 + (((lane & 7) ^ (row_l & 7)) << 4)));
                *reinterpret_cast<float4*>(dst) = v;
              }
              dst += 4 * static_cast<size_t>(ldd);
            }
          }
        }
      }
      if (half == 1) {
        s_best_v[r] = best_v;
        s_best_c[r] = best_c;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (half == 0 && row < n && !aborted) {
        const float v1 = s_best_v[r];
        const int c1 = s_best_c[r];
        // half 0 holds the lower 64 columns of every chunk: on equal values take the
        // lower column, on a smaller value take it
        if (c1 >= 0 && (best_c < 0 || v1 < best_v || (v1 == best_v && c1 < best_c))) {
          best_v = v1;
          best_c = c1;
        }
        if (best_c < 0) best_c = 0;
        const size_t o = static_cast<size_t>(head) * n + row;
        prop_g[o] = best_c;
        prop_v[o] = best_v;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (__any_sync(0xffffffffu, nonfinite && !aborted) && lane == 0) record_error(status, kErrNonFinite);
    }
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
  const size_t smem = kDtTile + 2ull * kDtTile * (split ? 2 : 1) + 8ull * kWarpStage + 1024 +
                      sizeof(float) * ceil_div(a.ncols, 128) * 128;
  if (smem > 227 * 1024 || ldd % 4 != 0 || ldd < a.ncols) return cudaErrorInvalidValue;
  auto kern = split ? dist_tc_kernel<true> : dist_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int total = a.heads * ceil_div(a.n, 128);
  const long long xrows = static_cast<long long>(a.heads) * a.n, wrows = static_cast<long long>(a.heads) * a.ncols;
  if (xrows > 0x7fffffffLL || wrows > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA coordinates are int32
  CUtensorMap tx, twh, twl;
  if (!bf16_map(&tx, a.X, xrows, 128) || !bf16_map(&twh, a.Bhi, wrows, 128) ||
      !bf16_map(&twl, split ? static_cast<const void*>(a.Blo) : static_cast<const void*>(a.Bhi), wrows, 128))
    return cudaErrorInvalidValue;
  kern<<<std::min(total, sms), kDtThreads, smem, st>>>(
      tx, a.n, twh, twl, a.ncols, ldd, a.nrm, a.ecol, a.tau2, a.Dout,
      a.prop_g, a.prop_v, a.seg_min, a.nseg, a.status, a.heads);
  return counted(cudaGetLastError(), 1);
}

}  // namespace spr
