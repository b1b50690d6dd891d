// Block-sparse (and dense) flash attention on 5th-generation tensor cores (sm_100a).
//
// Method (SparsePR abstract, arXiv 2608.18484, arxivdaily.com English abstract): each
// query block attends only to its routed key groups, softmax renormalised over that
// support.  One CTA per (query block of 128 rows, head); head dim 128; key groups of 128.
//
// Warp roles (256 threads, one CTA per SM):
//   warps 0-1  producers: gather the block's Q rows and each routed group's K and V rows
//              (through the permutations) with cp.async into 128B-swizzled UMMA tiles;
//              K and V double-buffered; arrival on mbarriers when the copies land.
//   warp 2     MMA issuer (one lane): S_j = Q K_j^T into TMEM (double-buffered, so S_{j+1}
//              overlaps the softmax of tile j), O += P_j V_j with P read from TMEM.
//   warps 4-7  softmax: thread i owns TMEM lane i (query row i); reads S_j, keeps the
//              running max / sum, writes P_j (bf16) back over S_j, rescales O only when
//              the row max grew by more than 2^8 (stale maxima are exact after the final
//              division), and writes the normalised row at the end.
// TMEM (512 columns): S0 [0,128), S1 [128,256), O [256,384).
// Every wait is bounded; on timeout the CTA records kErrTimeout, drains its MMAs and
// frees TMEM before exiting.
#include "attention.cuh"
#include "common.cuh"
#include "tcgen05.cuh"
#include "warp_mma.cuh"

namespace spr {
namespace {

constexpr int kTcThreads = 256;
constexpr int kTcProducers = 64;
constexpr uint32_t kTile = 128 * 128 * 2;  // one 128 x 128 bf16 tile
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kInf = __builtin_huge_valf();

enum : int {
  kQFull = 0, kKFull0 = 1, kVFull0 = 3, kKEmpty0 = 5, kVEmpty0 = 7, kSFull0 = 9,
  kPFull = 11, kOReady = 12, kOFinal = 13, kDrain = 14, kNumBars = 15
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
  const bool ok = tc::mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag (used to drain outstanding MMAs).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
}

template <bool DENSE>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                   const __nv_bfloat16* __restrict__ V, int N, int G, int k, const int* __restrict__ key_perm,
                   const int* __restrict__ key_gsize, const int* __restrict__ query_perm,
                   const int* __restrict__ qblock_size, const int* __restrict__ route, float scale_log2,
                   float* __restrict__ out, int* __restrict__ status) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x, head = blockIdx.y;
  const uint32_t sbase = (tc::saddr(dsmem) + 1023u) & ~1023u;
  const uint32_t sQ = sbase;
  const uint32_t sK[2] = {sbase + kTile, sbase + 2 * kTile};
  const uint32_t sV[2] = {sbase + 3 * kTile, sbase + 4 * kTile};
  auto bar = [&](int i) { return tc::saddr(&bars[i]); };

  if (tid == 0) {
    tc::mbar_init(bar(kQFull), kTcProducers);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(kKFull0 + s), kTcProducers);
      tc::mbar_init(bar(kVFull0 + s), kTcProducers);
      tc::mbar_init(bar(kKEmpty0 + s), 1);
      tc::mbar_init(bar(kVEmpty0 + s), 1);
      tc::mbar_init(bar(kSFull0 + s), 1);
    }
    tc::mbar_init(bar(kPFull), 128);
    tc::mbar_init(bar(kOReady), 1);
    tc::mbar_init(bar(kOFinal), 1);
    tc::mbar_init(bar(kDrain), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    tc::tmem_alloc(tc::saddr(&tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = tmem_slot;

  const size_t hoff = static_cast<size_t>(head) * N * 128;
  Q += hoff;
  K += hoff;
  V += hoff;
  out += hoff;
  const size_t goff = static_cast<size_t>(head) * G;
  const int nq = DENSE ? min(128, N - b * 128) : qblock_size[goff + b];
  const int* qperm = DENSE ? nullptr : query_perm + (goff + b) * 128;
  const int* kperm = DENSE ? nullptr : key_perm + goff * 128;
  const int n_tiles = DENSE ? G : k;
  const int* my_route = DENSE ? nullptr : route + (goff + b) * k;
  // per-tile key group and its size, staged once (the producers and the softmax read them)
  int* s_group = reinterpret_cast<int*>(dsmem + (sbase - tc::saddr(dsmem)) + 5 * kTile);
  int* s_size = s_group + n_tiles;
  for (int j = tid; j < n_tiles; j += kTcThreads) {
    const int g = DENSE ? j : __ldg(my_route + j);
    s_group[j] = g;
    s_size[j] = DENSE ? min(128, N - g * 128) : __ldg(key_gsize + goff + g);
  }
  __syncthreads();
  volatile int* abort_v = &abort_flag;

  if (warp < 2) {
    // ------------------------------------------------------------------ producers
    // Thread pt copies 16-byte chunk (pt & 15) of rows (pt >> 4) + 4 i, i < 32: 16 threads
    // cover one 256-byte row.  The 32 row indices are fetched before any copy is issued.
    const int pt = tid, ch = pt & 15, r0 = pt >> 4;
    int toks[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int r = r0 + 4 * i;
      toks[i] = r < nq ? (DENSE ? b * 128 + r : __ldg(qperm + r)) : -1;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int r = r0 + 4 * i;
      cp_async_16(sQ + tc::sw128_offset(r, ch), toks[i] >= 0 ? Q + static_cast<size_t>(toks[i]) * 128 + ch * 8 : Q,
                  toks[i] >= 0 ? 16 : 0);
    }
    tc::cp_async_arrive_noinc(bar(kQFull));
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1;
      const int g = s_group[j];
      const int gs = s_size[j];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = r0 + 4 * i;
        toks[i] = r < gs ? (DENSE ? g * 128 + r : __ldg(kperm + g * 128 + r)) : -1;
      }
      if (j >= 2 && !tc::mbar_wait(bar(kKEmpty0 + s), ((j >> 1) - 1) & 1, abort_v, status)) break;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = r0 + 4 * i;
        cp_async_16(sK[s] + tc::sw128_offset(r, ch),
                    toks[i] >= 0 ? K + static_cast<size_t>(toks[i]) * 128 + ch * 8 : K, toks[i] >= 0 ? 16 : 0);
      }
      tc::cp_async_arrive_noinc(bar(kKFull0 + s));
      if (j >= 2 && !tc::mbar_wait(bar(kVEmpty0 + s), ((j >> 1) - 1) & 1, abort_v, status)) break;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = r0 + 4 * i;
        cp_async_16(sV[s] + tc::sw128_offset(r, ch),
                    toks[i] >= 0 ? V + static_cast<size_t>(toks[i]) * 128 + ch * 8 : V, toks[i] >= 0 ? 16 : 0);
      }
      tc::cp_async_arrive_noinc(bar(kVFull0 + s));
    }
    cp_async_wait<0>();
  } else if (warp == 2) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdQK = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdPV = tc::idesc_bf16(128, 128, false, true);
      const uint32_t tS[2] = {tbase, tbase + 128};
      const uint32_t tO = tbase + 256;
      bool ok = tc::mbar_wait(bar(kQFull), 0, abort_v, status);
      tc::fence_proxy_async();
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        if (!tc::mbar_wait(bar(kKFull0 + s), (j >> 1) & 1, abort_v, status)) return false;
        tc::fence_proxy_async();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          tc::mma_ss(tS[s], tc::sdesc_sw128(sQ + koff, 16, 1024), tc::sdesc_sw128(sK[s] + koff, 16, 1024), kIdQK,
                     kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar(kKEmpty0 + s));
        tc::mma_commit(bar(kSFull0 + s));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_tiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j & 1;
        if (!tc::mbar_wait(bar(kPFull), j & 1, abort_v, status)) break;
        tc::fence_after_sync();
        if (!tc::mbar_wait(bar(kVFull0 + s), (j >> 1) & 1, abort_v, status)) break;
        tc::fence_proxy_async();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          tc::mma_ts(tO, tS[s] + kk * 8, tc::sdesc_sw128(sV[s] + kk * 2048, 128 * 128, 1024), kIdPV,
                     (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(bar(kVEmpty0 + s));
        tc::mma_commit(bar(kOReady));
        if (j + 2 < n_tiles && !issue_s(j + 2)) break;
        if (j == n_tiles - 1) tc::mma_commit(bar(kOFinal));
      }
      tc::mma_commit(bar(kDrain));
      drain_wait(bar(kDrain), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax
    const int r = tid - 128;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp - 4)) << 16;
    const int tok = r < nq ? (DENSE ? b * 128 + r : __ldg(qperm + r)) : -1;
    float m_run = -kInf, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1;
      if (!warp_wait(bar(kSFull0 + s), (j >> 1) & 1, abort_v, status)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t sbuf = tbase + lane_off + s * 128;
      uint32_t u[128];
      tc::tmem_ld32(sbuf, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
      tc::tmem_ld32(sbuf + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
      tc::tmem_ld32(sbuf + 64, *reinterpret_cast<uint32_t(*)[32]>(&u[64]));
      tc::tmem_ld32(sbuf + 96, *reinterpret_cast<uint32_t(*)[32]>(&u[96]));
      tc::tmem_wait_ld();
      const int nvalid = s_size[j];
      if (nvalid < 128) {  // short group (warp-uniform): mask the padding keys
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= nvalid) u[c] = __float_as_uint(-kInf);
      }
      // row max as a tree of 8 independent chains
      float mx8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mx8[t] = __uint_as_float(u[t]);
#pragma unroll
      for (int c = 8; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(u[c]));
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      mx *= scale_log2;
      const bool grow = mx > m_run + kRescaleLog2;
      const bool need_o = grow && m_run != -kInf;
      float alpha = 1.f;
      if (grow) {
        alpha = need_o ? ex2(m_run - mx) : 1.f;
        l_run *= alpha;
        m_run = mx;
      }
      if (__any_sync(0xffffffffu, need_o)) {
        if (!warp_wait(bar(kOReady), (j - 1) & 1, abort_v, status)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t obuf = tbase + lane_off + 256;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tc::tmem_ld32(obuf + q * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc::tmem_st32(obuf + q * 32, o);
        }
      }
      const float msafe = m_run == -kInf ? 0.f : m_run;
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2(fmaf(__uint_as_float(u[half * 64 + 2 * i]), scale_log2, -msafe));
          const float p1 = ex2(fmaf(__uint_as_float(u[half * 64 + 2 * i + 1]), scale_log2, -msafe));
          sum4[i & 3] += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tc::tmem_st32(sbuf + half * 32, pk);
      }
      l_run += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(bar(kPFull));
    }
    if (ok && warp_wait(bar(kOFinal), 0, abort_v, status)) {
      tc::fence_after_sync();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      const uint32_t obuf = tbase + lane_off + 256;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tc::tmem_ld32(obuf + q * 32, o);
        tc::tmem_wait_ld();
        if (tok >= 0) {
          float4* dst = reinterpret_cast<float4*>(out + static_cast<size_t>(tok) * 128 + q * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                 __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace

size_t attn_tc_smem_bytes(int n_tiles) { return 5ull * kTile + 1024 + 8ull * n_tiles; }

cudaError_t launch_attention_tc(const AttnArgs& a, bool dense, int* status, cudaStream_t st) {
  const size_t smem = attn_tc_smem_bytes(dense ? a.G : a.k);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  auto kern = dense ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.G, a.heads), kTcThreads, smem, st>>>(
      static_cast<const __nv_bfloat16*>(a.Q), static_cast<const __nv_bfloat16*>(a.K),
      static_cast<const __nv_bfloat16*>(a.V), a.N, a.G, a.k, a.key_perm, a.key_gsize, a.query_perm, a.qblock_size,
      a.route, a.scale_log2, a.out, status);
  return counted(cudaGetLastError(), 1);
}

}  // namespace spr
