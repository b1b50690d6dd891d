// Block-sparse (and dense) flash attention on 5th-generation tensor cores (sm_100a).
//
// Method (SparsePR abstract, arXiv 2608.18484, arxivdaily.com English abstract): each
// query block attends only to its routed key groups, softmax renormalised over that
// support.  One CTA per (query block of 128 rows, head); head dim 128; key groups of 128.
//
// The routed tiles j = 0 .. n-1 of a block are split into two streams, even and odd j.
// Each stream keeps its own S tile (TMEM), P tile (shared memory), running max / sum
// and O accumulator (TMEM), so that the two softmax warpgroups work on different tiles
// at the same time; the two partial results are merged at the end like a split-K
// softmax: O = (2^(m0-m) O0 + 2^(m1-m) O1) / (2^(m0-m) l0 + 2^(m1-m) l1), m = max(m0, m1).
// Within a stream, S is released as soon as the softmax holds it in registers, so QK of
// the stream's next tile runs while the softmax of the current one computes P.
//
// Warp roles (384 threads, one CTA per SM):
//   warp 0      gathers the block's Q rows through the query permutation (tile::gather4,
//               4 token rows per instruction; pad rows of a short block repeat its first
//               member), then loads K of every routed tile; warp 1 loads V.  Each tile is
//               two 64-column x 128-row TMA boxes of the group-ordered K / V copies
//               (sparse) or of K / V in token order (dense), into the buffer of its stream.
//   warps 2-3   MMA issuers, lane 0 of warp 2 + x drives stream x: S_x = Q K^T (TMEM),
//               and O_x += P V with P from shared memory.  With one issuer per stream,
//               one stream's waits and commits overlap the other stream's MMAs.
//   warps 4-7   softmax, stream 0; warps 8-11 softmax, stream 1.  Thread i of a
//               warpgroup owns TMEM lane i (query row i); it reads S, keeps the running
//               max / sum, writes P (bf16) into the 128B-swizzled P tile, rescales its O
//               only when the row max grew by more than 2^8 (stale maxima are exact after
//               the final division), and at the end merges the two streams for half the
//               columns.
// Warps 0-3 give registers to the softmax warpgroups (setmaxnreg).
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// Shared memory: Q, and per stream one K, one V and one P tile (7 x 32 KB).
// Every wait is bounded; on timeout the CTA records kErrTimeout, drains its MMAs and
// copies and frees TMEM before exiting.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <utility>
#include <vector>

#include "attention.cuh"
#include "common.cuh"
#include "tcgen05.cuh"
#include "warp_mma.cuh"

namespace spr {
namespace {

constexpr int kTcThreads = 384;
constexpr int kRegLow = 72;       // warps 0-3 after the re-split
constexpr int kRegSoftmax = 216;  // warps 4-11 after the re-split
constexpr uint32_t kTile = 128 * 128 * 2;  // one 128 x 128 bf16 tile
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kInf = __builtin_huge_valf();

// Barriers: Q landed; per stream x (index + x): K / V tile landed, S ready (QK done,
// which also frees the stream's K buffer), S loaded by the softmax (S may be
// overwritten), P written to shared memory, PV done (which frees the stream's V and P
// buffers and means O_x holds every finished tile), drain; and the last PV of both
// streams.
// Fused correction only: M (hi, lo) landed, the merged S tile (hi, lo) written, S M^T done.
enum : int {
  kQFull = 0, kKFull0 = 1, kVFull0 = 3, kSFull0 = 5, kSFree0 = 7, kPFull0 = 9, kVEmpty0 = 11, kDrain0 = 13,
  kOFinal = 15, kMFull = 16, kSFin = 17, kCorr = 18, kNumBars = 19
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed pairs of fp32 (one f32x2 instruction does two lanes' worth of FMA / add).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
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

// FUSED (sparse only): O = S + S M^T + beta is formed in the epilogue and written as
// bf16 to out_bf16; S itself never leaves the SM.  Otherwise S (fp32) goes to out.
template <bool DENSE, bool FUSED, bool VARLEN>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmM, int N, int G,
                   int k, const int* __restrict__ key_gsize, const int* __restrict__ query_perm,
                   const int* __restrict__ qblock_size, const int* __restrict__ route, float scale_log2,
                   float* __restrict__ out, const float* __restrict__ beta, __nv_bfloat16* __restrict__ out_bf16,
                   int* __restrict__ status) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x, head = blockIdx.y;
  // shared memory: Q, then per stream x a K, a V and a P tile (128 x 128 bf16 each,
  // 128B-swizzled, 1024-byte aligned)
  const uint32_t sbase = (tc::saddr(dsmem) + 1023u) & ~1023u;
  const uint32_t sQ = sbase;
  auto sK = [&](int x) { return sbase + (1 + x) * kTile; };
  auto sV = [&](int x) { return sbase + (3 + x) * kTile; };
  auto sP = [&](int x) { return sbase + (5 + x) * kTile; };
  uint8_t* const gsP0 = dsmem + (sP(0) - tc::saddr(dsmem));  // generic pointer to stream 0's P tile
  auto bar = [&](int i) { return tc::saddr(&bars[i]); };

  if (tid == 0) {
    tc::mbar_init(bar(kQFull), 1);
    for (int x = 0; x < 2; ++x) {
      tc::mbar_init(bar(kKFull0 + x), 1);
      tc::mbar_init(bar(kVFull0 + x), 1);
      tc::mbar_init(bar(kSFull0 + x), 1);
      tc::mbar_init(bar(kSFree0 + x), 128);
      tc::mbar_init(bar(kPFull0 + x), 128);
      tc::mbar_init(bar(kVEmpty0 + x), 1);
      tc::mbar_init(bar(kDrain0 + x), 1);
    }
    tc::mbar_init(bar(kOFinal), 2);
    tc::mbar_init(bar(kMFull), 1);
    tc::mbar_init(bar(kSFin), 256);
    tc::mbar_init(bar(kCorr), 1);
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

  const int row0 = head * N;  // first row of this head in the [heads * N, 128] tensor maps
  out += static_cast<size_t>(head) * N * 128;
  if (FUSED) out_bf16 += static_cast<size_t>(head) * N * 128;
  const size_t goff = static_cast<size_t>(head) * G;
  const int nq = DENSE ? min(128, N - b * 128) : qblock_size[goff + b];
  const int* qperm = DENSE ? nullptr : query_perm + (goff + b) * 128;
  const int* my_route = DENSE ? nullptr : route + (goff + b) * k;
  // VARLEN: route rows of capacity k = G that end with -1 (global pair budget); otherwise
  // every row holds exactly k groups and the count stays a kernel parameter
  const int n_tiles = DENSE ? G : VARLEN ? routed_len(my_route, k) : k;
  // key group of routed tile j and its number of members
  auto group_of = [&](int j) { return DENSE ? j : __ldg(my_route + j); };
  auto size_of = [&](int g) { return DENSE ? min(128, N - g * 128) : __ldg(key_gsize + goff + g); };
  volatile int* abort_v = &abort_flag;

  if (warp < 4) {
    tc::setmaxnreg_dec<kRegLow>();
    if (warp < 2) {
      // ------------------------------------------------------------------ producers
      if (warp == 0) {
        // Q: lane l gathers rows 4 l .. 4 l + 3 through the query permutation (two
        // gather4 per lane, one per 64-column half of the swizzled tile).
        const int rq = 4 * lane;
        int4 t;
        if (DENSE) {
          const int base = row0 + b * 128;
          t = make_int4(base + min(rq, nq - 1), base + min(rq + 1, nq - 1), base + min(rq + 2, nq - 1),
                        base + min(rq + 3, nq - 1));
        } else {
          const int4 v = __ldg(reinterpret_cast<const int4*>(qperm + rq));
          const int first = __shfl_sync(0xffffffffu, v.x, 0);
          t = make_int4(row0 + (rq < nq ? v.x : first), row0 + (rq + 1 < nq ? v.y : first),
                        row0 + (rq + 2 < nq ? v.z : first), row0 + (rq + 3 < nq ? v.w : first));
        }
        if (lane == 0) tc::mbar_arrive_expect_tx(bar(kQFull), kTile);
        __syncwarp();
        tc::tma_gather4(sQ + rq * 128, &tmQ, 0, t.x, t.y, t.z, t.w, bar(kQFull));
        tc::tma_gather4(sQ + 128 * 128 + rq * 128, &tmQ, 64, t.x, t.y, t.z, t.w, bar(kQFull));
      }
      // K (warp 0) and V (warp 1) of each routed group, tile after tile, into the buffer
      // of the tile's stream: two 64-column x 128-row boxes of the group-ordered copies
      // (sparse) or of K and V in token order (dense).  K of a stream's next tile waits
      // only for the stream's previous QK, V only for its previous PV.
      const bool isK = warp == 0;
      const int kvrow0 = DENSE ? row0 : head * G * 128;
      const CUtensorMap* tm = isK ? &tmK : &tmV;
      const int full0 = isK ? kKFull0 : kVFull0;
      // the stream's buffer is free once its previous QK (K) or PV (V) is done
      const int free0 = isK ? kSFull0 : kVEmpty0;
      int issued = 0;  // tiles whose copies were issued
      int g_next = n_tiles > 0 ? group_of(0) : 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int xs = j & 1, it = j >> 1;
        const int row = kvrow0 + g_next * 128;
        if (j + 1 < n_tiles) g_next = group_of(j + 1);
        if (it >= 1 && !warp_wait(bar(free0 + xs), (it - 1) & 1, abort_v, status)) break;
        if (lane == 0) {
          const uint32_t dst = isK ? sK(xs) : sV(xs);
          tc::mbar_arrive_expect_tx(bar(full0 + xs), kTile);
          tc::tma_load_2d(dst, tm, 0, row, bar(full0 + xs));
          tc::tma_load_2d(dst + 128 * 128, tm, 64, row, bar(full0 + xs));
        }
        issued = j + 1;
      }
      // Copies still in flight after an abort must land before the CTA exits: wait
      // (bounded) for the last phase of each stream's buffer and for Q.  On the normal
      // path these phases completed long ago and the waits return at once.
      if (lane == 0) {
        for (int j = max(0, issued - 2); j < issued; ++j) drain_wait(bar(full0 + (j & 1)), (j >> 1) & 1);
        if (isK) drain_wait(bar(kQFull), 0);
        // fused correction: M of this head (hi into K buffer 0, lo into K buffer 1) once
        // every MMA of the attention is done and the K buffers are free
        if (FUSED && isK && tc::mbar_wait(bar(kOFinal), 0, abort_v, status)) {
          tc::mbar_arrive_expect_tx(bar(kMFull), 2 * kTile);
          tc::tma_load_2d(sK(0), &tmM, 0, head * 128, bar(kMFull));
          tc::tma_load_2d(sK(0) + 128 * 128, &tmM, 64, head * 128, bar(kMFull));
          tc::tma_load_2d(sK(1), &tmM, 0, (gridDim.y + head) * 128, bar(kMFull));
          tc::tma_load_2d(sK(1) + 128 * 128, &tmM, 64, (gridDim.y + head) * 128, bar(kMFull));
          drain_wait(bar(kMFull), 0);  // the copies land before this thread can exit
        }
      }
      __syncwarp();
    } else if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuers
      // Lane 0 of warp 2 + x drives stream x.  Per tile: as soon as the softmax has
      // loaded S, S of the stream's next tile is computed (it overlaps the softmax);
      // then O_x += P V with P from shared memory.
      const int x = warp - 2;
      constexpr uint32_t kIdMma = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdPV = tc::idesc_bf16(128, 128, false, true);
      const uint32_t tS = tbase + 128 * x, tO = tbase + 256 + 128 * x;
      const int n_x = n_tiles > x ? (n_tiles - x + 1) / 2 : 0;  // tiles of this stream
      bool ok = tc::mbar_wait(bar(kQFull), 0, abort_v, status);
      auto issue_s = [&](int it) -> bool {
        if (!tc::mbar_wait(bar(kKFull0 + x), it & 1, abort_v, status)) return false;
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          tc::mma_ss(tS, tc::sdesc_sw128(sQ + koff, 16, 1024), tc::sdesc_sw128(sK(x) + koff, 16, 1024), kIdMma,
                     kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar(kSFull0 + x));
        return true;
      };
      if (ok && n_x > 0) ok = issue_s(0);
      for (int it = 0; ok && it < n_x; ++it) {
        if (it + 1 < n_x) {
          // S_x may be overwritten once the softmax holds tile it's scores in registers
          if (!tc::mbar_wait(bar(kSFree0 + x), it & 1, abort_v, status)) break;
          tc::fence_after_sync();
          if (!issue_s(it + 1)) break;
        }
        if (!tc::mbar_wait(bar(kPFull0 + x), it & 1, abort_v, status)) break;
        tc::fence_after_sync();
        if (!tc::mbar_wait(bar(kVFull0 + x), it & 1, abort_v, status)) break;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          tc::mma_ss(tO, tc::sdesc_sw128(sP(x) + koff, 16, 1024),
                     tc::sdesc_sw128(sV(x) + kk * 2048, 128 * 128, 1024), kIdPV, (it > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(bar(kVEmpty0 + x));
      }
      tc::mma_commit(bar(kOFinal));
      tc::mma_commit(bar(kDrain0 + x));
      drain_wait(bar(kDrain0 + x), 0);
      if (FUSED && x == 0 && ok && tc::mbar_wait(bar(kMFull), 0, abort_v, status) &&
          tc::mbar_wait(bar(kSFin), 0, abort_v, status)) {
        // S M^T into TMEM columns [0, 128) (S of stream 0, free now) in split precision:
        // S_hi M_hi + S_hi M_lo + S_lo M_hi, S tiles in the V buffers, M tiles in the K ones
        tc::fence_after_sync();
        const uint32_t sA[3] = {sV(0), sV(0), sV(1)}, sB[3] = {sK(0), sK(1), sK(0)};
#pragma unroll
        for (int t = 0; t < 3; ++t) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
            tc::mma_ss(tbase, tc::sdesc_sw128(sA[t] + koff, 16, 1024), tc::sdesc_sw128(sB[t] + koff, 16, 1024),
                       kIdMma, (t > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(bar(kCorr));
        tc::mma_commit(bar(kDrain0));
        drain_wait(bar(kDrain0), 1);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax
    tc::setmaxnreg_inc<kRegSoftmax>();
    const int x = (warp - 4) >> 2;  // stream: tiles x, x + 2, x + 4, ...
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t sbuf = tbase + lane_off + x * 128;
    const uint32_t obuf = tbase + lane_off + 256 + x * 128;
    const int tok = r < nq ? (DENSE ? b * 128 + r : __ldg(qperm + r)) : -1;
    float m_run = -kInf, l_run = 0.f;
    bool ok = true;
    int nv_next = x < n_tiles ? size_of(group_of(x)) : 0;
    for (int j = x, it = 0; j < n_tiles; j += 2, ++it) {
      const int nvalid = nv_next;
      if (j + 2 < n_tiles) nv_next = size_of(group_of(j + 2));  // in flight during this tile
      if (!warp_wait(bar(kSFull0 + x), it & 1, abort_v, status)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t u[128];
      tc::tmem_ld32(sbuf, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
      tc::tmem_ld32(sbuf + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
      tc::tmem_ld32(sbuf + 64, *reinterpret_cast<uint32_t(*)[32]>(&u[64]));
      tc::tmem_ld32(sbuf + 96, *reinterpret_cast<uint32_t(*)[32]>(&u[96]));
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      tc::mbar_arrive(bar(kSFree0 + x));  // S_x may now take the stream's next tile
      if (nvalid < 128) {  // short group (warp-uniform): mask the padding keys
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= nvalid) u[c] = __float_as_uint(-kInf);
      }
      // row max: 8 independent chains of 3-input maxima
      float mx8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mx8[t] = __uint_as_float(u[t]);
#pragma unroll
      for (int c = 8; c < 128; c += 2)
        mx8[(c >> 1) & 7] = fmax3(mx8[(c >> 1) & 7], __uint_as_float(u[c]), __uint_as_float(u[c + 1]));
      float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
      mx *= scale_log2;
      const bool grow = mx > m_run + kRescaleLog2;
      const bool need_o = grow && m_run != -kInf;
      float alpha = 1.f;
      if (grow) {
        alpha = need_o ? ex2(m_run - mx) : 1.f;
        l_run *= alpha;
        m_run = mx;
      }
      // The P tile is free, and O_x holds every earlier tile, once the previous PV is done.
      if (it >= 1 && !warp_wait(bar(kVEmpty0 + x), (it - 1) & 1, abort_v, status)) {
        ok = false;
        break;
      }
      if (__any_sync(0xffffffffu, need_o)) {
        tc::fence_after_sync();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tc::tmem_ld32(obuf + q * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc::tmem_st32(obuf + q * 32, o);
        }
        tc::tmem_wait_st();
      }
      const float msafe = m_run == -kInf ? 0.f : m_run;
      const uint64_t sc2 = f32x2(scale_log2, scale_log2), nm2 = f32x2(-msafe, -msafe);
      uint64_t acc2[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int c = half * 64 + 2 * i;
          float y0, y1;
          f32x2_split(ffma2(f32x2(__uint_as_float(u[c]), __uint_as_float(u[c + 1])), sc2, nm2), y0, y1);
          const float p0 = ex2(y0), p1 = ex2(y1);
          acc2[i & 1] = fadd2(acc2[i & 1], f32x2(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        // row r of the 128B-swizzled P tile (K-major A operand of the PV MMA)
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8)
          st_shared_v4(sP(x) + tc::sw128_offset(r, half * 8 + c8), pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2],
                       pk[4 * c8 + 3]);
      }
      float sum4[4];
      f32x2_split(acc2[0], sum4[0], sum4[1]);
      f32x2_split(acc2[1], sum4[2], sum4[3]);
      l_run += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      tc::fence_proxy_async();  // P (generic-proxy stores) visible to the tensor core
      tc::fence_before_sync();
      tc::mbar_arrive(bar(kPFull0 + x));
    }
    // ---- merge the two streams; warpgroup x writes columns [64 x, 64 x + 64)
    const bool fin = ok && warp_wait(bar(kOFinal), 0, abort_v, status);
    // every PV is done: the P tiles are free and hold each row's (max, sum) per stream
    float2* s_ml = reinterpret_cast<float2*>(gsP0);
    if (fin) s_ml[x * 128 + r] = make_float2(m_run, l_run);
    tc::named_bar_sync(1, 256);  // every softmax thread reaches this exactly once
    float sv[FUSED ? 64 : 1];  // this thread's 64 merged S values (fused correction)
    if (fin) {
      tc::fence_after_sync();
      const float2 a0 = s_ml[r], a1 = s_ml[128 + r];
      const float mm = fmaxf(a0.x, a1.x);
      const float f0 = a0.x == -kInf ? 0.f : ex2(a0.x - mm);
      const float f1 = a1.x == -kInf ? 0.f : ex2(a1.x - mm);
      const float den = a0.y * f0 + a1.y * f1;
      const float inv = den > 0.f ? 1.f / den : 0.f;
      const float g0 = f0 * inv, g1 = f1 * inv;
      const bool has1 = n_tiles > 1;  // stream 1 never wrote O1 otherwise
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int col = 64 * x + 32 * q;
        uint32_t o0[32], o1[32];
        tc::tmem_ld32(tbase + lane_off + 256 + col, o0);
        if (has1) tc::tmem_ld32(tbase + lane_off + 384 + col, o1);
        tc::tmem_wait_ld();
        if (!has1) {
#pragma unroll
          for (int i = 0; i < 32; ++i) o1[i] = 0u;
        }
        if (FUSED) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            sv[32 * q + i] = fmaf(__uint_as_float(o0[i]), g0, __uint_as_float(o1[i]) * g1);
        } else if (tok >= 0) {
          float4* dst = reinterpret_cast<float4*>(out + static_cast<size_t>(tok) * 128 + col);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float v[4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
              v[t] = fmaf(__uint_as_float(o0[4 * i + t]), g0, __uint_as_float(o1[4 * i + t]) * g1);
            dst[i] = make_float4(v[0], v[1], v[2], v[3]);
          }
        }
      }
    }
    if (FUSED) {
      // ---- the correction: row r of the merged S (columns [64 x, 64 x + 64)) as bf16
      // hi and lo into the V buffers (K-major A operands), S M^T on the tensor cores,
      // then O = S + S M^T + beta in bf16
      if (fin) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float a = sv[8 * c8 + 2 * t], b2 = sv[8 * c8 + 2 * t + 1];
            const __nv_bfloat16 ah = __float2bfloat16_rn(a), bh = __float2bfloat16_rn(b2);
            hi[t] = pack_bf16x2(a, b2);
            lo[t] = pack_bf16x2(a - __bfloat162float(ah), b2 - __bfloat162float(bh));
          }
          st_shared_v4(sV(0) + tc::sw128_offset(r, 8 * x + c8), hi[0], hi[1], hi[2], hi[3]);
          st_shared_v4(sV(1) + tc::sw128_offset(r, 8 * x + c8), lo[0], lo[1], lo[2], lo[3]);
        }
      }
      tc::fence_proxy_async();
      tc::mbar_arrive(bar(kSFin));
      if (fin && warp_wait(bar(kCorr), 0, abort_v, status)) {
        tc::fence_after_sync();
        const float* bh = beta + static_cast<size_t>(head) * 128 + 64 * x;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t c32[32];
          tc::tmem_ld32(tbase + lane_off + 64 * x + 32 * q, c32);
          tc::tmem_wait_ld();
          if (tok >= 0) {
            uint4* dst = reinterpret_cast<uint4*>(out_bf16 + static_cast<size_t>(tok) * 128 + 64 * x + 32 * q);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t w[4];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const int c = 8 * i + 2 * t;
                const float v0 = sv[32 * q + c] + __uint_as_float(c32[c]) + __ldg(bh + 32 * q + c);
                const float v1 = sv[32 * q + c + 1] + __uint_as_float(c32[c + 1]) + __ldg(bh + 32 * q + c + 1);
                w[t] = pack_bf16x2(v0, v1);
              }
              dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
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

// K and V rows of every key group, in group order: row r of group g of head h lands at
// row (h G + g) 128 + r of the copies; rows past the group's size are zero.  One CTA per
// (group, head); 16 threads copy one 256-byte row with 16-byte accesses.
struct KvTag {
  unsigned long long w[6];
};

__global__ void __launch_bounds__(256) kv_group_kernel(const uint4* __restrict__ K, const uint4* __restrict__ V,
                                                       int N, int G, const int* __restrict__ key_perm,
                                                       const int* __restrict__ key_gsize, uint4* __restrict__ Kg,
                                                       uint4* __restrict__ Vg, KvTag want,
                                                       const unsigned long long* __restrict__ have) {
  if (have != nullptr) {  // the copy in the workspace already comes from these inputs
    bool same = true;
#pragma unroll
    for (int i = 0; i < 6; ++i) same = same && have[i] == want.w[i];
    if (same) return;
  }
  const int g = blockIdx.x, head = blockIdx.y;
  const size_t grp = static_cast<size_t>(head) * G + g;
  const int gs = __ldg(key_gsize + grp);
  const int ch = threadIdx.x & 15;
#pragma unroll 4
  for (int r = threadIdx.x >> 4; r < 128; r += 16) {
    const int tok = r < gs ? __ldg(key_perm + grp * 128 + r) : -1;
    const size_t dst = (grp * 128 + r) * 16 + ch;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
    if (tok >= 0 && tok < N) {
      const size_t src = (static_cast<size_t>(head) * N + tok) * 16 + ch;
      kv = __ldg(K + src);
      vv = __ldg(V + src);
    }
    Kg[dst] = kv;
    Vg[dst] = vv;
  }
}

}  // namespace

// Q, and a K, a V and a P tile per stream, plus the 1024-byte alignment slack.
size_t attn_tc_smem_bytes(int) { return 7ull * kTile + 1024; }

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

// Map over a [rows, 128] bf16 tensor with 128-byte swizzle and a box of 64 columns x
// box_rows rows (1 for row gathers).
bool bf16_map(CUtensorMap* m, const void* base, long long rows, int box_rows) {
  auto fn = encode_tiled();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(base) & 15u) != 0 || rows <= 0) return false;
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {128 * sizeof(__nv_bfloat16)};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
__global__ void kv_tag_kernel(KvTag want, unsigned long long* have) {
  if (threadIdx.x < 6) have[threadIdx.x] = want.w[threadIdx.x];
}
}  // namespace

cudaError_t launch_kv_group(const void* K, const void* V, int N, int G, int heads, const int* key_perm,
                            const int* key_gsize, void* k_grouped, void* v_grouped, unsigned long long* kv_tag,
                            cudaStream_t st) {
  if (G <= 0 || heads <= 0) return cudaSuccess;
  const KvTag want{{reinterpret_cast<uintptr_t>(K), reinterpret_cast<uintptr_t>(V),
                    reinterpret_cast<uintptr_t>(key_perm), reinterpret_cast<uintptr_t>(key_gsize),
                    (static_cast<unsigned long long>(static_cast<unsigned>(N)) << 32) | static_cast<unsigned>(G),
                    static_cast<unsigned long long>(heads)}};
  kv_group_kernel<<<dim3(G, heads), 256, 0, st>>>(static_cast<const uint4*>(K), static_cast<const uint4*>(V), N, G,
                                                  key_perm, key_gsize, static_cast<uint4*>(k_grouped),
                                                  static_cast<uint4*>(v_grouped), want, kv_tag);
  cudaError_t e = counted(cudaGetLastError(), 1);
  if (e != cudaSuccess || kv_tag == nullptr) return e;
  kv_tag_kernel<<<1, 32, 0, st>>>(want, kv_tag);
  return counted(cudaGetLastError(), 1);
}

namespace {
std::mutex g_timing_mu;
bool g_timing_on = false;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_timing_pairs;  // recorded, not yet read
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_timing_free;   // reusable
}  // namespace

void attn_timing_enable(bool on) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  g_timing_on = on;
}

cudaError_t attn_timing_read(double* ms_total, long long* launches) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  double total = 0.0;
  cudaError_t err = cudaSuccess;
  for (auto& pr : g_timing_pairs) {
    cudaError_t e = cudaEventSynchronize(pr.second);
    float ms = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pr.first, pr.second);
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    total += ms;
    g_timing_free.push_back(pr);
  }
  if (launches) *launches = static_cast<long long>(g_timing_pairs.size());
  g_timing_pairs.clear();
  if (ms_total) *ms_total = total;
  return err;
}

cudaError_t launch_attention_tc(const AttnArgs& a, bool dense, int* status, cudaStream_t st) {
  const size_t smem = attn_tc_smem_bytes(dense ? a.G : a.k);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  const bool fused = !dense && a.m_hilo != nullptr;
  if (fused && (a.beta == nullptr || a.out_bf16 == nullptr)) return cudaErrorInvalidValue;
  const bool varlen = !dense && a.k == a.G;
  auto kern = dense    ? attn_tc_kernel<true, false, false>
              : fused  ? (varlen ? attn_tc_kernel<false, true, true> : attn_tc_kernel<false, true, false>)
                       : (varlen ? attn_tc_kernel<false, false, true> : attn_tc_kernel<false, false, false>);
  // The register re-split must fit in what the block is launched with, or the
  // setmaxnreg.inc of the softmax warpgroups would never be granted.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (128 * kRegLow + 256 * kRegSoftmax > fa.numRegs * kTcThreads) return cudaErrorInvalidConfiguration;
  const long long rows = static_cast<long long>(a.heads) * a.N;
  const long long grows = static_cast<long long>(a.heads) * a.G * 128;
  if (rows > 0x7fffffffLL || grows > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA coordinates are int32
  if (!dense && (a.k_grouped == nullptr || a.v_grouped == nullptr)) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, tm;
  const bool maps = bf16_map(&tq, a.Q, rows, 1) &&
                    (dense ? bf16_map(&tk, a.K, rows, 128) && bf16_map(&tv, a.V, rows, 128)
                           : bf16_map(&tk, a.k_grouped, grows, 128) && bf16_map(&tv, a.v_grouped, grows, 128));
  if (!maps) return cudaErrorInvalidValue;
  // M of every head as bf16 hi rows [0, 128 heads) then lo rows [128 heads, 256 heads)
  if (fused) {
    if (!bf16_map(&tm, a.m_hilo, 2LL * a.heads * 128, 128)) return cudaErrorInvalidValue;
  } else {
    tm = tk;  // unused
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (!dense) {
    e = launch_kv_group(a.K, a.V, a.N, a.G, a.heads, a.key_perm, a.key_gsize, a.k_grouped, a.v_grouped, a.kv_tag,
                        st);
    if (e != cudaSuccess) return e;
  }
  std::pair<cudaEvent_t, cudaEvent_t> ev{nullptr, nullptr};
  {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    if (g_timing_on) {
      if (!g_timing_free.empty()) {
        ev = g_timing_free.back();
        g_timing_free.pop_back();
      } else if (cudaEventCreate(&ev.first) != cudaSuccess || cudaEventCreate(&ev.second) != cudaSuccess) {
        return cudaErrorMemoryAllocation;
      }
    }
  }
  if (ev.first != nullptr && (e = cudaEventRecord(ev.first, st)) != cudaSuccess) return e;
  kern<<<dim3(a.G, a.heads), kTcThreads, smem, st>>>(
      tq, tk, tv, tm, a.N, a.G, a.k, a.key_gsize, a.query_perm, a.qblock_size, a.route, a.scale_log2, a.out,
      a.beta, static_cast<__nv_bfloat16*>(a.out_bf16), status);
  e = counted(cudaGetLastError(), 1);
  if (ev.first != nullptr) {
    cudaError_t e2 = cudaEventRecord(ev.second, st);
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timing_pairs.push_back(ev);
    if (e == cudaSuccess) e = e2;
  }
  return e;
}

}  // namespace spr
