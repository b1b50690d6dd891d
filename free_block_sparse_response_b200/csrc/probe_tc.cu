// Probe rows on 5th-generation tensor cores (sm_100a): for each probe query p of a head,
// the exact softmax attention over all N keys (dense) and over the key groups routed to
// p's query block (sparse), the two outputs the residual fit compares (SparsePR
// abstract, arXiv 2608.18484, arxivdaily.com English abstract: exact probe rows
// calibrate the correction).  The softmax weights enter the PV products as bf16 hi + lo
// (two products each), so the fit sees ~16-bit weights.
//
// CTA = (128 probe rows, one split of the key groups, head); 384 threads:
//   warp 0      gathers the 128 probe rows of Q (tile::gather4), then loads each key
//               group's K tile (two TMA boxes) from the group-ordered copy, two stages;
//   warp 2      the same for V;
//   warp 1      MMA issuer (one lane): S = Q K^T; once the softmax holds S the next S;
//               then O_d += P_d,hi V + P_d,lo V (P_d from TMEM) and O_s += P_s,hi V +
//               P_s,lo V (P_s from shared memory);
//   warps 4-11  softmax, two threads per probe row (columns 0-63 and 64-127 of the tile,
//               row maxima exchanged once per tile): running (max, sum) of the dense and of
//               the sparse state (the latter only on groups routed to the row's block;
//               zero weights elsewhere), lazy rescaling of O_d / O_s (max grows by > 2^8).
// The split of the key groups is at most 64 groups (membership is a 64-bit mask per row).
// At the end each row's unnormalised (m_d, l_d, m_s, l_s, O_d, O_s) of the split is
// written; a combine kernel merges the splits.
// TMEM (512 columns): S [0,128), O_d [128,256), O_s [256,384), P_d hi [384,448), lo [448,512).
// Shared memory: Q, K x2, V x2, P_s hi, P_s lo (7 x 32 KB).  Every wait is bounded.
#include <cuda.h>

#include "attention.cuh"
#include "common.cuh"
#include "tcgen05.cuh"
#include "warp_mma.cuh"

namespace spr {
namespace {

constexpr int kPtThreads = 384;
constexpr uint32_t kPtTile = 128 * 128 * 2;
constexpr uint32_t kPtTmemCols = 512;
constexpr float kPtRescaleLog2 = 8.0f;
constexpr float kPtInf = __builtin_huge_valf();

enum : int {
  kPQFull = 0, kPKFull0 = 1, kPVFull0 = 3, kPKEmpty0 = 5, kPVEmpty0 = 7, kPSFull = 9, kPSFree = 10,
  kPPFull = 11, kPPVDone = 12, kPDrain = 13, kPLx = 14, kPNumBars = 15
};

__device__ __forceinline__ float pt_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool pt_warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
  const bool ok = tc::mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void pt_drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
}

__device__ __forceinline__ void pt_st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__global__ void __launch_bounds__(kPtThreads, 1)
    probe_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, int N, int G, int k, int groups_per_split,
                    const int* __restrict__ probe_idx, int P, const int* __restrict__ key_gsize,
                    const int* __restrict__ route, const int* __restrict__ qblock_of_token, float scale_log2,
                    float* __restrict__ part, int* __restrict__ status) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bars[kPNumBars];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row_tile = blockIdx.x, split = blockIdx.y, head = blockIdx.z, nsplit = gridDim.y;
  const int g0 = split * groups_per_split, g1 = min(G, g0 + groups_per_split);
  const int n_tiles = max(g1 - g0, 0);
  const uint32_t sbase = (tc::saddr(dsmem) + 1023u) & ~1023u;
  const uint32_t sQ = sbase;
  auto sK = [&](int s) { return sbase + (1 + s) * kPtTile; };
  auto sV = [&](int s) { return sbase + (3 + s) * kPtTile; };
  const uint32_t sPh = sbase + 5 * kPtTile, sPl = sbase + 6 * kPtTile;
  auto bar = [&](int i) { return tc::saddr(&bars[i]); };

  if (tid == 0) {
    tc::mbar_init(bar(kPQFull), 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(kPKFull0 + s), 1);
      tc::mbar_init(bar(kPVFull0 + s), 1);
      tc::mbar_init(bar(kPKEmpty0 + s), 1);
      tc::mbar_init(bar(kPVEmpty0 + s), 1);
    }
    tc::mbar_init(bar(kPSFull), 1);
    tc::mbar_init(bar(kPSFree), 256);
    tc::mbar_init(bar(kPPFull), 256);
    tc::mbar_init(bar(kPLx), 256);
    tc::mbar_init(bar(kPPVDone), 1);
    tc::mbar_init(bar(kPDrain), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::saddr(&tmem_slot), kPtTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = tmem_slot;
  volatile int* abort_v = &abort_flag;
  const int row0 = head * N;            // first row of this head in the Q map
  const int kvrow0 = head * G * 128;    // first row of this head in the group-ordered maps
  const int* pidx = probe_idx + static_cast<size_t>(head) * P;
  const int prow0 = row_tile * 128;
  const int nrows = min(128, P - prow0);

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------------ producers
    const bool isK = warp == 0;
    if (isK) {
      // Q: lane l gathers probe rows 4 l .. 4 l + 3 (rows past P repeat the first one)
      const int rq = 4 * lane;
      int t[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) t[i] = row0 + __ldg(pidx + prow0 + (rq + i < nrows ? rq + i : 0));
      if (lane == 0) tc::mbar_arrive_expect_tx(bar(kPQFull), kPtTile);
      __syncwarp();
      tc::tma_gather4(sQ + rq * 128, &tmQ, 0, t[0], t[1], t[2], t[3], bar(kPQFull));
      tc::tma_gather4(sQ + 128 * 128 + rq * 128, &tmQ, 64, t[0], t[1], t[2], t[3], bar(kPQFull));
    }
    const CUtensorMap* tm = isK ? &tmK : &tmV;
    const int full0 = isK ? kPKFull0 : kPVFull0, empty0 = isK ? kPKEmpty0 : kPVEmpty0;
    int issued = 0;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1, it = j >> 1;
      if (it >= 1 && !pt_warp_wait(bar(empty0 + s), (it - 1) & 1, abort_v, status)) break;
      if (lane == 0) {
        const uint32_t dst = isK ? sK(s) : sV(s);
        const int row = kvrow0 + (g0 + j) * 128;
        tc::mbar_arrive_expect_tx(bar(full0 + s), kPtTile);
        tc::tma_load_2d(dst, tm, 0, row, bar(full0 + s));
        tc::tma_load_2d(dst + 128 * 128, tm, 64, row, bar(full0 + s));
      }
      __syncwarp();
      issued = j + 1;
    }
    // copies still in flight after an abort land before the CTA exits (bounded waits)
    if (lane == 0) {
      for (int j = max(0, issued - 2); j < issued; ++j) pt_drain_wait(bar(full0 + (j & 1)), (j >> 1) & 1);
      if (isK) pt_drain_wait(bar(kPQFull), 0);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdQK = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdPV = tc::idesc_bf16(128, 128, false, true);
      const uint32_t tS = tbase, tOd = tbase + 128, tOs = tbase + 256, tPh = tbase + 384, tPl = tbase + 448;
      bool ok = tc::mbar_wait(bar(kPQFull), 0, abort_v, status);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        if (!tc::mbar_wait(bar(kPKFull0 + s), (j >> 1) & 1, abort_v, status)) return false;
        tc::fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          tc::mma_ss(tS, tc::sdesc_sw128(sQ + koff, 16, 1024), tc::sdesc_sw128(sK(s) + koff, 16, 1024), kIdQK,
                     kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(bar(kPKEmpty0 + s));
        tc::mma_commit(bar(kPSFull));
        return true;
      };
      if (ok && n_tiles > 0) ok = issue_s(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j & 1;
        if (j + 1 < n_tiles) {  // S may take the next tile once the softmax holds it
          if (!tc::mbar_wait(bar(kPSFree), j & 1, abort_v, status)) break;
          tc::fence_after_sync();
          if (!issue_s(j + 1)) break;
        }
        if (!tc::mbar_wait(bar(kPPFull), j & 1, abort_v, status)) break;
        tc::fence_after_sync();
        if (!tc::mbar_wait(bar(kPVFull0 + s), (j >> 1) & 1, abort_v, status)) break;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t vdesc = tc::sdesc_sw128(sV(s) + kk * 2048, 128 * 128, 1024);
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          tc::mma_ts(tOd, tPh + kk * 8, vdesc, kIdPV, acc);
          tc::mma_ts(tOd, tPl + kk * 8, vdesc, kIdPV, 1u);
          tc::mma_ss(tOs, tc::sdesc_sw128(sPh + koff, 16, 1024), vdesc, kIdPV, acc);
          tc::mma_ss(tOs, tc::sdesc_sw128(sPl + koff, 16, 1024), vdesc, kIdPV, 1u);
        }
        tc::mma_commit(bar(kPVEmpty0 + s));
        tc::mma_commit(bar(kPPVDone));
      }
      tc::mma_commit(bar(kPDrain));
      pt_drain_wait(bar(kPDrain), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ softmax
    // Two threads per probe row: warp (quadrant q, half h) holds row 32 q + lane, columns
    // [64 h, 64 h + 64) of S and of P, and columns [64 h, 64 h + 64) of O_d / O_s.  Each
    // half also reads the other half of its row of S from TMEM for the row maximum (so
    // both take the same maximum), and keeps its own partial sums, added at the end.
    // Both states run in log2 units (scores x scale_log2).  The sparse weights reuse the
    // dense exponentials: 2^(y - m_s) = 2^(y - m_d) 2^(m_d - m_s), exact unless
    // 2^(y - m_d) underflows; a row whose sparse maximum trails the dense one by more than
    // 2^64 takes its own exponentials instead (warp-uniform branch).
    const int hf = (warp - 4) >> 2;
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tS = tbase + lane_off + 64 * hf, tSo = tbase + lane_off + 64 * (1 - hf), tOd = tbase + lane_off + 128 + 64 * hf,
                   tOs = tbase + lane_off + 256 + 64 * hf, tPh = tbase + lane_off + 384 + 32 * hf,
                   tPl = tbase + lane_off + 448 + 32 * hf;
    const int tok = __ldg(pidx + prow0 + (r < nrows ? r : 0));
    const int qb = __ldg(qblock_of_token + static_cast<size_t>(head) * N + tok);
    uint64_t member_bits = 0;  // bit (g - g0): group g routed to this row's query block
    {
      // the route row is sorted ascending (then -1 padding): eight independent loads per step
      const int* rt = route + (static_cast<size_t>(head) * G + qb) * k;
      for (int j0 = 0; j0 < k; j0 += 8) {
        int gg[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) gg[i] = j0 + i < k ? __ldg(rt + j0 + i) : -1;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (gg[i] >= g0 && gg[i] < g1) member_bits |= 1ull << (gg[i] - g0);
        if (gg[7] < 0 || gg[7] >= g1) break;  // -1 padding, or past this split's groups
      }
    }
    const int* gsz = key_gsize + static_cast<size_t>(head) * G;
    float m_d = -kPtInf, l_d = 0.f, m_s = -kPtInf, l_s = 0.f;  // l_*: this half's part
    bool ok = true, zeroed = false;
    int nv_next = n_tiles > 0 ? __ldg(gsz + g0) : 0;
    for (int t = 0; t < n_tiles; ++t) {
      const int nvalid = nv_next;
      if (t + 1 < n_tiles) nv_next = __ldg(gsz + g0 + t + 1);
      if (!pt_warp_wait(bar(kPSFull), t & 1, abort_v, status)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t u[64];
      tc::tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
      tc::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
      tc::tmem_wait_ld();
      if (nvalid < 128) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (64 * hf + c >= nvalid) u[c] = __float_as_uint(-kPtInf);
      }
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = __uint_as_float(u[i]);
#pragma unroll
      for (int c = 8; c < 64; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(u[c]));
      // the other half of the row (maximum only)
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        uint32_t w32[32];
        tc::tmem_ld32(tSo + 32 * q2, w32);
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (nvalid >= 128 || 64 * (1 - hf) + 32 * q2 + c < nvalid)
            mx8[c & 7] = fmaxf(mx8[c & 7], __uint_as_float(w32[c]));
      }
      tc::fence_before_sync();
      tc::mbar_arrive(bar(kPSFree));  // S may take the next tile once both halves hold it
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * scale_log2;
      // dense state: lazy rescale (the running max moves only when it grows by > 2^8)
      const bool grow_d = mx > m_d + kPtRescaleLog2;
      const bool need_od = grow_d && m_d != -kPtInf;
      float alpha_d = 1.f;
      if (grow_d) {
        alpha_d = need_od ? pt_ex2(m_d - mx) : 1.f;
        l_d *= alpha_d;
        m_d = mx;
      }
      // sparse state: only on groups routed to the row's block
      const bool member = (member_bits >> t) & 1ull;
      const bool grow_s = member && mx > m_s + kPtRescaleLog2;
      const bool need_os = grow_s && m_s != -kPtInf;
      float alpha_s = 1.f;
      if (grow_s) {
        alpha_s = need_os ? pt_ex2(m_s - mx) : 1.f;
        l_s *= alpha_s;
        m_s = mx;
      }
      const bool live_s = member && m_s != -kPtInf;
      const bool far = live_s && m_d - m_s > 64.f;
      const float csp = live_s && !far ? pt_ex2(m_d - m_s) : 0.f;
      const bool any_member = __any_sync(0xffffffffu, member);
      const bool any_far = __any_sync(0xffffffffu, far);
      const float md_safe = m_d == -kPtInf ? 0.f : m_d;
      const float ms_safe = m_s == -kPtInf ? 0.f : m_s;
      float sum_d = 0.f, sum_s = 0.f;
      if (!any_far) {
        // dense weights in place, while the previous tile's PV products still run
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float p0 = pt_ex2(fmaf(__uint_as_float(u[c]), scale_log2, -md_safe));
          const float p1 = pt_ex2(fmaf(__uint_as_float(u[c + 1]), scale_log2, -md_safe));
          u[c] = __float_as_uint(p0);
          u[c + 1] = __float_as_uint(p1);
          sum_d += p0 + p1;
        }
      }
      // P_d (TMEM), P_s (shared) and O_d / O_s are free once the previous PV is done
      if (t >= 1 && !pt_warp_wait(bar(kPPVDone), (t - 1) & 1, abort_v, status)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      if (__any_sync(0xffffffffu, need_od) || __any_sync(0xffffffffu, need_os)) {
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const float a = which == 0 ? alpha_d : alpha_s;
          if (!__any_sync(0xffffffffu, which == 0 ? need_od : need_os)) continue;
          const uint32_t ob = which == 0 ? tOd : tOs;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t o[32];
            tc::tmem_ld32(ob + q * 32, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
            tc::tmem_st32(ob + q * 32, o);
          }
        }
      }
      const float mem_f = live_s ? 1.f : 0.f;
      const bool write_s = any_member || !zeroed;
      // quarters of 32 keys of this half: 16 packed columns of P_d (hi, lo) and 4 16-byte
      // chunks of P_s
#pragma unroll
      for (int qt = 0; qt < 2; ++qt) {
        uint32_t hi[16], lo[16];
        const int ch0 = 8 * hf + 4 * qt;  // first 16-byte chunk of these keys in a P_s row
        if (any_far) {  // sparse weights from their own exponentials (before u is overwritten)
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = qt * 32 + 2 * i;
            const float p0 = mem_f * pt_ex2(fmaf(__uint_as_float(u[c]), scale_log2, -ms_safe));
            const float p1 = mem_f * pt_ex2(fmaf(__uint_as_float(u[c + 1]), scale_log2, -ms_safe));
            sum_s += p0 + p1;
            split_bf16x2(p0, p1, hi[i], lo[i]);
          }
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t off = tc::sw128_offset(r, ch0 + c4);
            pt_st_shared_v4(sPh + off, hi[4 * c4], hi[4 * c4 + 1], hi[4 * c4 + 2], hi[4 * c4 + 3]);
            pt_st_shared_v4(sPl + off, lo[4 * c4], lo[4 * c4 + 1], lo[4 * c4 + 2], lo[4 * c4 + 3]);
          }
        }
        // dense weights (computed above unless a row of the warp is far), kept in u
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = qt * 32 + 2 * i;
          float p0 = __uint_as_float(u[c]), p1 = __uint_as_float(u[c + 1]);
          if (any_far) {
            p0 = pt_ex2(fmaf(p0, scale_log2, -md_safe));
            p1 = pt_ex2(fmaf(p1, scale_log2, -md_safe));
            u[c] = __float_as_uint(p0);
            u[c + 1] = __float_as_uint(p1);
            sum_d += p0 + p1;
          }
          split_bf16x2(p0, p1, hi[i], lo[i]);
        }
        tc::tmem_st16(tPh + 16 * qt, hi);
        tc::tmem_st16(tPl + 16 * qt, lo);
        if (!any_far && write_s) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = qt * 32 + 2 * i;
            split_bf16x2(__uint_as_float(u[c]) * csp, __uint_as_float(u[c + 1]) * csp, hi[i], lo[i]);
          }
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t off = tc::sw128_offset(r, ch0 + c4);
            pt_st_shared_v4(sPh + off, hi[4 * c4], hi[4 * c4 + 1], hi[4 * c4 + 2], hi[4 * c4 + 3]);
            pt_st_shared_v4(sPl + off, lo[4 * c4], lo[4 * c4 + 1], lo[4 * c4 + 2], lo[4 * c4 + 3]);
          }
        }
      }
      zeroed = !any_member;
      l_d += sum_d;
      l_s += any_far ? sum_s : csp * sum_d;
      tc::tmem_wait_st();
      tc::fence_proxy_async();  // P_s (generic-proxy stores) visible to the tensor core
      tc::fence_before_sync();
      tc::mbar_arrive(bar(kPPFull));
    }
    // ---- partial records [m_d, l_d, m_s, l_s, O_d[128], O_s[128]] of this split; each half
    // writes its 64 columns of O_d and O_s, half 0 the (max, sum) header
    constexpr int kRec = 4 + 2 * 128;
    const bool have_rows = ok && n_tiles > 0 && pt_warp_wait(bar(kPPVDone), (n_tiles - 1) & 1, abort_v, status);
    float4* rec = reinterpret_cast<float4*>(
        part + ((static_cast<size_t>(head) * P + prow0 + r) * nsplit + split) * kRec);
    const bool mine = r < nrows;
    if (have_rows) {
      // the halves' (l_d, l_s) meet in the P_s buffer, free after the last PV product
      float2* s_l = reinterpret_cast<float2*>(dsmem + (sPh - tc::saddr(dsmem)));
      s_l[hf * 128 + r] = make_float2(l_d, l_s);
      tc::mbar_arrive(bar(kPLx));
      const bool got = pt_warp_wait(bar(kPLx), 0, abort_v, status);
      tc::fence_after_sync();
      if (got && mine && hf == 0) {
        const float2 o2 = s_l[128 + r];
        rec[0] = make_float4(m_d, l_d + o2.x, m_s, l_s + o2.y);
      }
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tc::tmem_ld32((q < 2 ? tOd : tOs) + (q & 1) * 32, o);
        tc::tmem_wait_ld();
        if (got && mine) {
          const int base = 1 + (q < 2 ? 0 : 32) + 16 * hf + 8 * (q & 1);  // float4 index in the record
#pragma unroll
          for (int i = 0; i < 8; ++i)
            rec[base + i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                        __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        }
      }
    } else if (ok && n_tiles == 0 && mine) {
      if (hf == 0) rec[0] = make_float4(-kPtInf, 0.f, -kPtInf, 0.f);
      for (int i = 0; i < 16; ++i) {
        rec[1 + 16 * hf + i] = make_float4(0.f, 0.f, 0.f, 0.f);   // O_d columns of this half
        rec[33 + 16 * hf + i] = make_float4(0.f, 0.f, 0.f, 0.f);  // O_s columns of this half
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, kPtTmemCols);
  }
}

}  // namespace

cudaError_t launch_probe_tc(const ProbeArgs& a, int nsplit, cudaStream_t st) {
  if (a.f32 || a.d != 128 || a.block != 128 || a.k_grouped == nullptr || a.v_grouped == nullptr ||
      a.status == nullptr || nsplit < 1)
    return cudaErrorInvalidValue;
  if (a.P <= 0 || a.heads <= 0) return cudaSuccess;
  const int gps = ceil_div(a.G, nsplit);
  if (gps > 64) return cudaErrorInvalidValue;  // membership is a 64-bit mask per row
  const long long rows = static_cast<long long>(a.heads) * a.N;
  const long long grows = static_cast<long long>(a.heads) * a.G * 128;
  if (rows > 0x7fffffffLL || grows > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA coordinates are int32
  CUtensorMap tq, tk, tv;
  if (!bf16_map(&tq, a.Q, rows, 1) || !bf16_map(&tk, a.k_grouped, grows, 128) ||
      !bf16_map(&tv, a.v_grouped, grows, 128))
    return cudaErrorInvalidValue;
  const size_t smem = 7ull * kPtTile + 1024;
  cudaError_t e = cudaFuncSetAttribute(probe_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  probe_tc_kernel<<<dim3(ceil_div(a.P, 128), nsplit, a.heads), kPtThreads, smem, st>>>(
      tq, tk, tv, a.N, a.G, a.k, gps, a.probe_idx, a.P, a.key_gsize, a.route, a.qblk, a.scale_log2, a.partial,
      a.status);
  return counted(cudaGetLastError(), 1);
}

}  // namespace spr
