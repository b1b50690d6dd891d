// Balanced k-means assignment on 5th-generation tensor cores (sm_100a): the capacity-B
// fill of one k-means iteration with every proposal round's distances recomputed on
// tcgen05, so that no distance matrix is ever stored.
//
// Source: SparsePR abstract (arXiv 2608.18484): keys are grouped by their responses to
// sampled queries, queries by their responses to the key-group centroids.  Both are the
// balanced k-means whose assignment is the proposal-round fill: every unplaced item
// proposes to its nearest group with room (ties to the lower group), every group takes
// its proposers in ascending (distance, token) order while it has room.  Distances are
//     D[i][g] = tau^2 (n_i - 2 x_i . w_g + e_g),   w_g = Gamma c_g,  e_g = c_g . w_g,
// the head-dim form of the squared response-space distance; w_g enters as bf16 hi + lo.
//
// One cooperative launch per iteration, one CTA per SM, all heads.  Each round:
//   A. proposals: the unplaced items of every head, 256 at a time, are multiplied with the
//      head's W in chunks of 128 groups (X by four 2-D TMA boxes in the first round; in
//      the later rounds the rows of the unplaced list, read by two loader warps with
//      coalesced loads, and W only the head's open groups, packed at the round's start
//      with a column -> group map; W hi and lo double-buffered and used for both 128-row
//      halves, which halves the W traffic from L2; two accumulators per stage, double-
//      buffered, fill the 512 TMEM columns); the epilogue forms D exactly as above and
//      keeps the first minimum over the OPEN groups (a full group's e_g is staged as +inf,
//      so its D never wins a strict '<' scan): the item's proposal;
//   B. per head: groups whose proposers fit their room take them all (room and full-group
//      bit updated here); the others get bucket offsets and join the overflow list;
//   C. every proposer of a group that takes all is placed; the others are scattered into
//      their group's bucket as (D, token) keys (slots reserved per distinct group of a
//      warp);
//   D. every overflowing group takes its room's worth of best proposers (radix select of
//      the kth key) and is full; the rejected join the head's list for the next round.
// A grid barrier separates the phases.  Every item's D row is the same fp32 numbers in
// every round (same operands, same MMA sequence, same epilogue arithmetic; a packed
// column is computed exactly as its group's full column), so the decisions are the
// fill's decisions on that one matrix.  Once few items are left, one round also stores
// their D rows; the tail's first proposals then run across the grid and its later rounds
// one head per CTA from those rows.  Warp roles in phase A: warp 0 issues the TMA loads,
// warps 1 and 3 load the gathered rows, warp 2 issues the MMAs, warps 4-11 run the
// epilogue (two threads per row pair: columns 0-63 and 64-127 of every chunk, rows r and
// r + 128); phases B-D use all 12 warps.  Per-head list lengths are staged in shared
// memory once per round.  Every wait is bounded.  With Dout set, the first round also
// stores every item's D row (row stride ldd) for the parity tests.  Norm mode (nrm_out
// set, W = Gamma, G = d): one pass over all items whose epilogue forms x_i^T Gamma x_i from
// the accumulator row and the item's own row of the X tile in shared memory, and no fill.
#include <cuda.h>

#include "attention.cuh"
#include "common.cuh"
#include "fill_select.cuh"
#include "partition.cuh"
#include "tcgen05.cuh"

namespace spr {
namespace {

constexpr int kAsThreads = 384;              // warp 0 loads, warp 2 issues MMAs, warps 4-11 epilogue
constexpr int kAsWarps = kAsThreads / 32;
constexpr int kAsEpi = kAsThreads - 128;     // epilogue threads: 2 per row, 64 columns each
constexpr int kAsRows = 256;                 // items per work item: two 128-row halves
constexpr uint32_t kAsTile = 128 * 128 * 2;  // 128 rows x 128 bf16: two 64-column swizzled boxes
constexpr uint32_t kAsXStage = 2 * kAsTile;  // one work item's X (two buffers)
constexpr uint32_t kAsWStage = kAsTile;      // half a chunk of W: its hi or its lo part
constexpr uint32_t kAsTmemCols = 512;        // 2 stages x 2 halves x 128 fp32 columns
constexpr int kAsMaxCols = 1024;             // groups per head
constexpr int kAsMaxHeads = 1024;            // heads per launch (the launcher splits larger calls)
constexpr float kAsInf = __builtin_huge_valf();

enum : int { kXFull0 = 0, kXEmpty0 = 2, kWFull0 = 4, kWEmpty0 = 6, kAccFull0 = 8, kAccEmpty0 = 10, kDrain = 12, kBars = 13 };

__device__ __forceinline__ uint64_t as_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void as_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t as_ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t as_fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Walks the heads in order for increasing positions (work items or list entries):
// position p -> (head, position within the head), given per-head counts in shared memory.
struct HeadWalk {
  int h = 0, base = 0;
  int ibase = 0;  // list entries of the heads passed (when `lens` is given)
  __device__ void seek(const int* cnt, int p, int& head, int& off, const int* lens = nullptr) {
    while (p >= base + cnt[h]) {
      base += cnt[h];
      if (lens != nullptr) ibase += lens[h];
      ++h;
    }
    head = h;
    off = p - base;
  }
};

// One 64-column half-chunk of a row: D from the accumulator columns u (u is overwritten
// with D), and the first minimum over the open groups merged into (best_v, best_c).  The
// half-chunk's minimum comes from four fminf chains (NaN never wins: fminf drops it; a
// full group's +inf never wins either); only when it is strictly below every earlier
// column's is the first column holding it looked for, so the result is the first minimum
// of the row in ascending column order, as a strict '<' scan would give (+-0 compare
// equal, so the first zero of either sign is the one kept).
__device__ __forceinline__ void scan_half_chunk(uint32_t (&u)[64], const float* s_e, int c0, float tnr, float m2t,
                                                float& best_v, int& best_c) {
  const float4* e4 = reinterpret_cast<const float4*>(s_e + c0);
  float mn[4] = {kAsInf, kAsInf, kAsInf, kAsInf};
  const uint64_t m2 = as_f32x2(m2t, m2t), tn2 = as_f32x2(tnr, tnr);
#pragma unroll
  for (int qq = 0; qq < 16; ++qq) {
    const float4 e = e4[qq];
    float v[4];
    as_split(as_fadd2(as_ffma2(as_f32x2(__uint_as_float(u[4 * qq]), __uint_as_float(u[4 * qq + 1])), m2, tn2),
                      as_f32x2(e.x, e.y)),
             v[0], v[1]);
    as_split(as_fadd2(as_ffma2(as_f32x2(__uint_as_float(u[4 * qq + 2]), __uint_as_float(u[4 * qq + 3])), m2, tn2),
                      as_f32x2(e.z, e.w)),
             v[2], v[3]);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      u[4 * qq + t] = __float_as_uint(v[t]);
      mn[t] = fminf(mn[t], v[t]);
    }
  }
  const float m = fminf(fminf(mn[0], mn[1]), fminf(mn[2], mn[3]));
  if (m < best_v) {  // chunks ascend: only a strictly smaller value can displace the best
    int idx = 0;
#pragma unroll
    for (int k = 63; k >= 0; --k)
      if (__uint_as_float(u[k]) == m) idx = k;
    best_v = m;
    best_c = c0 + idx;
  }
}

// Exclusive prefix sum of one value per thread over the CTA (kAsThreads threads): warp
// scans by shuffles, the warp totals scanned by warp 0 through `tmp` (kAsWarps ints), two
// CTA barriers.  Every thread of the CTA calls it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = lane < kAsWarps ? tmp[lane] : 0;
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    if (lane < kAsWarps) tmp[lane] = ti - t;
  }
  __syncthreads();
  return tmp[warp] + incl - v;
}

// Of a warp's chunk of an overflowing group's bucket (key u * 32 + lane in kb[u], the
// first valid_n valid), the keys <= thr join the group's member list and the others the
// head's next list.  One atomic per list reserves the chunk's slots; positions follow the
// warp's ballots.  Neither order affects a decision: the group update sorts the members,
// and an item's next proposal is its own whatever its place in the list.
__device__ __forceinline__ void accept_reject(const unsigned long long (&kb)[8], int valid_n, unsigned long long thr,
                                              int g, int* lab, int* members_g, int* msize_g, int* nlist, int* nlen) {
  const int lane = threadIdx.x & 31;
  unsigned int tk[8], rj[8];
  int ntk = 0, nrj = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const bool valid = u * 32 + lane < valid_n;
    const bool take = valid && kb[u] <= thr;
    tk[u] = __ballot_sync(0xffffffffu, take);
    rj[u] = __ballot_sync(0xffffffffu, valid && !take);
    ntk += __popc(tk[u]);
    nrj += __popc(rj[u]);
  }
  int bt = 0, br = 0;
  if (lane == 0) {
    if (ntk > 0) bt = atomicAdd(msize_g, ntk);
    if (nrj > 0) br = atomicAdd(nlen, nrj);
  }
  bt = __shfl_sync(0xffffffffu, bt, 0);
  br = __shfl_sync(0xffffffffu, br, 0);
  const unsigned int lt = (1u << lane) - 1u;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int i = static_cast<int>(kb[u] & 0xffffffffu);
    if ((tk[u] >> lane) & 1u) {
      lab[i] = g;
      members_g[bt + __popc(tk[u] & lt)] = i;
    } else if ((rj[u] >> lane) & 1u) {
      nlist[br + __popc(rj[u] & lt)] = i;
    }
    bt += __popc(tk[u]);
    br += __popc(rj[u]);
  }
}

// Tail proposals of the kTailItems items x0.. of head h's list hl (len items) from their
// stored D rows, by one warp, their row loads in flight together; clw: the head's
// full-group bitmap.  The rule is the epilogue's: the first minimum over the open groups
// (strict '<' in ascending column order, so +inf and NaN never win; none finite: the
// lowest open group at +inf).  The proposal's value is the winning key's (+-0 read as +0,
// which the decision keys do not tell apart).
constexpr int kTailItems = 4;
__device__ __forceinline__ void tail_propose(const AssignArgs& a, int h, const int* hl, int len, int x0,
                                             const unsigned int* clw) {
  const int lane = threadIdx.x & 31;
  const int n = a.n, G = a.G, words = ceil_div(G, 32);
  const int xl = x0 + lane;
  size_t my_grow = 0;
  long long my_row = -1;
  if (lane < kTailItems && xl < len) {
    my_grow = static_cast<size_t>(h) * n + __ldcg(hl + xl);
    my_row = static_cast<long long>(__ldcg(a.tailpos + my_grow)) * a.ldt;
  }
  const float* rows[kTailItems];
  unsigned long long best[kTailItems];
#pragma unroll
  for (int k = 0; k < kTailItems; ++k) {
    const long long ro = __shfl_sync(0xffffffffu, my_row, k);
    rows[k] = ro >= 0 ? a.Dtail + ro : nullptr;
    best[k] = ~0ull;
  }
  int first_open = G;
  for (int w0 = 0; w0 < words; w0 += 16) {  // 16 words of every row requested at once
    float v[kTailItems][16];
#pragma unroll
    for (int k = 0; k < kTailItems; ++k) {
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int g = (w0 + u) * 32 + lane;
        v[k][u] = (rows[k] != nullptr && g < G) ? __ldcg(rows[k] + g) : kAsInf;
      }
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int wd = w0 + u;
      const int g = wd * 32 + lane;
      const bool open = g < G && !((clw[wd < words ? wd : 0] >> lane) & 1u);
#pragma unroll
      for (int k = 0; k < kTailItems; ++k) {
        if (open && v[k][u] < kAsInf) {
          const unsigned long long key = decision_key(v[k][u], g);
          best[k] = key < best[k] ? key : best[k];
        }
      }
      const unsigned int om = __ballot_sync(0xffffffffu, open);
      if (first_open == G && om != 0u) first_open = wd * 32 + __ffs(om) - 1;
    }
  }
  unsigned long long mine = ~0ull;
#pragma unroll
  for (int k = 0; k < kTailItems; ++k) {
    best[k] = warp_min_u64(best[k]);
    if (lane == k) mine = best[k];
  }
  if (lane < kTailItems && xl < len) {
    int g;
    float pv;
    if (mine != ~0ull) {
      g = static_cast<int>(mine & 0xffffffffu);
      pv = float_from_order_key(static_cast<uint32_t>(mine >> 32));
    } else if (first_open < G) {
      g = first_open;
      pv = kAsInf;
    } else {  // no open group: more items than room (cannot happen)
      record_error(&a.hdr->status, kErrInvalidArg);
      g = 0;
      pv = kAsInf;
    }
    a.prop_g[my_grow] = g;
    a.prop_v[my_grow] = pv;
    atomicAdd(a.cnt + static_cast<size_t>(h) * G + g, 1);
  }
}

__global__ void __launch_bounds__(kAsThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmWhi, const __grid_constant__ CUtensorMap tmWlo,
                     const __grid_constant__ CUtensorMap tmWcHi, const __grid_constant__ CUtensorMap tmWcLo,
                     AssignArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kBars];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, s_enf, s_remaining, s_total;
  __shared__ float s_best_v[kAsRows];  // the upper column halves' partial results
  __shared__ int s_best_c[kAsRows];
  __shared__ int s_xidx[2][128];       // the loader warps' row items
  __shared__ int s_inch[4];            // W chunks of the producer's latest work items

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = (tc::saddr(smem_raw) + 1023u) & ~1023u;
  const uint32_t sX[2] = {sbase, sbase + kAsXStage};  // two work items, each two 128-row halves
  const uint32_t sW[2] = {sbase + 2 * kAsXStage, sbase + 2 * kAsXStage + kAsWStage};
  uint8_t* sgen = smem_raw + (sbase - tc::saddr(smem_raw)) + 2 * kAsXStage + 2 * kAsWStage;
  float* s_e = reinterpret_cast<float*>(sgen);                   // [kAsMaxCols]
  // phases B-D (and the per-head rounds) run with no copy or MMA in flight: their scratch
  // lives in the idle W stages
  int* scan_tmp = reinterpret_cast<int*>(smem_raw + (sW[1] - tc::saddr(smem_raw)));              // [kAsThreads]
  unsigned int (*hist)[256] = reinterpret_cast<unsigned int (*)[256]>(smem_raw + (sW[0] - tc::saddr(smem_raw)));
  int* s_len = reinterpret_cast<int*>(sgen + 4 * kAsMaxCols);     // [kAsMaxHeads] list lengths
  int* s_tiles = s_len + kAsMaxHeads;                             // [kAsMaxHeads] work items per head
  int* s_nch = s_tiles + kAsMaxHeads;                             // [kAsMaxHeads] W chunks per head
  int* s_g = s_nch + kAsMaxHeads;                                 // [kAsMaxCols] packed column -> group
  auto bar = [&](int i) { return tc::saddr(&bars[i]); };

  const int n = a.n, G = a.G, heads = a.heads;
  const int n_chunks = ceil_div(G, 128);
  const int words = ceil_div(G, 32);
  const unsigned int nblocks = gridDim.x;
  const int gthread = blockIdx.x * kAsThreads + tid, nthreads = nblocks * kAsThreads;
  const int gwarp = gthread >> 5, nwarps = nthreads >> 5;
  int* status = &a.hdr->status;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(kXFull0 + s), 2);  // TMA rounds: the producer twice; gathered: each loader warp
      tc::mbar_init(bar(kXEmpty0 + s), 1);
      tc::mbar_init(bar(kWFull0 + s), 1);
      tc::mbar_init(bar(kWEmpty0 + s), 1);
      tc::mbar_init(bar(kAccFull0 + s), 1);
      tc::mbar_init(bar(kAccEmpty0 + s), kAsEpi);
    }
    tc::mbar_init(bar(kDrain), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    tc::tmem_alloc(tc::saddr(&tmem_slot), kAsTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = tmem_slot;
  volatile int* abort_v = &abort_flag;

  const bool norm_mode = a.nrm_out != nullptr;
  // ---- fill state: nothing placed, every group open with room B, no lists yet
  if (!norm_mode) {
    const size_t items = static_cast<size_t>(heads) * n, groups = static_cast<size_t>(heads) * G;
    for (size_t x = gthread; x < items; x += nthreads) a.labels[x] = -1;
    for (size_t x = gthread; x < groups; x += nthreads) {
      a.room[x] = a.cap;
      a.cnt[x] = 0;
      a.cursor[x] = 0;
      a.msize[x] = 0;
    }
    for (size_t x = gthread; x < static_cast<size_t>(heads) * words; x += nthreads) a.closed[x] = 0u;
    for (int x = gthread; x < 2 * heads; x += nthreads) a.list_len[x] = 0;
    if (gthread < 2) a.ovf_total[gthread] = 0;
  }
  // Grid-wide step between phases: a CTA whose bounded wait gave up raises the abort
  // word first, so every CTA leaves the rounds together (the status word may already
  // hold another error, which the barrier alone would not stop on).
  auto sync_grid = [&]() -> bool {
    __syncthreads();
    if (tid == 0 && *abort_v) atomicExch(&a.hdr->grid_abort, 1);
    const bool ok = grid_barrier(a.hdr, nblocks);
    return ok && *reinterpret_cast<volatile int*>(&a.hdr->grid_abort) == 0;
  };
  bool alive = norm_mode ? true : sync_grid();

  // pipeline counters, continued across rounds: work items and W chunks seen by this CTA
  int it_prod = 0, it_mma = 0, it_epi = 0, it_x = 0;
  int qc_prod = 0, qc_mma = 0, qc_epi = 0;  // W chunks so far (each two ring stages, one accumulator stage)
  int last_q = -1, last_it = -1;  // producer: last W chunk and X tile issued
  const int max_rounds = n + 2;
  int cur = 0;
  // store_rows: this round's tensor-core pass also stores the unplaced items' D rows;
  // tail: this round proposes from the stored rows (every CTA takes the same decision)
  bool store_rows = false, tail = false;
  for (int round = 0; alive; ++round) {
    const bool first = round == 0;
    const int* list = a.list[cur];
    const int par = round & 1;
    // this round's list lengths and work items per head, and their total
    for (int h = tid; h < heads; h += kAsThreads) {
      const int len = first ? n : __ldcg(a.list_len + cur * heads + h);
      s_len[h] = len;
      s_tiles[h] = ceil_div(len, kAsRows);
    }
    __syncthreads();
    if (warp == 0) {
      int t = 0;
      for (int h = lane; h < heads; h += 32) t += s_tiles[h];
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) s_total = t;
    }
    __syncthreads();
    const int total = s_total;

    // ---- the rounds after the first multiply with the open groups' W only.  Each head's
    // open groups (ascending) are packed into wc_hi / wc_lo at the head's offset; the
    // round that stores the tail rows (whose rows the tail reads by group), and the tail,
    // keep the full W.
    const bool packed = !first && !norm_mode && !tail && !store_rows;
    if (packed) {
      __shared__ int s_wpre[32];
      __shared__ int s_nopen;
      for (int h = blockIdx.x; h < heads; h += nblocks) {
        const unsigned int* cl = a.closed + static_cast<size_t>(h) * words;
        if (warp == 0) {
          unsigned int open = 0u;
          if (lane < words) {
            open = ~__ldcg(cl + lane);
            if (lane == words - 1 && (G & 31) != 0) open &= (1u << (G & 31)) - 1u;
          }
          const int cnt = __popc(open);
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          s_wpre[lane] = incl - cnt;
          if (lane == 31) s_nopen = incl;
        }
        __syncthreads();
        for (int g = tid; g < G; g += kAsThreads) {
          const unsigned int open = ~__ldcg(cl + (g >> 5));
          if ((open >> (g & 31)) & 1u) s_g[s_wpre[g >> 5] + __popc(open & ((1u << (g & 31)) - 1u))] = g;
        }
        __syncthreads();
        const int nop = s_nopen;
        // a warp per open group: lanes 0-15 copy its hi row, lanes 16-31 its lo row
        for (int c = warp; c < nop; c += kAsWarps) {
          const int g = s_g[c];
          const __nv_bfloat16* src = (lane < 16 ? a.whi : a.wlo) + (static_cast<size_t>(h) * G + g) * 128;
          __nv_bfloat16* dst = (lane < 16 ? a.wc_hi : a.wc_lo) + (static_cast<size_t>(h) * G + c) * 128;
          reinterpret_cast<uint4*>(dst)[lane & 15] = __ldcg(reinterpret_cast<const uint4*>(src) + (lane & 15));
          if (lane == 0) a.open_g[static_cast<size_t>(h) * G + c] = g;
        }
        if (tid == 0) a.n_open[h] = nop;
        __syncthreads();
      }
      // the packed rows are read by other CTAs' TMA (the async proxy) after the barrier
      asm volatile("fence.proxy.async.global;" ::: "memory");
      alive = sync_grid();
      if (!alive) break;
    }
    for (int h = tid; h < heads; h += kAsThreads)
      s_nch[h] = packed ? ceil_div(__ldcg(a.n_open + h), 128) : n_chunks;
    __syncthreads();

    // ---------------------------------------------------------------- A. proposals
    if (tail) {
      // ---- the rest of the fill, one head per CTA.  Every unplaced item's D row is stored
      // (the previous round's tensor-core pass), and heads are independent problems, so
      // each CTA runs its heads' remaining rounds alone: proposals from the stored rows (a
      // warp per item: the first minimum over the open groups by the epilogue's rule --
      // strict '<' in ascending column order, so +inf and NaN never win; none finite: the
      // lowest open group at +inf), then the same group pass, placement and overflow
      // selection as the grid-wide rounds, separated by __syncthreads.  The X and W
      // buffers are idle now and hold the overflow list and the full-group bitmap.
      int* s_ovf = reinterpret_cast<int*>(smem_raw + (sX[0] - tc::saddr(smem_raw)));           // [G]
      unsigned int* s_cl = reinterpret_cast<unsigned int*>(smem_raw + (sX[1] - tc::saddr(smem_raw)));  // [words]
      __shared__ int s_novf, s_nlen;
      // The first proposals of the tail (every unplaced item once) use the whole grid,
      // one head after the other; the per-head rounds below start from them.
      {
        // batches of kTailItems items, numbered across the heads; warp w takes batches
        // w, w + nwarps, ... (its head walk moves forward only)
        int hh = 0, bbase = 0;
        for (int bi = gwarp;; bi += nwarps) {
          while (hh < heads && bi >= bbase + ceil_div(s_len[hh], kTailItems)) bbase += ceil_div(s_len[hh++], kTailItems);
          if (hh >= heads) break;
          tail_propose(a, hh, list + static_cast<size_t>(hh) * n, s_len[hh], (bi - bbase) * kTailItems,
                       a.closed + static_cast<size_t>(hh) * words);
        }
      }
      alive = sync_grid();
      if (!alive) break;
      for (int h = blockIdx.x; h < heads; h += nblocks) {
        int lc = cur;
        int len = __ldcg(a.list_len + lc * heads + h);
        int* cnt = a.cnt + static_cast<size_t>(h) * G;
        int* room = a.room + static_cast<size_t>(h) * G;
        int* offs = a.offs + static_cast<size_t>(h) * G;
        int* cursor = a.cursor + static_cast<size_t>(h) * G;
        unsigned int* cl = a.closed + static_cast<size_t>(h) * words;
        int* lab = a.labels + static_cast<size_t>(h) * n;
        for (int lr = 0; len > 0; ++lr) {
          if (lr > max_rounds) {
            if (tid == 0) record_error(status, kErrTimeout);
            break;
          }
          const int* hl = a.list[lc] + static_cast<size_t>(h) * n;
          int* nl = a.list[lc ^ 1] + static_cast<size_t>(h) * n;
          for (int wd = tid; wd < words; wd += kAsThreads) s_cl[wd] = __ldcg(cl + wd);
          if (tid == 0) {
            s_novf = 0;
            s_nlen = 0;
          }
          __syncthreads();
          // A. proposals (the first local round's came from the whole grid above)
          if (lr > 0)
            for (int x0 = warp * kTailItems; x0 < len; x0 += kAsWarps * kTailItems) tail_propose(a, h, hl, len, x0, s_cl);
          __syncthreads();
          // B. groups that take all their proposers; bucket offsets of the others
          {
            const int per = ceil_div(G, kAsThreads);
            const int g0 = tid * per, g1 = min(G, g0 + per);
            int local = 0;
            for (int g = g0; g < g1; ++g) {
              const int c = __ldcg(cnt + g);
              if (c > __ldcg(room + g)) local += c;
            }
            int run = block_exclusive_scan(local, scan_tmp);
            for (int g = g0; g < g1; ++g) {
              const int c = __ldcg(cnt + g), rm = __ldcg(room + g);
              if (c > rm) {
                offs[g] = run;
                run += c;
                s_ovf[atomicAdd(&s_novf, 1)] = g;
              } else {
                offs[g] = -1;
                if (c > 0) {
                  room[g] = rm - c;
                  cnt[g] = 0;
                  if (rm == c) atomicOr(cl + g / 32, 1u << (g % 32));
                }
              }
            }
          }
          __syncthreads();
          // C. place / scatter
          for (int x = tid; x < len; x += kAsThreads) {
            const int i = __ldcg(hl + x);
            const size_t item = static_cast<size_t>(h) * n + i;
            const int g = __ldcg(a.prop_g + item);
            const size_t gi = static_cast<size_t>(h) * G + g;
            const int o = __ldcg(offs + g);
            if (o < 0) {
              lab[i] = g;
              a.members[gi * a.cap + atomicAdd(a.msize + gi, 1)] = i;
            } else {
              const int slot = atomicAdd(cursor + g, 1);
              a.bucket[static_cast<size_t>(h) * n + o + slot] = decision_key(__ldcg(a.prop_v + item), i);
            }
          }
          __syncthreads();
          // D. overflowing groups
          for (int j2 = warp; j2 < s_novf; j2 += kAsWarps) {
            const int g = s_ovf[j2];
            const size_t x = static_cast<size_t>(h) * G + g;
            const int c = __ldcg(cnt + g), rm = __ldcg(room + g);
            const unsigned long long* bk = a.bucket + static_cast<size_t>(h) * n + __ldcg(offs + g);
            unsigned long long kr[8];
            if (c <= 256) {
#pragma unroll
              for (int u = 0; u < 8; ++u) kr[u] = u * 32 + lane < c ? __ldcg(bk + u * 32 + lane) : ~0ull;
            }
            const unsigned long long thr = rm == 0 ? 0ull
                                           : c <= 256 ? warp_select_kth_by(KeysInRegisters{kr}, c, rm, hist[warp])
                                                      : warp_select_kth(bk, c, rm, hist[warp]);
            for (int e0 = 0; e0 < c; e0 += 256) {
              unsigned long long kb[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * 32 + lane;
                kb[u] = c <= 256 ? kr[u] : (e < c ? __ldcg(bk + e) : ~0ull);
              }
              accept_reject(kb, c - e0, thr, g, lab, a.members + x * a.cap, a.msize + x, nl, &s_nlen);
            }
            __syncwarp();
            if (lane == 0) {
              room[g] = 0;
              cnt[g] = 0;
              cursor[g] = 0;
              atomicOr(cl + g / 32, 1u << (g % 32));
            }
          }
          __syncthreads();
          len = s_nlen;
          lc ^= 1;
          __syncthreads();
        }
      }
      break;
    } else if (warp == 0) {
      // producer: in the first round per work item the 256 rows of X into buffer it & 1
      // (lane 0, four 2-D boxes; the later rounds' rows come from the loader warps), then
      // per chunk of 128 groups its W hi part and its lo part, each one stage of a two-
      // stage ring.  The next item's X is issued right after this item's first lo part:
      // that stage was freed by the previous item's last MMAs, so the X buffer the next
      // item reuses is free, and its load overlaps all of this item's MMAs.
      auto issue_x = [&](int it, int h, int t) -> bool {
        if (!first) return true;  // the gathered rounds' X comes from the loader warps
        const int b = it & 1, off = t * kAsRows;
        int ok = 1;
        if (lane == 0 && it >= 2 && !tc::mbar_wait(bar(kXEmpty0 + b), ((it >> 1) - 1) & 1, abort_v, status)) ok = 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
        if (lane == 0) {
          tc::mbar_arrive_expect_tx(bar(kXFull0 + b), kAsXStage);
          tc::mbar_arrive(bar(kXFull0 + b));  // the phase's second arrival (the loader warps' two otherwise)
#pragma unroll
          for (int j2 = 0; j2 < 2; ++j2) {
            tc::tma_load_2d(sX[b] + j2 * kAsTile, &tmX, 0, h * n + off + 128 * j2, bar(kXFull0 + b));
            tc::tma_load_2d(sX[b] + j2 * kAsTile + 128 * 128, &tmX, 64, h * n + off + 128 * j2, bar(kXFull0 + b));
          }
        }
        __syncwarp();
        last_it = it;
        return true;
      };
      // every X box of the first round has landed by now (the MMAs waited for each), and
      // the later rounds' X is not TMA's: nothing of it is left for the final drain
      if (!first) last_it = -1;
      HeadWalk hw;
      int h = 0, t = 0;
      bool ok = true;
      if (static_cast<int>(blockIdx.x) < total) {
        hw.seek(s_tiles, blockIdx.x, h, t);
        ok = issue_x(it_prod, h, t);
      }
      for (int w = blockIdx.x; ok && w < total; w += nblocks, ++it_prod) {
        const int wn = w + nblocks;
        int hn = 0, tn = 0;
        if (wn < total) hw.seek(s_tiles, wn, hn, tn);
        const int nch = s_nch[h];
        if (lane == 0) s_inch[it_prod & 3] = nch;  // for the MMA issuer (read after this item's first W stage)
        for (int c = 0; ok && c < nch; ++c, ++qc_prod) {
          for (int part = 0; ok && part < 2; ++part) {
            int okc = 1;
            if (lane == 0) {
              const int q = qc_prod * 2 + part, st = q & 1;
              if (q >= 2 && !tc::mbar_wait(bar(kWEmpty0 + st), ((q >> 1) - 1) & 1, abort_v, status)) {
                okc = 0;
              } else {
                const CUtensorMap* tm = packed ? (part == 0 ? &tmWcHi : &tmWcLo) : (part == 0 ? &tmWhi : &tmWlo);
                const int wrow = h * G + c * 128;
                tc::mbar_arrive_expect_tx(bar(kWFull0 + st), kAsWStage);
                tc::tma_load_2d(sW[st], tm, 0, wrow, bar(kWFull0 + st));
                tc::tma_load_2d(sW[st] + 128 * 128, tm, 64, wrow, bar(kWFull0 + st));
                last_q = q;
              }
            }
            ok = __shfl_sync(0xffffffffu, okc, 0) != 0;
            if (ok && c == 0 && part == 1 && wn < total) ok = issue_x(it_prod + 1, hn, tn);
          }
        }
        h = hn;
        t = tn;
      }
    } else if (warp == 1 || warp == 3) {
      // X of the gathered rounds: the rows of the head's unplaced list, read with coalesced
      // 16-byte loads (two rows per warp instruction, 16 instructions in flight per lane)
      // and stored in the swizzled tile layout, warp 1 the item's rows 0-127 and warp 3
      // rows 128-255; rows past the list are zero (never used).  The TMA engine then
      // serves only W (the first round's contiguous rows come by TMA boxes instead).
      const int hx = warp >> 1;
      const int sub = lane >> 4, ch = lane & 15;  // row of the pair, 16-byte chunk of the row
      HeadWalk hw;
      for (int w = blockIdx.x; w < total; w += nblocks, ++it_x) {
        if (first) continue;  // (the items are still counted: every role numbers them alike)
        int h, t;
        hw.seek(s_tiles, w, h, t);
        const int b = it_x & 1, off = t * kAsRows + 128 * hx, len = s_len[h];
        int ok = 1;
        if (lane == 0 && it_x >= 2 && !tc::mbar_wait(bar(kXEmpty0 + b), ((it_x >> 1) - 1) & 1, abort_v, status))
          ok = 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        int* xidx = s_xidx[hx];  // the items of this half's 128 rows
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = off + 32 * k + lane;
          xidx[32 * k + lane] = e < len ? __ldcg(list + static_cast<size_t>(h) * n + e) : -1;
        }
        __syncwarp();
        uint8_t* dst = smem_raw + (sX[b] - tc::saddr(smem_raw)) + hx * kAsTile + (ch >> 3) * (128 * 128);
        const __nv_bfloat16* xh = a.x + static_cast<size_t>(h) * n * 128;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {  // 32 rows per batch
          uint4 v[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int ix = xidx[32 * q + 2 * k + sub];
            v[k] = ix >= 0 ? __ldcg(reinterpret_cast<const uint4*>(xh + static_cast<size_t>(ix) * 128) + ch)
                           : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int row = 32 * q + 2 * k + sub;
            *reinterpret_cast<uint4*>(dst + row * 128 + (((ch & 7) ^ (row & 7)) << 4)) = v[k];
          }
        }
        __syncwarp();  // every lane done with xidx before the next item overwrites it
        tc::fence_proxy_async();  // the stores, before the tensor core reads the tile
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(kXFull0 + b));
      }
    } else if (warp == 2) {
      // MMA issuer: per chunk, all hi products (8 k-steps of 16, both 128-row halves),
      // then all lo products, into the chunk's accumulator stage
      if (lane == 0) {
        constexpr uint32_t kId = tc::idesc_bf16(128, 128, false, false);
        for (int w = blockIdx.x; w < total; w += nblocks, ++it_mma) {
          const int b = it_mma & 1;
          if (!tc::mbar_wait(bar(kXFull0 + b), (it_mma >> 1) & 1, abort_v, status)) break;
          tc::fence_proxy_async();
          bool ok = true;
          // the item's chunk count, written by the producer before its first W stage (the
          // hi part of chunk qc is ring stage 0, phase qc)
          if (!tc::mbar_wait(bar(kWFull0), qc_mma & 1, abort_v, status)) break;
          const int nch = s_inch[it_mma & 3];
          for (int c = 0; ok && c < n_chunks; ++c) {
            if (c >= nch) break;  // (a loop-invariant bound keeps the register allocation of the issue loop)
            const int qc = qc_mma++, s = qc & 1;
            if (qc >= 2 && !tc::mbar_wait(bar(kAccEmpty0 + s), ((qc >> 1) - 1) & 1, abort_v, status)) {
              ok = false;
              break;
            }
            for (int part = 0; part < 2; ++part) {
              const int q = qc * 2 + part, st = q & 1;
              if (!tc::mbar_wait(bar(kWFull0 + st), (q >> 1) & 1, abort_v, status)) {
                ok = false;
                break;
              }
              tc::fence_proxy_async();
              tc::fence_after_sync();
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint32_t acc = tbase + s * 256 + j * 128;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const uint32_t koff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                  tc::mma_ss(acc, tc::sdesc_sw128(sX[b] + j * kAsTile + koff, 16, 1024),
                             tc::sdesc_sw128(sW[st] + koff, 16, 1024), kId, (part == 0 && kk == 0) ? 0u : 1u);
                }
              }
              tc::mma_commit(bar(kWEmpty0 + st));
            }
            if (ok) tc::mma_commit(bar(kAccFull0 + s));
          }
          if (!ok) break;
          if (!norm_mode) tc::mma_commit(bar(kXEmpty0 + b));  // norm mode: the epilogue frees X
        }
      }
      __syncwarp();
    } else if (warp >= 4) {
      // epilogue: for rows r and r + 128, D of the row's 64 columns of every chunk and the
      // first minimum over the open groups, halves of the columns merged at the end
      const int r = (warp & 3) * 32 + lane;  // row within each 128-row half == TMEM lane
      const int half = (warp - 4) >> 2;      // columns [64 half, 64 half + 64) of every chunk
      const int etid = tid - 128;
      const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
      const float tau2 = a.tau2, m2t = -2.f * tau2;
      int loaded_head = -1;
      bool aborted = *abort_v != 0;
      HeadWalk hw;
      // The rows of the next work items are read ahead, so that no load waits at an item's
      // start: the list entries two items ahead, the norms tau^2 n_i one item ahead (their
      // list entries arrived during the previous item).
      HeadWalk hwa;
      int ah1 = 0, ah2 = 0;
      int aidx1[2] = {0, 0}, aidx2[2] = {0, 0};
      bool aok1[2] = {false, false}, aok2[2] = {false, false};
      float atn1[2] = {0.f, 0.f};
      auto fetch_idx = [&](int w, int& hh, int (&idx)[2], bool (&ok)[2]) {
        if (w >= total) {
          ok[0] = ok[1] = false;
          return;
        }
        int tt;
        hwa.seek(s_tiles, w, hh, tt);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int e = tt * kAsRows + 128 * j + r;
          ok[j] = e < s_len[hh];
          idx[j] = ok[j] ? (first ? e : __ldcg(list + static_cast<size_t>(hh) * n + e)) : 0;
        }
      };
      auto fetch_nrm = [&]() {
#pragma unroll
        for (int j = 0; j < 2; ++j)
          atn1[j] = aok1[j] ? tau2 * __ldcg(a.nrm + static_cast<size_t>(ah1) * n + aidx1[j]) : 0.f;
      };
      if (!norm_mode) {
        fetch_idx(blockIdx.x, ah1, aidx1, aok1);
        fetch_nrm();
        fetch_idx(blockIdx.x + nblocks, ah2, aidx2, aok2);
      }
      for (int w = blockIdx.x; w < total; w += nblocks, ++it_epi) {
        int h, t;
        hw.seek(s_tiles, w, h, t, s_len);
        const int off = t * kAsRows;
        if (norm_mode) {
          // x_i^T Gamma x_i: this thread's 64 accumulator columns (the 64-column box
          // `half` of its row) dotted with the same columns of x_i from the X tile
          const uint8_t* xs = smem_raw + (sX[it_epi & 1] - tc::saddr(smem_raw)) + half * (128 * 128) + r * 128;
          float part[2] = {0.f, 0.f};
          const bool got = !aborted && tc::mbar_wait(bar(kAccFull0 + (it_epi & 1)), (it_epi >> 1) & 1, abort_v, status);
          if (!__all_sync(0xffffffffu, got)) {
            aborted = true;
          } else {
            tc::fence_after_sync();
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              uint32_t u[64];
              const uint32_t buf = tbase + lane_off + (it_epi & 1) * 256 + j * 128 + half * 64;
              tc::tmem_ld32(buf, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
              tc::tmem_ld32(buf + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
              tc::tmem_wait_ld();
              if (j == 1) {
                tc::fence_before_sync();
                tc::mbar_arrive(bar(kAccEmpty0 + (it_epi & 1)));
              }
#pragma unroll
              for (int ch = 0; ch < 8; ++ch) {
                const uint4 xv = *reinterpret_cast<const uint4*>(xs + j * kAsTile + ((ch ^ (r & 7)) << 4));
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[k]));
                  part[j] = fmaf(__uint_as_float(u[8 * ch + 2 * k]), xf.x, part[j]);
                  part[j] = fmaf(__uint_as_float(u[8 * ch + 2 * k + 1]), xf.y, part[j]);
                }
              }
            }
          }
          if (half == 1) {
            s_best_v[r] = part[0];
            s_best_v[128 + r] = part[1];
          }
          asm volatile("bar.sync 1, 256;" ::: "memory");  // every X read of this item done
          if (etid == 0 && !aborted) tc::mbar_arrive(bar(kXEmpty0 + (it_epi & 1)));
          if (half == 0 && !aborted) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int e = off + 128 * j + r;
              if (e < s_len[h]) a.nrm_out[static_cast<size_t>(h) * n + e] = part[j] + s_best_v[128 * j + r];
            }
          }
          asm volatile("bar.sync 1, 256;" ::: "memory");
          continue;
        }
        if (h != loaded_head) {  // tau^2 e_g of this head, +inf for full groups and past G
          asm volatile("bar.sync 1, 256;" ::: "memory");
          if (etid == 0) s_enf = 0;
          asm volatile("bar.sync 1, 256;" ::: "memory");
          const unsigned int* cl = a.closed + static_cast<size_t>(h) * words;
          const int nop = packed ? __ldcg(a.n_open + h) : G;
          for (int c = etid; c < s_nch[h] * 128; c += kAsEpi) {
            float v = kAsInf;
            int g = c;
            if (packed) {  // packed column c: the head's c-th open group
              if (c < nop) {
                g = __ldcg(a.open_g + static_cast<size_t>(h) * G + c);
                v = tau2 * __ldcg(a.ecol + static_cast<size_t>(h) * G + g);
                if (!isfinite(v)) s_enf = 1;
              }
            } else if (c < G) {
              const float e = tau2 * __ldcg(a.ecol + static_cast<size_t>(h) * G + c);
              if (!isfinite(e)) s_enf = 1;
              if (!((__ldcg(cl + (c >> 5)) >> (c & 31)) & 1u)) v = e;
            }
            s_e[c] = v;
            s_g[c] = g;
          }
          asm volatile("bar.sync 1, 256;" ::: "memory");
          loaded_head = h;
        }
        bool row_ok[2];
        size_t grow[2];
        float tnr[2], best_v[2] = {kAsInf, kAsInf};
        int best_c[2] = {-1, -1};
        bool nonfinite = false;
#pragma unroll
        for (int j = 0; j < 2; ++j) {  // this item's rows, read ahead (ah1 == h)
          row_ok[j] = aok1[j];
          grow[j] = static_cast<size_t>(h) * n + aidx1[j];
          tnr[j] = atn1[j];
          nonfinite |= row_ok[j] && (!isfinite(tnr[j]) || s_enf != 0);
        }
        // read ahead: the next item's norms, the list entries of the one after it
        ah1 = ah2;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          aidx1[j] = aidx2[j];
          aok1[j] = aok2[j];
        }
        fetch_nrm();
        fetch_idx(w + 2 * static_cast<int>(nblocks), ah2, aidx2, aok2);
        const int nch = s_nch[h];
        for (int c = 0; c < nch && !aborted; ++c) {
          const int q = qc_epi++, s = q & 1;
          const bool got = tc::mbar_wait(bar(kAccFull0 + s), (q >> 1) & 1, abort_v, status);
          if (!__all_sync(0xffffffffu, got)) {
            aborted = true;
            break;
          }
          tc::fence_after_sync();
          const int c0 = c * 128 + half * 64;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            uint32_t u[64];
            const uint32_t buf = tbase + lane_off + s * 256 + j * 128 + half * 64;
            tc::tmem_ld32(buf, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
            tc::tmem_ld32(buf + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
            tc::tmem_wait_ld();
            if (j == 1) {  // both halves read: the accumulator stage is free again
              tc::fence_before_sync();
              tc::mbar_arrive(bar(kAccEmpty0 + s));
            }
            scan_half_chunk(u, s_e, c0, tnr[j], m2t, best_v[j], best_c[j]);
            if (first && a.Dout != nullptr && row_ok[j]) {  // parity tests: the full row of D
              float* dst = a.Dout + grow[j] * a.ldd + c0;
#pragma unroll
              for (int k4 = 0; k4 < 16; ++k4) {
                if (c0 + 4 * k4 < a.ldd)
                  *reinterpret_cast<float4*>(dst + 4 * k4) =
                      make_float4(__uint_as_float(u[4 * k4]), __uint_as_float(u[4 * k4 + 1]),
                                  __uint_as_float(u[4 * k4 + 2]), __uint_as_float(u[4 * k4 + 3]));
              }
            }
            if (store_rows && row_ok[j]) {  // the tail's stored rows (ldt covers every chunk)
              float* dst = a.Dtail + static_cast<size_t>(hw.ibase + off + 128 * j + r) * a.ldt + c0;
#pragma unroll
              for (int k4 = 0; k4 < 16; ++k4)
                *reinterpret_cast<float4*>(dst + 4 * k4) =
                    make_float4(__uint_as_float(u[4 * k4]), __uint_as_float(u[4 * k4 + 1]),
                                __uint_as_float(u[4 * k4 + 2]), __uint_as_float(u[4 * k4 + 3]));
            }
          }
        }
        if (half == 1) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            s_best_v[128 * j + r] = best_v[j];
            s_best_c[128 * j + r] = best_c[j];
          }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (half == 0 && !aborted) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (!row_ok[j]) continue;
            float bv = best_v[j];
            int bc = best_c[j];
            const float v1 = s_best_v[128 * j + r];
            const int c1 = s_best_c[128 * j + r];
            // half 0 holds the lower 64 columns of every chunk: equal values go to it
            if (c1 >= 0 && (bc < 0 || v1 < bv || (v1 == bv && c1 < bc))) {
              bv = v1;
              bc = c1;
            }
            if (bc >= 0) bc = s_g[bc];  // the column's group (packed columns ascend with it)
            if (bc < 0) {  // every open group at +inf (or NaN): the lowest open group
              const unsigned int* cl = a.closed + static_cast<size_t>(h) * words;
              for (int wd = 0; wd < words && bc < 0; ++wd) {
                const unsigned int open = ~__ldcg(cl + wd);
                if (open != 0u) {
                  const int g = wd * 32 + __ffs(open) - 1;
                  if (g < G) bc = g;
                }
              }
              if (bc < 0) {  // no open group: more items than room (cannot happen)
                record_error(status, kErrInvalidArg);
                bc = 0;
              }
            }
            a.prop_g[grow[j]] = bc;
            a.prop_v[grow[j]] = bv;
            atomicAdd(a.cnt + static_cast<size_t>(h) * G + bc, 1);
            if (store_rows) a.tailpos[grow[j]] = hw.ibase + off + 128 * j + r;
          }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (__any_sync(0xffffffffu, nonfinite && !aborted) && lane == 0) record_error(status, kErrNonFinite);
        // after an abort the loop still runs to the end, skipping the work, so that every
        // epilogue warp passes the same named barriers
      }
    }
    __syncwarp();
    if (norm_mode) break;  // one pass, no fill
    alive = sync_grid();
    if (!alive) break;

    // ---------------------------------------------------------------- B. groups
    // A group whose proposers fit its room takes them all now; an overflowing group gets
    // the offset of its bucket (the head's overflow proposals are packed in group order)
    // and joins the overflow list.
    for (int h = blockIdx.x; h < heads; h += nblocks) {
      int* cnt = a.cnt + static_cast<size_t>(h) * G;
      int* room = a.room + static_cast<size_t>(h) * G;
      int* offs = a.offs + static_cast<size_t>(h) * G;
      const int per = ceil_div(G, kAsThreads);
      const int g0 = tid * per, g1 = min(G, g0 + per);
      int local = 0;
      for (int g = g0; g < g1; ++g) {
        const int c = __ldcg(cnt + g);
        if (c > __ldcg(room + g)) local += c;
      }
      int run = block_exclusive_scan(local, scan_tmp);
      for (int g = g0; g < g1; ++g) {
        const int c = __ldcg(cnt + g), rm = __ldcg(room + g);
        if (c > rm) {
          offs[g] = run;
          run += c;
          a.ovf_list[atomicAdd(a.ovf_total + par, 1)] = h * G + g;
        } else {
          offs[g] = -1;
          if (c > 0) {
            room[g] = rm - c;
            cnt[g] = 0;
            if (rm == c) atomicOr(a.closed + static_cast<size_t>(h) * words + g / 32, 1u << (g % 32));
          }
        }
      }
      __syncthreads();
    }
    alive = sync_grid();
    if (!alive) break;

    // ---------------------------------------------------------------- C. place / scatter
    {
      // three items per thread at a time, so that their dependent loads and atomics overlap
      constexpr int kCI = 3;
      int items = 0;
      for (int h = 0; h < heads; ++h) items += s_len[h];
      HeadWalk hw;
      for (int x0 = gthread; x0 - lane < items; x0 += nthreads * kCI) {  // warp-uniform trip count
        int hh[kCI], ii[kCI], gg[kCI], oo[kCI];
        float vv[kCI];
#pragma unroll
        for (int u = 0; u < kCI; ++u) {
          const int x = x0 + u * nthreads;
          hh[u] = -1;
          ii[u] = 0;
          if (x < items) {
            int e;
            hw.seek(s_len, x, hh[u], e);
            ii[u] = first ? e : __ldcg(list + static_cast<size_t>(hh[u]) * n + e);
          }
        }
#pragma unroll
        for (int u = 0; u < kCI; ++u) {
          gg[u] = 0;
          vv[u] = 0.f;
          if (hh[u] >= 0) {
            const size_t item = static_cast<size_t>(hh[u]) * n + ii[u];
            gg[u] = __ldcg(a.prop_g + item);
            vv[u] = __ldcg(a.prop_v + item);
          }
        }
#pragma unroll
        for (int u = 0; u < kCI; ++u)
          oo[u] = hh[u] >= 0 ? __ldcg(a.offs + static_cast<size_t>(hh[u]) * G + gg[u]) : 0;
#pragma unroll
        for (int u = 0; u < kCI; ++u) {
          // a warp's items are consecutive, often of one group: one atomic per distinct group
          // of the warp reserves its lanes' slots (a group either places or scatters all)
          const unsigned int act = __ballot_sync(0xffffffffu, hh[u] >= 0);
          if (hh[u] < 0) continue;
          const size_t gi = static_cast<size_t>(hh[u]) * G + gg[u];
          const unsigned int same = __match_any_sync(act, static_cast<unsigned long long>(gi));
          const int leader = __ffs(same) - 1;
          int base = 0;
          if (lane == leader) base = atomicAdd((oo[u] < 0 ? a.msize : a.cursor) + gi, __popc(same));
          const int slot = __shfl_sync(act, base, leader) + __popc(same & ((1u << lane) - 1u));
          const size_t item = static_cast<size_t>(hh[u]) * n + ii[u];
          if (oo[u] < 0) {
            a.labels[item] = gg[u];
            a.members[gi * a.cap + slot] = ii[u];
          } else {
            a.bucket[static_cast<size_t>(hh[u]) * n + oo[u] + slot] = decision_key(vv[u], ii[u]);
          }
        }
      }
    }
    alive = sync_grid();
    if (!alive) break;

    // ---------------------------------------------------------------- D. overflowing groups
    const int next = cur ^ 1;
    {
      const int novf = __ldcg(a.ovf_total + par);
      for (int j = gwarp; j < novf; j += nwarps) {
        const int x = __ldcg(a.ovf_list + j);
        const int h = x / G, g = x - h * G;
        const int c = __ldcg(a.cnt + x), rm = __ldcg(a.room + x);
        const unsigned long long* bk = a.bucket + static_cast<size_t>(h) * n + __ldcg(a.offs + x);
        int* lab = a.labels + static_cast<size_t>(h) * n;
        int* nlist = a.list[next] + static_cast<size_t>(h) * n;
        int* nlen = a.list_len + next * heads + h;
        // (rm = 0 only after a recorded error: nothing is taken then).  A bucket of at most
        // 256 keys is read once and selected in registers.
        unsigned long long kr[8];
        if (c <= 256) {
#pragma unroll
          for (int u = 0; u < 8; ++u) kr[u] = u * 32 + lane < c ? __ldcg(bk + u * 32 + lane) : ~0ull;
        }
        const unsigned long long thr = rm == 0 ? 0ull
                                       : c <= 256 ? warp_select_kth_by(KeysInRegisters{kr}, c, rm, hist[warp])
                                                  : warp_select_kth(bk, c, rm, hist[warp]);
        for (int e0 = 0; e0 < c; e0 += 256) {
          unsigned long long kb[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * 32 + lane;
            kb[u] = c <= 256 ? kr[u] : (e < c ? __ldcg(bk + e) : ~0ull);
          }
          accept_reject(kb, c - e0, thr, g, lab, a.members + static_cast<size_t>(x) * a.cap, a.msize + x, nlist, nlen);
        }
        __syncwarp();
        if (lane == 0) {
          a.room[x] = 0;
          a.cnt[x] = 0;
          a.cursor[x] = 0;
          atomicOr(a.closed + static_cast<size_t>(h) * words + g / 32, 1u << (g % 32));
        }
      }
      if (blockIdx.x == 0 && tid == 0) a.ovf_total[par ^ 1] = 0;  // the next round's list
    }
    alive = sync_grid();
    if (!alive) break;
    if (warp == 0) {
      int rem = 0;
      for (int h = lane; h < heads; h += 32) rem += __ldcg(a.list_len + next * heads + h);
      for (int o = 16; o > 0; o >>= 1) rem += __shfl_xor_sync(0xffffffffu, rem, o);
      if (lane == 0) s_remaining = rem;
    }
    __syncthreads();
    if (s_remaining == 0) break;
    if (store_rows) {
      store_rows = false;
      tail = true;
    } else if (!tail && s_remaining <= a.tail_cap) {
      store_rows = true;
    }
    if (round >= max_rounds) {
      if (gthread == 0) record_error(status, kErrTimeout);
      break;
    }
    if (blockIdx.x == 0)
      for (int h = tid; h < heads; h += kAsThreads) a.list_len[cur * heads + h] = 0;
    cur = next;
  }

  // ---- drain: copies still in flight after an abort land, MMAs complete, TMEM freed
  if (warp == 0 && lane == 0) {
    auto drain = [&](uint32_t b, uint32_t parity) {
      const uint64_t t0 = globaltimer_ns();
      while (!tc::mbar_try_wait(b, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      }
    };
    for (int q = last_q - 1; q <= last_q; ++q)
      if (q >= 0) drain(bar(kWFull0 + (q & 1)), (q >> 1) & 1);
    for (int it = last_it - 1; it <= last_it; ++it)
      if (it >= 0) drain(bar(kXFull0 + (it & 1)), (it >> 1) & 1);
  }
  if (warp == 2 && lane == 0) {
    tc::mma_commit(bar(kDrain));
    const uint64_t t0 = globaltimer_ns();
    while (!tc::mbar_try_wait(bar(kDrain), 0)) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, kAsTmemCols);
  }
}

}  // namespace

size_t assign_tc_smem_bytes() {
  return 1024 + 2ull * kAsXStage + 2ull * kAsWStage + sizeof(float) * kAsMaxCols + 3 * sizeof(int) * kAsMaxHeads +
         sizeof(int) * kAsMaxCols;
}

cudaError_t launch_assign_tc(const __nv_bfloat16* X, const __nv_bfloat16* Whi, const __nv_bfloat16* Wlo,
                             const AssignArgs& a, cudaStream_t st) {
  if (a.G < 1 || a.G > kAsMaxCols || a.n < 1 || a.heads < 1 || a.cap < 1 || (a.Dout != nullptr && a.ldd % 4 != 0) ||
      (a.tail_cap > 0 && (a.Dtail == nullptr || a.tailpos == nullptr || a.ldt < ceil_div(a.G, 128) * 128 ||
                          a.ldt % 4 != 0)))
    return cudaErrorInvalidValue;
  const size_t smem = assign_tc_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(assign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, assign_tc_kernel, kAsThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int words = ceil_div(a.G, 32);
  // at most kAsMaxHeads heads per launch: larger calls run head slices one after another
  for (int h0 = 0; h0 < a.heads; h0 += kAsMaxHeads) {
    const int hc = std::min(kAsMaxHeads, a.heads - h0);
    const size_t ni = static_cast<size_t>(h0) * a.n, gi = static_cast<size_t>(h0) * a.G;
    auto sl = [](auto* p, size_t k) { return p != nullptr ? p + k : p; };
    AssignArgs s = a;
    s.heads = hc;
    s.x = X + ni * 128;
    s.whi = Whi + gi * 128;
    s.wlo = Wlo + gi * 128;
    s.wc_hi = sl(a.wc_hi, gi * 128);
    s.wc_lo = sl(a.wc_lo, gi * 128);
    s.open_g = sl(a.open_g, gi);
    s.n_open = sl(a.n_open, static_cast<size_t>(h0));
    s.nrm = sl(a.nrm, ni);
    s.ecol = sl(a.ecol, gi);
    s.labels = sl(a.labels, ni);
    s.room = sl(a.room, gi);
    s.cnt = sl(a.cnt, gi);
    s.offs = sl(a.offs, gi);
    s.cursor = sl(a.cursor, gi);
    s.closed = sl(a.closed, static_cast<size_t>(h0) * words);
    s.bucket = sl(a.bucket, ni);
    s.list[0] = sl(a.list[0], ni);
    s.list[1] = sl(a.list[1], ni);
    s.list_len = sl(a.list_len, static_cast<size_t>(2) * h0);
    s.prop_g = sl(a.prop_g, ni);
    s.prop_v = sl(a.prop_v, ni);
    s.ovf_list = sl(a.ovf_list, gi);
    s.members = sl(a.members, gi * a.cap);
    s.msize = sl(a.msize, gi);
    s.tailpos = sl(a.tailpos, ni);
    s.nrm_out = sl(a.nrm_out, ni);
    s.Dout = sl(a.Dout, ni * a.ldd);
    const long long xrows = static_cast<long long>(hc) * a.n, wrows = static_cast<long long>(hc) * a.G;
    if (xrows > 0x7fffffffLL || wrows > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA coordinates are int32
    CUtensorMap tx, twh, twl, twch, twcl;
    const __nv_bfloat16* Xs = X + ni * 128;
    if (!bf16_map(&tx, Xs, xrows, 128) ||
        !bf16_map(&twh, Whi + gi * 128, wrows, 128) || !bf16_map(&twl, Wlo + gi * 128, wrows, 128))
      return cudaErrorInvalidValue;
    // the packed open groups' W (norm mode packs nothing: the maps then name W itself)
    if (!bf16_map(&twch, s.wc_hi != nullptr ? s.wc_hi : s.whi, wrows, 128) ||
        !bf16_map(&twcl, s.wc_lo != nullptr ? s.wc_lo : s.wlo, wrows, 128))
      return cudaErrorInvalidValue;
    e = cudaMemsetAsync(&a.hdr->barrier_count, 0, 2 * sizeof(unsigned int), st);
    if (e != cudaSuccess) return e;
    void* params[] = {&tx, &twh, &twl, &twch, &twcl, &s};
    e = cudaLaunchCooperativeKernel(reinterpret_cast<void*>(assign_tc_kernel), dim3(sms), dim3(kAsThreads), params,
                                    smem, st);
    if ((e = counted(e, 1)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_row_norms_tc(const __nv_bfloat16* X, const __nv_bfloat16* ghi, const __nv_bfloat16* glo,
                                int heads, int n, float* nrm, WorkspaceHeader* hdr, cudaStream_t st) {
  AssignArgs a{};
  a.heads = heads;
  a.n = n;
  a.G = 128;  // the columns of Gamma
  a.cap = 1;
  a.nrm_out = nrm;
  a.hdr = hdr;
  return launch_assign_tc(X, ghi, glo, a, st);
}

}  // namespace spr
