// Attention kernels of the SparsePR call (sm_100a):
//   * block-sparse softmax attention over routed (query block, key group) tiles, and
//     the dense comparator as the same kernel with every group routed;
//   * probe rows: exact dense attention and the row's own block-sparse output, with the
//     softmax weights carried as bf16 hi + lo (two products) for ~16-bit precision;
//   * fp32 (SIMT) variants of both for fp32 inputs.
// Method: the SparsePR abstract (arXiv 2608.18484, arxivdaily.com English abstract)
// computes attention only between selected groups and exact attention on a few probe
// rows; the routed softmax is renormalised over the routed support.
#include <algorithm>

#include "attention.cuh"
#include "common.cuh"
#include "warp_mma.cuh"

namespace spr {

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr float kNegInf = -__builtin_huge_valf();

// ------------------------------------------------------------------------------------
// bf16 block-sparse / dense attention.  One CTA per (query block, head); BQ = B rows,
// BQ/16 warps of 16 rows.  Keys stream in chunks of 64 (double-buffered cp.async,
// gathered row by row through key_perm).  S and P stay in registers.
// ------------------------------------------------------------------------------------
constexpr int kChunk = 64;

template <int D, int BQ, bool DENSE>
__global__ void __launch_bounds__(BQ * 2, 1)
    attn_mma_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                    const __nv_bfloat16* __restrict__ V, int N, int G, int k,
                    const int* __restrict__ key_perm, const int* __restrict__ key_gsize,
                    const int* __restrict__ query_perm, const int* __restrict__ qblock_size,
                    const int* __restrict__ route, float scale_log2, float* __restrict__ out) {
  constexpr int kThreads = BQ * 2;
  constexpr int kCh = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + BQ * D * 2;
  uint8_t* sV = sK + 2 * kChunk * D * 2;
  __shared__ int sTokQ[BQ];

  const int b = blockIdx.x;
  const int head = blockIdx.y;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const size_t hoff = static_cast<size_t>(head) * N * D;
  Q += hoff;
  K += hoff;
  V += hoff;
  out += hoff;
  const size_t goff = static_cast<size_t>(head) * G;
  const int nq = DENSE ? min(BQ, N - b * BQ) : qblock_size[goff + b];
  const int* qperm = query_perm + goff * BQ;
  const int* kperm = key_perm + goff * BQ;

  for (int x = tid; x < BQ * kCh; x += kThreads) {
    const int r = x / kCh, ch = x % kCh;
    const int tok = r < nq ? (DENSE ? b * BQ + r : qperm[b * BQ + r]) : -1;
    if (ch == 0) sTokQ[r] = tok;
    cp_async_16(smem_u32(sQ) + swz<D>(r, ch), tok >= 0 ? Q + static_cast<size_t>(tok) * D + ch * 8 : Q,
                tok >= 0 ? 16 : 0);
  }
  cp_async_commit();

  constexpr int kCpg = BQ / kChunk;  // chunks per key group
  const int* my_route = DENSE ? nullptr : route + (goff + b) * k;
  const int n_chunks = (DENSE ? k : routed_len(my_route, k)) * kCpg;

  auto chunk_group = [&](int t) { return DENSE ? t / kCpg : __ldg(my_route + t / kCpg); };
  auto chunk_valid = [&](int t) {
    const int g = chunk_group(t);
    const int gs = DENSE ? min(BQ, N - g * BQ) : __ldg(key_gsize + goff + g);
    return gs - (t % kCpg) * kChunk;
  };
  auto load_chunk = [&](int t) {
    const int stage = t & 1;
    const int g = chunk_group(t);
    const int gs = DENSE ? min(BQ, N - g * BQ) : __ldg(key_gsize + goff + g);
    const int j0 = (t % kCpg) * kChunk;
    const uint32_t kb = smem_u32(sK) + stage * kChunk * D * 2;
    const uint32_t vb = smem_u32(sV) + stage * kChunk * D * 2;
    for (int x = tid; x < kChunk * kCh; x += kThreads) {
      const int j = x / kCh, ch = x % kCh;
      const int slot = j0 + j;
      const int tok = slot < gs ? (DENSE ? g * BQ + slot : __ldg(kperm + g * BQ + slot)) : -1;
      const size_t off = tok >= 0 ? static_cast<size_t>(tok) * D + ch * 8 : 0;
      cp_async_16(kb + swz<D>(j, ch), K + off, tok >= 0 ? 16 : 0);
      cp_async_16(vb + swz<D>(j, ch), V + off, tok >= 0 ? 16 : 0);
    }
  };

  load_chunk(0);
  cp_async_commit();

  const int g8 = lane >> 2, t4 = lane & 3;
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {kNegInf, kNegInf};
  float l_run[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];

  for (int t = 0; t < n_chunks; ++t) {
    if (t + 1 < n_chunks) load_chunk(t + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldmatrix_x4(qf[kk], smem_u32(sQ) + swz<D>(r, kk * 2 + (lane >> 4)));
      }
    }
    const int stage = t & 1;
    const uint32_t kb = smem_u32(sK) + stage * kChunk * D * 2;
    const uint32_t vb = smem_u32(sV) + stage * kChunk * D * 2;

    float s[kChunk / 8][4];
#pragma unroll
    for (int i = 0; i < kChunk / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nt2 = 0; nt2 < kChunk / 16; ++nt2) {
        uint32_t bf[4];
        const int r = nt2 * 16 + (lane & 7) + (lane >> 4) * 8;
        ldmatrix_x4(bf, kb + swz<D>(r, kk * 2 + ((lane >> 3) & 1)));
        mma_bf16_16816(s[2 * nt2], qf[kk], &bf[0]);
        mma_bf16_16816(s[2 * nt2 + 1], qf[kk], &bf[2]);
      }
    }
    const int nvalid = chunk_valid(t);
#pragma unroll
    for (int nt = 0; nt < kChunk / 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int key = nt * 8 + 2 * t4 + (c & 1);
        s[nt][c] = key < nvalid ? s[nt][c] * scale_log2 : kNegInf;
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = kNegInf;
#pragma unroll
      for (int nt = 0; nt < kChunk / 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * h], s[nt][2 * h + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[h], mx);
      const float m_use = m_new == kNegInf ? 0.f : m_new;
      const float alpha = fast_exp2(m_run[h] - m_use);
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < kChunk / 8; ++nt) {
        s[nt][2 * h] = fast_exp2(s[nt][2 * h] - m_use);
        s[nt][2 * h + 1] = fast_exp2(s[nt][2 * h + 1] - m_use);
        sum += s[nt][2 * h] + s[nt][2 * h + 1];
      }
      l_run[h] = l_run[h] * alpha + sum;
      m_run[h] = m_new;
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        o[dt][2 * h] *= alpha;
        o[dt][2 * h + 1] *= alpha;
      }
    }
#pragma unroll
    for (int kk2 = 0; kk2 < kChunk / 16; ++kk2) {
      uint32_t a[4];
      a[0] = pack_bf16x2(s[2 * kk2][0], s[2 * kk2][1]);
      a[1] = pack_bf16x2(s[2 * kk2][2], s[2 * kk2][3]);
      a[2] = pack_bf16x2(s[2 * kk2 + 1][0], s[2 * kk2 + 1][1]);
      a[3] = pack_bf16x2(s[2 * kk2 + 1][2], s[2 * kk2 + 1][3]);
#pragma unroll
      for (int dt2 = 0; dt2 < D / 16; ++dt2) {
        uint32_t vf[4];
        const int r = kk2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldmatrix_x4_trans(vf, vb + swz<D>(r, dt2 * 2 + (lane >> 4)));
        mma_bf16_16816(o[2 * dt2], a, &vf[0]);
        mma_bf16_16816(o[2 * dt2 + 1], a, &vf[2]);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float l = l_run[h];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int r = warp * 16 + g8 + 8 * h;
    if (r < nq) {
      float* dst = out + static_cast<size_t>(sTokQ[r]) * D;
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        *reinterpret_cast<float2*>(dst + dt * 8 + 2 * t4) =
            make_float2(o[dt][2 * h] * inv, o[dt][2 * h + 1] * inv);
      }
    }
  }
}

// ------------------------------------------------------------------------------------
// Probe rows, bf16 inputs.  CTA = 64 probe rows (4 warps) x one split of the key groups
// (all N keys in key_perm order).  Two online-softmax states per row: dense (every
// key) and sparse (keys of the groups routed to the row's query block).  P enters the
// PV products as bf16 hi + lo.  Partial (m, l, O) per split; combined afterwards.
// ------------------------------------------------------------------------------------
constexpr int kProbeRows = 64;
constexpr int kProbeChunk = 32;

template <int D>
__global__ void __launch_bounds__(128)
    probe_mma_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                     const __nv_bfloat16* __restrict__ V, int N, int block, int G, int k,
                     const int* __restrict__ probe_idx, int P, const int* __restrict__ key_perm,
                     const int* __restrict__ key_gsize, const int* __restrict__ route,
                     const int* __restrict__ qblock_of_token, int groups_per_split,
                     float scale_log2, float* __restrict__ part) {
  constexpr int kCh = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kProbeRows * D * 2;
  uint8_t* sV = sK + 2 * kProbeChunk * D * 2;
  __shared__ uint32_t sMember[kProbeRows];  // bit (g - g0): group routed to row's block

  const int head = blockIdx.z;
  const int split = blockIdx.y;
  const int row0 = blockIdx.x * kProbeRows;
  const int nsplit = gridDim.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t hoff = static_cast<size_t>(head) * N * D;
  Q += hoff;
  K += hoff;
  V += hoff;
  const size_t goff = static_cast<size_t>(head) * G;
  const int* kperm = key_perm + goff * block;
  const int g0 = split * groups_per_split;
  const int g1 = min(G, g0 + groups_per_split);

  for (int x = tid; x < kProbeRows * kCh; x += 128) {
    const int r = x / kCh, ch = x % kCh;
    const int p = row0 + r;
    const int tok = p < P ? probe_idx[static_cast<size_t>(head) * P + p] : -1;
    cp_async_16(smem_u32(sQ) + swz<D>(r, ch), tok >= 0 ? Q + static_cast<size_t>(tok) * D + ch * 8 : Q,
                tok >= 0 ? 16 : 0);
  }
  cp_async_commit();
  if (tid < kProbeRows) {
    uint32_t bits = 0;
    const int p = row0 + tid;
    if (p < P) {
      const int tok = probe_idx[static_cast<size_t>(head) * P + p];
      const int blk = qblock_of_token[static_cast<size_t>(head) * N + tok];
      const int* rt = route + (goff + blk) * k;
      for (int j = 0; j < k; ++j) {
        const int g = rt[j];
        if (g < 0) break;  // -1 padding
        if (g >= g0 && g < g1) bits |= 1u << (g - g0);
      }
    }
    sMember[tid] = bits;
  }

  const int cpg = block / kProbeChunk;
  const int n_chunks = (g1 - g0) * cpg;
  auto load_chunk = [&](int t) {
    const int stage = t & 1;
    const int g = g0 + t / cpg;
    const int gs = __ldg(key_gsize + goff + g);
    const int j0 = (t % cpg) * kProbeChunk;
    const uint32_t kb = smem_u32(sK) + stage * kProbeChunk * D * 2;
    const uint32_t vb = smem_u32(sV) + stage * kProbeChunk * D * 2;
    for (int x = tid; x < kProbeChunk * kCh; x += 128) {
      const int j = x / kCh, ch = x % kCh;
      const int slot = j0 + j;
      const int tok = slot < gs ? __ldg(kperm + g * block + slot) : -1;
      const size_t off = tok >= 0 ? static_cast<size_t>(tok) * D + ch * 8 : 0;
      cp_async_16(kb + swz<D>(j, ch), K + off, tok >= 0 ? 16 : 0);
      cp_async_16(vb + swz<D>(j, ch), V + off, tok >= 0 ? 16 : 0);
    }
  };
  if (n_chunks > 0) load_chunk(0);
  cp_async_commit();

  const int g8 = lane >> 2, t4 = lane & 3;
  float od[D / 8][4], os[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    od[i][0] = od[i][1] = od[i][2] = od[i][3] = 0.f;
    os[i][0] = os[i][1] = os[i][2] = os[i][3] = 0.f;
  }
  float md[2] = {kNegInf, kNegInf}, ld[2] = {0.f, 0.f};
  float ms[2] = {kNegInf, kNegInf}, ls[2] = {0.f, 0.f};

  for (int t = 0; t < n_chunks; ++t) {
    if (t + 1 < n_chunks) load_chunk(t + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int stage = t & 1;
    const uint32_t kb = smem_u32(sK) + stage * kProbeChunk * D * 2;
    const uint32_t vb = smem_u32(sV) + stage * kProbeChunk * D * 2;
    const int g = g0 + t / cpg;
    const int nvalid = __ldg(key_gsize + goff + g) - (t % cpg) * kProbeChunk;
    bool member[2];
    member[0] = (sMember[warp * 16 + g8] >> (g - g0)) & 1u;
    member[1] = (sMember[warp * 16 + g8 + 8] >> (g - g0)) & 1u;

    float s[kProbeChunk / 8][4];
#pragma unroll
    for (int i = 0; i < kProbeChunk / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t qa[4];
      ldmatrix_x4(qa, smem_u32(sQ) + swz<D>(warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                                             kk * 2 + (lane >> 4)));
#pragma unroll
      for (int nt2 = 0; nt2 < kProbeChunk / 16; ++nt2) {
        uint32_t bf[4];
        ldmatrix_x4(bf, kb + swz<D>(nt2 * 16 + (lane & 7) + (lane >> 4) * 8, kk * 2 + ((lane >> 3) & 1)));
        mma_bf16_16816(s[2 * nt2], qa, &bf[0]);
        mma_bf16_16816(s[2 * nt2 + 1], qa, &bf[2]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < kProbeChunk / 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int key = nt * 8 + 2 * t4 + (c & 1);
        s[nt][c] = key < nvalid ? s[nt][c] * scale_log2 : kNegInf;
      }
    }
    float pd[kProbeChunk / 8][4], ps[kProbeChunk / 8][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = kNegInf;
#pragma unroll
      for (int nt = 0; nt < kProbeChunk / 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * h], s[nt][2 * h + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      {  // dense state
        const float m_new = fmaxf(md[h], mx);
        const float m_use = m_new == kNegInf ? 0.f : m_new;
        const float alpha = fast_exp2(md[h] - m_use);
        float sum = 0.f;
#pragma unroll
        for (int nt = 0; nt < kProbeChunk / 8; ++nt) {
          pd[nt][2 * h] = fast_exp2(s[nt][2 * h] - m_use);
          pd[nt][2 * h + 1] = fast_exp2(s[nt][2 * h + 1] - m_use);
          sum += pd[nt][2 * h] + pd[nt][2 * h + 1];
        }
        ld[h] = ld[h] * alpha + sum;
        md[h] = m_new;
#pragma unroll
        for (int dt = 0; dt < D / 8; ++dt) {
          od[dt][2 * h] *= alpha;
          od[dt][2 * h + 1] *= alpha;
        }
      }
      {  // sparse state: only rows whose block routes this group
        const float mxs = member[h] ? mx : kNegInf;
        const float m_new = fmaxf(ms[h], mxs);
        const float m_use = m_new == kNegInf ? 0.f : m_new;
        const float alpha = fast_exp2(ms[h] - m_use);
        float sum = 0.f;
#pragma unroll
        for (int nt = 0; nt < kProbeChunk / 8; ++nt) {
          ps[nt][2 * h] = member[h] ? fast_exp2(s[nt][2 * h] - m_use) : 0.f;
          ps[nt][2 * h + 1] = member[h] ? fast_exp2(s[nt][2 * h + 1] - m_use) : 0.f;
          sum += ps[nt][2 * h] + ps[nt][2 * h + 1];
        }
        ls[h] = ls[h] * alpha + sum;
        ms[h] = m_new;
#pragma unroll
        for (int dt = 0; dt < D / 8; ++dt) {
          os[dt][2 * h] *= alpha;
          os[dt][2 * h + 1] *= alpha;
        }
      }
    }
#pragma unroll
    for (int kk2 = 0; kk2 < kProbeChunk / 16; ++kk2) {
      uint32_t adh[4], adl[4], ash[4], asl[4];
      split_bf16x2(pd[2 * kk2][0], pd[2 * kk2][1], adh[0], adl[0]);
      split_bf16x2(pd[2 * kk2][2], pd[2 * kk2][3], adh[1], adl[1]);
      split_bf16x2(pd[2 * kk2 + 1][0], pd[2 * kk2 + 1][1], adh[2], adl[2]);
      split_bf16x2(pd[2 * kk2 + 1][2], pd[2 * kk2 + 1][3], adh[3], adl[3]);
      split_bf16x2(ps[2 * kk2][0], ps[2 * kk2][1], ash[0], asl[0]);
      split_bf16x2(ps[2 * kk2][2], ps[2 * kk2][3], ash[1], asl[1]);
      split_bf16x2(ps[2 * kk2 + 1][0], ps[2 * kk2 + 1][1], ash[2], asl[2]);
      split_bf16x2(ps[2 * kk2 + 1][2], ps[2 * kk2 + 1][3], ash[3], asl[3]);
#pragma unroll
      for (int dt2 = 0; dt2 < D / 16; ++dt2) {
        uint32_t vf[4];
        ldmatrix_x4_trans(vf, vb + swz<D>(kk2 * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                                          dt2 * 2 + (lane >> 4)));
        mma_bf16_16816(od[2 * dt2], adh, &vf[0]);
        mma_bf16_16816(od[2 * dt2], adl, &vf[0]);
        mma_bf16_16816(od[2 * dt2 + 1], adh, &vf[2]);
        mma_bf16_16816(od[2 * dt2 + 1], adl, &vf[2]);
        mma_bf16_16816(os[2 * dt2], ash, &vf[0]);
        mma_bf16_16816(os[2 * dt2], asl, &vf[0]);
        mma_bf16_16816(os[2 * dt2 + 1], ash, &vf[2]);
        mma_bf16_16816(os[2 * dt2 + 1], asl, &vf[2]);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // partial layout per (head, row, split): [m_d, l_d, m_s, l_s, O_d[D], O_s[D]]
  constexpr int kRec = 4 + 2 * D;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float l1 = ld[h], l2 = ls[h];
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    l2 += __shfl_xor_sync(0xffffffffu, l2, 1);
    l2 += __shfl_xor_sync(0xffffffffu, l2, 2);
    const int p = row0 + warp * 16 + g8 + 8 * h;
    if (p < P) {
      float* rec = part + ((static_cast<size_t>(head) * P + p) * nsplit + split) * kRec;
      if (t4 == 0) {
        rec[0] = md[h];
        rec[1] = l1;
        rec[2] = ms[h];
        rec[3] = l2;
      }
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        rec[4 + dt * 8 + 2 * t4] = od[dt][2 * h];
        rec[4 + dt * 8 + 2 * t4 + 1] = od[dt][2 * h + 1];
        rec[4 + D + dt * 8 + 2 * t4] = os[dt][2 * h];
        rec[4 + D + dt * 8 + 2 * t4 + 1] = os[dt][2 * h + 1];
      }
    }
  }
}

// Combine the per-split partials of one probe row (one CTA of D threads per row).
template <int D>
__global__ void probe_combine_kernel(const float* __restrict__ part, int P, int nsplit,
                                     float* __restrict__ probe_out, float* __restrict__ probe_sparse) {
  constexpr int kRec = 4 + 2 * D;
  const int p = blockIdx.x, head = blockIdx.y, e = threadIdx.x;
  const float* base = part + (static_cast<size_t>(head) * P + p) * nsplit * kRec;
  for (int which = 0; which < 2; ++which) {
    float m = kNegInf;
    for (int s = 0; s < nsplit; ++s) m = fmaxf(m, base[s * kRec + 2 * which]);
    float l = 0.f, acc = 0.f;
    if (m != kNegInf) {
      for (int s = 0; s < nsplit; ++s) {
        const float ms = base[s * kRec + 2 * which];
        if (ms == kNegInf) continue;
        const float f = fast_exp2(ms - m);
        l += base[s * kRec + 2 * which + 1] * f;
        acc += base[s * kRec + 4 + which * D + e] * f;
      }
    }
    float* dst = (which == 0 ? probe_out : probe_sparse) + (static_cast<size_t>(head) * P + p) * D;
    dst[e] = l > 0.f ? acc / l : 0.f;
  }
}

// ------------------------------------------------------------------------------------
// fp32 inputs: exact fp32 SIMT attention, one warp per query row.
// ------------------------------------------------------------------------------------
template <int D>
struct RowState {
  float q[D / 32], o[D / 32];
  float m, l;
  __device__ void init(const float* qrow, int lane) {
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      q[i] = qrow[lane + 32 * i];
      o[i] = 0.f;
    }
    m = kNegInf;
    l = 0.f;
  }
  __device__ void add_key(const float* krow, const float* vrow, int lane, float scale_log2) {
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) dot += q[i] * krow[lane + 32 * i];
    const float sc = warp_sum(dot) * scale_log2;
    const float m_new = fmaxf(m, sc);
    const float alpha = exp2f(m - m_new);
    const float p = exp2f(sc - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) o[i] = o[i] * alpha + p * vrow[lane + 32 * i];
    m = m_new;
  }
  __device__ void store(float* dst, int lane) const {
#pragma unroll
    for (int i = 0; i < D / 32; ++i) dst[lane + 32 * i] = l > 0.f ? o[i] / l : 0.f;
  }
};

template <int D, bool DENSE>
__global__ void attn_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                                const float* __restrict__ V, int N, int block, int G, int k,
                                const int* __restrict__ key_perm, const int* __restrict__ key_gsize,
                                const int* __restrict__ query_perm, const int* __restrict__ qblock_size,
                                const int* __restrict__ route, float scale_log2, float* __restrict__ out) {
  const int b = blockIdx.x, head = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const size_t hoff = static_cast<size_t>(head) * N * D;
  const size_t goff = static_cast<size_t>(head) * G;
  const int nq = DENSE ? min(block, N - b * block) : qblock_size[goff + b];
  for (int r = warp; r < nq; r += nwarps) {
    const int tok = DENSE ? b * block + r : query_perm[(goff + b) * block + r];
    RowState<D> st;
    st.init(Q + hoff + static_cast<size_t>(tok) * D, lane);
    const int ng = DENSE ? G : routed_len(route + (goff + b) * k, k);
    for (int x = 0; x < ng; ++x) {
      const int g = DENSE ? x : route[(goff + b) * k + x];
      const int gs = DENSE ? min(block, N - g * block) : key_gsize[goff + g];
      for (int j = 0; j < gs; ++j) {
        const int kt = DENSE ? g * block + j : key_perm[(goff + g) * block + j];
        st.add_key(K + hoff + static_cast<size_t>(kt) * D, V + hoff + static_cast<size_t>(kt) * D, lane,
                   scale_log2);
      }
    }
    st.store(out + hoff + static_cast<size_t>(tok) * D, lane);
  }
}

template <int D>
__global__ void probe_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                                 const float* __restrict__ V, int N, int block, int G, int k,
                                 const int* __restrict__ probe_idx, int P,
                                 const int* __restrict__ key_perm, const int* __restrict__ key_gsize,
                                 const int* __restrict__ route, const int* __restrict__ qblock_of_token,
                                 float scale_log2, float* __restrict__ probe_out,
                                 float* __restrict__ probe_sparse) {
  const int head = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (p >= P) return;
  const size_t hoff = static_cast<size_t>(head) * N * D;
  const size_t goff = static_cast<size_t>(head) * G;
  const int tok = probe_idx[static_cast<size_t>(head) * P + p];
  RowState<D> dense, sparse;
  dense.init(Q + hoff + static_cast<size_t>(tok) * D, lane);
  sparse.init(Q + hoff + static_cast<size_t>(tok) * D, lane);
  for (int j = 0; j < N; ++j)
    dense.add_key(K + hoff + static_cast<size_t>(j) * D, V + hoff + static_cast<size_t>(j) * D, lane,
                  scale_log2);
  const int blk = qblock_of_token[static_cast<size_t>(head) * N + tok];
  const int nr = routed_len(route + (goff + blk) * k, k);
  for (int x = 0; x < nr; ++x) {
    const int g = route[(goff + blk) * k + x];
    const int gs = key_gsize[goff + g];
    for (int j = 0; j < gs; ++j) {
      const int kt = key_perm[(goff + g) * block + j];
      sparse.add_key(K + hoff + static_cast<size_t>(kt) * D, V + hoff + static_cast<size_t>(kt) * D, lane,
                     scale_log2);
    }
  }
  dense.store(probe_out + (static_cast<size_t>(head) * P + p) * D, lane);
  sparse.store(probe_sparse + (static_cast<size_t>(head) * P + p) * D, lane);
}

// Probe rows: midpoint stride floor((2p+1) N / (2P)) in token order, same for every head.
__global__ void probe_rows_kernel(int N, int P, int heads, int* __restrict__ probe_idx) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= heads * P) return;
  const long long p = x % P;
  probe_idx[x] = static_cast<int>(((2 * p + 1) * N) / (2ll * P));
}

cudaError_t launch_probe_rows(int N, int P, int heads, int* probe_idx, cudaStream_t st) {
  probe_rows_kernel<<<ceil_div(heads * P, 256), 256, 0, st>>>(N, P, heads, probe_idx);
  return counted(cudaGetLastError(), 1);
}

// token -> query block, from query_perm.
__global__ void qblock_of_token_kernel(const int* __restrict__ query_perm, int N, int block, int G,
                                       int* __restrict__ qblk) {
  const int head = blockIdx.y;
  const int slots = G * block;
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < slots; s += gridDim.x * blockDim.x) {
    const int tok = query_perm[static_cast<size_t>(head) * slots + s];
    if (tok >= 0) qblk[static_cast<size_t>(head) * N + tok] = s / block;
  }
}

// ------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------
template <int D, int BQ, bool DENSE>
static cudaError_t launch_attn_mma_t(const AttnArgs& a, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(BQ) * D * 2 + 4ull * kChunk * D * 2;
  auto kern = attn_mma_kernel<D, BQ, DENSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.G, a.heads);
  kern<<<grid, BQ * 2, smem, st>>>(static_cast<const __nv_bfloat16*>(a.Q), static_cast<const __nv_bfloat16*>(a.K),
                                   static_cast<const __nv_bfloat16*>(a.V), a.N, a.G, a.k, a.key_perm,
                                   a.key_gsize, a.query_perm, a.qblock_size, a.route, a.scale_log2, a.out);
  return counted(cudaGetLastError(), 1);
}

template <int D, bool DENSE>
static cudaError_t launch_attn_f32_t(const AttnArgs& a, cudaStream_t st) {
  dim3 grid(a.G, a.heads);
  attn_f32_kernel<D, DENSE><<<grid, 256, 0, st>>>(
      static_cast<const float*>(a.Q), static_cast<const float*>(a.K), static_cast<const float*>(a.V), a.N,
      a.block, a.G, a.k, a.key_perm, a.key_gsize, a.query_perm, a.qblock_size, a.route, a.scale_log2, a.out);
  return counted(cudaGetLastError(), 1);
}

cudaError_t launch_attention(const AttnArgs& a, bool dense, cudaStream_t st) {
  if (!a.f32 && a.d == 128 && a.block == 128) return launch_attention_tc(a, dense, a.status, st);
  if (a.f32) {
    if (a.d == 64) return dense ? launch_attn_f32_t<64, true>(a, st) : launch_attn_f32_t<64, false>(a, st);
    return dense ? launch_attn_f32_t<128, true>(a, st) : launch_attn_f32_t<128, false>(a, st);
  }
  if (a.d == 64) {
    if (a.block == 64) return dense ? launch_attn_mma_t<64, 64, true>(a, st) : launch_attn_mma_t<64, 64, false>(a, st);
    return dense ? launch_attn_mma_t<64, 128, true>(a, st) : launch_attn_mma_t<64, 128, false>(a, st);
  }
  if (a.block == 64) return dense ? launch_attn_mma_t<128, 64, true>(a, st) : launch_attn_mma_t<128, 64, false>(a, st);
  return dense ? launch_attn_mma_t<128, 128, true>(a, st) : launch_attn_mma_t<128, 128, false>(a, st);
}

int probe_groups_per_split(int G) { return G < 32 ? G : 32; }

size_t probe_partial_bytes(int heads, int P, int G, int d) {
  const int gps = probe_groups_per_split(G);
  const int nsplit = ceil_div(G, gps);
  return static_cast<size_t>(heads) * P * nsplit * (4 + 2 * d) * sizeof(float);
}

// Splits of the key groups for the tensor-core probe kernel (one CTA per SM): at most
// 64 groups a split, at most max_splits (the partial buffer's room), and the count that
// minimises waves x groups per CTA over 148 SMs, with ~4 groups of fixed cost per CTA.
static int probe_tc_splits(int G, int units, int max_splits) {
  const int lo = ceil_div(G, 64);
  int best = std::max(lo, 1), best_cost = -1;
  for (int n = std::max(lo, 1); n <= std::max(max_splits, lo); ++n) {
    const int waves = ceil_div(units * n, 148);
    const int cost = waves * (ceil_div(G, n) + 4);
    if (best_cost < 0 || cost < best_cost) {
      best = n;
      best_cost = cost;
    }
  }
  return best;
}

template <int D>
static cudaError_t launch_probe_t(const ProbeArgs& a, cudaStream_t st) {
  qblock_of_token_kernel<<<dim3(ceil_div(a.G * a.block, 256), a.heads), 256, 0, st>>>(
      a.query_perm, a.N, a.block, a.G, a.qblk);
  if (a.f32) {
    probe_f32_kernel<D><<<dim3(ceil_div(a.P, 4), a.heads), 128, 0, st>>>(
        static_cast<const float*>(a.Q), static_cast<const float*>(a.K), static_cast<const float*>(a.V), a.N,
        a.block, a.G, a.k, a.probe_idx, a.P, a.key_perm, a.key_gsize, a.route, a.qblk, a.scale_log2,
        a.probe_out, a.probe_sparse);
    return counted(cudaGetLastError(), 2);
  }
  const int gps = probe_groups_per_split(a.G);
  const int nsplit = ceil_div(a.G, gps);
  if (D == 128 && a.block == 128 && a.k_grouped != nullptr && a.v_grouped != nullptr && a.status != nullptr) {
    // tensor-core path: K / V in group order, then one CTA per (128 probe rows, split, head)
    cudaError_t e = launch_kv_group(a.K, a.V, a.N, a.G, a.heads, a.key_perm, a.key_gsize, a.k_grouped,
                                    a.v_grouped, a.kv_tag, st);
    if (e != cudaSuccess) return e;
    const int ns = probe_tc_splits(a.G, a.heads * ceil_div(a.P, 128), nsplit);
    if ((e = launch_probe_tc(a, ns, st)) != cudaSuccess) return e;
    probe_combine_kernel<D><<<dim3(a.P, a.heads), D, 0, st>>>(a.partial, a.P, ns, a.probe_out, a.probe_sparse);
    return counted(cudaGetLastError(), 2);
  }
  const size_t smem = static_cast<size_t>(kProbeRows) * D * 2 + 4ull * kProbeChunk * D * 2;
  auto kern = probe_mma_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<dim3(ceil_div(a.P, kProbeRows), nsplit, a.heads), 128, smem, st>>>(
      static_cast<const __nv_bfloat16*>(a.Q), static_cast<const __nv_bfloat16*>(a.K),
      static_cast<const __nv_bfloat16*>(a.V), a.N, a.block, a.G, a.k, a.probe_idx, a.P, a.key_perm,
      a.key_gsize, a.route, a.qblk, gps, a.scale_log2, a.partial);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  probe_combine_kernel<D><<<dim3(a.P, a.heads), D, 0, st>>>(a.partial, a.P, nsplit, a.probe_out, a.probe_sparse);
  return counted(cudaGetLastError(), 3);
}

cudaError_t launch_probe(const ProbeArgs& a, cudaStream_t st) {
  return a.d == 64 ? launch_probe_t<64>(a, st) : launch_probe_t<128>(a, st);
}

}  // namespace spr
