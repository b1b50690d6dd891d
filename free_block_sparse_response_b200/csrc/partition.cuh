// Launch interface of the partition kernels (internal to the library).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace spr {

struct RowGemmArgs {
  const void* X;  // [heads, n, d] bf16 or f32
  bool f32;
  int heads, n, d, ncols;
  const __nv_bfloat16* Bhi;  // [heads, ncols, d] (bf16 path)
  const __nv_bfloat16* Blo;  // optional low part (split precision)
  const float* Bf32;         // [heads, ncols, d] (fp32 path)
  const float* nrm;          // DIST: [heads, n]
  const float* ecol;         // DIST: [heads, ncols]
  float tau2;
  float* Dout;               // DIST: [heads, n, ldd]
  int ldd;                   // DIST: row stride of Dout (>= ncols)
  int* prop_g;               // DIST: [heads, n]
  float* prop_v;
  float* nrm_out;            // NORM: [heads, n]
  int* status;
};

struct FillArgs {
  const float* D;       // [heads, n, ldd]
  int ldd;              // row stride of D (>= G)
  const int* prop_g0;   // optional first proposals [heads, n]
  const float* prop_v0;
  int heads, n, G, cap;
  int* labels;          // [heads, n]
  int* room;            // [heads, G]
  int* cnt;
  int* offs;
  int* cursor;
  unsigned int* closed;  // [heads, ceil(G/32)] bit g set once group g is full
  unsigned long long* bucket;  // [heads, n]
  int* list0;           // [heads * n]
  int* list1;
  int* list_len;        // [2]
  int* prop_g;          // [heads, n]
  float* prop_v;
  WorkspaceHeader* hdr;
  int stage_closed;     // set by the launcher: bitmaps fit in shared memory
  int d_vec4;           // set by the launcher: D rows start on 16-byte boundaries
};

// One balanced k-means assignment (the capacity fill) with the distances recomputed on
// tcgen05 in every proposal round (bf16 items, d = 128, at most 1024 groups per head).
struct AssignArgs {
  int heads, n, G, cap;
  float tau2;
  const __nv_bfloat16* x;       // [heads, n, 128]  the items (set by the launcher)
  const __nv_bfloat16* whi;     // [heads, G, 128]  W = C Gamma, bf16 hi / lo (set by the launcher)
  const __nv_bfloat16* wlo;
  const float* nrm;             // [heads, n]  x_i^T Gamma x_i
  const float* ecol;            // [heads, G]  c_g^T Gamma c_g
  int* labels;                  // [heads, n]  out: the group of every item
  int* room;                    // [heads, G]
  int* cnt;
  int* offs;
  int* cursor;
  unsigned int* closed;         // [heads, ceil(G/32)]
  unsigned long long* bucket;   // [heads, n]
  int* list[2];                 // [heads, n] each: per-head lists of unplaced items
  int* list_len;                // [2, heads]
  int* prop_g;                  // [heads, n]
  float* prop_v;
  int* members;                 // [heads, G, cap]: every group's members, in placement order
  int* msize;                   // [heads, G]: their counts
  int* ovf_list;                // [heads, G]: the round's groups with more proposers than room
  int* ovf_total;               // [2]: its length, alternating between rounds
  float* nrm_out;               // norm mode: [heads, n] x_i^T Gamma x_i with W = Gamma, no fill
  float* Dout;                  // optional [heads, n, ldd]: the first round's D rows
  int ldd;
  // Tail of the fill: once at most tail_cap items are unplaced, the next round's tensor-
  // core pass also stores each one's D row (closed groups as +inf) at Dtail[pos * ldt],
  // pos in tailpos[item]; the rounds after it propose from the stored rows.
  float* Dtail;                 // [tail_cap, ldt], ldt = ceil(G / 128) * 128
  int ldt;
  int tail_cap;
  int* tailpos;                 // [heads, n]
  // Rounds after the first multiply the rows with the open groups' W only: each round
  // starts by packing every head's open groups (ascending) into wc_hi / wc_lo at the same
  // per-head offsets, open_g mapping packed column -> group and n_open counting them.
  __nv_bfloat16* wc_hi;         // [heads, G, 128]
  __nv_bfloat16* wc_lo;
  int* open_g;                  // [heads, G]
  int* n_open;                  // [heads]
  WorkspaceHeader* hdr;
};
cudaError_t launch_assign_tc(const __nv_bfloat16* X, const __nv_bfloat16* Whi, const __nv_bfloat16* Wlo,
                             const AssignArgs& a, cudaStream_t st);
// nrm[h, i] = x_i^T Gamma_h x_i on the same pipeline (bf16 X, d = 128, Gamma as bf16 hi + lo)
cudaError_t launch_row_norms_tc(const __nv_bfloat16* X, const __nv_bfloat16* ghi, const __nv_bfloat16* glo,
                                int heads, int n, float* nrm, WorkspaceHeader* hdr, cudaStream_t st);

cudaError_t launch_midpoint_stride(int* idx, int n, int count, cudaStream_t st);
// gamma [heads, d, d] = identity (the metric of the semantic partition)
cudaError_t launch_identity(float* gamma, int heads, int d, cudaStream_t st);
cudaError_t launch_gram(const void* X, bool f32, size_t head_stride, const int* rows, int nrows, int heads,
                        int d, float* gamma, cudaStream_t st);
cudaError_t launch_split_bf16(const float* src, __nv_bfloat16* hi, __nv_bfloat16* lo, size_t count,
                              cudaStream_t st);
cudaError_t launch_chunk_perm(int* perm, int* sizes, int n, int G, int cap, int heads, cudaStream_t st);
cudaError_t launch_centroid(const void* X, bool f32, int n, const int* perm, const int* sizes, int G, int cap,
                            int heads, int d, float* cent, cudaStream_t st);
cudaError_t launch_wmat(const float* cent, const float* gamma, int G, int heads, int d, float* wf,
                        __nv_bfloat16* whi, __nv_bfloat16* wlo, float* eg, cudaStream_t st);
cudaError_t launch_rowgemm(const RowGemmArgs& a, bool dist, cudaStream_t st);
cudaError_t launch_fill(const FillArgs& a, cudaStream_t st);
cudaError_t launch_build_perm(const int* labels, int n, int G, int cap, int heads, int* cursor, int* tmp,
                              int* perm, int* sizes, int* status, cudaStream_t st);
// Members (unsorted tmp lists, cursor counts) -> sorted perm and sizes, the member means
// cent, and W = cent Gamma (fp32, bf16 hi/lo), e_g = c_g . w_g for the next iteration.
cudaError_t launch_group_update(const void* X, bool f32, int n, const int* cursor, const int* tmp, int G, int cap,
                                int heads, int d, const float* gamma, int* perm, int* sizes, float* cent, float* wf,
                                __nv_bfloat16* whi, __nv_bfloat16* wlo, float* eg, cudaStream_t st);
// labels -> unsorted member lists tmp[g * cap + slot] and their counts cursor[g]
cudaError_t launch_perm_scatter(const int* labels, int n, int G, int cap, int heads, int* cursor, int* tmp,
                                int* status, cudaStream_t st);
cudaError_t launch_block_scores(const float* qbar, const float* mu, int G, int heads, int d, float tau,
                                float* sc, cudaStream_t st);

}  // namespace spr
