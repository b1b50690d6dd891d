// Launch interface of the attention kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace spr {

struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  bool f32;
  int heads, N, d, block, G, k;
  const int* key_perm;
  const int* key_gsize;
  const int* query_perm;
  const int* qblock_size;
  const int* route;
  float scale_log2;  // tau * log2(e)
  float* out;
  int* status;       // device status word (bounded waits of the tensor-core kernel)
  // Group-ordered copies of K and V ([heads, G * 128, 128] bf16 each, pad rows zero),
  // written by the sparse tensor-core path before its attention kernel; null otherwise.
  void* k_grouped;
  void* v_grouped;
  // Fused correction (sparse, bf16, d = 128 only): when m_hilo is set the kernel writes
  // O = S + S M^T + beta as bf16 to out_bf16 instead of S to out.  m_hilo holds M (per
  // head [128, 128]) as bf16 hi parts for all heads, then the lo parts.
  const void* m_hilo;
  const float* beta;
  void* out_bf16;
};

struct ProbeArgs {
  const void* Q;
  const void* K;
  const void* V;
  bool f32;
  int heads, N, d, block, G, k, P;
  const int* probe_idx;
  const int* key_perm;
  const int* key_gsize;
  const int* query_perm;
  const int* route;
  float scale_log2;
  float* probe_out;
  float* probe_sparse;
  int* qblk;       // workspace [heads, N]
  float* partial;  // workspace, probe_partial_bytes()
};

cudaError_t launch_attention(const AttnArgs& a, bool dense, cudaStream_t st);
cudaError_t launch_attention_tc(const AttnArgs& a, bool dense, int* status, cudaStream_t st);
// Event pairs around the tensor-core attention kernel (measurement hook).
void attn_timing_enable(bool on);
cudaError_t attn_timing_read(double* ms_total, long long* launches);
size_t attn_tc_smem_bytes(int n_tiles);
cudaError_t launch_probe(const ProbeArgs& a, cudaStream_t st);
size_t probe_partial_bytes(int heads, int P, int G, int d);
cudaError_t launch_probe_rows(int N, int P, int heads, int* probe_idx, cudaStream_t st);

}  // namespace spr
