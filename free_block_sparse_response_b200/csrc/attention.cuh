// Launch interface of the attention kernels (internal to the library).
#pragma once

#include <cuda.h>
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
  unsigned long long* kv_tag;  // workspace header's copy tag (null: always copy)
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
  // tensor-core path (bf16, d = 128, B = 128): K and V in key-group order (workspace,
  // written by the probe call) and the device status word for its bounded waits
  void* k_grouped;
  void* v_grouped;
  unsigned long long* kv_tag;  // workspace header's copy tag (null: always copy)
  int* status;
};

cudaError_t launch_attention(const AttnArgs& a, bool dense, cudaStream_t st);
// TMA map over a [rows, 128] bf16 tensor, 128-byte swizzle, box 64 columns x box_rows rows
// (box_rows = 1 for row gathers); false if the driver entry point or the encode fails.
bool bf16_map(CUtensorMap* m, const void* base, long long rows, int box_rows);
// Group-ordered copies of K and V ([heads, G * 128, 128] bf16, pad rows zero).  With a
// tag (the workspace header's kv_tag) the copy is skipped on the device when the tag
// names the same K, V, key_perm, key_gsize and shape, and the tag is set afterwards.
cudaError_t launch_kv_group(const void* K, const void* V, int N, int G, int heads, const int* key_perm,
                            const int* key_gsize, void* k_grouped, void* v_grouped, unsigned long long* kv_tag,
                            cudaStream_t st);
// Probe rows on the tensor cores (bf16, d = 128, B = 128); partial records in the
// layout probe_combine_kernel reads, nsplit splits of the key groups.
cudaError_t launch_probe_tc(const ProbeArgs& a, int nsplit, cudaStream_t st);
cudaError_t launch_attention_tc(const AttnArgs& a, bool dense, int* status, cudaStream_t st);
// Event pairs around the tensor-core attention kernel (measurement hook).
void attn_timing_enable(bool on);
cudaError_t attn_timing_read(double* ms_total, long long* launches);
size_t attn_tc_smem_bytes(int n_tiles);
cudaError_t launch_probe(const ProbeArgs& a, cudaStream_t st);
size_t probe_partial_bytes(int heads, int P, int G, int d);
cudaError_t launch_probe_rows(int N, int P, int heads, int* probe_idx, cudaStream_t st);

}  // namespace spr
