// Launch interface of the fit and apply kernels (internal to the library).
#pragma once
#include <cuda_bf16.h>

#include <cuda_runtime.h>
#include <stddef.h>

namespace spr {

// weight_mode of the fit: the probe weights in the low byte (0 inverse squared norm, 1
// uniform), kRidgeRelative set for lambda relative to the mean diagonal of X_c^T W X_c.
constexpr int kWeightModeMask = 0xff;
constexpr int kRidgeRelative = 0x100;

__host__ __device__ size_t fit_scratch_doubles(int P, int d);
size_t fit_smem_bytes(int d, int P);
// Largest probe count the fit kernel takes at head dimension d (its shared memory).
int fit_max_probes(int d);
cudaError_t launch_fit(const float* xs, const float* dp, const float* weights, int heads, int d, int P,
                       double lambda, int rank, int weight_mode, double* scratch, float* M, float* beta,
                       int* status, cudaStream_t st);
// Probe rows of a bf16 output (d = 128) set to the exact probe outputs.
cudaError_t launch_probe_overwrite_bf16(const int* probe_idx, const float* probe_out, int heads, int N, int P,
                                       __nv_bfloat16* O, cudaStream_t st);
cudaError_t launch_apply(const float* S, const float* M, const float* beta, const int* probe_idx,
                         const float* probe_out, int heads, int N, int d, int P, void* O, bool out_f32,
                         cudaStream_t st);

cudaError_t launch_row_errors(const void* O, bool o_f32, const float* ref, int heads, int N, int d,
                              const int* probe_idx, int P, float* err, cudaStream_t st);

}  // namespace spr
