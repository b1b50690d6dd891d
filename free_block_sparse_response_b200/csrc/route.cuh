// Launch interface of the routing kernel (internal to the library).
#pragma once

#include <cuda_runtime.h>

namespace spr {

// pairs may be null (selection only, e.g. on injected scores).
cudaError_t launch_route(const float* sc, int heads, int Gq, int G, int k, int* route, const int* key_gsize,
                         const int* qblock_size, long long* pairs, long long probe_pairs, int* status,
                         cudaStream_t st);
// Global budget allocation: every block keeps its best group, the other (block, group)
// pairs in descending score order while the head's pair budget lasts; route [heads, Gq, G]
// holds each block's groups in ascending order then -1.  key_gsize and qblock_size are
// required (the pair costs).
cudaError_t launch_route_global(const float* sc, int heads, int Gq, int G, long long budget, int* route,
                                const int* key_gsize, const int* qblock_size, long long* pairs, long long probe_pairs,
                                int* status, cudaStream_t st);
// Replace (LSE, mode 2) or correct (size, mode 1) the centroid block scores sc [heads,
// Gq, G]; qbar [heads, Gq, 128] are the query-block means, K bf16 with d = 128.
cudaError_t launch_route_scores(int mode, float* sc, const void* K, int N, int heads, int Gq, int G,
                                const int* key_perm, const int* key_gsize, const float* qbar, float tau,
                                cudaStream_t st);

}  // namespace spr
