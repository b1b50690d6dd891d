// Launch interface of the routing kernel (internal to the library).
#pragma once

#include <cuda_runtime.h>

namespace spr {

// pairs may be null (selection only, e.g. on injected scores).
cudaError_t launch_route(const float* sc, int heads, int Gq, int G, int k, int* route, const int* key_gsize,
                         const int* qblock_size, long long* pairs, long long probe_pairs, int* status,
                         cudaStream_t st);

}  // namespace spr
