// la_phi_map.cuh — phi(q) and phi(k) written out elementwise, for the
// forward paths that do not store them from their own tiles (non-causal,
// D != 64, float32, segment-split runs of the D = 64 causal kernel store
// them themselves).  Same feature map as those paths: phi_fast rounded to
// bf16 for bf16 tensors, phi_exact for float32.
#pragma once

#include "la_common.cuh"

namespace la {

template <typename T, int PHI>
__global__ void __launch_bounds__(256)
phi_map_kernel(const T* __restrict__ q, const T* __restrict__ k, T* __restrict__ pq,
               T* __restrict__ pk, int64_t n) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float a = to_f32(q[i]), b = to_f32(k[i]);
        if constexpr (sizeof(T) == 4) {
            pq[i] = from_f32<T>(phi_exact<PHI>(a));
            pk[i] = from_f32<T>(phi_exact<PHI>(b));
        } else {
            pq[i] = from_f32<T>(phi_fast<PHI>(a));
            pk[i] = from_f32<T>(phi_fast<PHI>(b));
        }
    }
}

}  // namespace la
