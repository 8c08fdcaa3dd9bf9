// la_pad.cuh — row copies between feature widths, for attention whose
// feature vectors and value vectors differ in length (m features of
// q and k, head size D of v): the narrower operand is widened with zero
// columns into the workspace, and the wider result is narrowed back.  Zero
// value columns add zero output columns; zero feature columns add nothing to
// a_i . b_j, S or z (with the identity feature map, whose features are given).
#pragma once

#include "la_common.cuh"

namespace la {

// dst[r][c] = src[r][c] for c < min(ws, wd), 0 for ws <= c < wd; rows of
// `ws` and `wd` bf16 elements, both multiples of 8 (16-byte units).
__global__ void __launch_bounds__(256)
copy_cols_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t rows, int ws8,
                 int wd8) {
    const int64_t total = rows * wd8;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t r = i / wd8;
        const int c = int(i - r * wd8);
        dst[i] = c < ws8 ? src[r * ws8 + c] : make_uint4(0u, 0u, 0u, 0u);
    }
}

}  // namespace la
