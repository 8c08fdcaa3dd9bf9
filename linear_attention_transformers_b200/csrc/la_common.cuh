// la_common.cuh — element types, the feature map and small device helpers
// shared by the CUDA kernels of liblinattn.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace la {

enum : int { PHI_ELU1 = 0, PHI_RELU_EPS = 1, PHI_IDENTITY = 2 };

// Error word for bounded waits (set by a kernel that gave up waiting).  The
// library is one translation unit, so the definition lives here.
__device__ unsigned int g_device_error = 0;

// ---------------------------------------------------------------- feature map
// phi is elementwise: elu(x)+1 (x+1 for x > 0, exp(x) otherwise) or
// max(x,0)+1e-6.  The pages leave phi generic ("Efficient Transformers
// Survey", Proposition "Linear Attention via Kernel Decomposition": any
// phi: R^d -> R^m); m = D here.  PHI_IDENTITY: the inputs are feature
// vectors already (the Performer's positive random features, computed by
// la_favor_features), phi(x) = x and phi' = 1.

// Accurate variant (libm expf) for the reference-quality kernels.
template <int PHI>
__device__ __forceinline__ float phi_exact(float x) {
    if (PHI == PHI_ELU1) return x > 0.f ? x + 1.f : expf(x);
    if (PHI == PHI_IDENTITY) return x;
    return fmaxf(x, 0.f) + 1e-6f;
}
template <int PHI>
__device__ __forceinline__ float dphi_exact(float x) {
    if (PHI == PHI_ELU1) return x > 0.f ? 1.f : expf(x);
    if (PHI == PHI_IDENTITY) return 1.f;
    return x > 0.f ? 1.f : 0.f;
}

// e^x for the streaming kernels, from the identity e^x = 2^(x log2 e) on the
// hardware base-2 exponential (ex2.approx.ftz.f32: relative error near 2^-22,
// results below 2^-126 flush to zero).  Its results are rounded to bf16
// right after, so that error never shows.  On B200 the phi pass over a tile
// runs about 1.6x faster with it than with __expf, which also handles
// denormal results.
__device__ __forceinline__ float exp_fast(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x * 1.4426950408889634f));
    return r;
}

// Fast variant of the feature map and its derivative.
template <int PHI>
__device__ __forceinline__ float phi_fast(float x) {
    if (PHI == PHI_ELU1) return x > 0.f ? x + 1.f : exp_fast(x);
    if (PHI == PHI_IDENTITY) return x;
    return fmaxf(x, 0.f) + 1e-6f;
}
template <int PHI>
__device__ __forceinline__ float dphi_fast(float x) {
    if (PHI == PHI_ELU1) return x > 0.f ? 1.f : exp_fast(x);
    if (PHI == PHI_IDENTITY) return 1.f;
    return x > 0.f ? 1.f : 0.f;
}

// ------------------------------------------------ grouped key/value heads
// With grouped-query attention G = kv_group query heads share one key/value
// head ("Attention Optimization", Advanced Techniques: Multi-Query and
// Grouped-Query Attention): flattened query head `head` = b*H + h reads
// key/value head b*Hkv + h/G = head / G, and the state (a function of k and
// v only) belongs to that key/value head.
__device__ __forceinline__ int kv_head_of(int head, int kv_group) {
    return head / (kv_group > 0 ? kv_group : 1);
}
// The group's first query head writes the key/value head's state.
__device__ __forceinline__ bool writes_kv_state(int head, int kv_group) {
    return kv_group <= 1 || head % kv_group == 0;
}

// ------------------------------------------------ decayed (gated) recurrence
// S_i = gamma S_{i-1} + b_i v_i^T, z_i = gamma z_{i-1} + b_i with one gamma
// per head (the gating / decay factors of "Efficient Transformers Survey",
// Common Confusions, "Watch Out").  Passed by value to the kernels that take
// it; H = 0 means no decay (gamma = 1, and gamma * x is then exactly x).
constexpr int kMaxDecayHeads = 256;
struct DecayArg {
    int H;
    float gamma[kMaxDecayHeads];
};
// gamma of flattened head b*H + h
__device__ __forceinline__ float decay_of(const DecayArg& d, size_t head) {
    return d.H > 0 ? d.gamma[head % size_t(d.H)] : 1.f;
}

// ---------------------------------------------------------------- elements
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace la
