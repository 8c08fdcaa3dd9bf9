// la_state.cuh — small kernels over per-segment states.
//
// States are additive: the state after a run of tokens is the sum of the
// states of its pieces (S and z are sums over tokens, "Efficient
// Transformers Survey", Proposition "Linear Attention via Kernel
// Decomposition", Statement).  A record holds S [D][D] (row = key feature)
// followed by z [D], float32; records are laid out [head][segment][R] with
// R = D*D + D.  Every sum below runs over segments in a fixed order, so the
// results are bitwise reproducible.
#pragma once

#include "la_common.cuh"

namespace la {

constexpr int kStateThreads = 256;
constexpr int kStateBatch = 8;  // segments whose loads are issued together

// The kernels below run over float4 columns of the records (R = D*D + D is
// a multiple of 4 for every supported D; record arrays start 16-byte
// aligned): thread e of a head's blocks owns elements 4e..4e+3 of every
// record of that head, so each access is one 16-byte load or store and a
// launch has a quarter of the threads of an element-per-thread layout
// (measured on B200: the exclusive scan of 64 heads x 2 segments of D = 128
// records 11.7 -> 6.2 us back to back).

__device__ __forceinline__ float4 f4add(float4 a, float4 b) {
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
__device__ __forceinline__ float4 f4fma(float f, float4 a, float4 b) {  // f * a + b
    return make_float4(fmaf(f, a.x, b.x), fmaf(f, a.y, b.y), fmaf(f, a.z, b.z),
                       fmaf(f, a.w, b.w));
}

// Up to kStateBatch float4s p0, p0 + step, ... (n of them) of a column of
// records (stride R4 float4s), loaded before any is stored so their
// latencies overlap.
__device__ __forceinline__ void load_batch(const float4* base, int p0, int step, int n, size_t R4,
                                           float4* x) {
#pragma unroll
    for (int i = 0; i < kStateBatch; ++i)
        if (i < n) x[i] = base[size_t(p0 + i * step) * R4];
}

// rec[h][p] <- init[h] + sum_{p' < p} rec[h][p'] (exclusive prefix, in
// place; init is the state the head starts from, null = zero, e.g. the sum
// of the states of the tokens other ranks hold before this rank's).  With a
// decay factor per head (decayed recurrence; every segment before the last
// holds seg_len tokens and its record is its state at its end) the prefix
// is run_p = gamma^seg_len run_{p-1} + rec[p-1]; without one the factor is
// 1 and the sum is the plain one, bit for bit.  R4 = R / 4.
__global__ void __launch_bounds__(kStateThreads)
state_exclusive_scan_kernel(float* __restrict__ rec, int nseg, int R4, int blocks_per_head,
                            const DecayArg dec, int seg_len, const float* __restrict__ init) {
    const size_t h = blockIdx.x / blocks_per_head;
    const int e = (blockIdx.x % blocks_per_head) * kStateThreads + threadIdx.x;
    if (e >= R4) return;
    float4* base = reinterpret_cast<float4*>(rec) + h * size_t(nseg) * R4 + e;
    const float fac = dec.H > 0 ? powf(decay_of(dec, h), float(seg_len)) : 1.f;
    float4 run = init ? reinterpret_cast<const float4*>(init)[h * size_t(R4) + e]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < nseg; p0 += kStateBatch) {
        const int n = min(kStateBatch, nseg - p0);
        float4 x[kStateBatch];
        load_batch(base, p0, 1, n, R4, x);
#pragma unroll
        for (int i = 0; i < kStateBatch; ++i)
            if (i < n) {
                base[size_t(p0 + i) * R4] = run;
                run = f4fma(fac, run, x[i]);
            }
    }
}

// Segment starts of a causal pass from sub-segment records:
// starts[h][p] <- init[h] + sum_{s < p * ratio} sub[h][s] for p < nseg.
// sub holds the states of the (nseg - 1) * ratio equal pieces of the tokens
// before the last segment (its own state is never a start), ratio pieces
// per segment; added in increasing s.  init null = zero.
__global__ void __launch_bounds__(kStateThreads)
state_segment_starts_kernel(const float* __restrict__ sub, float* __restrict__ starts, int nseg,
                            int ratio, int R4, int blocks_per_head,
                            const float* __restrict__ init) {
    const size_t h = blockIdx.x / blocks_per_head;
    const int e = (blockIdx.x % blocks_per_head) * kStateThreads + threadIdx.x;
    if (e >= R4) return;
    const int nsub = (nseg - 1) * ratio;
    const float4* src = reinterpret_cast<const float4*>(sub) + h * size_t(nsub) * R4 + e;
    float4* dst = reinterpret_cast<float4*>(starts) + h * size_t(nseg) * R4 + e;
    float4 run = init ? reinterpret_cast<const float4*>(init)[h * size_t(R4) + e]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < nseg; ++p) {
        dst[size_t(p) * R4] = run;
        if (p + 1 == nseg) break;
        for (int s0 = p * ratio; s0 < (p + 1) * ratio; s0 += kStateBatch) {
            const int n = min(kStateBatch, (p + 1) * ratio - s0);
            float4 x[kStateBatch];
            load_batch(src, s0, 1, n, R4, x);
#pragma unroll
            for (int i = 0; i < kStateBatch; ++i)
                if (i < n) run = f4add(run, x[i]);
        }
    }
}

// rec[h][p] <- init[h] + sum_{p' > p} rec[h][p'] (exclusive suffix, in
// place; init null = zero).
__global__ void __launch_bounds__(kStateThreads)
state_exclusive_rscan_kernel(float* __restrict__ rec, int nseg, int R4, int blocks_per_head,
                             const float* __restrict__ init) {
    const size_t h = blockIdx.x / blocks_per_head;
    const int e = (blockIdx.x % blocks_per_head) * kStateThreads + threadIdx.x;
    if (e >= R4) return;
    float4* base = reinterpret_cast<float4*>(rec) + h * size_t(nseg) * R4 + e;
    float4 run = init ? reinterpret_cast<const float4*>(init)[h * size_t(R4) + e]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = nseg - 1; p0 >= 0; p0 -= kStateBatch) {
        const int n = min(kStateBatch, p0 + 1);
        float4 x[kStateBatch];
        load_batch(base, p0, -1, n, R4, x);
#pragma unroll
        for (int i = 0; i < kStateBatch; ++i)
            if (i < n) {
                base[size_t(p0 - i) * R4] = run;
                run = f4add(run, x[i]);
            }
    }
}

// out[h] <- sum_p rec[h][p]; out record stride R.
__global__ void __launch_bounds__(kStateThreads)
state_sum_kernel(const float* __restrict__ rec, float* __restrict__ out, int nseg, int R4,
                 int blocks_per_head) {
    const size_t h = blockIdx.x / blocks_per_head;
    const int e = (blockIdx.x % blocks_per_head) * kStateThreads + threadIdx.x;
    if (e >= R4) return;
    const float4* base = reinterpret_cast<const float4*>(rec) + h * size_t(nseg) * R4 + e;
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < nseg; p0 += kStateBatch) {
        const int n = min(kStateBatch, nseg - p0);
        float4 x[kStateBatch];
        load_batch(base, p0, 1, n, R4, x);
#pragma unroll
        for (int i = 0; i < kStateBatch; ++i)
            if (i < n) run = f4add(run, x[i]);
    }
    reinterpret_cast<float4*>(out)[h * size_t(R4) + e] = run;
}

// out[h] <- sum_{lo <= p < hi} recs[p][h] for records laid out [P][heads][R]
// (one block of records per rank, in rank order, as an all-gather leaves
// them), added in increasing p; lo >= hi gives zero.  The state a rank of a
// sequence split across ranks starts from is the sum over the ranks before
// it (causal) or over all ranks (non-causal); the suffix over the ranks
// after it is the backward's.
__global__ void __launch_bounds__(kStateThreads)
state_range_sum_kernel(const float* __restrict__ recs, float* __restrict__ out, int lo, int hi,
                       int64_t heads, int R4, int blocks_per_head) {
    const size_t h = blockIdx.x / blocks_per_head;
    const int e = (blockIdx.x % blocks_per_head) * kStateThreads + threadIdx.x;
    if (e >= R4) return;
    const size_t stride = size_t(heads) * size_t(R4);
    const float4* base = reinterpret_cast<const float4*>(recs) + h * size_t(R4) + e;
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = lo; p0 < hi; p0 += kStateBatch) {
        const int n = min(kStateBatch, hi - p0);
        float4 x[kStateBatch];
#pragma unroll
        for (int i = 0; i < kStateBatch; ++i)
            if (i < n) x[i] = base[size_t(p0 + i) * stride];
#pragma unroll
        for (int i = 0; i < kStateBatch; ++i)
            if (i < n) run = f4add(run, x[i]);
    }
    reinterpret_cast<float4*>(out)[h * size_t(R4) + e] = run;
}

// Split records into the caller's S [h][D][D] and z [h][D] arrays; output
// h takes record h * rec_step (with grouped key/value heads the records are
// per query head and every group's first one holds the key/value head's
// state).
__global__ void __launch_bounds__(kStateThreads)
state_unpack_kernel(const float* __restrict__ rec, float* __restrict__ S, float* __restrict__ z,
                    int D, int blocks_per_head, int rec_step) {
    const size_t h = blockIdx.x / blocks_per_head;
    const int R = D * D + D;
    const int e = (blockIdx.x % blocks_per_head) * kStateThreads + threadIdx.x;
    if (e >= R) return;
    const float x = rec[h * size_t(rec_step) * size_t(R) + e];
    if (e < D * D) {
        if (S) S[h * size_t(D) * D + e] = x;
    } else if (z) {
        z[h * size_t(D) + (e - D * D)] = x;
    }
}

// out[h][e] <- sum_{g < G} part[h*G + g][e] for the n elements of each head:
// the float32 per-query-head dK, dV of a key/value head's group, added in a
// fixed order and rounded once to the output type.  Four elements per
// thread (n is a multiple of 4: n = N*D with D a multiple of 16).
template <typename T>
__global__ void __launch_bounds__(256)
group_sum_kernel(const float* __restrict__ part, T* __restrict__ out, int64_t n, int G,
                 int64_t total4) {
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    const int64_t n4 = n / 4;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total4; i += stride) {
        const int64_t h = i / n4, e = i % n4;
        const float4* src = reinterpret_cast<const float4*>(part) + h * G * n4 + e;
        float4 acc = __ldcs(src);
        for (int g = 1; g < G; ++g) {
            const float4 x = __ldcs(src + g * n4);
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        T* dst = out + 4 * i;
        dst[0] = from_f32<T>(acc.x);
        dst[1] = from_f32<T>(acc.y);
        dst[2] = from_f32<T>(acc.z);
        dst[3] = from_f32<T>(acc.w);
    }
}

}  // namespace la
