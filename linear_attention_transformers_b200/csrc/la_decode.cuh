// la_decode.cuh — one recurrent decode step, in place, for every (b, h):
//     S += phi(k) v^T,  z += phi(k),  o = S^T phi(q) / (phi(q) . z)
// ("Efficient Transformers Survey", Proposition "Linear Attention via Kernel
// Decomposition", "Why It Matters": S and z updated token by token with
// constant memory per step).  With a decay factor gamma per head (DecayArg)
// the step is S = gamma S + phi(k) v^T, z = gamma z + phi(k); gamma = 1
// gives bitwise the undecayed step.
//
// The step is a single streaming pass over the float32 state: each S element
// is read once and written once (8 bytes per element), so the kernel is HBM
// bound.  One thread block per head; 2*D threads; thread (rg, cg) owns
// columns 4*cg..4*cg+3 (one 16-byte vector) of rows rg, rg+8, ..., so a warp
// reads whole 128-byte segments.  All of a thread's loads are issued before
// any arithmetic so a block keeps D*D*4 bytes in flight; loads and stores
// use the streaming cache hint because the state is not reused within the
// step.  The partial numerators of the 8 row groups are summed through
// shared memory in a fixed order (deterministic).
#pragma once

#include "la_common.cuh"

namespace la {

template <typename T, int PHI, int D>
__global__ void __launch_bounds__(2 * D)
decode_step_kernel(float* __restrict__ S, float* __restrict__ z,
                   const T* __restrict__ q, const T* __restrict__ k,
                   const T* __restrict__ v, T* __restrict__ o, const DecayArg dec) {
    constexpr int CG = D / 4;    // 16-byte column groups
    constexpr int RG = 8;        // row groups
    constexpr int RPT = D / RG;  // rows per thread
    constexpr int NT = 2 * D;
    constexpr bool kExact = sizeof(T) == sizeof(float);
    static_assert(CG * RG == NT, "thread layout");
    __shared__ float a_s[D], b_s[D];
    __shared__ float4 v_s4[CG];
    __shared__ float4 part[RG][CG];
    __shared__ float den_part[NT / 32];

    const size_t h = blockIdx.x;
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float4* Sh = reinterpret_cast<float4*>(S + h * D * D);
    const float gm = decay_of(dec, h);

    // Issue the state loads first; the vectors arrive while they are in flight.
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) s[r] = __ldcs(Sh + (rg + RG * r) * CG + cg);

    float znew = 0.f;
    if (tid < D) {
        // float32 tensors take libm's expf, as the float32 forward and
        // backward do; bf16 ones the base-2 form (rounded away right after)
        const float xq = to_f32(q[h * D + tid]), xk = to_f32(k[h * D + tid]);
        const float af = kExact ? phi_exact<PHI>(xq) : phi_fast<PHI>(xq);
        const float bf = kExact ? phi_exact<PHI>(xk) : phi_fast<PHI>(xk);
        a_s[tid] = af;
        b_s[tid] = bf;
        reinterpret_cast<float*>(v_s4)[tid] = to_f32(v[h * D + tid]);
        znew = fmaf(gm, z[h * D + tid], bf);
        z[h * D + tid] = znew;
        znew *= af;  // this thread's term of phi(q) . z
    }
    const float wsum = warp_sum(znew);
    if ((tid & 31) == 0) den_part[tid >> 5] = wsum;
    __syncthreads();

    const float4 vv = v_s4[cg];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int f = rg + RG * r;
        const float bf = b_s[f], af = a_s[f];
        float4 x = s[r];
        x.x = fmaf(bf, vv.x, gm * x.x);
        x.y = fmaf(bf, vv.y, gm * x.y);
        x.z = fmaf(bf, vv.z, gm * x.z);
        x.w = fmaf(bf, vv.w, gm * x.w);
        __stcs(Sh + f * CG + cg, x);
        acc.x = fmaf(af, x.x, acc.x);
        acc.y = fmaf(af, x.y, acc.y);
        acc.z = fmaf(af, x.z, acc.z);
        acc.w = fmaf(af, x.w, acc.w);
    }
    part[rg][cg] = acc;
    __syncthreads();
    if (tid < D) {
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) den += den_part[w];
        const float* pf = reinterpret_cast<const float*>(&part[0][0]);
        float num = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) num += pf[g * D + tid];
        o[h * D + tid] = from_f32<T>(num / den);
    }
}

// The same step with G query heads per key/value head (grouped-query or
// multi-query attention, "Attention Optimization", Advanced Techniques): one
// block per key/value head updates its state once, S += phi(k) v^T and
// z += phi(k), then answers the group's G queries from the updated state,
// o_h = S^T phi(q_h) / (phi(q_h) . z).  The state, the step's dominant
// traffic, is read and written once per group instead of once per query
// head.  Queries are taken QB at a time with the updated state slice kept
// in registers.
template <typename T, int PHI, int D>
__global__ void __launch_bounds__(2 * D)
decode_step_gqa_kernel(float* __restrict__ S, float* __restrict__ z,
                       const T* __restrict__ q, const T* __restrict__ k,
                       const T* __restrict__ v, T* __restrict__ o, int G) {
    constexpr int CG = D / 4;
    constexpr int RG = 8;
    constexpr int RPT = D / RG;
    constexpr int NT = 2 * D;
    constexpr int QB = 4;
    constexpr bool kExact = sizeof(T) == sizeof(float);
    static_assert(CG * RG == NT, "thread layout");
    __shared__ float a_s[QB][D], b_s[D], z_s[D];
    __shared__ float4 v_s4[CG];
    __shared__ float4 part[QB][RG][CG];
    __shared__ float den_s[QB];

    const size_t hk = blockIdx.x;  // key/value head
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float4* Sh = reinterpret_cast<float4*>(S + hk * D * D);

    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) s[r] = __ldcs(Sh + (rg + RG * r) * CG + cg);
    // the queries of batch g0 (QB of them), loaded one batch ahead so that
    // their latency hides behind the state loads and the previous batch
    float xq[QB];
    auto load_q = [&](int g0) {
        if (tid < D) {
#pragma unroll
            for (int i = 0; i < QB; ++i)
                xq[i] = g0 + i < G ? to_f32(q[(hk * G + g0 + i) * D + tid]) : 0.f;
        }
    };
    load_q(0);
    if (tid < D) {
        const float xk = to_f32(k[hk * D + tid]);
        const float bf = kExact ? phi_exact<PHI>(xk) : phi_fast<PHI>(xk);
        b_s[tid] = bf;
        reinterpret_cast<float*>(v_s4)[tid] = to_f32(v[hk * D + tid]);
        const float zn = z[hk * D + tid] + bf;
        z[hk * D + tid] = zn;
        z_s[tid] = zn;
    }
    __syncthreads();
    const float4 vv = v_s4[cg];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int f = rg + RG * r;
        const float bf = b_s[f];
        float4 x = s[r];
        x.x = fmaf(bf, vv.x, x.x);
        x.y = fmaf(bf, vv.y, x.y);
        x.z = fmaf(bf, vv.z, x.z);
        x.w = fmaf(bf, vv.w, x.w);
        __stcs(Sh + f * CG + cg, x);
        s[r] = x;
    }
    for (int g0 = 0; g0 < G; g0 += QB) {
        const int nq = min(QB, G - g0);
        __syncthreads();  // a_s, part, den_s of the previous batch are consumed
        if (tid < D) {
#pragma unroll
            for (int i = 0; i < QB; ++i)
                if (i < nq) a_s[i][tid] = kExact ? phi_exact<PHI>(xq[i]) : phi_fast<PHI>(xq[i]);
        }
        if (g0 + QB < G) load_q(g0 + QB);
        __syncthreads();
        // denominators phi(q) . z, query i by warp i mod (warps), fixed order
        for (int i = tid >> 5; i < nq; i += NT / 32) {
            const int l = tid & 31;
            float d = 0.f;
            for (int f = l; f < D; f += 32) d = fmaf(a_s[i][f], z_s[f], d);
            d = warp_sum(d);
            if (l == 0) den_s[i] = d;
        }
        for (int i = 0; i < nq; ++i) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float af = a_s[i][rg + RG * r];
                acc.x = fmaf(af, s[r].x, acc.x);
                acc.y = fmaf(af, s[r].y, acc.y);
                acc.z = fmaf(af, s[r].z, acc.z);
                acc.w = fmaf(af, s[r].w, acc.w);
            }
            part[i][rg][cg] = acc;
        }
        __syncthreads();
        if (tid < D) {
            const float* pf = reinterpret_cast<const float*>(&part[0][0][0]);
            for (int i = 0; i < nq; ++i) {
                float num = 0.f;
#pragma unroll
                for (int gr = 0; gr < RG; ++gr) num += pf[(i * RG + gr) * D + tid];
                o[(hk * G + g0 + i) * D + tid] = from_f32<T>(num / den_s[i]);
            }
        }
    }
}

}  // namespace la
