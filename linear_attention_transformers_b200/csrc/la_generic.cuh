// la_generic.cuh — token-sequential kernels that serve every dtype and head
// size (D <= 128): the float32 path, and the path for shapes the tensor-core
// kernels do not take.  One thread block per (b, h); the running state lives
// in shared memory and is updated one token at a time, which is the
// recurrent form of "Efficient Transformers Survey", Proposition "Linear
// Attention via Kernel Decomposition" ("Why It Matters": S and z updated
// incrementally).  Accumulation is float32 with libm expf in phi.
#pragma once

#include "la_common.cuh"

namespace la {

constexpr int kGenericThreads = 128;

__host__ __device__ inline size_t generic_smem_bytes(int D) {
    // state (D*D) + z (D) + four D-vectors + reduction scratch (32)
    return (size_t(D) * D + 5 * size_t(D) + 32) * sizeof(float);
}

__device__ __forceinline__ float block_sum_128(float x, float* red) {
    x = warp_sum(x);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = x;
    __syncthreads();
    return red[0] + red[1] + red[2] + red[3];
}

// Forward.  S_out/z_out (nullable) receive the state after all N tokens.
template <typename T, int PHI>
__global__ void __launch_bounds__(kGenericThreads)
fwd_generic_kernel(const T* __restrict__ q, const T* __restrict__ k,
                   const T* __restrict__ v, T* __restrict__ o,
                   float* __restrict__ S_out, float* __restrict__ z_out,
                   float* __restrict__ g_out, int N, int D, int causal, int G,
                   const DecayArg dec) {
    extern __shared__ float sm[];
    float* S = sm;
    float* z = S + D * D;
    float* a = z + D;
    float* b = a + D;
    float* vv = b + D;
    const int tid = threadIdx.x, nt = blockDim.x;
    const size_t head = blockIdx.x;
    const size_t base = head * size_t(N) * D;
    const size_t kvh = head / size_t(G);  // key/value head of this query head
    const T* qh = q + base;
    const T* kh = k + kvh * size_t(N) * D;
    const T* vh = v + kvh * size_t(N) * D;
    T* oh = o + base;
    const float gm = decay_of(dec, head);  // causal only: scales the state per token

    for (int t = tid; t < D * D; t += nt) S[t] = 0.f;
    for (int t = tid; t < D; t += nt) z[t] = 0.f;
    __syncthreads();

    if (!causal) {
        for (int j = 0; j < N; ++j) {
            for (int t = tid; t < D; t += nt) {
                b[t] = phi_exact<PHI>(to_f32(kh[size_t(j) * D + t]));
                vv[t] = to_f32(vh[size_t(j) * D + t]);
            }
            __syncthreads();
            for (int t = tid; t < D * D; t += nt) S[t] = fmaf(b[t / D], vv[t % D], S[t]);
            for (int t = tid; t < D; t += nt) z[t] += b[t];
            __syncthreads();
        }
    }
    for (int i = 0; i < N; ++i) {
        const size_t row = size_t(i) * D;
        for (int t = tid; t < D; t += nt) {
            a[t] = phi_exact<PHI>(to_f32(qh[row + t]));
            if (causal) {
                b[t] = phi_exact<PHI>(to_f32(kh[row + t]));
                vv[t] = to_f32(vh[row + t]);
            }
        }
        __syncthreads();
        if (causal) {
            for (int t = tid; t < D * D; t += nt) S[t] = fmaf(b[t / D], vv[t % D], gm * S[t]);
            for (int t = tid; t < D; t += nt) z[t] = fmaf(gm, z[t], b[t]);
            __syncthreads();
        }
        for (int e = tid; e < D; e += nt) {
            float num = 0.f, den = 0.f;
            for (int f = 0; f < D; ++f) {
                num = fmaf(a[f], S[f * D + e], num);
                den = fmaf(a[f], z[f], den);
            }
            oh[row + e] = from_f32<T>(num / den);
            if (g_out && e == 0) g_out[head * size_t(N) + i] = den;
        }
        __syncthreads();
    }
    // the state belongs to the key/value head: its group's first query head
    // writes it
    if (head % G == 0) {
        if (S_out)
            for (int t = tid; t < D * D; t += nt) S_out[kvh * D * D + t] = S[t];
        if (z_out)
            for (int t = tid; t < D; t += nt) z_out[kvh * D + t] = z[t];
    }
}

// Backward of sum(dO * O).  Sweep 1 (token order) rebuilds the forward
// state, forms g_i = a_i.z_i, o_i, du_i = dO_i/g_i, dg_i = -(dO_i.o_i)/g_i and
// dQ_i = (S_i du_i + z_i dg_i) * phi'(q_i), saving g and dg.  Sweep 2
// (reverse order) accumulates R = sum a_i du_i^T and r = sum a_i dg_i over
// the queries that see key j: dK_j = (R v_j + r) * phi'(k_j), dV_j = R^T b_j.
// TO: the dK, dV element type (float for per-query-head partials that the
// caller sums over a key/value group before rounding).
template <typename T, int PHI, typename TO = T>
__global__ void __launch_bounds__(kGenericThreads)
bwd_generic_kernel(const T* __restrict__ q, const T* __restrict__ k,
                   const T* __restrict__ v, const T* __restrict__ dO,
                   T* __restrict__ dq, TO* __restrict__ dk, TO* __restrict__ dv,
                   float* __restrict__ gbuf, float* __restrict__ dgbuf,
                   int N, int D, int causal, int G, const DecayArg dec) {
    extern __shared__ float sm[];
    float* M = sm;            // S in sweep 1, R in sweep 2
    float* zr = M + D * D;    // z in sweep 1, r in sweep 2
    float* a = zr + D;
    float* b = a + D;
    float* vv = b + D;
    float* du = vv + D;
    float* red = du + D;
    const int tid = threadIdx.x, nt = blockDim.x;
    const size_t head = blockIdx.x;
    const size_t base = head * size_t(N) * D;
    // k, v of the query head's group; dK, dV are written per query head
    const size_t kvbase = (head / size_t(G)) * size_t(N) * D;
    const T *qh = q + base, *kh = k + kvbase, *vh = v + kvbase, *gh = dO + base;
    T* dqh = dq + base;
    TO *dkh = dk + base, *dvh = dv + base;
    float* gb = gbuf + head * size_t(N);
    float* dgb = dgbuf + head * size_t(N);
    // decay (causal only): the prefix state S, z and the suffix sums R, r
    // are scaled by gamma per token
    const float gm = decay_of(dec, head);

    // ---------------- sweep 1
    for (int t = tid; t < D * D; t += nt) M[t] = 0.f;
    for (int t = tid; t < D; t += nt) zr[t] = 0.f;
    __syncthreads();
    if (!causal) {
        for (int j = 0; j < N; ++j) {
            for (int t = tid; t < D; t += nt) {
                b[t] = phi_exact<PHI>(to_f32(kh[size_t(j) * D + t]));
                vv[t] = to_f32(vh[size_t(j) * D + t]);
            }
            __syncthreads();
            for (int t = tid; t < D * D; t += nt) M[t] = fmaf(b[t / D], vv[t % D], M[t]);
            for (int t = tid; t < D; t += nt) zr[t] += b[t];
            __syncthreads();
        }
    }
    for (int i = 0; i < N; ++i) {
        const size_t row = size_t(i) * D;
        for (int t = tid; t < D; t += nt) {
            a[t] = phi_exact<PHI>(to_f32(qh[row + t]));
            du[t] = to_f32(gh[row + t]);
            if (causal) {
                b[t] = phi_exact<PHI>(to_f32(kh[row + t]));
                vv[t] = to_f32(vh[row + t]);
            }
        }
        __syncthreads();
        if (causal) {
            for (int t = tid; t < D * D; t += nt) M[t] = fmaf(b[t / D], vv[t % D], gm * M[t]);
            for (int t = tid; t < D; t += nt) zr[t] = fmaf(gm, zr[t], b[t]);
            __syncthreads();
        }
        float g = 0.f;
        for (int f = 0; f < D; ++f) g = fmaf(a[f], zr[f], g);
        float part = 0.f;
        for (int e = tid; e < D; e += nt) {
            float u = 0.f;
            for (int f = 0; f < D; ++f) u = fmaf(a[f], M[f * D + e], u);
            part = fmaf(du[e], u / g, part);
        }
        const float dot = block_sum_128(part, red);
        const float dg = -dot / g;
        for (int e = tid; e < D; e += nt) du[e] = du[e] / g;
        __syncthreads();
        for (int f = tid; f < D; f += nt) {
            float da = zr[f] * dg;
            for (int e = 0; e < D; ++e) da = fmaf(M[f * D + e], du[e], da);
            dqh[row + f] = from_f32<T>(da * dphi_exact<PHI>(to_f32(qh[row + f])));
        }
        if (tid == 0) {
            gb[i] = g;
            dgb[i] = dg;
        }
        __syncthreads();
    }

    // ---------------- sweep 2
    for (int t = tid; t < D * D; t += nt) M[t] = 0.f;
    for (int t = tid; t < D; t += nt) zr[t] = 0.f;
    __syncthreads();
    if (!causal) {
        for (int i = 0; i < N; ++i) {
            const size_t row = size_t(i) * D;
            const float g = gb[i];
            const float dg = dgb[i];
            for (int t = tid; t < D; t += nt) {
                a[t] = phi_exact<PHI>(to_f32(qh[row + t]));
                du[t] = to_f32(gh[row + t]) / g;
            }
            __syncthreads();
            for (int t = tid; t < D * D; t += nt) M[t] = fmaf(a[t / D], du[t % D], M[t]);
            for (int t = tid; t < D; t += nt) zr[t] = fmaf(a[t], dg, zr[t]);
            __syncthreads();
        }
    }
    for (int j = N - 1; j >= 0; --j) {
        const size_t row = size_t(j) * D;
        const float g = gb[j];
        const float dg = dgb[j];
        for (int t = tid; t < D; t += nt) {
            b[t] = phi_exact<PHI>(to_f32(kh[row + t]));
            vv[t] = to_f32(vh[row + t]);
            if (causal) {
                a[t] = phi_exact<PHI>(to_f32(qh[row + t]));
                du[t] = to_f32(gh[row + t]) / g;
            }
        }
        __syncthreads();
        if (causal) {
            for (int t = tid; t < D * D; t += nt) M[t] = fmaf(a[t / D], du[t % D], gm * M[t]);
            for (int t = tid; t < D; t += nt) zr[t] = fmaf(a[t], dg, gm * zr[t]);
            __syncthreads();
        }
        for (int f = tid; f < D; f += nt) {
            float db = zr[f];
            for (int e = 0; e < D; ++e) db = fmaf(M[f * D + e], vv[e], db);
            dkh[row + f] = from_f32<TO>(db * dphi_exact<PHI>(to_f32(kh[row + f])));
        }
        for (int e = tid; e < D; e += nt) {
            float acc = 0.f;
            for (int f = 0; f < D; ++f) acc = fmaf(M[f * D + e], b[f], acc);
            dvh[row + e] = from_f32<TO>(acc);
        }
        __syncthreads();
    }
}

}  // namespace la
