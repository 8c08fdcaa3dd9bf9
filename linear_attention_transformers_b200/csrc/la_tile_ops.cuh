// la_tile_ops.cuh — elementwise passes over swizzled bf16 row tiles in
// shared memory (see la_sm100.cuh for the layout), shared by the chunked
// kernels.
#pragma once

#include "la_common.cuh"
#include "la_sm100.cuh"

namespace la {

// elu(x)+1 on a pair of bf16 values, to bf16: max(x, 0) + e^min(x, 0),
// with the min/max and the final add on the packed pair (exact for bf16:
// one of the two terms is 0 or, for x > 0, e^0 = 1 and 1 + x is exact in
// fp32 before the add rounds), so only the exponential runs in fp32.  The
// results equal rounding fp32 elu(x)+1 to bf16; about 5 instructions per
// element instead of 6.5.
__device__ __forceinline__ uint32_t phi2_elu1(uint32_t w) {
    uint32_t m, big, r;
    asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(w), "r"(0u));
    asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(big) : "r"(w), "r"(0u));
    const uint32_t e = sm100::pack_bf16(exp_fast(__uint_as_float(m << 16)),
                                        exp_fast(__uint_as_float(m & 0xffff0000u)));
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(e), "r"(big));
    return r;
}

// The same map less its value at 0 minus the x > 0 slope's offset:
// elu(x) = phi(x) - 1 (x for x > 0, exp(x) - 1 otherwise), to bf16.  The
// exponential and the subtraction run in fp32 before the one rounding, so
// the small deviations of phi from 1 keep bf16's relative precision instead
// of being rounded against the 1.
__device__ __forceinline__ uint32_t phi2_elu1_centered(uint32_t w) {
    uint32_t m, big, r;
    asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(w), "r"(0u));
    asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(big) : "r"(w), "r"(0u));
    const uint32_t e = sm100::pack_bf16(exp_fast(__uint_as_float(m << 16)) - 1.f,
                                        exp_fast(__uint_as_float(m & 0xffff0000u)) - 1.f);
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(e), "r"(big));
    return r;
}

// The constant c with phi = c + (a map whose typical values are small): the
// feature vectors of elu(x)+1 on small inputs sit near the all-ones vector,
// so products of them are formed from phi - 1 plus rank-one terms in c;
// relu(x)+1e-6 has no such offset.
template <int PHI>
__host__ __device__ constexpr float phi_center() {
    return PHI == PHI_ELU1 ? 1.f : 0.f;
}

// Apply the feature map in place to a [C][D] bf16 row tile.  The T threads
// calling this split the tile's C*D/8 16-byte chunks evenly; each thread
// loads all of its chunks before it computes so their latencies overlap.
// Rows >= nvalid are written as zero when `zero_tail` (a partial last chunk:
// those keys must not reach the state).  CENTER: write phi - phi_center
// instead (see phi2_elu1_centered).
template <int PHI, int C, int D, int T, bool CENTER = false>
__device__ __forceinline__ void phi_tile(uint8_t* tile, int t, int nvalid, bool zero_tail) {
    using namespace sm100;
    constexpr int CH = D / 8;
    constexpr int PER = (C * CH) / T;
    static_assert(PER >= 1 && (C * CH) % T == 0 && CH % PER == 0, "work split");
    const int first = t * PER;
    const int row = first / CH, q0 = first % CH;
    uint4 x[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i)
        x[i] = *reinterpret_cast<const uint4*>(tile + tile_chunk_off(C, row, q0 + i));
    const bool zero = zero_tail && row >= nvalid;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (PHI == PHI_ELU1) {
                w[k] = zero ? 0u : (CENTER ? phi2_elu1_centered(w[k]) : phi2_elu1(w[k]));
            } else {
                const float2 f = unpack_bf16(w[k]);
                w[k] = zero ? 0u : pack_bf16(phi_fast<PHI>(f.x), phi_fast<PHI>(f.y));
            }
        }
        x[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
        *reinterpret_cast<uint4*>(tile + tile_chunk_off(C, row, q0 + i)) = x[i];
}

// phi_tile for the decayed recurrence: row r of the tile becomes
// phi(x_r) * 2^(lg * (sgn * r + off)), evaluated in fp32 and rounded to bf16
// once.  With lg = log2(gamma) the chunked kernels give query rows the
// factor gamma^(r + 1 - m) and key rows gamma^(m - 1 - r), so that a query
// row times a key row carries gamma^(i - j) (the decay weight between them),
// with every factor within gamma^(+-C/2).  Rows >= nvalid are zero when
// zero_tail.
template <int PHI, int C, int D, int T, bool CENTER = false>
__device__ __forceinline__ void phi_tile_scaled(uint8_t* tile, int t, int nvalid, bool zero_tail,
                                                float lg, float sgn, float off) {
    constexpr float kc = CENTER ? phi_center<PHI>() : 0.f;  // centred: (phi - c) * factor
    using namespace sm100;
    constexpr int CH = D / 8;
    constexpr int PER = (C * CH) / T;
    static_assert(PER >= 1 && (C * CH) % T == 0 && CH % PER == 0, "work split");
    constexpr int GRP = PER > 4 ? 4 : PER;  // 16-byte chunks converted at a time
    const int first = t * PER;
    const int row = first / CH, q0 = first % CH;
    const bool zero = zero_tail && row >= nvalid;
    const float sc = exp2f(lg * fmaf(sgn, float(row), off));
#pragma unroll
    for (int g0 = 0; g0 < PER; g0 += GRP) {
        uint4 x[GRP];
#pragma unroll
        for (int i = 0; i < GRP; ++i)
            x[i] = *reinterpret_cast<const uint4*>(tile + tile_chunk_off(C, row, q0 + g0 + i));
#pragma unroll
        for (int i = 0; i < GRP; ++i) {
            uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = unpack_bf16(w[k]);
                w[k] = zero ? 0u
                            : pack_bf16((phi_fast<PHI>(f.x) - kc) * sc,
                                        (phi_fast<PHI>(f.y) - kc) * sc);
            }
            x[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
#pragma unroll
        for (int i = 0; i < GRP; ++i)
            *reinterpret_cast<uint4*>(tile + tile_chunk_off(C, row, q0 + g0 + i)) = x[i];
    }
}

// Rows of a [C][D] bf16 row tile times 2^(lg * (sgn * r + off)) in place
// (rows >= nvalid become zero): the decay factors of a tile the feature map
// does not touch.  Same work split as phi_tile.
template <int C, int D, int T>
__device__ __forceinline__ void scale_tile_rows_exp2(uint8_t* tile, int t, int nvalid, float lg,
                                                     float sgn, float off) {
    using namespace sm100;
    constexpr int CH = D / 8;
    constexpr int PER = (C * CH) / T;
    static_assert(PER >= 1 && (C * CH) % T == 0 && CH % PER == 0, "work split");
    const int first = t * PER;
    const int row = first / CH, q0 = first % CH;
    uint4 x[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i)
        x[i] = *reinterpret_cast<const uint4*>(tile + tile_chunk_off(C, row, q0 + i));
    const float sc = row < nvalid ? exp2f(lg * fmaf(sgn, float(row), off)) : 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = unpack_bf16(w[k]);
            w[k] = pack_bf16(f.x * sc, f.y * sc);
        }
        x[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
        *reinterpret_cast<uint4*>(tile + tile_chunk_off(C, row, q0 + i)) = x[i];
}

// Sum of row `row` of a [C][D] bf16 row tile (fp32, fixed order).
template <int C, int D>
__device__ __forceinline__ float tile_row_sum(const uint8_t* tile, int row) {
    using namespace sm100;
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
        const uint4 x = *reinterpret_cast<const uint4*>(tile + tile_chunk_off(C, row, q));
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = unpack_bf16(w[k]);
            acc += f.x + f.y;
        }
    }
    return acc;
}

// Scale rows of a [C][D] bf16 row tile in place: row r times rs[r] (rows >=
// nvalid become zero).  Same work split as phi_tile.
template <int C, int D, int T>
__device__ __forceinline__ void scale_tile_rows(uint8_t* tile, int t, int nvalid, const float* rs) {
    using namespace sm100;
    constexpr int CH = D / 8;
    constexpr int PER = (C * CH) / T;
    static_assert(PER >= 1 && (C * CH) % T == 0 && CH % PER == 0, "work split");
    const int first = t * PER;
    const int row = first / CH, q0 = first % CH;
    uint4 x[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i)
        x[i] = *reinterpret_cast<const uint4*>(tile + tile_chunk_off(C, row, q0 + i));
    const float sc = row < nvalid ? rs[row] : 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        uint32_t w[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = unpack_bf16(w[k]);
            w[k] = pack_bf16(f.x * sc, f.y * sc);
        }
        x[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
        *reinterpret_cast<uint4*>(tile + tile_chunk_off(C, row, q0 + i)) = x[i];
}

// Write n x 16 fp32 values of row `row` (columns col0..col0+16n-1) as bf16
// into a row tile with `rows` rows.
template <int NV>
__device__ __forceinline__ void store_row_bf16(uint8_t* tile, int rows, int row, int col0,
                                               const float* v) {
    using namespace sm100;
#pragma unroll
    for (int j = 0; j < NV / 8; ++j) {
        const float* x = v + 8 * j;
        *reinterpret_cast<uint4*>(tile + tile_chunk_off(rows, row, (col0 >> 3) + j)) =
            make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                       pack_bf16(x[6], x[7]));
    }
}

// Row `row` of a float32 state record (rec + row * D, 16-byte aligned; null
// or row < 0 = zeros), times `scale`, into row `row` of the bf16 operand tile
// (rows = D) and, when `to_tmem`, into the TMEM columns from `tm` of this
// thread's lane as float32 (warp-collective then: every lane calls it).  One
// read of the row, 32 columns (eight 16-byte loads in flight) per round trip.
template <int D>
__device__ __forceinline__ void load_record_row(const float* rec, int row, float scale,
                                                uint8_t* tile, uint32_t tm, bool to_tmem) {
    constexpr int W = D < 32 ? D : 32;
    const bool valid = rec != nullptr && row >= 0;
    const float4* src = reinterpret_cast<const float4*>(rec + (valid ? size_t(row) * D : 0));
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += W) {
        float v[W];
#pragma unroll
        for (int j = 0; j < W / 4; ++j) {
            const float4 x = valid ? __ldg(src + c0 / 4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * j] = x.x * scale;
            v[4 * j + 1] = x.y * scale;
            v[4 * j + 2] = x.z * scale;
            v[4 * j + 3] = x.w * scale;
        }
        if (row >= 0) store_row_bf16<W>(tile, D, row, c0, v);
        if (to_tmem) {
#pragma unroll
            for (int h = 0; h < W / 16; ++h) sm100::tmem_st16(tm + c0 + 16 * h, v + 16 * h);
        }
    }
    if (to_tmem) sm100::tmem_wait_st();
}

// Load NV consecutive TMEM columns of this thread's lane (NV multiple of 16).
template <int NV>
__device__ __forceinline__ void tmem_load(uint32_t taddr, float* v) {
#pragma unroll
    for (int j = 0; j < NV / 16; ++j) sm100::tmem_ld16(taddr + 16 * j, v + 16 * j);
    sm100::tmem_wait_ld();
}

}  // namespace la
