// la_favor.cuh — the Performer's positive random features (FAVOR+) and their
// gradient ("Efficient Transformers Survey", Low-Rank Approximations,
// Performer):
//
//     phi(x) = m^-1/2 exp(-|x|^2 / 2) [exp(w_1^T x), ..., exp(w_m^T x)]
//
// for rows x of q or k (pre-normalised by the caller) and the m random
// directions w_i (rows of omega [m][D], drawn by the caller).  The features
// then go through the linear-attention kernels as already-mapped inputs
// (PHI_IDENTITY).  The gradient of sum(dphi * phi) is
//
//     dx = sum_i dphi_i phi_i w_i - x sum_i dphi_i phi_i = G omega - x s,
//
// G = dphi * phi (elementwise), s its row sum.
//
// Forward: per 128-row tile one tensor-core product P = X W^T ([128 x D] x
// [D x m], exact in fp32 for bf16 inputs) and the epilogue exp(P - |x|^2/2 -
// ln(m)/2), rounded to bf16 once.  Backward: the same product recomputes
// phi in fp32 (no stored features are read, and none of their rounding
// enters dx), G is formed in fp32 and split into two bf16 parts G_hi + G_lo
// (each rounded once), and G_hi W + G_lo W accumulate in TMEM; the epilogue
// subtracts x s.  The MMAs are nearly free: the kernels do 2 D m / (D + m)
// flops per byte moved (32 to 64), a tenth of the tensor cores' balance
// point, so they run at the speed of HBM.  tcgen05 MMAs with TMEM
// accumulators (two buffers), TMA-fed stages, omega held in shared memory
// for the whole persistent kernel, one CTA per SM looping over the 128-row
// tiles of every head.  D and m are each 64 or 128.
#pragma once

#include "la_chunk_bwd.cuh"

namespace la {

struct FavorParams {
    CUtensorMap tm_x;     // x [heads][N][D] bf16, box (64, 128, 1)
    CUtensorMap tm_w;     // omega [1][m][D] bf16, box (64, m, 1)
    CUtensorMap tm_phi;   // forward: phi [heads][N][m] (output)
    CUtensorMap tm_dphi;  // backward: dphi [heads][N][m]
    CUtensorMap tm_dx;    // backward: dx [heads][N][D] (output)
    int tiles_per_head;   // ceil(N / 128)
    int ntiles;           // heads * tiles_per_head
    float log_scale;      // -ln(m) / 2
};

// Head size D, M = m features.  Forward: per stage one x tile [128][D] and
// the output [128][M], staged over x when M <= D (once each row's |x|^2 is
// read), else in its own tile.  Backward: per stage the x tile and two
// [128][M] tiles: G_hi is formed over dphi, G_lo in the third tile; dx is
// staged over x (each thread reads its row's x before it writes that row).
// TMEM: per buffer b the product P (M columns) and, backward, the dx
// accumulator (D columns).
template <int D, int M, bool BWD>
struct FavorCfg {
    static constexpr int R = 128;
    static constexpr int NS = BWD ? 2 : 3;
    static constexpr int XT = R * D * 2;                 // x / dx tile
    static constexpr int PT = R * M * 2;                 // phi / dphi / G tile
    static constexpr int OFF_OUT = (!BWD && M > D) ? XT : 0;  // forward output staging
    static constexpr int STAGE = BWD ? XT + 2 * PT : XT + (M > D ? PT : 0);
    static constexpr int OFF_W = NS * STAGE;            // omega [M][D] row tile
    static constexpr int OFF_S = OFF_W + M * D * 2;     // backward: row sums s [NS][R] float
    static constexpr int OFF_BAR = OFF_S + (BWD ? NS * R * 4 : 0);
    static constexpr int NBAR = 4 * NS + 7;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int ACC = BWD ? M + D : M;  // TMEM columns per buffer
    static constexpr int T_COLS = 2 * ACC <= 128 ? 128 : (2 * ACC <= 256 ? 256 : 512);
    static constexpr int THREADS = BWD ? 320 : 192;
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(2 * ACC <= 512, "TMEM budget");
};

template <int D, int M, bool BWD>
__global__ void __launch_bounds__(FavorCfg<D, M, BWD>::THREADS, 1)
favor_kernel(const __grid_constant__ FavorParams prm) {
    using namespace sm100;
    using Cfg = FavorCfg<D, M, BWD>;
    constexpr int R = Cfg::R, NS = Cfg::NS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;               // [NS] TMA landed                   (1 + tx)
    uint64_t* prep = bars + NS;          // [NS] backward: G, s formed        (128)
    uint64_t* empty = bars + 2 * NS;     // [NS] MMAs + store done            (2)
    uint64_t* acc_full = bars + 3 * NS;  // [2] output accumulator complete   (commit)
    uint64_t* acc_free = acc_full + 2;   // [2] output accumulator read       (128)
    uint64_t* p_full = acc_full + 4;     // [2] backward: P = X W^T complete  (commit)
    uint64_t* w_full = acc_full + 6;     // omega landed                      (1 + tx)
    uint64_t* drain = w_full + 1;        // every MMA finished                (commit)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
    float* srow = reinterpret_cast<float*>(smem + Cfg::OFF_S);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // tiles of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
    const int my_tiles = prm.ntiles > int(blockIdx.x)
                             ? (prm.ntiles - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x)
                             : 0;
    auto tile_of = [&](int i) { return int(blockIdx.x) + i * int(gridDim.x); };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&prep[s], 128);
            mbar_init(&empty[s], 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_free[b], 128);
            mbar_init(&p_full[b], 1);
        }
        mbar_init(w_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::T_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&prm.tm_x);
            tma_prefetch_desc(&prm.tm_w);
            if (BWD) tma_prefetch_desc(&prm.tm_dphi);
            mbar_arrive_expect_tx(w_full, uint32_t(M * D * 2));
#pragma unroll
            for (int a = 0; a < D / 64; ++a)
                tma_load_3d(smem + Cfg::OFF_W + a * M * 128, &prm.tm_w, w_full, a * 64, 0, 0);
            constexpr uint32_t bytes = uint32_t(BWD ? Cfg::XT + Cfg::PT : Cfg::XT);
            int issued = 0;
            for (int i = 0; i < my_tiles; ++i) {
                const int s = i % NS;
                if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1, abort_flag)) break;
                const int t = tile_of(i);
                const int head = t / prm.tiles_per_head, row0 = (t % prm.tiles_per_head) * R;
                uint8_t* st = smem + s * Cfg::STAGE;
                mbar_arrive_expect_tx(&full[s], bytes);
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tma_load_3d(st + a * R * 128, &prm.tm_x, &full[s], a * 64, row0, head);
                if (BWD) {
#pragma unroll
                    for (int a = 0; a < M / 64; ++a)
                        tma_load_3d(st + Cfg::XT + a * R * 128, &prm.tm_dphi, &full[s], a * 64,
                                    row0, head);
                }
                issued = i + 1;
            }
            for (int i = max(0, issued - NS); i < issued; ++i)
                mbar_wait_drain(&full[i % NS], (i / NS) & 1);
            mbar_wait_drain(w_full, 0);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idP = idesc_bf16(R, M, 0, 0);  // X W^T (K = D, both K-major)
            constexpr uint32_t idG = idesc_bf16(R, D, 0, 1);  // G W (W MN-major: rows = m = K)
            const uint32_t wt = sbase + Cfg::OFF_W;
            const uint64_t wk = desc_k_base(wt), wm = desc_mn_base(wt, M);
            bool ok = mbar_wait(w_full, 0, abort_flag);
            for (int i = 0; ok && i < my_tiles; ++i) {
                const int s = i % NS, b = i & 1;
                const uint32_t st = sbase + s * Cfg::STAGE;
                const uint32_t accP = tmem + uint32_t(b * Cfg::ACC);  // P (forward: the output)
                if (!(ok = mbar_wait(&full[s], (i / NS) & 1, abort_flag))) break;
                // forward: the buffer's previous output read; backward: its
                // previous P was read before that tile's G was formed (prep)
                if (!BWD && i >= 2 &&
                    !(ok = mbar_wait(&acc_free[b], ((i >> 1) - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                const uint64_t xa = desc_k_base(st);
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(accP, xa + kstep_k(R, k), wk + kstep_k(M, k), idP, k > 0);
                if constexpr (BWD) {
                    umma_commit(&p_full[b]);
                    if (!(ok = mbar_wait(&prep[s], (i / NS) & 1, abort_flag))) break;
                    if (i >= 2 && !(ok = mbar_wait(&acc_free[b], ((i >> 1) - 1) & 1, abort_flag)))
                        break;
                    tc_fence_after();
                    const uint32_t accG = accP + uint32_t(M);
                    const uint64_t gh = desc_k_base(st + Cfg::XT);            // G_hi
                    const uint64_t gl = desc_k_base(st + Cfg::XT + Cfg::PT);  // G_lo
#pragma unroll
                    for (int k = 0; k < M; k += 16)
                        umma_bf16(accG, gh + kstep_k(R, k), wm + kstep_mn(k), idG, k > 0);
#pragma unroll
                    for (int k = 0; k < M; k += 16)
                        umma_bf16(accG, gl + kstep_k(R, k), wm + kstep_mn(k), idG, 1u);
                }
                umma_commit(&acc_full[b]);
                umma_commit(&empty[s]);
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (BWD && warp < 6) {
        // ------- backward prep: phi (fp32) from P, G = dphi * phi -> hi, lo, s
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int r = 32 * sp + lane;  // tile row = accumulator lane
        for (int i = 0; i < my_tiles; ++i) {
            const int s = i % NS, b = i & 1;
            // the stage's tiles (read here directly) and this tile's P
            if (!mbar_wait(&full[s], (i / NS) & 1, abort_flag)) break;
            if (!mbar_wait(&p_full[b], (i >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint8_t* xt = smem + s * Cfg::STAGE;
            uint8_t* gt = smem + s * Cfg::STAGE + Cfg::XT;             // dphi -> G_hi
            uint8_t* lt = smem + s * Cfg::STAGE + Cfg::XT + Cfg::PT;   // G_lo
            float hsq = 0.f;
#pragma unroll 4
            for (int q = 0; q < D / 8; ++q) {
                float x8[8];
                load_chunk8(xt, R, r, q, x8);
#pragma unroll
                for (int j = 0; j < 8; ++j) hsq = fmaf(x8[j], x8[j], hsq);
            }
            const float shift = prm.log_scale - 0.5f * hsq;
            const uint32_t accP = tmem + lane_base + uint32_t(b * Cfg::ACC);
            float sum = 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < M; c0 += 32) {
                float pv[32];
                tmem_load<32>(accP + c0, pv);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4* gp = reinterpret_cast<uint4*>(gt + tile_chunk_off(R, r, (c0 >> 3) + q));
                    const uint4 d4 = *gp;
                    uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w}, lw[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 fd = unpack_bf16(dw[j]);
                        const float g0 = fd.x * exp_fast(pv[8 * q + 2 * j] + shift);
                        const float g1 = fd.y * exp_fast(pv[8 * q + 2 * j + 1] + shift);
                        sum += g0 + g1;
                        const uint32_t hi = pack_bf16(g0, g1);
                        const float2 fh = unpack_bf16(hi);
                        dw[j] = hi;
                        lw[j] = pack_bf16(g0 - fh.x, g1 - fh.y);
                    }
                    *gp = make_uint4(dw[0], dw[1], dw[2], dw[3]);
                    *reinterpret_cast<uint4*>(lt + tile_chunk_off(R, r, (c0 >> 3) + q)) =
                        make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
            srow[s * R + r] = sum;
            tc_fence_before();
            fence_proxy_async_smem();
            mbar_arrive(&prep[s]);
        }
    } else if (warp >= (BWD ? 6 : 2)) {
        // ----------------------------------------------------------- epilogue
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int r = 32 * sp + lane;  // tile row = accumulator lane
        const int e = tid - (BWD ? 192 : 64);
        for (int i = 0; i < my_tiles; ++i) {
            const int s = i % NS, b = i & 1;
            const int t = tile_of(i);
            const int head = t / prm.tiles_per_head, row0 = (t % prm.tiles_per_head) * R;
            if (!named_bar_all(1, 128, mbar_wait(&acc_full[b], (i >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            uint8_t* xt = smem + s * Cfg::STAGE;
            const uint32_t acc = tmem + lane_base + uint32_t(b * Cfg::ACC) + (BWD ? uint32_t(M) : 0u);
            uint8_t* ot = xt + Cfg::OFF_OUT;  // output staging (dx: over x)
            if constexpr (BWD) {
                // dx = G W - x s
                const float sr = srow[s * R + r];
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float v[32];
                    tmem_load<32>(acc + c0, v);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float x8[8];
                        load_chunk8(xt, R, r, (c0 >> 3) + q, x8);
#pragma unroll
                        for (int j = 0; j < 8; ++j) v[8 * q + j] = fmaf(-x8[j], sr, v[8 * q + j]);
                    }
                    store_row_bf16<32>(ot, R, r, c0, v);
                }
            } else {
                // phi = exp(w.x - |x|^2/2 - ln(m)/2), staged over this row of x
                float hsq = 0.f;
#pragma unroll 4
                for (int q = 0; q < D / 8; ++q) {
                    float x8[8];
                    load_chunk8(xt, R, r, q, x8);
#pragma unroll
                    for (int j = 0; j < 8; ++j) hsq = fmaf(x8[j], x8[j], hsq);
                }
                const float shift = prm.log_scale - 0.5f * hsq;
#pragma unroll 1
                for (int c0 = 0; c0 < M; c0 += 32) {
                    float v[32];
                    tmem_load<32>(acc + c0, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = exp_fast(v[j] + shift);
                    store_row_bf16<32>(ot, R, r, c0, v);
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_free[b]);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (e == 0) {
#pragma unroll
                for (int a = 0; a < (BWD ? D : M) / 64; ++a)
                    tma_store_3d(BWD ? &prm.tm_dx : &prm.tm_phi, ot + a * R * 128, a * 64, row0,
                                 head);
                bulk_commit();
                bulk_wait_read0();
                mbar_arrive(&empty[s]);
            }
        }
        if (e == 0) bulk_wait0();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::T_COLS);
}

}  // namespace la
