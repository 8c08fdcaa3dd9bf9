// la_reduce.cuh — the state record of a token range for head size 128 in a
// compact block: [S | z] = sum_j (phi(k_j) - c) [v_j^T | 1] over the range
// (S and z are sums over tokens, "Efficient Transformers Survey",
// Proposition "Linear Attention via Kernel Decomposition", Statement).
//
// The chunked forward kernel's REDUCE mode computes the same record but
// carries the whole causal pass's shared-memory and TMEM plan (one block per
// SM).  This block holds only what the sum needs: three stages of k and v
// tiles, the [16][C] ones operand for z, 144 TMEM columns (S, then z in
// column 128), so two blocks share an SM and one block's start-up and
// record write-out overlap the other's streaming.  Per 64-token chunk: phi
// (centred when asked) on the k tile in place, then S += B^T V (4 MMAs,
// N = 128) and z += B^T 1 (4 MMAs, N = 16, the ones row of the E operand).
#pragma once

#include "la_chunk_fwd.cuh"

namespace la {

struct Reduce128Cfg {
    static constexpr int D = 128, C = 64;
    static constexpr int NSTAGE = 3;
    static constexpr int ATOM = C * 128;         // [C][64] bf16 = 8 KB
    static constexpr int STAGE = 4 * ATOM;        // k (2 atoms), then v (2 atoms)
    static constexpr int OFF_E = NSTAGE * STAGE;  // [16][C] K-major ones operand, row 0 = 1
    static constexpr int OFF_BAR = OFF_E + 16 * C * 2;
    static constexpr int NBAR = 3 * NSTAGE + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
    static constexpr int T_S = 0, T_Z = D;
    static constexpr int T_COLS = 256;
    static_assert(2 * SMEM <= 227 * 1024, "two blocks per SM");
    static_assert(OFF_E % 1024 == 0, "swizzled tiles on 1 KB");
};

constexpr int kReduce128Threads = 320;  // TMA producer, MMA issuer, 8 feature-map warps (4 read out)

// Grid: heads x prm.nseg blocks; block b sums tokens [seg * seg_len,
// min(N, (seg + 1) * seg_len)) of head b / nseg (its key/value head with
// kv_group) and writes S to prm.S_out + b * stride_S (row f = key feature)
// and z to prm.z_out + b * stride_z.  prm.center: sum phi(k) - phi_center.
template <int PHI>
__global__ void __launch_bounds__(kReduce128Threads, 2)
reduce128_kernel(const __grid_constant__ ChunkParams prm) {
    using namespace sm100;
    using Cfg = Reduce128Cfg;
    constexpr int C = Cfg::C, D = Cfg::D, NS = Cfg::NSTAGE;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;                // TMA landed           (1 + tx)
    uint64_t* phi_done = bars + NS;       // phi applied          (256)
    uint64_t* empty = bars + 2 * NS;      // MMAs done with stage (commit)
    uint64_t* done = bars + 3 * NS;       // every MMA finished   (commit)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x / prm.nseg, seg = blockIdx.x % prm.nseg;
    const int kv_head = kv_head_of(head, prm.kv_group);
    const int tok0 = seg * prm.seg_len;
    const int tok1 = min(prm.N, tok0 + prm.seg_len);
    const int nchunks = (tok1 - tok0 + C - 1) / C;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&phi_done[s], 256);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
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
            tma_prefetch_desc(&prm.tm_k);
            tma_prefetch_desc(&prm.tm_v);
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                if (c >= NS && !mbar_wait(&empty[s], ((c / NS) - 1) & 1, abort_flag)) break;
                uint8_t* st = smem + s * Cfg::STAGE;
                mbar_arrive_expect_tx(&full[s], uint32_t(Cfg::STAGE));
                const int row = tok0 + c * C;
#pragma unroll
                for (int a = 0; a < D / 64; ++a) {
                    tma_load_3d(st + a * Cfg::ATOM, &prm.tm_k, &full[s], a * 64, row, kv_head);
                    tma_load_3d(st + (2 + a) * Cfg::ATOM, &prm.tm_v, &full[s], a * 64, row,
                                kv_head);
                }
                issued = c + 1;
            }
            // never leave the block with copies in flight
            for (int c = max(0, issued - NS); c < issued; ++c)
                mbar_wait_drain(&full[c % NS], (c / NS) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(D, D, 1, 1);   // B^T V, both MN-major
            constexpr uint32_t idZ = idesc_bf16(D, 16, 1, 0);  // B^T E, E K-major
            const uint32_t eop = sbase + Cfg::OFF_E;
            bool ok = true;
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c % NS;
                if (!(ok = mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                tc_fence_after();
                const uint32_t ks = sbase + s * Cfg::STAGE, vs = ks + 2 * Cfg::ATOM;
#pragma unroll
                for (int k = 0; k < C; k += 16) {
                    const uint32_t acc = (c > 0 || k > 0) ? 1u : 0u;
                    umma_bf16(tmem + Cfg::T_S, desc_mnmajor(ks, C, k), desc_mnmajor(vs, C, k),
                              idS, acc);
                    umma_bf16(tmem + Cfg::T_Z, desc_mnmajor(ks, C, k), desc_kmajor(eop, 16, k),
                              idZ, acc);
                }
                umma_commit(&empty[s]);
            }
            // every MMA issued above completes before the readout and the
            // TMEM release (a failed wait still commits, so nothing waits on
            // a phase that never comes)
            umma_commit(done);
        }
    } else {
        // ---------------------- feature map on k, then the record readout
        const int u = tid - 64;  // 0..255
        uint8_t* eop = smem + Cfg::OFF_E;
        for (int idx = u; idx < 16 * C; idx += 256) {
            const int r = idx / C, cc = idx % C;
            *reinterpret_cast<__nv_bfloat16*>(eop + tile_off(16, r, cc)) =
                __float2bfloat16_rn(r == 0 ? 1.f : 0.f);
        }
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            if (!(ok = mbar_wait(&full[s], (c / NS) & 1, abort_flag))) break;
            uint8_t* kt = smem + s * Cfg::STAGE;
            const int nvalid = min(C, tok1 - (tok0 + c * C));
            if (prm.center)
                phi_tile<PHI, C, D, 256, true>(kt, u, nvalid, true);
            else
                phi_tile<PHI, C, D, 256>(kt, u, nvalid, true);
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
        }
        // warps 2-5 cover the four TMEM lane quarters of the record
        if (warp < 6 && ok && mbar_wait(done, 0, abort_flag)) {
            tc_fence_after();
            const int sp = warp & 3;
            const uint32_t lane_base = uint32_t(32 * sp) << 16;
            const int frow = 32 * sp + lane;  // key feature (accumulator row)
            float* srow = prm.S_out + size_t(blockIdx.x) * prm.stride_S + size_t(frow) * D;
            float zv[16];
            tmem_ld16(tmem + lane_base + Cfg::T_Z, zv);
#pragma unroll 1
            for (int v0 = 0; v0 < D; v0 += 32) {
                float sv[32];
                tmem_load<32>(tmem + lane_base + Cfg::T_S + v0, sv);
                float4* dst = reinterpret_cast<float4*>(srow + v0);
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    dst[t] = make_float4(sv[4 * t], sv[4 * t + 1], sv[4 * t + 2], sv[4 * t + 3]);
            }
            prm.z_out[size_t(blockIdx.x) * prm.stride_z + frow] = zv[0];
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        // the MMA thread's last commit may still be pending if a wait gave
        // up: wait for it (bounded) before releasing the columns
        if (lane == 0) mbar_wait_drain(done, 0);
        __syncwarp();
        tmem_dealloc(tmem, Cfg::T_COLS);
    }
}

}  // namespace la
