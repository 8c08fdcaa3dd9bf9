// la_chunk_bwd64.cuh — causal backward pass 2 (dK, dV) for head size D = 64,
// chunk C = 128, as a software pipeline over chunks.
//
// Same mathematics as bwd_dkdv_kernel in la_chunk_bwd.cuh (reverse token
// order, R/r = suffix state of the later chunks):
//
//   X1 = (B A^T).M^T,  X2 = (V dU^T + 1 dg^T).M^T
//   dV = X1 dU + B R,  dB = X2 A + V R^T + 1 r^T,  dK = dB * phi'(k)
//   R += A^T dU,  r += A^T dg
//
// but laid out so that no chunk waits for the previous one to drain:
//  * the raw products X1, X2, the packed masked operands (in place, bf16
//    pairs, read by MMAs with A from TMEM), the dV/dB accumulators and the
//    state accumulators each have their own TMEM columns, so the MMAs of
//    chunk t+1 start while the epilogue still reads chunk t;
//  * three input stages (q, k, v, dO tiles); dV and dK are staged in place
//    over the chunk's V and K tiles (dead once dV, dB are complete) and
//    stored by TMA from a warp of their own, which frees the stage once the
//    store has read it (prefetching later chunks into L2 as well was measured
//    slower: 0.179 vs 0.144 ms for the dQ pass at B8 H16 N8192);
//  * masking skips whole 32-column blocks (all-zero below the diagonal block,
//    unmasked above it).
//
// Warp roles (608 threads): 0 TMA producer, 1 MMA issuer (one thread), 2-9
// feature map / dU scaling, 10-13 mask-and-pack of X1 and X2, 14-17 dV/dK
// epilogue and state readout, 18 TMA stores.  Every wait is bounded
// (la_sm100.cuh).
#pragma once

#include "la_chunk_bwd.cuh"

namespace la {

struct Bwd2x64Cfg {
    static constexpr int C = 128, D = 64;
    static constexpr int NSTAGE = 3;
    static constexpr int TILE = C * D * 2;             // 16 KB
    static constexpr int OFF_DGF = 4 * TILE;           // in-stage: dg float [C]
    static constexpr int OFF_RINV = OFF_DGF + C * 4;   // in-stage: 1/g float [C]
    static constexpr int STAGE = ((OFF_RINV + C * 4) + 1023) / 1024 * 1024;
    static constexpr int OFF_RP = NSTAGE * STAGE;      // R, bf16 [D][D] row tile (row f)
    static constexpr int OFF_RF = OFF_RP + D * D * 2;  // r, float [D]
    static constexpr int OFF_RPART = OFF_RF + D * 4;   // partial sums of A^T dg, float [2][D]
    static constexpr int OFF_RCH = OFF_RPART + 2 * D * 4;  // A^T dg per step, ring of 4, float [4][D]
    static constexpr int OFF_BAR = OFF_RCH + 4 * D * 4;
    static constexpr int NBAR = 4 * NSTAGE + 12;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    // TMEM columns
    static constexpr int T_X1 = 0, T_X2 = C, T_DV = 2 * C, T_DB = 2 * C + D;
    static constexpr int T_R = 2 * C + 2 * D;
    static constexpr int T_COLS = 512;
    static_assert(T_R + D <= T_COLS, "TMEM budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(OFF_RP % 1024 == 0, "swizzled tiles on 1 KB");
};
constexpr int kBwd64Threads = 608;

// Mask and pack one C x C product in place in TMEM (rows = key j in this
// thread's lane, columns = query i; keep i >= j), optionally adding dg_i to
// the kept entries.  Columns i, i+1 go to column i/2 as a bf16 pair.  Warp
// `sp` holds rows 32sp..32sp+31, so 32-column block b is all-zero for b < sp,
// the diagonal block for b == sp and unmasked for b > sp.  Block b is read
// before columns 16b.. are written, and writes only reach columns of blocks
// already read.
__device__ __forceinline__ void mask_pack_upper(uint32_t reg, int sp, int jrow, const float* dgf,
                                                float dscale = 1.f) {
    using namespace sm100;
#pragma unroll 1
    for (int b = 0; b < 4; ++b) {
        const int i0 = 32 * b;
        float pk[16];
        if (b < sp) {
#pragma unroll
            for (int t = 0; t < 16; ++t) pk[t] = 0.f;
        } else {
            float v[32];
            tmem_load<32>(reg + i0, v);
            if (dgf) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 d4 = reinterpret_cast<const float4*>(dgf + i0)[q];
                    v[4 * q] = fmaf(dscale, d4.x, v[4 * q]);
                    v[4 * q + 1] = fmaf(dscale, d4.y, v[4 * q + 1]);
                    v[4 * q + 2] = fmaf(dscale, d4.z, v[4 * q + 2]);
                    v[4 * q + 3] = fmaf(dscale, d4.w, v[4 * q + 3]);
                }
            }
            if (b == sp) {
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int i = i0 + 2 * t;
                    pk[t] = __uint_as_float(
                        pack_bf16(i >= jrow ? v[2 * t] : 0.f, i + 1 >= jrow ? v[2 * t + 1] : 0.f));
                }
            } else {
#pragma unroll
                for (int t = 0; t < 16; ++t) pk[t] = __uint_as_float(pack_bf16(v[2 * t], v[2 * t + 1]));
            }
        }
        tmem_st16(reg + i0 / 2, pk);
    }
    tmem_wait_st();
}

// The same for a product with rows = query i and columns = key j, keeping
// j <= i and adding the row's dg to the kept entries (pass 1's W').
__device__ __forceinline__ void mask_pack_lower(uint32_t reg, int sp, int irow, float dg) {
    using namespace sm100;
#pragma unroll 1
    for (int b = 0; b < 4; ++b) {
        const int j0 = 32 * b;
        float pk[16];
        if (b > sp) {
#pragma unroll
            for (int t = 0; t < 16; ++t) pk[t] = 0.f;
        } else {
            float v[32];
            tmem_load<32>(reg + j0, v);
            if (b == sp) {
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int j = j0 + 2 * t;
                    pk[t] = __uint_as_float(pack_bf16(j <= irow ? v[2 * t] + dg : 0.f,
                                                      j + 1 <= irow ? v[2 * t + 1] + dg : 0.f));
                }
            } else {
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    pk[t] = __uint_as_float(pack_bf16(v[2 * t] + dg, v[2 * t + 1] + dg));
            }
        }
        tmem_st16(reg + j0 / 2, pk);
    }
    tmem_wait_st();
}

// PIN: the q and k maps hold phi(q), phi(k) from the forward (no feature
// map is evaluated here).
// PART: grouped key/value heads, dK and dV stored as float32 per-query-head
// partials (prm.dk_part, dv_part) instead of the bf16 tiles.
// DECAY: the decayed recurrence (one segment per head, phi evaluated here).
// Within a chunk of L tokens, m = L/2, query rows a_i carry gamma^(i-m) and
// key and value rows b_j, v_j carry beta_j = gamma^(m-j), so X1, X2 and the
// products with dU, A carry gamma^(i-j) (the dg_i added to X2 takes beta_j
// too); the suffix state accumulator (and r) hold gamma^(L-m) R of the
// later tokens and are rescaled once per step; dK takes beta_j on r and
// phi'(k) from b / beta_j.
template <int PHI, bool PIN, bool PART = false, bool DECAY = false>
__global__ void __launch_bounds__(kBwd64Threads, 1)
bwd_dkdv64_kernel(const __grid_constant__ BwdParams prm) {
    static_assert(!(DECAY && PIN), "decay evaluates phi itself");
    using namespace sm100;
    using Cfg = Bwd2x64Cfg;
    constexpr int C = Cfg::C, D = Cfg::D, NS = Cfg::NSTAGE;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;                 // TMA
    uint64_t* phi_done = bars + NS;        // 256 feature-map threads
    uint64_t* empty = bars + 2 * NS;       // MMA commit + the store warp
    uint64_t* x1_full = bars + 3 * NS;     // commit: B A^T
    uint64_t* x2_full = x1_full + 1;       // commit: V dU^T
    uint64_t* x1p_full = x1_full + 2;      // 128: X1 packed
    uint64_t* x2p_full = x1_full + 3;      // 128: X2 packed
    uint64_t* d_full = x1_full + 4;        // commit: dV, dB complete
    uint64_t* d_free = x1_full + 5;        // 128: dV, dB read
    uint64_t* r_full = x1_full + 6;        // commit: state update complete
    uint64_t* rx_full = x1_full + 7;       // 128: R operand and r written
    uint64_t* drain = x1_full + 8;
    uint64_t* rch_full = x1_full + 9;      // [2] 128: the step's A^T dg in the ring (by step parity)
    uint64_t* staged = x1_full + 11;       // [NS] 128: dV, dK rows of the stage's step staged
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x / prm.nseg, seg = blockIdx.x % prm.nseg;
    const int kv_head = kv_head_of(head, prm.kv_group);  // k, v head of this query head
    const int tok0 = seg * prm.seg_len;
    const int tok1 = min(prm.N, tok0 + prm.seg_len);
    const int nchunks = (tok1 - tok0 + C - 1) / C;
    const float* st_in =
        prm.state_in ? prm.state_in + size_t(prm.in_per_head ? head : blockIdx.x) * size_t(D * D + D)
                     : nullptr;
    // chunk processed at step t (reverse token order)
    auto row_of = [&](int t) { return tok0 + (nchunks - 1 - t) * C; };
    float lg = 0.f;  // log2(gamma) of this head
    if constexpr (DECAY) lg = log2f(decay_of(prm.dec, head));

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&phi_done[s], 256);
            mbar_init(&empty[s], 2);
        }
        mbar_init(x1_full, 1);
        mbar_init(x2_full, 1);
        mbar_init(x1p_full, 128);
        mbar_init(x2p_full, 128);
        mbar_init(d_full, 1);
        mbar_init(d_free, 128);
        mbar_init(r_full, 1);
        mbar_init(rx_full, 128);
        mbar_init(drain, 1);
        for (int i = 0; i < NS; ++i) mbar_init(&staged[i], 128);
        for (int i = 0; i < 2; ++i) mbar_init(&rch_full[i], 128);
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
        if (lane == 0) {
            tma_prefetch_desc(&prm.tm_q);
            tma_prefetch_desc(&prm.tm_k);
            tma_prefetch_desc(&prm.tm_v);
            tma_prefetch_desc(&prm.tm_do);
            int issued = 0;
            for (int t = 0; t < nchunks; ++t) {
                const int s = t % NS;
                if (t >= NS && !mbar_wait(&empty[s], ((t / NS) - 1) & 1, abort_flag)) break;
                uint8_t* st = smem + s * Cfg::STAGE;
                mbar_arrive_expect_tx(&full[s], 4 * Cfg::TILE);
                const int row = row_of(t);
                tma_load_3d(st, &prm.tm_q, &full[s], 0, row, head);
                tma_load_3d(st + Cfg::TILE, &prm.tm_k, &full[s], 0, row, kv_head);
                tma_load_3d(st + 2 * Cfg::TILE, &prm.tm_v, &full[s], 0, row, kv_head);
                tma_load_3d(st + 3 * Cfg::TILE, &prm.tm_do, &full[s], 0, row, head);
                issued = t + 1;
            }
            for (int t = max(0, issued - NS); t < issued; ++t)
                mbar_wait_drain(&full[t % NS], (t / NS) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t tX1 = tmem + Cfg::T_X1, tX2 = tmem + Cfg::T_X2;
            const uint32_t tDV = tmem + Cfg::T_DV, tDB = tmem + Cfg::T_DB;
            const uint32_t tR = tmem + Cfg::T_R;
            const uint32_t rp = sbase + Cfg::OFF_RP;
            constexpr uint32_t idCC = idesc_bf16(C, C, 0, 0);     // B A^T, V dU^T
            constexpr uint32_t idCD_mn = idesc_bf16(C, D, 0, 1);  // B operand rows = K
            constexpr uint32_t idCD_k = idesc_bf16(C, D, 0, 0);   // B operand K-major
            constexpr uint32_t idDD = idesc_bf16(D, D, 1, 1);     // A^T dU
            const bool has_init = st_in != nullptr;
            // base descriptors (k = 0), stepped along K by constant offsets,
            // so each MMA costs the issuing thread few instructions
            const uint64_t krp = desc_k_base(rp), mrp = desc_mn_base(rp, D);
            // X1 = B A^T, X2 = V dU^T (raw, fp32) of step t
            auto x_raw = [&](int t) -> bool {
                const int s = t % NS;
                const uint32_t qs = sbase + s * Cfg::STAGE, ks = qs + Cfg::TILE;
                const uint32_t vs = qs + 2 * Cfg::TILE, dus = qs + 3 * Cfg::TILE;
                const uint64_t kq = desc_k_base(qs), kk = desc_k_base(ks);
                const uint64_t kv = desc_k_base(vs), kdu = desc_k_base(dus);
                if (!mbar_wait(&phi_done[s], (t / NS) & 1, abort_flag)) return false;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tX1, kk + kstep_k(C, k), kq + kstep_k(C, k), idCC, k > 0);
                umma_commit(x1_full);
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tX2, kv + kstep_k(C, k), kdu + kstep_k(C, k), idCC, k > 0);
                umma_commit(x2_full);
                return true;
            };
            // Order per step t (software-pipelined): dV = X1 dU and dB = X2 A
            // first (they start the accumulators), then the state terms
            // dV += B R, dB += V R^T, then step t+1's raw products, then the
            // state update with step t.  The packed X1/X2 of step t are read
            // before step t+1's raw products overwrite them (MMAs run in
            // issue order); the state accumulator is read out (rx_full)
            // before its next update.
            bool ok = nchunks == 0 || x_raw(0);
            for (int t = 0; ok && t < nchunks; ++t) {
                const int s = t % NS;
                const uint32_t qs = sbase + s * Cfg::STAGE, ks = qs + Cfg::TILE;
                const uint32_t vs = qs + 2 * Cfg::TILE, dus = qs + 3 * Cfg::TILE;
                const uint64_t mq = desc_mn_base(qs, C), mdu = desc_mn_base(dus, C);
                const uint64_t kk = desc_k_base(ks), kv = desc_k_base(vs);
                if (t > 0 && !(ok = mbar_wait(d_free, (t - 1) & 1, abort_flag))) break;
                if (!(ok = mbar_wait(x1p_full, t & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C; k += 16)
                    umma_bf16_ts(tDV, tX1 + k / 2, mdu + kstep_mn(k), idCD_mn, k > 0);
                if (!(ok = mbar_wait(x2p_full, t & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C; k += 16)
                    umma_bf16_ts(tDB, tX2 + k / 2, mq + kstep_mn(k), idCD_mn, k > 0);
                // dV += B R, dB += V R^T from the state of the later chunks
                if (!(ok = mbar_wait(rx_full, t & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D; k += 16) {
                    umma_bf16(tDV, kk + kstep_k(C, k), mrp + kstep_mn(k), idCD_mn, 1);
                    umma_bf16(tDB, kv + kstep_k(C, k), krp + kstep_k(D, k), idCD_k, 1);
                }
                umma_commit(d_full);
                if (t + 1 < nchunks) {
                    if (!(ok = x_raw(t + 1))) break;
                    // R += A^T dU (r += A^T dg is summed by the feature-map warps)
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16(tR, mq + kstep_mn(k), mdu + kstep_mn(k), idDD,
                                  (t > 0 || has_init || k > 0) ? 1u : 0u);
                    umma_commit(r_full);
                }
                umma_commit(&empty[s]);
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < 10) {
        // per chunk: dg and 1/g, phi on Q and K in place (unless given),
        // dU = dO / g in place
        const int u = tid - 64;  // 0..255
        const float* gb = prm.gbuf + size_t(head) * prm.N;
        const float* dgb = prm.dgbuf + size_t(head) * prm.N;
        // g and dg of the next chunk are loaded one chunk ahead
        float g_nx = 1.f, dg_nx = 0.f;
        auto load_gdg = [&](int t) {
            if (u < C && t < nchunks) {
                const int tok = row_of(t) + u;
                if (tok < tok1) {
                    g_nx = gb[tok];
                    dg_nx = dgb[tok];
                } else {
                    g_nx = 1.f;
                    dg_nx = 0.f;
                }
            }
        };
        load_gdg(0);
        // with the forward's feature maps (PIN) warps 2-5 also mask and pack
        // X2 (the X warpgroup then packs X1 only); a failed wait there is
        // carried into the next group barrier so all eight warps leave together
        bool ok_x2 = true;
        for (int t = 0; t < nchunks; ++t) {
            const int s = t % NS;
            const int row0 = row_of(t);
            const int nvalid = min(C, tok1 - row0);
            const float g = g_nx, dg = dg_nx;
            load_gdg(t + 1);
            if (!named_bar_all(3, 256, ok_x2 && mbar_wait(&full[s], (t / NS) & 1, abort_flag))) break;
            uint8_t* st = smem + s * Cfg::STAGE;
            float* dgf = reinterpret_cast<float*>(st + Cfg::OFF_DGF);
            float* rinv = reinterpret_cast<float*>(st + Cfg::OFF_RINV);
            if (u < C) {
                const bool valid = u < nvalid;
                const float d = valid ? dg : 0.f;
                rinv[u] = valid ? 1.f / g : 0.f;
                dgf[u] = d;
            }
            named_bar_sync(3, 256);  // rinv ready
            if constexpr (DECAY) {
                const float m = 0.5f * float(nvalid);
                if (u < 128)
                    phi_tile_scaled<PHI, C, D, 128>(st, u, nvalid, true, lg, 1.f, -m);
                else
                    phi_tile_scaled<PHI, C, D, 128>(st + Cfg::TILE, u - 128, nvalid, true, lg,
                                                    -1.f, m);
                scale_tile_rows_exp2<C, D, 256>(st + 2 * Cfg::TILE, u, nvalid, lg, -1.f, m);
            } else if constexpr (!PIN) {
                if (u < 128)
                    phi_tile<PHI, C, D, 128>(st, u, nvalid, true);
                else
                    phi_tile<PHI, C, D, 128>(st + Cfg::TILE, u - 128, nvalid, true);
            }
            scale_tile_rows<C, D, 256>(st + 3 * Cfg::TILE, u, nvalid, rinv);
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
            if (PIN && warp < 6) {
                const int sp = warp & 3;
                ok_x2 = named_bar_all(4, 128, mbar_wait(x2_full, t & 1, abort_flag));
                if (ok_x2) {
                    tc_fence_after();
                    mask_pack_upper(tmem + (uint32_t(32 * sp) << 16) + Cfg::T_X2, sp, 32 * sp + lane,
                                    dgf);
                    tc_fence_before();
                    mbar_arrive(x2p_full);
                }
            }
        }
    } else if (warp < 14) {
        // mask and pack X1 (keep i >= j) and, without PIN, X2 (+ dg_i) in
        // place; sum the step's r term A^T dg
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int jrow = 32 * sp + lane;
        float* rpart = reinterpret_cast<float*>(smem + Cfg::OFF_RPART);
        float* rch = reinterpret_cast<float*>(smem + Cfg::OFF_RCH);
        for (int t = 0; t < nchunks; ++t) {
            const int s = t % NS;
            const float* dgf = reinterpret_cast<const float*>(smem + s * Cfg::STAGE + Cfg::OFF_DGF);
            if (!named_bar_all(1, 128, mbar_wait(x1_full, t & 1, abort_flag))) break;
            tc_fence_after();
            mask_pack_upper(tmem + lane_base + Cfg::T_X1, sp, jrow, nullptr);
            tc_fence_before();
            mbar_arrive(x1p_full);
            {
                // this step's r term A^T dg into ring slot t % 4 (read by the
                // state readout of step t; the slot is written again at step
                // t + 4, which cannot start before that readout): column f,
                // half of the rows per thread, then the two halves summed
                const int e = tid - 320, f = e & 63, r0 = (e >> 6) * 64;
                const uint8_t* at = smem + s * Cfg::STAGE;
                float acc = 0.f;
#pragma unroll 8
                for (int i = r0; i < r0 + 64; ++i)
                    acc = fmaf(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(at + tile_off(C, i, f))),
                               dgf[i], acc);
                rpart[(e >> 6) * D + f] = acc;
                named_bar_sync(1, 128);
                if (e < D) rch[(t & 3) * D + e] = rpart[e] + rpart[D + e];
                mbar_arrive(&rch_full[t & 1]);
            }
            if (PIN) continue;  // X2 is packed by feature-map warps 2-5
            if (!named_bar_all(1, 128, mbar_wait(x2_full, t & 1, abort_flag))) break;
            tc_fence_after();
            if constexpr (DECAY) {
                const float m = 0.5f * float(min(C, tok1 - row_of(t)));
                mask_pack_upper(tmem + lane_base + Cfg::T_X2, sp, jrow, dgf,
                                exp2f(lg * (m - float(jrow))));
            } else {
                mask_pack_upper(tmem + lane_base + Cfg::T_X2, sp, jrow, dgf);
            }
            tc_fence_before();
            mbar_arrive(x2p_full);
        }
    } else if (warp < 18) {
        // dV / dK epilogue (rows staged in place over the V and K tiles) and
        // the state readout
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int jrow = 32 * sp + lane;
        const int frow = acc_row<D>(sp, lane);  // row of the M = 64 state accumulators
        uint8_t* rp = smem + Cfg::OFF_RP;
        float* rf = reinterpret_cast<float*>(smem + Cfg::OFF_RF);

        // initial state: R operand, r, and (with an initial state) the accumulators
        if (frow >= 0) {
            float r0;
            load_state_row<D>(st_in, frow, rp, &r0);
            rf[frow] = r0;
        }
        if (st_in) {
#pragma unroll 1
            for (int f0 = 0; f0 < D; f0 += 16) {
                float v16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v16[i] = frow >= 0 ? st_in[size_t(frow) * D + f0 + i] : 0.f;
                tmem_st16(tmem + lane_base + Cfg::T_R + f0, v16);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(rx_full);

        for (int t = 0; t < nchunks; ++t) {
            const int s = t % NS;
            uint8_t* kt = smem + s * Cfg::STAGE + Cfg::TILE;   // B, then dK
            uint8_t* vt = smem + s * Cfg::STAGE + 2 * Cfg::TILE;  // dV
            // decay: this row's beta_j (r term) and 1 / beta_j (phi' from b)
            float beta = 1.f, binv = 1.f, m = 0.f;
            if constexpr (DECAY) {
                m = 0.5f * float(min(C, tok1 - row_of(t)));
                beta = exp2f(lg * (m - float(jrow)));
                binv = exp2f(lg * (float(jrow) - m));
            }
            if (!named_bar_all(2, 128, mbar_wait(d_full, t & 1, abort_flag))) break;
            tc_fence_after();
            // NB 16-column groups of dV and dB per TMEM round trip (one
            // for the float32-partials variant, whose registers are tighter)
            constexpr int NB = PART ? 1 : 2;
#pragma unroll 1
            for (int c2 = 0; c2 < D; c2 += 16 * NB) {
                float dvx[16 * NB], dbx[16 * NB];
#pragma unroll
                for (int hh = 0; hh < NB; ++hh) {
                    tmem_ld16(tmem + lane_base + Cfg::T_DV + c2 + 16 * hh, dvx + 16 * hh);
                    tmem_ld16(tmem + lane_base + Cfg::T_DB + c2 + 16 * hh, dbx + 16 * hh);
                }
                tmem_wait_ld();
#pragma unroll
                for (int hh = 0; hh < NB; ++hh) {
                const int c0 = c2 + 16 * hh;
                float* dv16 = dvx + 16 * hh;
                const float* db16 = dbx + 16 * hh;
                float b8a[8], b8b[8];
                load_chunk8(kt, C, jrow, c0 >> 3, b8a);
                load_chunk8(kt, C, jrow, (c0 >> 3) + 1, b8b);
                float r16[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 x = reinterpret_cast<const float4*>(rf + c0)[q];
                    r16[4 * q] = x.x;
                    r16[4 * q + 1] = x.y;
                    r16[4 * q + 2] = x.z;
                    r16[4 * q + 3] = x.w;
                }
                float dk16[16];
                if constexpr (DECAY) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        dk16[i] = fmaf(beta, r16[i], db16[i]) *
                                  dphi_from_scaled_phi<PHI>(b8a[i], beta, binv);
                        dk16[8 + i] = fmaf(beta, r16[8 + i], db16[8 + i]) *
                                      dphi_from_scaled_phi<PHI>(b8b[i], beta, binv);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        dk16[i] = (db16[i] + r16[i]) * dphi_from_phi<PHI>(b8a[i]);
                        dk16[8 + i] = (db16[8 + i] + r16[8 + i]) * dphi_from_phi<PHI>(b8b[i]);
                    }
                }
                if constexpr (PART) {
                    if (row_of(t) + jrow < prm.N) {
                        const size_t off = (size_t(head) * prm.N + row_of(t) + jrow) * D + c0;
                        store16_f32(prm.dv_part + off, dv16);
                        store16_f32(prm.dk_part + off, dk16);
                    }
                } else {
                    // this thread's row of B is read before it is overwritten
                    store_row16_bf16(vt, C, jrow, c0, dv16);
                    store_row16_bf16(kt, C, jrow, c0, dk16);
                }
                }
            }
            tc_fence_before();
            mbar_arrive(d_free);
            fence_proxy_async_smem();
            mbar_arrive(&staged[s]);
            if (t + 1 == nchunks) break;
            // state after this chunk -> operands of the next (earlier) chunk
            if (!named_bar_all(2, 128, mbar_wait(r_full, t & 1, abort_flag))) break;
            tc_fence_after();
            // decay: the accumulator holds gamma^(-m) R of this chunk's
            // start; the next (earlier, full) chunk wants gamma^(C/2) R
            const float fr = DECAY ? exp2f(lg * (0.5f * float(C) + m)) : 1.f;
#pragma unroll 1
            for (int v0 = 0; v0 < D; v0 += 32) {
                float rv[32];
                tmem_load<32>(tmem + lane_base + Cfg::T_R + v0, rv);
                if constexpr (DECAY) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) rv[i] *= fr;
                    tmem_st16(tmem + lane_base + Cfg::T_R + v0, rv);
                    tmem_st16(tmem + lane_base + Cfg::T_R + v0 + 16, rv + 16);
                }
                if (frow >= 0) {
                    store_row16_bf16(rp, D, frow, v0, rv);
                    store_row16_bf16(rp, D, frow, v0 + 16, rv + 16);
                }
            }
            if constexpr (DECAY) tmem_wait_st();
            if (!named_bar_all(2, 128, mbar_wait(&rch_full[t & 1], (t >> 1) & 1, abort_flag))) break;
            if constexpr (DECAY) {
                if (frow >= 0)
                    rf[frow] = fr * (rf[frow] + reinterpret_cast<const float*>(
                                                     smem + Cfg::OFF_RCH)[(t & 3) * D + frow]);
            } else {
                if (frow >= 0) rf[frow] += reinterpret_cast<const float*>(smem + Cfg::OFF_RCH)[(t & 3) * D + frow];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(rx_full);
        }
    } else if (warp == 18) {
        // TMA stores of the staged dV, dK rows; the stage is free once they
        // have been read
        if (lane == 0) {
            for (int t = 0; t < nchunks; ++t) {
                const int s = t % NS;
                const int row0 = row_of(t);
                uint8_t* st = smem + s * Cfg::STAGE;
                if (!mbar_wait(&staged[s], (t / NS) & 1, abort_flag)) break;
                if constexpr (!PART) {  // else the epilogue stored float32 partials
                    tma_store_3d(&prm.tm_dv, st + 2 * Cfg::TILE, 0, row0, head);
                    tma_store_3d(&prm.tm_dk, st + Cfg::TILE, 0, row0, head);
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(&empty[s]);
            }
            bulk_wait0();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::T_COLS);
}

// ======================================================================
// Pass 1 (dQ), causal, with the forward's saved O and g, one segment per
// head.  Per chunk c (token order), S / z = state of the earlier chunks:
//
//   dU = dO / g,  dg = -(dO . o) / g          (feature-map warps)
//   W  = dU V^T,  W' = (W + dg 1^T).M         (M: keep key j <= query i)
//   dA = dU S^T + W' B,  dQ = (dA + dg z^T) * phi'(q)
//   T  = [V | 1]^T B accumulated: rows 0..63 = S^T, row 64 = z^T
//
// No product reads A = phi(q): the epilogue forms phi'(q) from the q tile
// (raw q, or with PIN the forward's phi(q), phi' = dphi_from_phi) and then
// stages dQ in place over it.  The k tile always comes from k and holds the
// centred features B = phi(k) - c (phi_center): with elu+1 on small inputs
// phi(k) is close to 1 and its bf16 rounding would lose most of phi(k) - 1.
// W' B and dU S^T (S, z summed from the same centred features) then differ
// from the true dA only along the all-ones vector, which the epilogue
// restores exactly from <dA_i, phi(q_i)> = 0.  Same warp roles and hand-offs as
// bwd_dkdv64_kernel; W and dA are double-buffered in TMEM.
// ======================================================================
struct Bwd1x64Cfg {
    static constexpr int C = 128, D = 64;
    static constexpr int NSTAGE = 3;
    static constexpr int TILE = C * D * 2;             // 16 KB
    static constexpr int OFF_DGF = 4 * TILE;           // in-stage: dg float [C]
    static constexpr int STAGE = ((OFF_DGF + C * 4) + 1023) / 1024 * 1024;
    static constexpr int OFF_ONES = NSTAGE * STAGE;    // [C][64] atom, column 0 = 1
    static constexpr int OFF_SX = OFF_ONES + TILE;     // S^T, bf16 [D][D] row tile (row v)
    static constexpr int OFF_ZF = OFF_SX + D * D * 2;  // z, float [2][D] (by chunk parity)
    static constexpr int OFF_BAR = OFF_ZF + 2 * D * 4;
    static constexpr int NBAR = 4 * NSTAGE + 10;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    // TMEM columns: W [2][C], dA [2][D], T [D]
    static constexpr int T_W = 0, T_DA = 2 * C, T_T = 2 * C + 2 * D;
    static constexpr int T_COLS = 512;
    static_assert(T_T + D <= T_COLS, "TMEM budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(OFF_ONES % 1024 == 0 && OFF_SX % 1024 == 0, "swizzled tiles on 1 KB");
};

// DECAY: the decayed recurrence (phi(q) evaluated here).  Within a chunk of
// L tokens, m = L/2, dU rows and dg_i carry gamma^(i+1-m) and the centred
// key rows gamma^(m-1-j), so W' B' carries gamma^(i-j); the state
// accumulator holds gamma^(m-L) S' after the chunk and is rescaled in TMEM
// to gamma^(m') S' (the next chunk's m') with the operand and z.
template <int PHI, bool PIN, bool DECAY = false>
__global__ void __launch_bounds__(kBwd64Threads, 1)
bwd_dq64_kernel(const __grid_constant__ BwdParams prm) {
    static_assert(!(DECAY && PIN), "decay evaluates phi itself");
    using namespace sm100;
    using Cfg = Bwd1x64Cfg;
    constexpr int C = Cfg::C, D = Cfg::D, NS = Cfg::NSTAGE;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;                // TMA
    uint64_t* phi_done = bars + NS;       // 256 feature-map threads
    uint64_t* empty = bars + 2 * NS;      // MMA commit + the store warp
    uint64_t* w_full = bars + 3 * NS;     // commit: W
    uint64_t* wp_full = w_full + 1;       // 128: W' packed
    uint64_t* t_full = w_full + 2;        // commit: state update
    uint64_t* sx_full = w_full + 3;       // 128: S^T operand and z written
    uint64_t* da_full = w_full + 4;       // [2] commit: dA complete
    uint64_t* da_free = w_full + 6;       // [2] 128: dA read
    uint64_t* drain = w_full + 8;
    uint64_t* staged = w_full + 9;        // [NS] 128: dQ rows of the stage's step staged
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x / prm.nseg, seg = blockIdx.x % prm.nseg;
    const int kv_head = kv_head_of(head, prm.kv_group);  // k, v head of this query head
    const int tok0 = seg * prm.seg_len;
    const int tok1 = min(prm.N, tok0 + prm.seg_len);
    const int nchunks = (tok1 - tok0 + C - 1) / C;
    auto row_of = [&](int c) { return tok0 + c * C; };
    float lg = 0.f;  // log2(gamma) of this head
    if constexpr (DECAY) lg = log2f(decay_of(prm.dec, head));

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&phi_done[s], 256);
            mbar_init(&empty[s], 2);
        }
        mbar_init(w_full, 1);
        mbar_init(wp_full, 128);
        mbar_init(t_full, 1);
        mbar_init(sx_full, 128);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&da_full[b], 1);
            mbar_init(&da_free[b], 128);
        }
        for (int i = 0; i < NS; ++i) mbar_init(&staged[i], 128);
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
        if (lane == 0) {
            tma_prefetch_desc(&prm.tm_q);
            tma_prefetch_desc(&prm.tm_k);
            tma_prefetch_desc(&prm.tm_v);
            tma_prefetch_desc(&prm.tm_do);
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                if (c >= NS && !mbar_wait(&empty[s], ((c / NS) - 1) & 1, abort_flag)) break;
                uint8_t* st = smem + s * Cfg::STAGE;
                mbar_arrive_expect_tx(&full[s], 4 * Cfg::TILE);
                const int row = row_of(c);
                tma_load_3d(st, &prm.tm_q, &full[s], 0, row, head);
                tma_load_3d(st + Cfg::TILE, &prm.tm_k, &full[s], 0, row, kv_head);
                tma_load_3d(st + 2 * Cfg::TILE, &prm.tm_v, &full[s], 0, row, kv_head);
                tma_load_3d(st + 3 * Cfg::TILE, &prm.tm_do, &full[s], 0, row, head);
                issued = c + 1;
            }
            for (int c = max(0, issued - NS); c < issued; ++c)
                mbar_wait_drain(&full[c % NS], (c / NS) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t tW = tmem + Cfg::T_W, tDA = tmem + Cfg::T_DA, tT = tmem + Cfg::T_T;
            const uint32_t sx = sbase + Cfg::OFF_SX, ones = sbase + Cfg::OFF_ONES;
            constexpr uint32_t idCC = idesc_bf16(C, C, 0, 0);     // dU V^T
            constexpr uint32_t idCD_mn = idesc_bf16(C, D, 0, 1);  // B operand rows = K
            constexpr uint32_t idT = idesc_bf16(128, D, 1, 1);    // [V | 1]^T B
            const uint64_t msx = desc_mn_base(sx, D);
            bool ok = true;
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c % NS, b = c & 1;
                const uint32_t qs = sbase + s * Cfg::STAGE, ks = qs + Cfg::TILE;
                const uint32_t vs = qs + 2 * Cfg::TILE, dus = qs + 3 * Cfg::TILE;
                // base descriptors (k = 0), stepped along K by constant offsets
                const uint64_t kdu = desc_k_base(dus), kv = desc_k_base(vs), mk = desc_mn_base(ks, C);
                if (!(ok = mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                tc_fence_after();
                // W = dU V^T
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tW + b * C, kdu + kstep_k(C, k), kv + kstep_k(C, k), idCC, k > 0);
                umma_commit(w_full);
                // dA = dU S^T (state of the earlier chunks), then the state update
                if (!(ok = mbar_wait(sx_full, c & 1, abort_flag))) break;
                if (c >= 2 && !(ok = mbar_wait(&da_free[b], ((c >> 1) - 1) & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tDA + b * D, kdu + kstep_k(C, k), msx + kstep_mn(k), idCD_mn, k > 0);
                if (c + 1 < nchunks) {
                    const uint64_t dvx = sdesc_sw128(vs, ones - vs, 1024);
                    const uint64_t dkm = desc_mn_base(ks, C);
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16(tT, dvx + kstep_mn(k), dkm + kstep_mn(k), idT, (c > 0 || k > 0) ? 1u : 0u);
                    umma_commit(t_full);
                }
                // dA += W' B (W' packed in TMEM)
                if (!(ok = mbar_wait(wp_full, c & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C; k += 16)
                    umma_bf16_ts(tDA + b * D, tW + b * C + k / 2, mk + kstep_mn(k), idCD_mn, 1);
                umma_commit(&da_full[b]);
                umma_commit(&empty[s]);
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < 10) {
        // phi on K in place, then dU = dO / g in place and dg = -(dO . o) / g
        // (two threads per row), all eight warps on each
        const int u = tid - 64;  // 0..255
        const int r = u >> 1, part = u & 1;
        const float* gb = prm.gbuf + size_t(head) * prm.N;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            const int row0 = row_of(c);
            const int nvalid = min(C, tok1 - row0);
            const bool valid = r < nvalid;
            // this row's o and g, loaded while the tiles land
            const uint4* orow =
                reinterpret_cast<const uint4*>(prm.o_in + (size_t(head) * prm.N + row0 + r) * D) + 4 * part;
            const float g = valid ? gb[row0 + r] : 1.f;
            uint4 ov[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) ov[j] = valid ? __ldg(orow + j) : make_uint4(0u, 0u, 0u, 0u);
            if (!named_bar_all(3, 256, mbar_wait(&full[s], (c / NS) & 1, abort_flag))) break;
            uint8_t* st = smem + s * Cfg::STAGE;
            // k -> phi(k) - c, the centred key features (from k even when the
            // forward's phi(k) is available: it is rounded once, from k)
            const float m = 0.5f * float(nvalid);
            if constexpr (DECAY)
                phi_tile_scaled<PHI, C, D, 256, true>(st + Cfg::TILE, u, nvalid, true, lg, -1.f,
                                                      m - 1.f);
            else
                phi_tile<PHI, C, D, 256, true>(st + Cfg::TILE, u, nvalid, true);
            uint8_t* dot = st + 3 * Cfg::TILE;
            float dotp = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 x = *reinterpret_cast<const uint4*>(dot + tile_chunk_off(C, r, 4 * part + j));
                const uint32_t a[4] = {x.x, x.y, x.z, x.w};
                const uint32_t bb[4] = {ov[j].x, ov[j].y, ov[j].z, ov[j].w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 fa = unpack_bf16(a[t]), fb = unpack_bf16(bb[t]);
                    dotp = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, dotp));
                }
            }
            dotp += __shfl_xor_sync(0xffffffffu, dotp, 1);
            // decay: dU and dg of row r carry gamma^(r+1-m)
            const float sr = DECAY ? exp2f(lg * (float(r) + 1.f - m)) : 1.f;
            const float ginv = 1.f / g;
            const float dg = valid ? -dotp * ginv : 0.f;
            const float gs = ginv * sr;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4* px = reinterpret_cast<uint4*>(dot + tile_chunk_off(C, r, 4 * part + j));
                const uint4 x = *px;
                uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 f = unpack_bf16(w[t]);
                    w[t] = valid ? pack_bf16(f.x * gs, f.y * gs) : 0u;
                }
                *px = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (part == 0) {
                reinterpret_cast<float*>(st + Cfg::OFF_DGF)[r] = dg * sr;
                if (valid) prm.dgbuf[size_t(head) * prm.N + row0 + r] = dg;
            }
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
        }
    } else if (warp < 14) {
        // W' = (W + dg) masked, packed in place
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int irow = 32 * sp + lane;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS, b = c & 1;
            if (!named_bar_all(1, 128, mbar_wait(w_full, c & 1, abort_flag))) break;
            tc_fence_after();
            const float dg = reinterpret_cast<const float*>(smem + s * Cfg::STAGE + Cfg::OFF_DGF)[irow];
            mask_pack_lower(tmem + lane_base + Cfg::T_W + b * C, sp, irow, dg);
            tc_fence_before();
            mbar_arrive(wp_full);
        }
    } else if (warp < 18) {
        // state readout (S^T operand, z) and the dQ epilogue (staged in place
        // over the raw q tile)
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int irow = 32 * sp + lane;  // token row; lane of T = v
        uint8_t* sxp = smem + Cfg::OFF_SX;
        uint8_t* ones = smem + Cfg::OFF_ONES;
        float* zf = reinterpret_cast<float*>(smem + Cfg::OFF_ZF);  // [2][D]
        {
            float v8[8] = {1.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            const float z8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int q = 0; q < 8; ++q) store_row_bf16<8>(ones, C, irow, 8 * q, q == 0 ? v8 : z8);
            if (irow < D) {
                for (int q = 0; q < 8; ++q) store_row_bf16<8>(sxp, D, irow, 8 * q, z8);
                zf[irow] = 0.f;
                zf[D + irow] = 0.f;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(sx_full);

        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS, b = c & 1;
            uint8_t* qt = smem + s * Cfg::STAGE;
            if (c + 1 < nchunks) {
                // state after this chunk -> operands of the next chunk
                if (!named_bar_all(2, 128, mbar_wait(t_full, c & 1, abort_flag))) break;
                tc_fence_after();
                // decay: gamma^(m-C) S' (this full chunk) -> gamma^(m') S'
                const float fs =
                    DECAY ? exp2f(lg * (0.5f * float(C) + 0.5f * float(min(C, tok1 - row_of(c + 1)))))
                          : 1.f;
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    float col[32];
                    tmem_load<32>(tmem + lane_base + Cfg::T_T + 32 * h, col);
                    if constexpr (DECAY) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) col[i] *= fs;
                        tmem_st16(tmem + lane_base + Cfg::T_T + 32 * h, col);
                        tmem_st16(tmem + lane_base + Cfg::T_T + 32 * h + 16, col + 16);
                    }
                    if (irow < D) {
                        store_row_bf16<32>(sxp, D, irow, 32 * h, col);
                    } else if (irow == D) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) zf[((c + 1) & 1) * D + 32 * h + i] = col[i];
                    }
                }
                if constexpr (DECAY) tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(sx_full);
            }
            // dQ = (T + t 1) * phi'(q): T = dA + dg z formed with the centred
            // key features, which differ from the true dA only along the
            // all-ones vector; t restores that component from
            // <dA_i, a_i> = 0 (t = -(T . a_i) / (1 . a_i)).  a = phi(q): the
            // forward's map (PIN) or evaluated here from q.
            if (!named_bar_all(2, 128, mbar_wait(&da_full[b], (c >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            const float dg = reinterpret_cast<const float*>(qt + Cfg::OFF_DGF)[irow];
            const float* z = zf + (c & 1) * D;
            constexpr float kc = phi_center<PHI>();
            float tcoef = 0.f;
            if (kc != 0.f) {
                float dot = 0.f, sa = 0.f;
#pragma unroll 1
                for (int f0 = 0; f0 < D; f0 += 32) {
                    float tv[32];
                    tmem_load<32>(tmem + lane_base + Cfg::T_DA + b * D + f0, tv);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float a8[8];
                        load_chunk8(qt, C, irow, (f0 >> 3) + q, a8);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float a = PIN ? a8[i] : phi_fast<PHI>(a8[i]);
                            dot = fmaf(fmaf(dg, z[f0 + 8 * q + i], tv[8 * q + i]), a, dot);
                            sa += a;
                        }
                    }
                }
                tcoef = -kc * dot / sa;
            }
#pragma unroll 1
            for (int f0 = 0; f0 < D; f0 += 32) {
                float tv[32];
                tmem_load<32>(tmem + lane_base + Cfg::T_DA + b * D + f0, tv);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float q8[8];
                    load_chunk8(qt, C, irow, (f0 >> 3) + q, q8);
                    uint32_t w[4];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        q8[i] = PIN ? dphi_from_phi<PHI>(q8[i]) : dphi_fast<PHI>(q8[i]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int f = f0 + 8 * q + 2 * i;
                        w[i] = pack_bf16((fmaf(dg, z[f], tv[8 * q + 2 * i]) + tcoef) * q8[2 * i],
                                         (fmaf(dg, z[f + 1], tv[8 * q + 2 * i + 1]) + tcoef) *
                                             q8[2 * i + 1]);
                    }
                    // this thread's row of q is read before it is overwritten
                    *reinterpret_cast<uint4*>(qt + tile_chunk_off(C, irow, (f0 >> 3) + q)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&da_free[b]);
            fence_proxy_async_smem();
            mbar_arrive(&staged[s]);
        }
    } else if (warp == 18) {
        // TMA stores of the staged dQ rows; the stage is free once they have
        // been read
        if (lane == 0) {
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                if (!mbar_wait(&staged[s], (c / NS) & 1, abort_flag)) break;
                tma_store_3d(&prm.tm_dq, smem + s * Cfg::STAGE, 0, row_of(c), head);
                bulk_commit();
                bulk_wait_read0();
                mbar_arrive(&empty[s]);
            }
            bulk_wait0();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::T_COLS);
}

}  // namespace la
