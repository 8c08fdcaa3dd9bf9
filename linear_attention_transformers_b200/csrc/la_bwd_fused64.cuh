// la_bwd_fused64.cuh — the causal backward in one pass over the sequence, for
// head size D = 64 (chunks of C = 128 tokens), one thread block per head.
//
// Gradients of L = sum(dO * O) (derived from the Statement of the
// Proposition "Linear Attention via Kernel Decomposition", "Efficient
// Transformers Survey"; see la_chunk_bwd.cuh for the per-token form).  With
// a = phi(q), b = phi(k), g_i = a_i . z_i, du_i = dO_i / g_i and
// dg_i = -(dO_i . o_i) / g_i:
//
//   dA_i = sum_{j<=i} b_j (v_j.du_i + dg_i)      dQ = dA * phi'(q)
//   dB_j = sum_{i>=j} a_i (v_j.du_i + dg_i)      dK = dB * phi'(k)
//   dV_j = sum_{i>=j} (a_i.b_j) du_i
//
// The chunks are walked from the last to the first.  The suffix sums over
// the chunks already walked give dK and dV directly (R = sum a_i du_i^T,
// r = sum a_i dg_i over later chunks):
//   dV_c = X1 dU + B R,  dB_c = X2 A + V R^T + r
//   X1 = (B A^T) keeping i >= j,  X2 = (V dU^T + 1 dg^T) keeping i >= j
// and the prefix state the dQ term needs is the final state minus the
// states of the chunks walked so far, this one included (states are sums
// over tokens, so they subtract):
//   dA_c = dU Sig^T + dg zeta^T + X2^T B,  Sig, zeta = state before the chunk.
// Every input (q, k, v, dO, o, g) is read once and every gradient written
// once; no N x D x D tensor exists.
//
// Precision.  With phi = elu+1 on small inputs every feature vector is close
// to the all-ones vector, and dA_i (orthogonal to a_i: <dA_i, a_i> = 0
// exactly) is a small difference of such vectors: rounding b = 1 + beta to
// bf16 would lose most of beta.  So the key side is kept centred: the k
// tile holds b' = phi(k) - c (c = 1 for elu+1, 0 for relu+eps; see
// phi_center), the states are sums of b', and the terms in c are restored
// exactly where they matter:
//   X1 = B' A^T + c 1 sa^T (sa_i = sum_f a_if, added by the mask warps),
//   B R = B' R + c 1 rho^T (rho = column sums of R, summed on CUDA cores),
// while in dA every c-term lies along the all-ones direction, as does any
// per-value-column constant in Sig (its mean over features is removed
// before the bf16 rounding); the component of dA along 1 is then restored
// from the identity: dA = T + t 1 with t = -(T . a) / (1 . a).
//
// Tensor-core layout (tcgen05, accumulators in TMEM, 512 columns):
//   X1 = B' A^T and E' = (-V) dU^T: raw C x C products (128 columns each);
//   the mask warps pack X1 + c sa (i >= j) and X2' = E' - dg (i >= j, = -X2)
//   in place as bf16 pairs, read by the dV / dB MMAs as A from TMEM, and
//   write X2 to shared memory as the MN-major operand of dA (its zero block,
//   i >= 64 > j, comes from a 2 KB zero block through the atom stride).  V is
//   negated in shared memory once per chunk so that one M = 128 state MMA
//   gives both states:
//   RS = [A | 0]^T dU  (rows 0..63: R)  +  [0 | -V]^T B'  (rows 64..127)
//   with rows 64..127 started at the centred final state S'^T, so after the
//   chunk's MMA they hold Sig^T.  dB' = X2' A + (-V) R^T = -dB_c (negated
//   back in the epilogue).  60 MMAs per chunk: X1 4, E' 4, dV 8 + 4,
//   dB 8 + 4, dA 4 + 8, RS 16.
//
// Warp roles (608 threads): 0 TMA producer, 1 MMA issuer (one thread),
// 2-9 feature map / -V / dU, dg (8 warps), 10-13 masks and the chunk's sums
// of b', a dg and sa du, 14-17 state readout and the dV, dK, dQ epilogues
// (staged in place over the chunk's v, k and q tiles), 18 TMA stores.  Every
// wait is bounded (la_sm100.cuh).
#pragma once

#include "la_chunk_bwd64.cuh"

namespace la {

struct BwdFused64Cfg {
    static constexpr int C = 128, D = 64;
    static constexpr int NS = 3;    // q, k, v stages
    static constexpr int NDO = 2;   // dO stages (free earlier: after the chunk's dA)
    static constexpr int TILE = C * D * 2;  // 16 KB, [C][64] bf16
    // Shared memory.  Operand order (atom strides are positive):
    // q tiles < ZERO < v tiles (state MMA); WL0 < WL1 and ZERO < WL1 (dA).
    static constexpr int OFF_Q = 0;                        // [NS] q -> A -> dQ
    static constexpr int OFF_WL0 = OFF_Q + NS * TILE;      // X2 rows j 0..63, i 0..63
    static constexpr int OFF_ZERO = OFF_WL0 + TILE / 2;    // 16 zero rows (2 KB)
    static constexpr int OFF_V = OFF_ZERO + 2048;          // [NS] v -> -V -> dV
    static constexpr int OFF_WL1 = OFF_V + NS * TILE;      // X2 rows j 0..127, i 64..127
    static constexpr int OFF_K = OFF_WL1 + TILE;           // [NS] k -> B' -> dK
    static constexpr int OFF_DO = OFF_K + NS * TILE;       // [NDO] dO -> dU
    static constexpr int OFF_SIGT = OFF_DO + NDO * TILE;   // Sig^T bf16 [D][D], row v
    static constexpr int OFF_R = OFF_SIGT + D * D * 2;     // R bf16 [D][D], row f
    static constexpr int OFF_DGF = OFF_R + D * D * 2;      // dg float [NS][C]
    static constexpr int OFF_SA = OFF_DGF + NS * C * 4;    // sa float [NS][C]
    static constexpr int OFF_ZETA = OFF_SA + NS * C * 4;   // zeta float [2][D]
    static constexpr int OFF_RN = OFF_ZETA + 2 * D * 4;    // r float [2][D]
    static constexpr int OFF_RHO = OFF_RN + 2 * D * 4;     // rho float [2][D]
    static constexpr int OFF_SUMS = OFF_RHO + 2 * D * 4;   // chunk sums [2][3][D]
    static constexpr int OFF_BAR = OFF_SUMS + 6 * D * 4;
    static constexpr int NBAR = 3 * NS + 2 * NDO + 13 + NS;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    // TMEM columns
    static constexpr int T_X1 = 0, T_E = 128, T_DV = 256, T_DB = 320, T_DA = 384, T_RS = 448;
    static constexpr int T_COLS = 512;
    static_assert(T_RS + D <= T_COLS, "TMEM budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(OFF_WL0 % 1024 == 0 && OFF_ZERO % 1024 == 0 && OFF_V % 1024 == 0 &&
                      OFF_WL1 % 1024 == 0 && OFF_K % 1024 == 0 && OFF_DO % 1024 == 0 &&
                      OFF_SIGT % 1024 == 0 && OFF_R % 1024 == 0,
                  "swizzled tiles on 1 KB");
    static_assert(OFF_Q + NS * TILE <= OFF_ZERO && OFF_ZERO < OFF_V && OFF_WL0 < OFF_WL1 &&
                      OFF_ZERO < OFF_WL1,
                  "operand order");
};
constexpr int kBwdFused64Threads = 608;

// E' row j of the chunk (this thread's TMEM lane): Y = E' - dg_i, kept for
// i >= j.  Y is packed in place as bf16 pairs (the X2' operand, read by MMAs
// with A from TMEM) and -Y = X2 is written to the dA operand in shared
// memory: row j, columns i < 64 in WL0 (rows j < 64 only: for j >= 64 those
// entries are zero and come from the zero block), columns i >= 64 in WL1.
// Warp `sp` holds rows 32sp.., so 32-column block b lies wholly below the
// diagonal (b < sp, dropped), on it (b == sp) or above it (b > sp, kept).
// Block b is read before columns 16b.. are written.
__device__ __forceinline__ void mask_split_e(uint32_t reg, int sp, int jrow, const float* dgf,
                                             uint8_t* wl0, uint8_t* wl1) {
    using namespace sm100;
#pragma unroll 1
    for (int b = 0; b < 4; ++b) {
        const int i0 = 32 * b;
        float y[32];
        if (b < sp) {
#pragma unroll
            for (int t = 0; t < 32; ++t) y[t] = 0.f;
        } else {
            tmem_load<32>(reg + i0, y);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 d4 = reinterpret_cast<const float4*>(dgf + i0)[q];
                y[4 * q] -= d4.x;
                y[4 * q + 1] -= d4.y;
                y[4 * q + 2] -= d4.z;
                y[4 * q + 3] -= d4.w;
            }
            if (b == sp) {
#pragma unroll
                for (int t = 0; t < 32; ++t) y[t] = i0 + t >= jrow ? y[t] : 0.f;
            }
        }
        float pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[t] = __uint_as_float(pack_bf16(y[2 * t], y[2 * t + 1]));
        tmem_st16(reg + i0 / 2, pk);
#pragma unroll
        for (int t = 0; t < 32; ++t) y[t] = -y[t];
        if (b >= 2)
            store_row_bf16<32>(wl1, 128, jrow, i0 - 64, y);
        else if (jrow < 64)
            store_row_bf16<32>(wl0, 64, jrow, i0, y);
    }
    tmem_wait_st();
}

template <int PHI>
__global__ void __launch_bounds__(kBwdFused64Threads, 1)
bwd_fused64_kernel(const __grid_constant__ BwdParams prm) {
    using namespace sm100;
    using Cfg = BwdFused64Cfg;
    constexpr int C = Cfg::C, D = Cfg::D, NS = Cfg::NS, NDO = Cfg::NDO;
    constexpr float kc = phi_center<PHI>();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* qkv_full = bars;                // [NS] TMA
    uint64_t* qkv_empty = bars + NS;          // [NS] store warp
    uint64_t* phi_done = bars + 2 * NS;       // [NS] 256 elementwise threads
    uint64_t* do_full = bars + 3 * NS;        // [NDO] TMA
    uint64_t* do_empty = do_full + NDO;       // [NDO] commit after the chunk's dA
    uint64_t* x1_full = bars + 3 * NS + 2 * NDO;  // commit: X1 raw
    uint64_t* e_full = x1_full + 1;           // commit: E' raw
    uint64_t* x1p_full = x1_full + 2;         // 128: X1 packed
    uint64_t* x2p_full = x1_full + 3;         // 128: X2' packed, X2 written to smem
    uint64_t* sum_full = x1_full + 4;         // 128: the chunk's sums
    uint64_t* rs_full = x1_full + 5;          // commit: state MMA
    uint64_t* rs_read = x1_full + 6;          // 128: state accumulator read
    uint64_t* sig_full = x1_full + 7;         // 128: Sig^T operand written
    uint64_t* r_full = x1_full + 8;           // 128: R operand, r, rho written
    uint64_t* da_full = x1_full + 9;          // commit: dV, dB, dA complete
    uint64_t* d_free = x1_full + 10;          // 128: dV, dB read
    uint64_t* da_free = x1_full + 11;         // 128: dA read
    uint64_t* drain = x1_full + 12;
    uint64_t* stg = x1_full + 13;             // [NS] 128: outputs of the stage staged
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);
    float* dgf_all = reinterpret_cast<float*>(smem + Cfg::OFF_DGF);  // [NS][C]
    float* sa_all = reinterpret_cast<float*>(smem + Cfg::OFF_SA);    // [NS][C]
    float* sums = reinterpret_cast<float*>(smem + Cfg::OFF_SUMS);    // [2][3][D]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x;
    const int N = prm.N;
    const int nch = (N + C - 1) / C;
    // chunk processed at step t (reverse token order)
    auto row_of = [&](int t) { return (nch - 1 - t) * C; };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&qkv_full[s], 1);
            mbar_init(&qkv_empty[s], 1);
            mbar_init(&phi_done[s], 256);
            mbar_init(&stg[s], 128);
        }
        for (int d = 0; d < NDO; ++d) {
            mbar_init(&do_full[d], 1);
            mbar_init(&do_empty[d], 1);
        }
        mbar_init(x1_full, 1);
        mbar_init(e_full, 1);
        mbar_init(x1p_full, 128);
        mbar_init(x2p_full, 128);
        mbar_init(sum_full, 128);
        mbar_init(rs_full, 1);
        mbar_init(rs_read, 128);
        mbar_init(sig_full, 128);
        mbar_init(r_full, 128);
        mbar_init(da_full, 1);
        mbar_init(d_free, 128);
        mbar_init(da_free, 128);
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
            for (int t = 0; t < nch; ++t) {
                const int s = t % NS, d = t % NDO;
                if (t >= NS && !mbar_wait(&qkv_empty[s], ((t / NS) - 1) & 1, abort_flag)) break;
                if (t >= NDO && !mbar_wait(&do_empty[d], ((t / NDO) - 1) & 1, abort_flag)) break;
                const int row = row_of(t);
                mbar_arrive_expect_tx(&qkv_full[s], 3 * Cfg::TILE);
                tma_load_3d(smem + Cfg::OFF_Q + s * Cfg::TILE, &prm.tm_q, &qkv_full[s], 0, row, head);
                tma_load_3d(smem + Cfg::OFF_K + s * Cfg::TILE, &prm.tm_k, &qkv_full[s], 0, row, head);
                tma_load_3d(smem + Cfg::OFF_V + s * Cfg::TILE, &prm.tm_v, &qkv_full[s], 0, row, head);
                mbar_arrive_expect_tx(&do_full[d], Cfg::TILE);
                tma_load_3d(smem + Cfg::OFF_DO + d * Cfg::TILE, &prm.tm_do, &do_full[d], 0, row, head);
                issued = t + 1;
            }
            for (int t = max(0, issued - NS); t < issued; ++t)
                mbar_wait_drain(&qkv_full[t % NS], (t / NS) & 1);
            for (int t = max(0, issued - NDO); t < issued; ++t)
                mbar_wait_drain(&do_full[t % NDO], (t / NDO) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t tX1 = tmem + Cfg::T_X1, tE = tmem + Cfg::T_E;
            const uint32_t tDV = tmem + Cfg::T_DV, tDB = tmem + Cfg::T_DB;
            const uint32_t tDA = tmem + Cfg::T_DA, tRS = tmem + Cfg::T_RS;
            const uint32_t zero = sbase + Cfg::OFF_ZERO;
            const uint32_t wl0 = sbase + Cfg::OFF_WL0, wl1 = sbase + Cfg::OFF_WL1;
            constexpr uint32_t idCC = idesc_bf16(C, C, 0, 0);     // B' A^T, (-V) dU^T
            constexpr uint32_t idCD_mn = idesc_bf16(C, D, 0, 1);  // B operand rows = K
            constexpr uint32_t idCD_k = idesc_bf16(C, D, 0, 0);   // B operand K-major
            constexpr uint32_t idMN = idesc_bf16(C, D, 1, 1);     // A and B MN-major
            const uint64_t sig_mn = desc_mn_base(sbase + Cfg::OFF_SIGT, D);
            const uint64_t r_mn = desc_mn_base(sbase + Cfg::OFF_R, D);
            const uint64_t r_k = desc_k_base(sbase + Cfg::OFF_R);
            auto qs = [&](int t) { return sbase + Cfg::OFF_Q + (t % NS) * Cfg::TILE; };
            auto ks = [&](int t) { return sbase + Cfg::OFF_K + (t % NS) * Cfg::TILE; };
            auto vs = [&](int t) { return sbase + Cfg::OFF_V + (t % NS) * Cfg::TILE; };
            auto dus = [&](int t) { return sbase + Cfg::OFF_DO + (t % NDO) * Cfg::TILE; };
            // X1 = B' A^T and E' = (-V) dU^T of step t
            auto x_raw = [&](int t) -> bool {
                if (!mbar_wait(&phi_done[t % NS], (t / NS) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint64_t kq = desc_k_base(qs(t)), kk = desc_k_base(ks(t));
                const uint64_t kv = desc_k_base(vs(t)), kdu = desc_k_base(dus(t));
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tX1, kk + kstep_k(C, k), kq + kstep_k(C, k), idCC, k > 0);
                umma_commit(x1_full);
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tE, kv + kstep_k(C, k), kdu + kstep_k(C, k), idCC, k > 0);
                umma_commit(e_full);
                return true;
            };
            bool ok = nch == 0 || x_raw(0);
            for (int t = 0; ok && t < nch; ++t) {
                const uint32_t q_s = qs(t), k_s = ks(t), v_s = vs(t), du_s = dus(t);
                const uint64_t mdu = desc_mn_base(du_s, C), kdu = desc_k_base(du_s);
                const uint64_t mq = desc_mn_base(q_s, C), mk = desc_mn_base(k_s, C);
                const uint64_t kk = desc_k_base(k_s), kv = desc_k_base(v_s);
                // RS += [A | 0]^T dU + [0 | -V]^T B' (this chunk), once the
                // previous value has been read out (or, at t = 0, set)
                if (!(ok = mbar_wait(rs_read, t & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C; k += 16) {
                    const uint32_t a = q_s + 128u * uint32_t(k);
                    umma_bf16(tRS, sdesc_sw128(a, zero - a, 1024), mdu + kstep_mn(k), idMN, 1);
                }
#pragma unroll
                for (int k = 0; k < C; k += 16) {
                    const uint32_t v = v_s + 128u * uint32_t(k);
                    umma_bf16(tRS, sdesc_sw128(zero, v - zero, 1024), mk + kstep_mn(k), idMN, 1);
                }
                umma_commit(rs_full);
                // dV = X1 dU + B' R  (+ c rho in the epilogue)
                if (!(ok = mbar_wait(r_full, t & 1, abort_flag))) break;
                if (!(ok = mbar_wait(x1p_full, t & 1, abort_flag))) break;
                if (t > 0 && !(ok = mbar_wait(d_free, (t - 1) & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C; k += 16)
                    umma_bf16_ts(tDV, tX1 + k / 2, mdu + kstep_mn(k), idCD_mn, k > 0);
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tDV, kk + kstep_k(C, k), r_mn + kstep_mn(k), idCD_mn, 1);
                // dB' = X2' A + (-V) R^T  (= -dB of the chunk, without r)
                if (!(ok = mbar_wait(x2p_full, t & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C; k += 16)
                    umma_bf16_ts(tDB, tE + k / 2, mq + kstep_mn(k), idCD_mn, k > 0);
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tDB, kv + kstep_k(C, k), r_k + kstep_k(D, k), idCD_k, 1);
                // dA = dU Sig^T + X2^T B'  (Sig: the state before this chunk)
                if (!(ok = mbar_wait(sig_full, t & 1, abort_flag))) break;
                if (t > 0 && !(ok = mbar_wait(da_free, (t - 1) & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tDA, kdu + kstep_k(C, k), sig_mn + kstep_mn(k), idCD_mn, k > 0);
#pragma unroll
                for (int k = 0; k < C; k += 16) {
                    const uint32_t a = k < 64 ? wl0 + 128u * uint32_t(k) : zero;
                    const uint32_t lbo = k < 64 ? wl1 - wl0 : wl1 + 128u * uint32_t(k) - zero;
                    umma_bf16(tDA, sdesc_sw128(a, lbo, 1024), mk + kstep_mn(k), idMN, 1);
                }
                umma_commit(da_full);
                umma_commit(&do_empty[t % NDO]);
                if (t + 1 < nch && !(ok = x_raw(t + 1))) break;
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < 10) {
        // per chunk: phi(q) in place and its row sums, phi(k) - c in place,
        // V negated, dU = dO / g in place and dg = -(dO . o) / g (two
        // threads per row)
        const int u = tid - 64;  // 0..255
        const int r = u >> 1, part = u & 1;
        const float* gb = prm.gbuf + size_t(head) * N;
        for (int t = 0; t < nch; ++t) {
            const int s = t % NS, d = t % NDO;
            const int row0 = row_of(t);
            const int nvalid = min(C, N - row0);
            const bool valid = r < nvalid;
            // this row's o and g, loaded while the tiles land
            const uint4* orow =
                reinterpret_cast<const uint4*>(prm.o_in + (size_t(head) * N + row0 + r) * D) + 4 * part;
            const float g = valid ? gb[row0 + r] : 1.f;
            uint4 ov[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) ov[j] = valid ? __ldg(orow + j) : make_uint4(0u, 0u, 0u, 0u);
            const bool landed = mbar_wait(&qkv_full[s], (t / NS) & 1, abort_flag) &&
                                mbar_wait(&do_full[d], (t / NDO) & 1, abort_flag);
            if (!named_bar_all(3, 256, landed)) break;
            uint8_t* qt = smem + Cfg::OFF_Q + s * Cfg::TILE;
            uint8_t* kt = smem + Cfg::OFF_K + s * Cfg::TILE;
            uint8_t* vt = smem + Cfg::OFF_V + s * Cfg::TILE;
            uint8_t* dot = smem + Cfg::OFF_DO + d * Cfg::TILE;
            if (u < 128) {
                phi_tile<PHI, C, D, 128>(qt, u, nvalid, false);
                sa_all[s * C + u] = tile_row_sum<C, D>(qt, u);
            } else {
                phi_tile<PHI, C, D, 128, true>(kt, u - 128, nvalid, true);
            }
            // -V (sign bits of the bf16 pairs)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4* p = reinterpret_cast<uint4*>(vt) + 4 * u + j;
                uint4 x = *p;
                x.x ^= 0x80008000u;
                x.y ^= 0x80008000u;
                x.z ^= 0x80008000u;
                x.w ^= 0x80008000u;
                *p = x;
            }
            float dotp = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 x = *reinterpret_cast<const uint4*>(dot + tile_chunk_off(C, r, 4 * part + j));
                const uint32_t a[4] = {x.x, x.y, x.z, x.w};
                const uint32_t bb[4] = {ov[j].x, ov[j].y, ov[j].z, ov[j].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 fa = unpack_bf16(a[e]), fb = unpack_bf16(bb[e]);
                    dotp = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, dotp));
                }
            }
            dotp += __shfl_xor_sync(0xffffffffu, dotp, 1);
            const float ginv = 1.f / g;
            const float dg = valid ? -dotp * ginv : 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4* px = reinterpret_cast<uint4*>(dot + tile_chunk_off(C, r, 4 * part + j));
                const uint4 x = *px;
                uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = unpack_bf16(w[e]);
                    w[e] = valid ? pack_bf16(f.x * ginv, f.y * ginv) : 0u;
                }
                *px = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (part == 0) dgf_all[s * C + r] = dg;
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
        }
    } else if (warp < 14) {
        // masks of X1 and E', and the chunk's sums z = sum_j b'_j,
        // r = sum_i a_i dg_i, rho = sum_i sa_i du_i
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int jrow = 32 * sp + lane;
        uint8_t* wl0 = smem + Cfg::OFF_WL0;
        uint8_t* wl1 = smem + Cfg::OFF_WL1;
        // sums: warp sp takes features 16sp..16sp+15; lane = 8 * rg + pair:
        // rows rg, rg + 4, ... of feature pair (16sp + 2 pair, + 1), then the
        // four row groups are added across lanes (fixed order)
        const int rg = lane >> 3, f0 = 16 * sp + 2 * (lane & 7);
        for (int t = 0; t < nch; ++t) {
            const int s = t % NS, d = t % NDO;
            const float* dgf = dgf_all + s * C;
            const float* sa = sa_all + s * C;
            if (!named_bar_all(1, 128, mbar_wait(x1_full, t & 1, abort_flag))) break;
            tc_fence_after();
            mask_pack_upper(tmem + lane_base + Cfg::T_X1, sp, jrow, kc != 0.f ? sa : nullptr);
            tc_fence_before();
            mbar_arrive(x1p_full);
            {
                const uint8_t* at = smem + Cfg::OFF_Q + s * Cfg::TILE;
                const uint8_t* bt = smem + Cfg::OFF_K + s * Cfg::TILE;
                const uint8_t* ut = smem + Cfg::OFF_DO + d * Cfg::TILE;
                float acc[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
                for (int jj = 0; jj < 32; ++jj) {
                    const int row = 4 * jj + rg;
                    const uint32_t off = tile_off(C, row, f0);
                    const float2 b2 = unpack_bf16(*reinterpret_cast<const uint32_t*>(bt + off));
                    const float2 a2 = unpack_bf16(*reinterpret_cast<const uint32_t*>(at + off));
                    const float2 u2 = unpack_bf16(*reinterpret_cast<const uint32_t*>(ut + off));
                    const float dg = dgf[row], sr = sa[row];
                    acc[0] += b2.x;
                    acc[1] += b2.y;
                    acc[2] = fmaf(a2.x, dg, acc[2]);
                    acc[3] = fmaf(a2.y, dg, acc[3]);
                    acc[4] = fmaf(sr, u2.x, acc[4]);
                    acc[5] = fmaf(sr, u2.y, acc[5]);
                }
#pragma unroll
                for (int i = 0; i < 6; ++i) {
                    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
                    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
                }
                if (rg == 0) {
                    float* out = sums + (t & 1) * 3 * D;
                    out[f0] = acc[0];
                    out[f0 + 1] = acc[1];
                    out[D + f0] = acc[2];
                    out[D + f0 + 1] = acc[3];
                    out[2 * D + f0] = acc[4];
                    out[2 * D + f0 + 1] = acc[5];
                }
                mbar_arrive(sum_full);
            }
            if (!named_bar_all(1, 128, mbar_wait(e_full, t & 1, abort_flag))) break;
            tc_fence_after();
            mask_split_e(tmem + lane_base + Cfg::T_E, sp, jrow, dgf, wl0, wl1);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(x2p_full);
        }
    } else if (warp < 18) {
        // state readout and the dV, dK, dQ epilogues
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int row = 32 * sp + lane;  // token row; row of the state accumulator
        const int e = tid - 448;         // 0..127
        uint8_t* sigt = smem + Cfg::OFF_SIGT;
        uint8_t* rt = smem + Cfg::OFF_R;
        float* zeta = reinterpret_cast<float*>(smem + Cfg::OFF_ZETA);  // [2][D]
        float* rn = reinterpret_cast<float*>(smem + Cfg::OFF_RN);      // [2][D]
        float* rho = reinterpret_cast<float*>(smem + Cfg::OFF_RHO);    // [2][D]
        const float* Sf = prm.S_fin + size_t(head) * prm.stride_S;
        const float* zf = prm.z_fin + size_t(head) * prm.stride_z;
        // RS starts at [0 ; S'^T] (the centred final state); the R operand of
        // step 0 is zero; zeta = z', r = rho = 0.  The zero block of the
        // state and dA operands is written here too: the first state MMA
        // waits for this group (rs_read).
        reinterpret_cast<uint4*>(smem + Cfg::OFF_ZERO)[e] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
            float v16[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v16[i] = row >= D ? Sf[size_t(c0 + i) * D + (row - D)] : 0.f;
            tmem_st16(tmem + lane_base + Cfg::T_RS + c0, v16);
            if (row < D) store_row16_bf16(rt, D, row, c0, v16);
        }
        tmem_wait_st();
        if (e < D) {
            zeta[e] = zf[e];
            rn[e] = 0.f;
            rho[e] = 0.f;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(2, 128);
        mbar_arrive(rs_read);
        mbar_arrive(r_full);

        for (int t = 0; t < nch; ++t) {
            const int s = t % NS;
            const int b = t & 1;
            uint8_t* qt = smem + Cfg::OFF_Q + s * Cfg::TILE;
            uint8_t* kt = smem + Cfg::OFF_K + s * Cfg::TILE;
            uint8_t* vt = smem + Cfg::OFF_V + s * Cfg::TILE;
            // the state after this chunk's MMA: rows 64.. are Sig^T, the
            // state before the chunk (read by this chunk's dA); rows 0..63
            // are R with this chunk (the next chunk's R operand)
            if (!named_bar_all(2, 128, mbar_wait(rs_full, t & 1, abort_flag))) break;
            tc_fence_after();
            // (warps 2, 3 of the group hold rows 64.., so the branches on
            // row >= D are warp-uniform, as tcgen05.ld requires)
            uint32_t pk[D / 2];
            if (row >= D) {
                // a constant along the features of a value column only moves
                // dA along the all-ones direction, which the epilogue restores
                // exactly: remove the column's mean before rounding to bf16
                float m = 0.f;
                if (kc != 0.f) {
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 16) {
                        float v16[16];
                        tmem_ld16(tmem + lane_base + Cfg::T_RS + c0, v16);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) m += v16[i];
                    }
                    m *= 1.f / D;
                }
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 16) {
                    float v16[16];
                    tmem_ld16(tmem + lane_base + Cfg::T_RS + c0, v16);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v16[i] -= m;
                    store_row16_bf16(sigt, D, row - D, c0, v16);
                }
                tc_fence_before();
                mbar_arrive(rs_read);
                fence_proxy_async_smem();
            } else {
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 16) {
                    float v16[16];
                    tmem_ld16(tmem + lane_base + Cfg::T_RS + c0, v16);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i) pk[c0 / 2 + i] = pack_bf16(v16[2 * i], v16[2 * i + 1]);
                }
                tc_fence_before();
                mbar_arrive(rs_read);
            }
            mbar_arrive(sig_full);
            // the chunk's products are complete: the next step's R operand
            // may be written and the stage's tiles reused as staging
            const bool ready = mbar_wait(da_full, t & 1, abort_flag) &&
                               mbar_wait(sum_full, t & 1, abort_flag);
            if (!named_bar_all(2, 128, ready)) break;
            tc_fence_after();
            if (row < D) {
#pragma unroll
                for (int q = 0; q < D / 8; ++q)
                    *reinterpret_cast<uint4*>(rt + tile_chunk_off(D, row, q)) =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
            {
                const float* cs = sums + b * 3 * D;  // z', r, rho of this chunk
                if (e < D) {
                    zeta[(b ^ 1) * D + e] = zeta[b * D + e] - cs[e];
                    rn[(b ^ 1) * D + e] = rn[b * D + e] + cs[D + e];
                } else {
                    const int f = e - D;
                    rho[(b ^ 1) * D + f] = rho[b * D + f] + cs[2 * D + f];
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(2, 128);
            tc_fence_before();
            mbar_arrive(r_full);
            // dV (+ c rho) and dK = (r - dB') * phi'(k), staged over the v and
            // k tiles
            const float* r_now = rn + b * D;
            const float* rho_now = rho + b * D;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 16) {
                float dv16[16], db16[16];
                tmem_ld16(tmem + lane_base + Cfg::T_DV + c0, dv16);
                tmem_ld16(tmem + lane_base + Cfg::T_DB + c0, db16);
                tmem_wait_ld();
                float b8a[8], b8b[8];
                load_chunk8(kt, C, row, c0 >> 3, b8a);
                load_chunk8(kt, C, row, (c0 >> 3) + 1, b8b);
                float dk16[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    dk16[i] = (r_now[c0 + i] - db16[i]) * dphi_from_phi<PHI>(b8a[i] + kc);
                    dk16[8 + i] = (r_now[c0 + 8 + i] - db16[8 + i]) * dphi_from_phi<PHI>(b8b[i] + kc);
                }
                if (kc != 0.f) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) dv16[i] = fmaf(kc, rho_now[c0 + i], dv16[i]);
                }
                // this thread's row of B' is read before it is overwritten
                store_row16_bf16(vt, C, row, c0, dv16);
                store_row16_bf16(kt, C, row, c0, dk16);
            }
            tc_fence_before();
            mbar_arrive(d_free);
            // dQ: T = dA + dg zeta (zeta: state before the chunk), then the
            // all-ones component from <dA_i, a_i> = 0, times phi'(q)
            const float dg = dgf_all[s * C + row];
            const float* z_prev = zeta + (b ^ 1) * D;
            float tcoef = 0.f;
            if (kc != 0.f) {
                float dot = 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 16) {
                    float av[16];
                    tmem_ld16(tmem + lane_base + Cfg::T_DA + c0, av);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float a8[8];
                        load_chunk8(qt, C, row, (c0 >> 3) + h, a8);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dot = fmaf(fmaf(dg, z_prev[c0 + 8 * h + i], av[8 * h + i]), a8[i], dot);
                    }
                }
                tcoef = -dot / sa_all[s * C + row];
            }
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 16) {
                float av[16];
                tmem_ld16(tmem + lane_base + Cfg::T_DA + c0, av);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float a8[8];
                    load_chunk8(qt, C, row, (c0 >> 3) + h, a8);
                    uint32_t w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int f = c0 + 8 * h + 2 * i;
                        const float d0 = fmaf(dg, z_prev[f], av[8 * h + 2 * i]) + kc * tcoef;
                        const float d1 = fmaf(dg, z_prev[f + 1], av[8 * h + 2 * i + 1]) + kc * tcoef;
                        w[i] = pack_bf16(d0 * dphi_from_phi<PHI>(a8[2 * i]),
                                         d1 * dphi_from_phi<PHI>(a8[2 * i + 1]));
                    }
                    *reinterpret_cast<uint4*>(qt + tile_chunk_off(C, row, (c0 >> 3) + h)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            tc_fence_before();
            mbar_arrive(da_free);
            fence_proxy_async_smem();
            mbar_arrive(&stg[s]);
        }
    } else if (warp == 18) {
        // TMA stores of the staged dQ, dK, dV rows; the stage is free once
        // they have been read
        if (lane == 0) {
            for (int t = 0; t < nch; ++t) {
                const int s = t % NS;
                if (!mbar_wait(&stg[s], (t / NS) & 1, abort_flag)) break;
                const int row0 = row_of(t);
                tma_store_3d(&prm.tm_dq, smem + Cfg::OFF_Q + s * Cfg::TILE, 0, row0, head);
                tma_store_3d(&prm.tm_dk, smem + Cfg::OFF_K + s * Cfg::TILE, 0, row0, head);
                tma_store_3d(&prm.tm_dv, smem + Cfg::OFF_V + s * Cfg::TILE, 0, row0, head);
                bulk_commit();
                bulk_wait_read0();
                mbar_arrive(&qkv_empty[s]);
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
