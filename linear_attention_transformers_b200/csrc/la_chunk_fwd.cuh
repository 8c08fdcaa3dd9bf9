// la_chunk_fwd.cuh — chunked linear-attention forward on sm_100a tensor cores.
//
// One kernel template, three modes, one thread block per (head, segment):
//
//  CAUSAL  the causal forward over a run of C-token chunks.  Per chunk c,
//          with A = phi(Q_c), B = phi(K_c) and the state S (D x D), z (D) of
//          every earlier token:
//              P   = A B^T                           (C x C)
//              [num | den] = A [S | z] + (P . tril) [V_c | 1]
//              O_c = num / den
//              [S | z] += B^T [V_c | 1]              (fp32 accumulators in TMEM)
//          Inside a chunk this is the quadratic form, across chunks the
//          associativity reorder (QK^T)V = Q(K^T V) of "Efficient Transformers
//          Survey", Proposition "Linear Attention via Kernel Decomposition"
//          (Intuition), with S and z carried chunk to chunk as in its "Why It
//          Matters" paragraph.
//  REDUCE  only [S | z] += B^T [V | 1] over the segment; writes the segment's
//          (S, z) record (non-causal totals, causal segment sums).
//  QUERY   O = A S / (A z) against a fixed (S, z) record (the non-causal
//          query pass: "each attention output costs O(md)").
//
// The denominator rides in the same MMAs as the numerator: the B operands
// are 144 columns wide, [S | z_hi z_lo 0..] (z split into two bf16 terms)
// and [V | 1] (V followed by a constant atom whose first column is ones), so
// a chunk takes 8 (A B^T) + 8 (A [S|z]) + 4 (state) + 4 (P~ [V|1]) = 24
// tcgen05.mma instructions; below N = 128 an instruction costs about the
// same whatever its width, so the count is what matters.
//
// Warp roles (18 warps): a TMA producer warp; a single-thread tcgen05.mma
// issuer; 8 feature-map warps that apply phi in place to the landed tiles;
// a "P" warpgroup that masks P and writes it back as a bf16 operand; an "O"
// warpgroup that converts the running state into the next chunk's bf16
// operand and forms O = num / den, stored with TMA.  The O accumulator is
// double-buffered in TMEM so the next chunk's products start while the
// current O is being read; the serial chain per chunk is state conversion ->
// (A [S|z], state) MMAs.  All handshakes are mbarriers with bounded waits.

#pragma once

#include "la_common.cuh"
#include "la_sm100.cuh"
#include "la_tile_ops.cuh"

namespace la {

enum : int { MODE_CAUSAL = 0, MODE_REDUCE = 1, MODE_QUERY = 2 };

struct ChunkParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_o;  // 3-D (D, N, heads), box (64, C, 1), bf16
    int N;                                // tokens per head
    int seg_len;                          // tokens per segment (multiple of C)
    int nseg;                             // segments per head
    // Initial / fixed state: record = S [D][D] row-major (row = key feature)
    // followed by z [D], float32.  Record index = head (in_per_head) or block.
    const float* state_in;
    int in_per_head;
    // Output state: S to S_out + idx*stride_S, z to z_out + idx*stride_z,
    // where idx = head (CAUSAL: written by the head's last segment; S_out may
    // be null) or block (REDUCE).
    float* S_out;
    float* z_out;
    int64_t stride_S, stride_z;
    // Optional [heads][N] output of the denominators g_i = phi(q_i) . z_i
    // (CAUSAL and QUERY), which lets the backward skip recomputing them.
    float* g_out;
    // Optional outputs phi(q), phi(k) (same layout as q, k): the bf16 tiles
    // the products read, stored by TMA (D = 64 CAUSAL kernel, store_phi != 0).
    CUtensorMap tm_pq, tm_pk;
    int store_phi;
    // REDUCE: sum phi(k) - phi_center (the centred state the backward's dQ
    // products use) instead of phi(k)
    int center;
    // query heads per key/value head (grouped-query attention; 1 = one each):
    // query head `head` reads k, v head head / kv_group, and the final state
    // (per key/value head) is written by the group's first query head
    int kv_group;
    // decay factor per head (read by the DECAY kernels only; causal)
    DecayArg dec;
};


// Shared-memory and TMEM plan of the kernel below (head size 128, 64-token
// chunks).  Stage tiles live in 19 slots of one [C][64] bf16 atom (8 KB).
// Slot 18 is the ones atom E; stage s puts its two V atoms at slots
// 18 - 2 l_s and 18 - l_s (l = 1, 3, 7), so V atom 0, V atom 1 and E are
// equally spaced and [V | 1] is a single MN-major operand whose atom stride
// (LBO) is l_s slots; Q and K fill the remaining adjacent slot pairs.
template <int D, int C>
struct ChunkCfg {
    static_assert(D == 128 && C == 64, "laid out for head size 128, 64-token chunks");
    static constexpr int NSTAGE = 3;
    static constexpr int NO = 2;            // O buffers in TMEM
    static constexpr int ATOM = C * 128;    // one [C][64] bf16 atom
    static constexpr int NSLOT = 19;
    static constexpr int E_SLOT = 18;
    __host__ __device__ static constexpr int q_slot(int s) { return s == 0 ? 0 : (s == 1 ? 5 : 9); }
    __host__ __device__ static constexpr int k_slot(int s) { return s == 0 ? 2 : (s == 1 ? 7 : 13); }
    __host__ __device__ static constexpr int v_l(int s) { return s == 0 ? 1 : (s == 1 ? 3 : 7); }
    __host__ __device__ static constexpr int v_slot(int s, int a) {
        return E_SLOT - (2 - a) * v_l(s);
    }
    // [D][192] row tile: S (columns 0..127), z_hi, z_lo (columns 128, 129)
    static constexpr int OFF_SX = NSLOT * ATOM;
    static constexpr int OFF_PT = OFF_SX + 3 * D * 128;  // [C][C] masked P
    static constexpr int OFF_OST = OFF_PT + C * C * 2;   // [C][D] output staging
    static constexpr int OFF_BAR = OFF_OST + C * D * 2;
    static constexpr int NBAR = 3 * NSTAGE + 7 + 2 * NO;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
    // TMEM columns: P, O[NO] (D + 16 each: numerator, then the two halves of
    // the denominator), [S | z] (D + 16)
    static constexpr int T_P = 0;
    static constexpr int T_O = C;
    static constexpr int T_S = C + NO * (D + 16);
    static constexpr int T_Z = T_S + D;
    static constexpr int T_COLS = 512;
    static_assert(T_Z + 16 <= T_COLS, "TMEM budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

constexpr int kChunkThreads = 576;  // producer, MMA, 8 phi warps, P and O warpgroups

// DECAY: the decayed recurrence, arranged as in chunk_fwd64_kernel (row
// factors gamma^(t+1-m) on queries and gamma^(m-1-j) on keys; the state
// accumulator rescaled in TMEM once per chunk; REDUCE decayed to the
// segment's end).
template <int D, int C, int PHI, int MODE, bool DECAY = false>
__global__ void __launch_bounds__(kChunkThreads, 1)
chunk_fwd_kernel(const __grid_constant__ ChunkParams prm) {
    static_assert(!DECAY || MODE != MODE_QUERY, "decay is causal");
    using namespace sm100;
    using Cfg = ChunkCfg<D, C>;
    constexpr int NS = Cfg::NSTAGE, NO = Cfg::NO;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;                // TMA landed                 (1 + tx)
    uint64_t* phi_done = bars + NS;       // phi applied                (256)
    uint64_t* empty = bars + 2 * NS;      // MMAs done with the stage   (commit)
    uint64_t* p_full = bars + 3 * NS;     // P = A B^T in TMEM          (commit)
    uint64_t* p_free = p_full + 1;        // P read by the P group      (128)
    uint64_t* pt_full = p_full + 2;       // masked P in smem           (128)
    uint64_t* pt_free = p_full + 3;       // masked P consumed          (commit)
    uint64_t* s_full = p_full + 4;        // state operand written      (128)
    uint64_t* s_done = p_full + 5;        // A [S|z], state update done (commit)
    uint64_t* drain = p_full + 6;         // every MMA finished         (commit)
    uint64_t* o_full = p_full + 7;        // [NO] O complete            (commit)
    uint64_t* o_free = o_full + NO;       // [NO] O read                (128)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x / prm.nseg;
    // grouped key/value heads: the k, v head this query head reads, and
    // whether it writes that head's final state (the group's first one does)
    const int kv_head = kv_head_of(head, prm.kv_group);
    const bool state_writer = writes_kv_state(head, prm.kv_group);
    const int seg = blockIdx.x % prm.nseg;
    const int tok0 = seg * prm.seg_len;
    const int tok1 = min(prm.N, tok0 + prm.seg_len);
    const int nchunks = (tok1 - tok0 + C - 1) / C;
    const float* st_in = prm.state_in
                             ? prm.state_in + size_t(prm.in_per_head ? head : blockIdx.x) *
                                                  size_t(D * D + D)
                             : nullptr;
    float lg = 0.f;  // log2(gamma) of this head
    if constexpr (DECAY) lg = log2f(decay_of(prm.dec, head));

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&phi_done[s], 256);
            mbar_init(&empty[s], 1);
        }
        mbar_init(p_full, 1);
        mbar_init(p_free, 128);
        mbar_init(pt_full, 128);
        mbar_init(pt_free, 1);
        mbar_init(s_full, 128);
        mbar_init(s_done, 1);
        mbar_init(drain, 1);
        for (int b = 0; b < NO; ++b) {
            mbar_init(&o_full[b], 1);
            mbar_init(&o_free[b], 128);
        }
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

    constexpr bool kQ = MODE != MODE_REDUCE;
    constexpr bool kKV = MODE != MODE_QUERY;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            if (kQ) tma_prefetch_desc(&prm.tm_q);
            if (kKV) {
                tma_prefetch_desc(&prm.tm_k);
                tma_prefetch_desc(&prm.tm_v);
            }
            constexpr uint32_t bytes = 2 * Cfg::ATOM * ((kQ ? 1 : 0) + (kKV ? 2 : 0));
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                if (c >= NS && !mbar_wait(&empty[s], ((c / NS) - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], bytes);
                const int row = tok0 + c * C;
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    if (kQ)
                        tma_load_3d(smem + (Cfg::q_slot(s) + a) * Cfg::ATOM, &prm.tm_q, &full[s],
                                    a * 64, row, head);
                    if (kKV) {
                        tma_load_3d(smem + (Cfg::k_slot(s) + a) * Cfg::ATOM, &prm.tm_k, &full[s],
                                    a * 64, row, kv_head);
                        tma_load_3d(smem + Cfg::v_slot(s, a) * Cfg::ATOM, &prm.tm_v, &full[s],
                                    a * 64, row, kv_head);
                    }
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
            constexpr uint32_t idP = idesc_bf16(C, C, 0, 0);       // A B^T
            constexpr uint32_t idO = idesc_bf16(C, D + 16, 0, 1);  // A [S|z] ; P~ [V|1]
            constexpr uint32_t idS = idesc_bf16(D, D + 16, 1, 1);  // B^T [V|1]
            const uint64_t dSx = desc_mn_base(sbase + Cfg::OFF_SX, D);
            const uint64_t dPt = desc_k_base(sbase + Cfg::OFF_PT);
            const bool has_init = st_in != nullptr;
            auto stage_q = [&](int s) { return desc_k_base(sbase + Cfg::q_slot(s) * Cfg::ATOM); };
            auto stage_k = [&](int s) { return desc_k_base(sbase + Cfg::k_slot(s) * Cfg::ATOM); };
            auto stage_kmn = [&](int s) {
                return desc_mn_base(sbase + Cfg::k_slot(s) * Cfg::ATOM, C);
            };
            // [V | 1]: V atom 0, V atom 1 and the ones atom, l_s slots apart
            auto stage_vx = [&](int s) {
                return sdesc_sw128(sbase + Cfg::v_slot(s, 0) * Cfg::ATOM,
                                   uint32_t(Cfg::v_l(s) * Cfg::ATOM), 1024);
            };
            bool ok = true;
            // P = A B^T for chunk c (one TMEM buffer: the P group has read
            // chunk c-1's long before chunk c's is issued)
            auto p_part = [&](int c) -> bool {
                const int s = c % NS;
                if (!mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag)) return false;
                if (c >= 1 && !mbar_wait(p_free, (c - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint64_t dq = stage_q(s), dk = stage_k(s);
                const uint32_t tP = tmem + Cfg::T_P;
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tP, dq + kstep_k(C, k), dk + kstep_k(C, k), idP, k > 0);
                umma_commit(p_full);
                return true;
            };
            if (MODE == MODE_CAUSAL) {
                if (nchunks > 0) ok = p_part(0);
                for (int c = 0; ok && c < nchunks; ++c) {
                    const int s = c % NS, bo = c % NO;
                    const uint32_t tO = tmem + Cfg::T_O + bo * (D + 16);
                    if (!(ok = mbar_wait(s_full, c & 1, abort_flag))) break;
                    if (c >= NO && !(ok = mbar_wait(&o_free[bo], ((c / NO) - 1) & 1, abort_flag)))
                        break;
                    tc_fence_after();
                    const uint64_t dq = stage_q(s), dkm = stage_kmn(s), dvx = stage_vx(s);
#pragma unroll
                    for (int k = 0; k < D; k += 16)
                        umma_bf16(tO, dq + kstep_k(C, k), dSx + kstep_mn(k), idO, k > 0);
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16(tmem + Cfg::T_S, dkm + kstep_mn(k), dvx + kstep_mn(k), idS,
                                  (c > 0 || has_init || k > 0) ? 1u : 0u);
                    umma_commit(s_done);
                    if (c + 1 < nchunks && !(ok = p_part(c + 1))) break;
                    if (!(ok = mbar_wait(pt_full, c & 1, abort_flag))) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16(tO, dPt + kstep_k(C, k), dvx + kstep_mn(k), idO, 1);
                    umma_commit(&o_full[bo]);
                    umma_commit(pt_free);
                    umma_commit(&empty[s]);
                }
            } else if (MODE == MODE_QUERY) {
                ok = mbar_wait(s_full, 0, abort_flag);
                for (int c = 0; ok && c < nchunks; ++c) {
                    const int s = c % NS, bo = c % NO;
                    const uint32_t tO = tmem + Cfg::T_O + bo * (D + 16);
                    if (!(ok = mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                    if (c >= NO && !(ok = mbar_wait(&o_free[bo], ((c / NO) - 1) & 1, abort_flag)))
                        break;
                    tc_fence_after();
                    const uint64_t dq = stage_q(s);
#pragma unroll
                    for (int k = 0; k < D; k += 16)
                        umma_bf16(tO, dq + kstep_k(C, k), dSx + kstep_mn(k), idO, k > 0);
                    umma_commit(&o_full[bo]);
                    umma_commit(&empty[s]);
                }
            } else {  // REDUCE
                ok = mbar_wait(s_full, 0, abort_flag);
                for (int c = 0; ok && c < nchunks; ++c) {
                    const int s = c % NS;
                    if (!(ok = mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                    tc_fence_after();
                    const uint64_t dkm = stage_kmn(s), dvx = stage_vx(s);
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16(tmem + Cfg::T_S, dkm + kstep_mn(k), dvx + kstep_mn(k), idS,
                                  (c > 0 || k > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(s_done);
            }
            // every MMA issued above completes before TMEM is released
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < 10) {
        // ------------------------------------------------ feature-map warps
        const int u = tid - 64;  // 0..255
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            if (!mbar_wait(&full[s], (c / NS) & 1, abort_flag)) break;
            uint8_t* qt = smem + Cfg::q_slot(s) * Cfg::ATOM;
            uint8_t* kt = smem + Cfg::k_slot(s) * Cfg::ATOM;
            const int nvalid = min(C, tok1 - (tok0 + c * C));
            if (DECAY && MODE == MODE_CAUSAL) {
                const float m = 0.5f * float(nvalid);
                if (u < 128)
                    phi_tile_scaled<PHI, C, D, 128>(qt, u, nvalid, false, lg, 1.f, 1.f - m);
                else
                    phi_tile_scaled<PHI, C, D, 128>(kt, u - 128, nvalid, true, lg, -1.f, m - 1.f);
            } else if (DECAY) {  // REDUCE: decayed to the segment's end
                phi_tile_scaled<PHI, C, D, 256>(kt, u, nvalid, true, lg, -1.f,
                                                float(tok1 - tok0 - 1 - c * C));
            } else if (MODE == MODE_CAUSAL) {
                if (u < 128)
                    phi_tile<PHI, C, D, 128>(qt, u, nvalid, false);
                else
                    phi_tile<PHI, C, D, 128>(kt, u - 128, nvalid, true);
            } else if (MODE == MODE_QUERY) {
                phi_tile<PHI, C, D, 256>(qt, u, nvalid, false);
            } else if (prm.center) {
                phi_tile<PHI, C, D, 256, true>(kt, u, nvalid, true);
            } else {
                phi_tile<PHI, C, D, 256>(kt, u, nvalid, true);
            }
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
        }
    } else if (warp < 14) {
        // ----------------------------------------- P group: mask P -> bf16
        if (MODE == MODE_CAUSAL) {
            const int sp = warp & 3;
            const uint32_t lane_base = uint32_t(32 * sp) << 16;
            const int irow = acc_row<C>(sp, lane);
            uint8_t* pt = smem + Cfg::OFF_PT;
            for (int c = 0; c < nchunks; ++c) {
                bool ok = c == 0 || mbar_wait(pt_free, (c - 1) & 1, abort_flag);
                ok = ok && mbar_wait(p_full, c & 1, abort_flag);
                if (!named_bar_all(1, 128, ok)) break;
                tc_fence_after();
#pragma unroll 1
                for (int j0 = 0; j0 < C; j0 += 32) {
                    float pv[32];
                    tmem_load<32>(tmem + lane_base + Cfg::T_P + j0, pv);
                    if (irow >= 0) {
#pragma unroll
                        for (int t = 0; t < 32; ++t)
                            if (j0 + t > irow) pv[t] = 0.f;
                        store_row_bf16<32>(pt, C, irow, j0, pv);
                    }
                }
                tc_fence_before();
                mbar_arrive(p_free);
                fence_proxy_async_smem();
                mbar_arrive(pt_full);
            }
        }
    } else {
        // ------------------------- O group: state operand, O = num / den
        const int e = tid - 448;  // 0..127
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int irow = acc_row<C>(sp, lane);  // token row of this thread (or -1)
        const int frow = acc_row<D>(sp, lane);  // state row of this thread (or -1)
        uint8_t* sx = smem + Cfg::OFF_SX;
        uint8_t* eop = smem + Cfg::E_SLOT * Cfg::ATOM;
        uint8_t* ost = smem + Cfg::OFF_OST;

        // ---- constant ones atom E (column 0) and the zero z atom of Sx
        for (int r = e; r < C + D; r += 128) {
            float v8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            const float z8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (r < C) {
                v8[0] = 1.f;
                for (int q = 0; q < 8; ++q) store_row_bf16<8>(eop, C, r, 8 * q, q == 0 ? v8 : z8);
            } else {
                for (int q = 0; q < 8; ++q) store_row_bf16<8>(sx, D, r - C, D + 8 * q, z8);
            }
        }
        named_bar_sync(2, 128);  // zero z atom written before its columns 128/129 below
        // ---- z into columns 128 (z_hi) and 129 (z_lo) of Sx, zeros after
        auto put_z = [&](float zf) {
            float z16[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) z16[t] = 0.f;
            z16[0] = zf;
            z16[1] = zf - __bfloat162float(__float2bfloat16_rn(zf));
            store_row_bf16<16>(sx, D, frow, D, z16);
        };
        // decay: the initial state enters as gamma^(m_0) S_0
        float s0 = 1.f;
        if constexpr (DECAY) s0 = exp2f(lg * 0.5f * float(min(C, tok1 - tok0)));
        // ---- initial state: bf16 operand (+ TMEM accumulator in CAUSAL mode)
        if (MODE != MODE_REDUCE) {
            // one read of the record row feeds the operand and the accumulator
            const bool to_tmem = MODE == MODE_CAUSAL && st_in != nullptr;
            load_record_row<D>(st_in, frow, s0, sx, tmem + lane_base + Cfg::T_S, to_tmem);
            const float z0 = (st_in && frow >= 0) ? s0 * st_in[size_t(D) * D + frow] : 0.f;
            if (frow >= 0) put_z(z0);
            if (to_tmem) {
                float z16[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) z16[t] = t == 0 ? z0 : 0.f;
                tmem_st16(tmem + lane_base + Cfg::T_Z, z16);
                tmem_wait_st();
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(s_full);

        if (MODE == MODE_REDUCE) {
            if (named_bar_all(2, 128, mbar_wait(s_done, 0, abort_flag))) {
                tc_fence_after();
                const size_t idx = blockIdx.x;
                for (int cc = 0; cc < D; cc += 16) {
                    float v16[16];
                    tmem_load<16>(tmem + lane_base + Cfg::T_S + cc, v16);
                    if (frow >= 0) {
                        float4* dst = reinterpret_cast<float4*>(
                            prm.S_out + idx * prm.stride_S + size_t(frow) * D + cc);
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            dst[t] = make_float4(v16[4 * t], v16[4 * t + 1], v16[4 * t + 2],
                                                 v16[4 * t + 3]);
                    }
                }
                float z16[16];
                tmem_load<16>(tmem + lane_base + Cfg::T_Z, z16);
                if (frow >= 0) prm.z_out[idx * prm.stride_z + frow] = z16[0];
            }
        } else {
            for (int c = 0; c < nchunks; ++c) {
                const int bo = c % NO;
                const int row0 = tok0 + c * C;
                if (MODE == MODE_CAUSAL) {
                    // ---- S_{<=c} -> bf16 operand of chunk c+1 (and the final state)
                    if (!named_bar_all(2, 128, mbar_wait(s_done, c & 1, abort_flag))) break;
                    tc_fence_after();
                    const bool last = c == nchunks - 1;
                    const bool write_final = last && seg == prm.nseg - 1 && prm.S_out != nullptr &&
                                             state_writer;
                    const size_t sidx = size_t(kv_head);
                    if (DECAY && (!last || write_final)) {
                        // accumulator gamma^(m-L) S -> gamma^(m') S for the
                        // next chunk (operand and accumulator), S at the end
                        const int L = min(C, tok1 - row0);
                        const float m = 0.5f * float(L);
                        const float f = last ? exp2f(lg * (float(L) - m))
                                             : exp2f(lg * (float(L) - m +
                                                           0.5f * float(min(C, tok1 - row0 - C))));
#pragma unroll 1
                        for (int v0 = 0; v0 < D; v0 += 16) {
                            float sv[16];
                            tmem_load<16>(tmem + lane_base + Cfg::T_S + v0, sv);
#pragma unroll
                            for (int t = 0; t < 16; ++t) sv[t] *= f;
                            if (!last) tmem_st16(tmem + lane_base + Cfg::T_S + v0, sv);
                            if (frow >= 0) {
                                if (last)
                                    for (int t = 0; t < 16; ++t)
                                        prm.S_out[sidx * prm.stride_S + size_t(frow) * D + v0 + t] =
                                            sv[t];
                                else
                                    store_row_bf16<16>(sx, D, frow, v0, sv);
                            }
                        }
                        float zv[16];
                        tmem_load<16>(tmem + lane_base + Cfg::T_Z, zv);
#pragma unroll
                        for (int t = 0; t < 16; ++t) zv[t] *= f;
                        if (!last) tmem_st16(tmem + lane_base + Cfg::T_Z, zv);
                        if (frow >= 0) {
                            if (!last)
                                put_z(zv[0]);
                            else if (prm.z_out)
                                prm.z_out[sidx * prm.stride_z + frow] = zv[0];
                        }
                        tmem_wait_st();
                    } else if (!last || write_final) {
                        // 32 state columns per TMEM round trip, z with the first
                        float zv[16];
                        sm100::tmem_ld16(tmem + lane_base + Cfg::T_Z, zv);
#pragma unroll 1
                        for (int v0 = 0; v0 < D; v0 += 32) {
                            float sv[32];
                            tmem_load<32>(tmem + lane_base + Cfg::T_S + v0, sv);
                            if (frow >= 0) {
                                store_row_bf16<32>(sx, D, frow, v0, sv);
                                if (write_final) {
                                    // S_out, its head stride and D * 4 are
                                    // multiples of 16 bytes
                                    float4* dst = reinterpret_cast<float4*>(
                                        prm.S_out + sidx * prm.stride_S + size_t(frow) * D + v0);
#pragma unroll
                                    for (int t = 0; t < 8; ++t)
                                        dst[t] = make_float4(sv[4 * t], sv[4 * t + 1],
                                                             sv[4 * t + 2], sv[4 * t + 3]);
                                }
                            }
                        }
                        if (frow >= 0) {
                            put_z(zv[0]);
                            if (write_final && prm.z_out)
                                prm.z_out[sidx * prm.stride_z + frow] = zv[0];
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(s_full);
                }
                // ---- O = num / den -> smem -> TMA store
                if (!named_bar_all(2, 128, mbar_wait(&o_full[bo], (c / NO) & 1, abort_flag))) break;
                tc_fence_after();
                if (e == 0) bulk_wait_read0();
                named_bar_sync(2, 128);
                const uint32_t tO = tmem + lane_base + Cfg::T_O + bo * (D + 16);
                // the denominator columns ride along with the first 32
                // numerator columns (one TMEM round trip for both)
                float oz[16], ov[32];
                sm100::tmem_ld16(tO + D, oz);
                sm100::tmem_ld16(tO, ov);
                sm100::tmem_ld16(tO + 16, ov + 16);
                sm100::tmem_wait_ld();
                const float inv = 1.f / (oz[0] + oz[1]);
                if (prm.g_out && irow >= 0 && row0 + irow < tok1)
                    prm.g_out[size_t(head) * prm.N + row0 + irow] = oz[0] + oz[1];
#pragma unroll 1
                for (int v0 = 0; v0 < D; v0 += 32) {
                    if (v0 > 0) tmem_load<32>(tO + v0, ov);
                    if (irow >= 0) {
#pragma unroll
                        for (int t = 0; t < 32; ++t) ov[t] *= inv;
                        store_row_bf16<32>(ost, C, irow, v0, ov);
                    }
                }
                tc_fence_before();
                mbar_arrive(&o_free[bo]);
                fence_proxy_async_smem();
                named_bar_sync(2, 128);
                if (e == 0) {
#pragma unroll
                    for (int a = 0; a < D / 64; ++a)
                        tma_store_3d(&prm.tm_o, ost + a * C * 128, a * 64, row0, head);
                    bulk_commit();
                }
            }
            if (e == 0) bulk_wait0();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::T_COLS);
}

}  // namespace la
