// la_chunk_fwd64.cuh — the chunked forward for head size D = 64 (C = 128).
//
// Same three modes and warp roles as la_chunk_fwd.cuh, with the state kept
// transposed and augmented so that every product runs as one M = 128 MMA
// with no 16-wide side products (tcgen05.mma costs a fixed ~60 cycles per
// instruction below N = 128 on this part, so instruction count is what
// matters):
//
//   state accumulator  T = [V | 1]^T B        (M = 128: rows 0..63 = S^T,
//                                              row 64 = z^T; K = tokens)
//   state operand      Sx = [S^T ; z_hi ; z_lo ; 0]    (80 x 64, bf16)
//   output accumulator O = A Sx^T + (P . tril) [V | 1] (N = 80: columns
//                                              0..63 numerator, 64..65 the
//                                              two halves of the denominator)
//
// The masked P~ is packed to bf16 in place over P in TMEM by the P warpgroup
// and read back by tcgen05.mma with A from TMEM, so it never touches shared
// memory.  "[V | 1]" is the V tile followed, at a per-stage descriptor stride, by one
// constant 64-column atom whose first column is ones; the same atom serves as
// extra M rows (state) and extra N columns (output).  Per chunk: 4 + 4 + 8 +
// 8 = 24 MMAs (A B^T, A Sx^T, [V|1]^T B, P [V|1]).  The mathematics is the
// one of la_chunk_fwd.cuh ("Efficient Transformers Survey", Proposition
// "Linear Attention via Kernel Decomposition": S, z as running sums, O as
// the normalised query).
#pragma once

#include "la_chunk_fwd.cuh"

namespace la {

struct Chunk64Cfg {
    static constexpr int C = 128, D = 64;
    static constexpr int NSTAGE = 3;
    static constexpr int TILE = C * D * 2;  // 16 KB
    static constexpr int STAGE = 3 * TILE;  // Q, K, V
    static constexpr int OFF_ONES = NSTAGE * STAGE;       // [C][64] atom, column 0 = 1
    static constexpr int OFF_SX = OFF_ONES + C * 128;      // [80][64] state operand
    static constexpr int OFF_PT = OFF_SX + 80 * D * 2;     // [C][C] masked P
    static constexpr int OFF_OST = OFF_PT + C * C * 2;     // [C][D] output staging
    static constexpr int OFF_BAR = OFF_OST + C * D * 2;
    static constexpr int NBAR = 3 * NSTAGE + 9 + 4;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int NO = 2;
    static constexpr int T_P = 0;            // [2][C]
    static constexpr int T_O = 2 * C;        // [2][80]
    static constexpr int T_S = 2 * C + 160;  // [64]  (lanes: S^T rows, z at lane 64)
    static constexpr int T_COLS = 512;
    static_assert(T_S + 64 <= T_COLS, "TMEM budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// Warp 18 stores phi(q), phi(k) when asked (CAUSAL): it waits for the
// feature map of each chunk, stores the two tiles by TMA and releases the
// stage once the stores have read it.
constexpr int kChunk64Threads = 608;

// DECAY: the decayed recurrence S_i = gamma S_{i-1} + b_i v_i^T (CAUSAL and
// REDUCE).  Within a chunk of L tokens, m = L/2, query row t carries
// gamma^(t+1-m) and key row j gamma^(m-1-j) (phi_tile_scaled), so P and the
// state products carry the decay weights; the state accumulator then holds
// gamma^(m-L) S after the chunk, and the state epilogue rescales it in TMEM
// to gamma^(m') S for the next chunk (m' of that chunk) before the next
// accumulation, writing the same values as the next operand.  REDUCE scales
// key row j of a segment of L_s tokens by gamma^(L_s-1-j) (the segment's
// state at its end; factors <= 1).  The host takes this path only for
// gamma >= 2^(-64/C), which keeps every scaled value below 2^64.
template <int PHI, int MODE, bool DECAY = false>
__global__ void __launch_bounds__(kChunk64Threads, 1)
chunk_fwd64_kernel(const __grid_constant__ ChunkParams prm) {
    static_assert(!DECAY || MODE != MODE_QUERY, "decay is causal");
    using namespace sm100;
    using Cfg = Chunk64Cfg;
    constexpr int C = Cfg::C, D = Cfg::D, NS = Cfg::NSTAGE, NO = Cfg::NO;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* phi_done = bars + NS;
    uint64_t* empty = bars + 2 * NS;
    uint64_t* p_full = bars + 3 * NS;  // [2]
    uint64_t* p_free = p_full + 2;     // [2]
    uint64_t* pt_full = p_full + 4;
    uint64_t* pt_free = p_full + 5;
    uint64_t* s_full = p_full + 6;
    uint64_t* s_done = p_full + 7;
    uint64_t* drain = p_full + 8;
    uint64_t* o_full = p_full + 9;  // [2]
    uint64_t* o_free = o_full + NO;  // [2]
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
            mbar_init(&empty[s], (MODE == MODE_CAUSAL && prm.store_phi) ? 2 : 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&p_full[b], 1);
            mbar_init(&p_free[b], 1);  // P buffer consumed by the P~ [V|1] MMAs
            mbar_init(&o_full[b], 1);
            mbar_init(&o_free[b], 128);
        }
        mbar_init(pt_full, 128);
        mbar_init(pt_free, 1);
        mbar_init(s_full, 128);
        mbar_init(s_done, 1);
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

    constexpr bool kQ = MODE != MODE_REDUCE;
    constexpr bool kKV = MODE != MODE_QUERY;

    if (warp == 0) {
        if (lane == 0) {
            if (kQ) tma_prefetch_desc(&prm.tm_q);
            if (kKV) {
                tma_prefetch_desc(&prm.tm_k);
                tma_prefetch_desc(&prm.tm_v);
            }
            constexpr uint32_t bytes = Cfg::TILE * ((kQ ? 1 : 0) + (kKV ? 2 : 0));
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                if (c >= NS && !mbar_wait(&empty[s], ((c / NS) - 1) & 1, abort_flag)) break;
                uint8_t* st = smem + s * Cfg::STAGE;
                mbar_arrive_expect_tx(&full[s], bytes);
                const int row = tok0 + c * C;
                if (kQ) tma_load_3d(st, &prm.tm_q, &full[s], 0, row, head);
                if (kKV) {
                    tma_load_3d(st + Cfg::TILE, &prm.tm_k, &full[s], 0, row, kv_head);
                    tma_load_3d(st + 2 * Cfg::TILE, &prm.tm_v, &full[s], 0, row, kv_head);
                }
                issued = c + 1;
            }
            for (int c = max(0, issued - NS); c < issued; ++c)
                mbar_wait_drain(&full[c % NS], (c / NS) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idP = idesc_bf16(C, C, 0, 0);   // A B^T
            constexpr uint32_t idO = idesc_bf16(C, 80, 0, 0);  // A Sx^T
            constexpr uint32_t idPV = idesc_bf16(C, 80, 0, 1); // (P.tril) [V|1]
            constexpr uint32_t idS = idesc_bf16(128, D, 1, 1); // [V|1]^T B
            const uint64_t dSx = desc_k_base(sbase + Cfg::OFF_SX);
            const uint32_t ones = sbase + Cfg::OFF_ONES;
            const bool has_init = st_in != nullptr;
            auto dq_of = [&](int s) { return desc_k_base(sbase + s * Cfg::STAGE); };
            auto dk_of = [&](int s) { return desc_k_base(sbase + s * Cfg::STAGE + Cfg::TILE); };
            auto dkmn_of = [&](int s) {
                return desc_mn_base(sbase + s * Cfg::STAGE + Cfg::TILE, C);
            };
            // [V | 1] as an MN-major operand: the ones atom one LBO after V
            auto dvx_of = [&](int s) {
                const uint32_t v = sbase + s * Cfg::STAGE + 2 * Cfg::TILE;
                return sdesc_sw128(v, ones - v, 1024);
            };
            bool ok = true;
            auto p_part = [&](int c) -> bool {
                const int s = c % NS;
                if (!mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag)) return false;
                if (c >= 2 && !mbar_wait(&p_free[c & 1], ((c >> 1) - 1) & 1, abort_flag))
                    return false;
                tc_fence_after();
                const uint64_t dq = dq_of(s), dk = dk_of(s);
                const uint32_t tP = tmem + Cfg::T_P + (c & 1) * C;
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tP, dq + kstep_k(C, k), dk + kstep_k(C, k), idP, k > 0);
                umma_commit(&p_full[c & 1]);
                return true;
            };
            if (MODE == MODE_CAUSAL) {
                if (nchunks > 0) ok = p_part(0);
                for (int c = 0; ok && c < nchunks; ++c) {
                    const int s = c % NS, bo = c & 1;
                    const uint32_t tO = tmem + Cfg::T_O + bo * 80;
                    if (!(ok = mbar_wait(s_full, c & 1, abort_flag))) break;
                    if (c >= NO && !(ok = mbar_wait(&o_free[bo], ((c >> 1) - 1) & 1, abort_flag)))
                        break;
                    tc_fence_after();
                    const uint64_t dq = dq_of(s), dkm = dkmn_of(s), dvx = dvx_of(s);
#pragma unroll
                    for (int k = 0; k < D; k += 16)
                        umma_bf16(tO, dq + kstep_k(C, k), dSx + kstep_k(80, k), idO, k > 0);
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16(tmem + Cfg::T_S, dvx + kstep_mn(k), dkm + kstep_mn(k), idS,
                                  (c > 0 || has_init || k > 0) ? 1u : 0u);
                    umma_commit(s_done);
                    if (c + 1 < nchunks && !(ok = p_part(c + 1))) break;
                    if (!(ok = mbar_wait(pt_full, c & 1, abort_flag))) break;
                    tc_fence_after();
                    // P~ is in TMEM (bf16 pairs over P's columns): A from TMEM
                    const uint32_t tPt = tmem + Cfg::T_P + (c & 1) * C;
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16_ts(tO, tPt + k / 2, dvx + kstep_mn(k), idPV, 1);
                    umma_commit(&o_full[bo]);
                    umma_commit(&p_free[c & 1]);
                    umma_commit(&empty[s]);
                }
            } else if (MODE == MODE_QUERY) {
                ok = mbar_wait(s_full, 0, abort_flag);
                for (int c = 0; ok && c < nchunks; ++c) {
                    const int s = c % NS, bo = c & 1;
                    const uint32_t tO = tmem + Cfg::T_O + bo * 80;
                    if (!(ok = mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                    if (c >= NO && !(ok = mbar_wait(&o_free[bo], ((c >> 1) - 1) & 1, abort_flag)))
                        break;
                    tc_fence_after();
                    const uint64_t dq = dq_of(s);
#pragma unroll
                    for (int k = 0; k < D; k += 16)
                        umma_bf16(tO, dq + kstep_k(C, k), dSx + kstep_k(80, k), idO, k > 0);
                    umma_commit(&o_full[bo]);
                    umma_commit(&empty[s]);
                }
            } else {  // REDUCE
                ok = mbar_wait(s_full, 0, abort_flag);
                for (int c = 0; ok && c < nchunks; ++c) {
                    const int s = c % NS;
                    if (!(ok = mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                    tc_fence_after();
                    const uint64_t dkm = dkmn_of(s), dvx = dvx_of(s);
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16(tmem + Cfg::T_S, dvx + kstep_mn(k), dkm + kstep_mn(k), idS,
                                  (c > 0 || k > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(s_done);
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < 10) {
        const int u = tid - 64;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            if (!mbar_wait(&full[s], (c / NS) & 1, abort_flag)) break;
            uint8_t* st = smem + s * Cfg::STAGE;
            const int nvalid = min(C, tok1 - (tok0 + c * C));
            if (DECAY && MODE == MODE_CAUSAL) {
                const float m = 0.5f * float(nvalid);
                if (u < 128)
                    phi_tile_scaled<PHI, C, D, 128>(st, u, nvalid, false, lg, 1.f, 1.f - m);
                else
                    phi_tile_scaled<PHI, C, D, 128>(st + Cfg::TILE, u - 128, nvalid, true, lg,
                                                    -1.f, m - 1.f);
            } else if (DECAY) {  // REDUCE: decayed to the segment's end
                phi_tile_scaled<PHI, C, D, 256>(st + Cfg::TILE, u, nvalid, true, lg, -1.f,
                                                float(tok1 - tok0 - 1 - c * C));
            } else if (MODE == MODE_CAUSAL) {
                if (u < 128)
                    phi_tile<PHI, C, D, 128>(st, u, nvalid, false);
                else
                    phi_tile<PHI, C, D, 128>(st + Cfg::TILE, u - 128, nvalid, true);
            } else if (MODE == MODE_QUERY) {
                phi_tile<PHI, C, D, 256>(st, u, nvalid, false);
            } else if (prm.center) {
                phi_tile<PHI, C, D, 256, true>(st + Cfg::TILE, u, nvalid, true);
            } else {
                phi_tile<PHI, C, D, 256>(st + Cfg::TILE, u, nvalid, true);
            }
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
        }
    } else if (warp < 14) {
        if (MODE == MODE_CAUSAL) {
            // mask P and pack it to bf16 pairs in place (TMEM): block j0 is
            // read before columns j0/2.. are overwritten
            const int sp = warp & 3;
            const uint32_t lane_base = uint32_t(32 * sp) << 16;
            const int irow = 32 * sp + lane;
            for (int c = 0; c < nchunks; ++c) {
                const int b = c & 1;
                if (!named_bar_all(1, 128, mbar_wait(&p_full[b], (c >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                const uint32_t reg = tmem + lane_base + Cfg::T_P + b * C;
#pragma unroll 1
                for (int j0 = 0; j0 < C; j0 += 32) {
                    float pv[32];
                    tmem_load<32>(reg + j0, pv);
                    float pk[16];
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int j = j0 + 2 * t;
                        pk[t] = __uint_as_float(pack_bf16(j <= irow ? pv[2 * t] : 0.f,
                                                          j + 1 <= irow ? pv[2 * t + 1] : 0.f));
                    }
                    tmem_st16(reg + j0 / 2, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(pt_full);
            }
        }
    } else if (warp < 18) {
        const int e = tid - 448;
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int row = 32 * sp + lane;  // token row of O; row of the state accumulator
        uint8_t* sx = smem + Cfg::OFF_SX;
        uint8_t* ones = smem + Cfg::OFF_ONES;
        uint8_t* ost = smem + Cfg::OFF_OST;

        // ---- ones atom (column 0) and the zero rows 66..79 of Sx
        for (int r = e; r < C; r += 128) {
            float v8[8] = {1.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            float z8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int q = 0; q < 8; ++q) store_row_bf16<8>(ones, C, r, 8 * q, q == 0 ? v8 : z8);
        }
        for (int idx = e; idx < 14 * 8; idx += 128) {
            const float z8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            store_row_bf16<8>(sx, 80, 66 + idx / 8, 8 * (idx % 8), z8);
        }
        // Sx row v <- S[:, v] for v < 64; rows 64, 65 <- z split in two bf16.
        // `half` selects columns 32*half .. 32*half+31.
        auto put_state = [&](int v, int half, const float* col) {
            if (v < D) {
                store_row_bf16<32>(sx, 80, v, 32 * half, col);
            } else if (v == D) {
#pragma unroll
                for (int f0 = 0; f0 < 32; f0 += 16) {
                    float hi[16], lo[16];
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        hi[t] = __bfloat162float(__float2bfloat16_rn(col[f0 + t]));
                        lo[t] = col[f0 + t] - hi[t];
                    }
                    store_row_bf16<16>(sx, 80, D, 32 * half + f0, hi);
                    store_row_bf16<16>(sx, 80, D + 1, 32 * half + f0, lo);
                }
            }
        };
        // column `row` of the state accumulator -> S[:, row] (or z), fp32
        auto write_state = [&](float* S_dst, float* z_dst, int half, const float* col) {
            if (row < D) {
                if (S_dst)
                    for (int t = 0; t < 32; ++t) S_dst[(32 * half + t) * D + row] = col[t];
            } else if (row == D && z_dst) {
                for (int t = 0; t < 32; ++t) z_dst[32 * half + t] = col[t];
            }
        };
        // decay: the initial state enters as gamma^(m_0) S_0 (m_0: half the
        // first chunk's tokens)
        float s0 = 1.f;
        if constexpr (DECAY) s0 = exp2f(lg * 0.5f * float(min(C, tok1 - tok0)));
        // initial / fixed state, transposed: column v of S (row 64: z)
        if (MODE != MODE_REDUCE && row <= D) {
            for (int half = 0; half < 2; ++half) {
                float col[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const int f = 32 * half + t;
                    col[t] = st_in ? s0 * (row < D ? st_in[f * D + row] : st_in[D * D + f]) : 0.f;
                }
                put_state(row, half, col);
            }
        }
        if (MODE == MODE_CAUSAL && st_in) {
            // the state accumulator starts at the initial state
            for (int f0 = 0; f0 < 64; f0 += 16) {
                float v16[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int f = f0 + t;
                    v16[t] = s0 * (row < D ? st_in[f * D + row] : (row == D ? st_in[D * D + f] : 0.f));
                }
                tmem_st16(tmem + lane_base + Cfg::T_S + f0, v16);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(s_full);

        if (MODE == MODE_REDUCE) {
            if (named_bar_all(2, 128, mbar_wait(s_done, 0, abort_flag))) {
                tc_fence_after();
                const size_t idx = blockIdx.x;
                for (int half = 0; half < 2; ++half) {
                    float col[32];
                    tmem_load<32>(tmem + lane_base + Cfg::T_S + 32 * half, col);
                    write_state(prm.S_out + idx * prm.stride_S, prm.z_out + idx * prm.stride_z,
                                half, col);
                }
            }
        } else {
            for (int c = 0; c < nchunks; ++c) {
                const int bo = c & 1;
                const int row0 = tok0 + c * C;
                if (MODE == MODE_CAUSAL) {
                    if (!named_bar_all(2, 128, mbar_wait(s_done, c & 1, abort_flag))) break;
                    tc_fence_after();
                    const bool last = c == nchunks - 1;
                    const bool write_final = last && seg == prm.nseg - 1 && prm.S_out != nullptr &&
                                             state_writer;
                    const size_t sidx = size_t(kv_head);
                    if (DECAY && (!last || write_final)) {
                        // the accumulator holds gamma^(m-L) S: the next chunk
                        // wants gamma^(m') S (operand and accumulator), the
                        // final state S itself
                        const int L = min(C, tok1 - row0);
                        const float m = 0.5f * float(L);
                        const float f = last ? exp2f(lg * (float(L) - m))
                                             : exp2f(lg * (float(L) - m +
                                                           0.5f * float(min(C, tok1 - row0 - C))));
                        float* S_dst = prm.S_out ? prm.S_out + sidx * prm.stride_S : nullptr;
                        float* z_dst = prm.z_out ? prm.z_out + sidx * prm.stride_z : nullptr;
#pragma unroll 1
                        for (int q4 = 0; q4 < 4; ++q4) {  // 16 columns at a time
                            float col[16];
                            tmem_load<16>(tmem + lane_base + Cfg::T_S + 16 * q4, col);
#pragma unroll
                            for (int t = 0; t < 16; ++t) col[t] *= f;
                            if (last) {
                                if (row < D && S_dst) {
                                    for (int t = 0; t < 16; ++t) S_dst[(16 * q4 + t) * D + row] = col[t];
                                } else if (row == D && z_dst) {
                                    for (int t = 0; t < 16; ++t) z_dst[16 * q4 + t] = col[t];
                                }
                            } else {
                                tmem_st16(tmem + lane_base + Cfg::T_S + 16 * q4, col);
                                if (row < D) {
                                    store_row_bf16<16>(sx, 80, row, 16 * q4, col);
                                } else if (row == D) {
                                    float hi[16], lo[16];
#pragma unroll
                                    for (int t = 0; t < 16; ++t) {
                                        hi[t] = __bfloat162float(__float2bfloat16_rn(col[t]));
                                        lo[t] = col[t] - hi[t];
                                    }
                                    store_row_bf16<16>(sx, 80, D, 16 * q4, hi);
                                    store_row_bf16<16>(sx, 80, D + 1, 16 * q4, lo);
                                }
                            }
                        }
                        tmem_wait_st();
                    } else if (!last || write_final) {
#pragma unroll 1
                        for (int half = 0; half < 2; ++half) {
                            float col[32];
                            tmem_load<32>(tmem + lane_base + Cfg::T_S + 32 * half, col);
                            put_state(row, half, col);
                            if (write_final)
                                write_state(prm.S_out + sidx * prm.stride_S,
                                            prm.z_out ? prm.z_out + sidx * prm.stride_z : nullptr,
                                            half, col);
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(s_full);
                }
                if (!named_bar_all(2, 128, mbar_wait(&o_full[bo], (c >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                if (e == 0) bulk_wait_read0();
                named_bar_sync(2, 128);
                const uint32_t tO = tmem + lane_base + Cfg::T_O + bo * 80;
                float den[16];
                tmem_load<16>(tO + 64, den);
                const float inv = 1.f / (den[0] + den[1]);
                if (prm.g_out && row0 + row < tok1)
                    prm.g_out[size_t(head) * prm.N + row0 + row] = den[0] + den[1];
#pragma unroll 1
                for (int v0 = 0; v0 < D; v0 += 32) {
                    float ov[32];
                    tmem_load<32>(tO + v0, ov);
#pragma unroll
                    for (int t = 0; t < 32; ++t) ov[t] *= inv;
                    store_row_bf16<32>(ost, C, row, v0, ov);
                }
                tc_fence_before();
                mbar_arrive(&o_free[bo]);
                fence_proxy_async_smem();
                named_bar_sync(2, 128);
                if (e == 0) {
                    tma_store_3d(&prm.tm_o, ost, 0, row0, head);
                    bulk_commit();
                }
            }
            if (e == 0) bulk_wait0();
        }
    } else if (warp == 18) {
        if (MODE == MODE_CAUSAL && prm.store_phi && lane == 0) {
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                if (!mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag)) break;
                const uint8_t* st = smem + s * Cfg::STAGE;
                tma_store_3d(&prm.tm_pq, st, 0, tok0 + c * C, head);
                tma_store_3d(&prm.tm_pk, st + Cfg::TILE, 0, tok0 + c * C, head);
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
