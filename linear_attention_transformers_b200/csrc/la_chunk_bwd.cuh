// la_chunk_bwd.cuh — chunked linear-attention backward on sm_100a tensor cores.
//
// Gradients of L = sum(dO * O) (the pages print none; derived from the
// definition in "Efficient Transformers Survey", Proposition "Linear
// Attention via Kernel Decomposition", Statement).  Per head, with
// a = phi(q), b = phi(k), g_i = a_i.z_i and o_i = S_i^T a_i / g_i:
//
//   du_i = dO_i / g_i,   dg_i = -(dO_i . o_i) / g_i
//   dA_i = S_i du_i + z_i dg_i              = sum_{j<=i} b_j (v_j.du_i + dg_i)
//   dB_j = R_j v_j + r_j                    = sum_{i>=j} a_i (v_j.du_i + dg_i)
//   dV_j = R_j^T b_j                        = sum_{i>=j} (a_i.b_j) du_i
//   dQ = dA * phi'(q),  dK = dB * phi'(k)
//
// with the suffix sums R_j = sum_{i>=j} a_i du_i^T, r_j = sum_{i>=j} a_i dg_i
// (non-causal: every sum runs over all tokens).  Neither pass stores an
// N x D x D tensor; the prefix (S, z) and suffix (R, r) states are rebuilt
// chunk by chunk, in the spirit of the abstract of "Transformer Based Linear
// Attention with Optimized GPU Kernel Implementation" (an O(N D^2) forward and
// backward).
//
// Pass 1 (token order) per C-token chunk, S/z = state of earlier chunks:
//   P = A B^T, num = (P.M) V + A S, g = rowsum(P.M) + A z, o = num / g
//   du, dg;  W' = ((dU V^T) + dg 1^T).M;  dA = W' B + dU S^T + dg z^T
//   S += B^T V, z += B^T 1;  saves g, dg;  optionally R += A^T dU, r += A^T dg
// Pass 2 (reverse token order), R/r = state of later chunks:
//   X1 = (B A^T).M^T,  X2 = (V dU^T + 1 dg^T).M^T
//   dV = X1 dU + B R,  dB = X2 A + V R^T + 1 r^T;  R += A^T dU, r += A^T dg
// (M = lower-triangular mask with the diagonal.)  Both passes use the same
// warp roles as the forward: TMA producer, phi warpgroup, single-thread MMA
// issuer, epilogue warpgroup; all waits are bounded.
#pragma once

#include "la_common.cuh"
#include "la_sm100.cuh"
#include "la_tile_ops.cuh"

namespace la {

struct BwdParams {
    CUtensorMap tm_q, tm_k, tm_v, tm_do, tm_dq, tm_dk, tm_dv;
    int N, seg_len, nseg;
    // pass 1: initial (S, z) record; pass 2: initial (R, r) record.  Record =
    // [D][D] row-major (row = key feature) then [D].  Index = head
    // (in_per_head) or block; null = zero state.
    const float* state_in;
    int in_per_head;
    float* gbuf;     // [heads][N] g_i (pass 1 writes, pass 2 reads)
    float* dgbuf;    // [heads][N] dg_i
    float* rec_out;  // pass 1: (R, r) of the block's tokens, record per block (nullable)
    // pass 1 with saved forward statistics: the forward's output O (bf16
    // [heads][N][D]); gbuf then holds the forward's denominators g.
    const __nv_bfloat16* o_in;
    // query heads per key/value head: k and v are read at head / kv_group
    int kv_group;
    // kv_group > 1: dK, dV of each query head in float32 ([heads][N][D]),
    // stored by the epilogue threads in place of the bf16 tiles, so that the
    // caller's sum over each group rounds to bf16 once
    float* dk_part;
    float* dv_part;
    // decay factor per head (read by the DECAY kernels only; causal)
    DecayArg dec;
};

template <int D, int C>
struct Bwd1Cfg {
    static constexpr int NSTAGE = 2;
    static constexpr int TILE = C * D * 2;
    // Q, K, V, dO tiles, then (saved-statistics mode) the chunk's DG operand
    // [16][C] and its dg values [C]
    static constexpr int OFF_SDG = 4 * TILE;
    static constexpr int OFF_SDGF = OFF_SDG + 16 * C * 2;
    static constexpr int STAGE = ((OFF_SDGF + C * 4) + 1023) / 1024 * 1024;
    static constexpr int OFF_SPREV = NSTAGE * STAGE;
    static constexpr int OFF_ZOP = OFF_SPREV + D * D * 2;
    static constexpr int OFF_E = OFF_ZOP + 16 * D * 2;
    static constexpr int OFF_X = OFF_E + 16 * C * 2;
    static constexpr int OFF_DU = OFF_X + C * C * 2;
    static constexpr int OFF_DG = OFF_DU + C * D * 2;
    static constexpr int OFF_STG = OFF_DG + 16 * C * 2;
    static constexpr int OFF_ZF = OFF_STG + C * D * 2;
    // z as float, two copies (chunk parity): with the state readout on its
    // own warp group, chunk c's dQ reads one while chunk c's readout writes
    // the other
    static constexpr int OFF_BAR = OFF_ZF + 2 * (((D * 4 + 15) / 16) * 16);
    static constexpr int NBAR = 6 * NSTAGE + 10;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    static constexpr int T_P = 0, T_O = C, T_OZ = C + D, T_S = C + D + 16, T_Z = C + 2 * D + 16;
    // masked C x C operands (P~, W') packed in place in TMEM and read by MMAs
    // with A from TMEM (needs M = C = 128 rows); otherwise through smem
    static constexpr bool XT = C == 128 && D == 64;
    static constexpr int T_R = C + 2 * D + 32, T_RZ = C + 3 * D + 32;
    static constexpr int T_COLS = 512;
    static_assert(T_RZ + 16 <= T_COLS, "TMEM budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

template <int D, int C>
struct Bwd2Cfg {
    static constexpr int NSTAGE = 2;
    static constexpr int TILE = C * D * 2;
    static constexpr int OFF_DGT = 4 * TILE;           // in-stage: DG operand [16][C]
    static constexpr int OFF_DGF = 4 * TILE + 16 * C * 2;  // in-stage: dg float [C]
    static constexpr int OFF_RINV = OFF_DGF + C * 4;       // in-stage: 1/g float [C]
    static constexpr int STAGE = ((OFF_RINV + C * 4) + 1023) / 1024 * 1024;
    static constexpr int OFF_RPREV = NSTAGE * STAGE;
    static constexpr int OFF_RF = OFF_RPREV + D * D * 2;
    static constexpr int OFF_X1 = OFF_RF + 1024;
    static constexpr int OFF_X2 = OFF_X1 + C * C * 2;
    static constexpr bool STG_ALIAS = C >= D;  // dV/dK staging reuses X1/X2
    static constexpr int OFF_STGV = STG_ALIAS ? OFF_X1 : OFF_X2 + C * C * 2;
    static constexpr int OFF_STGK = STG_ALIAS ? OFF_X2 : OFF_STGV + C * D * 2;
    static constexpr int OFF_BAR = STG_ALIAS ? OFF_X2 + C * C * 2 : OFF_STGK + C * D * 2;
    static constexpr int NBAR = 3 * NSTAGE + 6;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;
    // X in TMEM (C = 128): X1, X2 are packed to bf16 in place over the low
    // halves of T1, T2 and feed MMAs with A from TMEM; dV and dB accumulate in
    // the high halves.  Otherwise X1, X2 go through shared memory and dV, dB
    // reuse T1/T2's columns.
    static constexpr bool XT = C == 128 && D == 64;
    static constexpr int T_1 = 0, T_2 = C;
    static constexpr int T_3 = XT ? C / 2 : 0, T_4 = XT ? C + C / 2 : D;
    static constexpr int T_R = (2 * C > 2 * D ? 2 * C : 2 * D), T_RZ = T_R + D;
    static constexpr int T_COLS = 512;
    static_assert(T_RZ + 16 <= T_COLS, "TMEM budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// phi'(x) from the bf16 value a = phi(x) that the MMAs read:
// elu+1: 1 for x > 0 (a > 1), exp(x) = a otherwise -> min(a, 1);
// relu+eps: 1 where x > 0, i.e. where a exceeds the x <= 0 value bf16(1e-6).
template <int PHI>
__device__ __forceinline__ float dphi_from_phi(float a) {
    if (PHI == PHI_ELU1) return fminf(a, 1.f);
    if (PHI == PHI_IDENTITY) return 1.f;
    const float floor_val = __bfloat162float(__float2bfloat16_rn(1e-6f));
    return a > floor_val ? 1.f : 0.f;
}

// phi'(k) from the bf16 value b = bf16(phi(k) * beta) of a key row scaled
// by the decay factor beta (the decayed passes): elu+1 takes min(b / beta, 1);
// for relu+eps, k <= 0 left exactly bf16(1e-6 * beta) in the tile (the same
// product, rounded the same way), so b above it means k > 0.
template <int PHI>
__device__ __forceinline__ float dphi_from_scaled_phi(float b, float beta, float binv) {
    if (PHI == PHI_ELU1) return fminf(b * binv, 1.f);
    if (PHI == PHI_IDENTITY) return 1.f;
    return b > __bfloat162float(__float2bfloat16_rn(1e-6f * beta)) ? 1.f : 0.f;
}

// Load a state record into the bf16 operand tile [D][D] (row f) and return
// row f's last entry (z_f or r_f) in *last.  Rows outside [0, D) skip.
template <int D>
__device__ __forceinline__ void load_state_row(const float* rec, int frow, uint8_t* tile,
                                               float* last) {
    using namespace sm100;
    for (int q = 0; q < D / 8; ++q) {
        float v8[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) v8[t] = rec ? rec[size_t(frow) * D + q * 8 + t] : 0.f;
        *reinterpret_cast<uint4*>(tile + tile_chunk_off(D, frow, q)) =
            make_uint4(pack_bf16(v8[0], v8[1]), pack_bf16(v8[2], v8[3]), pack_bf16(v8[4], v8[5]),
                       pack_bf16(v8[6], v8[7]));
    }
    *last = rec ? rec[size_t(D) * D + frow] : 0.f;
}

// Write 16 fp32 TMEM values of row `row` as bf16 into a row tile.
__device__ __forceinline__ void store_row16_bf16(uint8_t* tile, int rows, int row, int col0,
                                                 const float* v) {
    using namespace sm100;
    *reinterpret_cast<uint4*>(tile + tile_chunk_off(rows, row, col0 >> 3)) =
        make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                   pack_bf16(v[6], v[7]));
    *reinterpret_cast<uint4*>(tile + tile_chunk_off(rows, row, (col0 >> 3) + 1)) =
        make_uint4(pack_bf16(v[8], v[9]), pack_bf16(v[10], v[11]), pack_bf16(v[12], v[13]),
                   pack_bf16(v[14], v[15]));
}

// Write 16 fp32 values to global memory (16-byte aligned destination).
__device__ __forceinline__ void store16_f32(float* dst, const float* v) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Read 8 bf16 values (columns 8q..8q+7) of row `row` of a row tile.
__device__ __forceinline__ void load_chunk8(const uint8_t* tile, int rows, int row, int q,
                                            float* out) {
    using namespace sm100;
    const uint4 x = *reinterpret_cast<const uint4*>(tile + tile_chunk_off(rows, row, q));
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float2 f = unpack_bf16(w[t]);
        out[2 * t] = f.x;
        out[2 * t + 1] = f.y;
    }
}

// ======================================================================
// Pass 1: dQ (token order), g and dg saved for pass 2.
// ======================================================================
constexpr int kBwdThreads = 448;  // producer, MMA, 8 phi warps, 4 epilogue warps

// SAVED = the forward's O and g are given: no forward recompute; the
// feature-map warps form dU = dO / g and dg = -(dO . O) / g directly.
//
// SPLIT (causal, saved, D = 128): the state readout (S -> the bf16 operand
// of the next chunk, z, the segment's (R, r)) runs on the key half of the
// feature-map warps (warps 6-9) while the epilogue warps form dQ, so the two
// TMEM readouts of a chunk overlap instead of following each other; and the
// MMA thread issues the next chunk's W = dU V^T as soon as its tiles are
// ready (W has its own TMEM columns), so W is done when the epilogue comes
// to mask it.
template <int D, int C, int PHI, bool CAUSAL, bool SAVED>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dq_kernel(const __grid_constant__ BwdParams prm) {
    using namespace sm100;
    using Cfg = Bwd1Cfg<D, C>;
    constexpr int NS = Cfg::NSTAGE;
    constexpr bool SPLIT = SAVED && CAUSAL && D == 128 && !Cfg::XT;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* phi_done = bars + NS;
    uint64_t* empty = bars + 2 * NS;     // released by the epilogue (count 128)
    uint64_t* p_ready = bars + 3 * NS;   // commit: P, A S, A z
    uint64_t* pt_ready = p_ready + 1;    // 128: masked P in X
    uint64_t* o_ready = p_ready + 2;     // commit: num complete
    uint64_t* du_ready = p_ready + 3;    // 128: dU, DG written
    uint64_t* w_ready = p_ready + 4;     // commit: dU V^T
    uint64_t* wt_ready = p_ready + 5;    // 128: W' in X
    uint64_t* da_ready = p_ready + 6;    // commit: dA, state updates
    uint64_t* s_ready = p_ready + 7;     // 128: state operand for next chunk
    uint64_t* drain = p_ready + 8;
    uint64_t* st_ready = p_ready + 9;    // commit (SPLIT): S, z, R, r updated
    // SPLIT: the stage's q tile has barriers of its own (k, v, dO are
    // released by the products' commit, q by the epilogue once dQ is formed)
    uint64_t* fullq = p_ready + 10;       // TMA landed (q)
    uint64_t* phiq_done = fullq + NS;     // 128: phi(q) applied
    uint64_t* emptyq = fullq + 2 * NS;    // 128: epilogue done with q
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
    const bool rec = prm.rec_out != nullptr;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&phi_done[s], 256);
            mbar_init(&empty[s], SPLIT ? 1 : 128);
            mbar_init(&fullq[s], 1);
            mbar_init(&phiq_done[s], 128);
            mbar_init(&emptyq[s], 128);
        }
        mbar_init(p_ready, 1);
        mbar_init(pt_ready, 128);
        mbar_init(o_ready, 1);
        mbar_init(du_ready, 128);
        mbar_init(w_ready, 1);
        mbar_init(wt_ready, 128);
        mbar_init(da_ready, 1);
        mbar_init(s_ready, SPLIT ? 256 : 128);
        mbar_init(drain, 1);
        mbar_init(st_ready, 1);
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
            int issued = 0, issued_q = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                if (c >= NS && !mbar_wait(&empty[s], ((c / NS) - 1) & 1, abort_flag)) break;
                uint8_t* st = smem + s * Cfg::STAGE;
                mbar_arrive_expect_tx(&full[s], (SPLIT ? 3 : 4) * Cfg::TILE);
                const int row = tok0 + c * C;
#pragma unroll
                for (int a = 0; a < D / 64; ++a) {
                    if (!SPLIT)
                        tma_load_3d(st + a * C * 128, &prm.tm_q, &full[s], a * 64, row, head);
                    tma_load_3d(st + Cfg::TILE + a * C * 128, &prm.tm_k, &full[s], a * 64, row,
                                kv_head);
                    tma_load_3d(st + 2 * Cfg::TILE + a * C * 128, &prm.tm_v, &full[s], a * 64, row,
                                kv_head);
                    tma_load_3d(st + 3 * Cfg::TILE + a * C * 128, &prm.tm_do, &full[s], a * 64, row,
                                head);
                }
                issued = c + 1;
                if (SPLIT) {
                    // q of chunk c, once the epilogue is done with chunk c - NS
                    if (c >= NS && !mbar_wait(&emptyq[s], ((c / NS) - 1) & 1, abort_flag)) break;
                    mbar_arrive_expect_tx(&fullq[s], Cfg::TILE);
#pragma unroll
                    for (int a = 0; a < D / 64; ++a)
                        tma_load_3d(st + a * C * 128, &prm.tm_q, &fullq[s], a * 64, row, head);
                    issued_q = c + 1;
                }
            }
            for (int c = max(0, issued - NS); c < issued; ++c)
                mbar_wait_drain(&full[c % NS], (c / NS) & 1);
            for (int c = max(0, issued_q - NS); c < issued_q; ++c)
                mbar_wait_drain(&fullq[c % NS], (c / NS) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t tP = tmem + Cfg::T_P, tO = tmem + Cfg::T_O, tOZ = tmem + Cfg::T_OZ;
            const uint32_t tS = tmem + Cfg::T_S, tZ = tmem + Cfg::T_Z;
            const uint32_t tR = tmem + Cfg::T_R, tRZ = tmem + Cfg::T_RZ;
            const uint32_t sprev = sbase + Cfg::OFF_SPREV, zop = sbase + Cfg::OFF_ZOP;
            const uint32_t eop = sbase + Cfg::OFF_E, xop = sbase + Cfg::OFF_X;
            const uint32_t duop_g = sbase + Cfg::OFF_DU, dgop_g = sbase + Cfg::OFF_DG;
            constexpr uint32_t idCC = idesc_bf16(C, C, 0, 0);   // [C x C] from two K-major
            constexpr uint32_t idCD_mn = idesc_bf16(C, D, 0, 1);
            constexpr uint32_t idCD_k = idesc_bf16(C, D, 0, 0);
            constexpr uint32_t idOZ = idesc_bf16(C, 16, 0, 0);
            constexpr uint32_t idDD = idesc_bf16(D, D, 1, 1);
            constexpr uint32_t idD16 = idesc_bf16(D, 16, 1, 0);
            const bool has_init = st_in != nullptr;
            bool ok = true;
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c % NS;
                const uint32_t qs = sbase + s * Cfg::STAGE, ks = qs + Cfg::TILE;
                const uint32_t vs = qs + 2 * Cfg::TILE;
                // dU and the DG operand: the scaled dO tile and the stage's DG
                // (saved mode) or the epilogue-written tiles
                const uint32_t duop = SAVED ? qs + 3 * Cfg::TILE : duop_g;
                const uint32_t dgop = SAVED ? qs + Cfg::OFF_SDG : dgop_g;
                if (!(ok = mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                // SPLIT: W needs only this chunk's tiles (its columns were
                // last read by the previous chunk's mask); the state operand
                // is waited for just before dU S^T
                if (!SPLIT && !(ok = mbar_wait(s_ready, c & 1, abort_flag))) break;
                tc_fence_after();
                if (!SAVED) {
                    if (CAUSAL) {
#pragma unroll
                        for (int k = 0; k < D; k += 16)
                            umma_bf16(tP, desc_kmajor(qs, C, k), desc_kmajor(ks, C, k), idCC, k > 0);
                    }
#pragma unroll
                    for (int k = 0; k < D; k += 16) {
                        umma_bf16(tO, desc_kmajor(qs, C, k), desc_mnmajor(sprev, D, k), idCD_mn,
                                  k > 0);
                        umma_bf16(tOZ, desc_kmajor(qs, C, k), desc_kmajor(zop, 16, k), idOZ, k > 0);
                    }
                    if (CAUSAL) {
                        umma_commit(p_ready);
                        if (!(ok = mbar_wait(pt_ready, c & 1, abort_flag))) break;
                        tc_fence_after();
                        if (Cfg::XT) {
#pragma unroll
                            for (int k = 0; k < C; k += 16)
                                umma_bf16_ts(tO, tP + k / 2, desc_mnmajor(vs, C, k), idCD_mn, 1);
                        } else {
#pragma unroll
                            for (int k = 0; k < C; k += 16)
                                umma_bf16(tO, desc_kmajor(xop, C, k), desc_mnmajor(vs, C, k), idCD_mn,
                                          1);
                        }
                    }
                    umma_commit(o_ready);
                    if (!(ok = mbar_wait(du_ready, c & 1, abort_flag))) break;
                    tc_fence_after();
                }
                if (CAUSAL) {
                    // W = dU V^T
#pragma unroll
                    for (int k = 0; k < D; k += 16)
                        umma_bf16(tP, desc_kmajor(duop, C, k), desc_kmajor(vs, C, k), idCC, k > 0);
                    umma_commit(w_ready);
                    if (!(ok = mbar_wait(wt_ready, c & 1, abort_flag))) break;
                    if (SPLIT && !(ok = mbar_wait(s_ready, c & 1, abort_flag))) break;
                    tc_fence_after();
                    // dA = W' B
                    if (Cfg::XT) {
#pragma unroll
                        for (int k = 0; k < C; k += 16)
                            umma_bf16_ts(tO, tP + k / 2, desc_mnmajor(ks, C, k), idCD_mn, k > 0);
                    } else {
#pragma unroll
                        for (int k = 0; k < C; k += 16)
                            umma_bf16(tO, desc_kmajor(xop, C, k), desc_mnmajor(ks, C, k), idCD_mn,
                                      k > 0);
                    }
                }
                // dA += dU S^T
#pragma unroll
                for (int k = 0; k < D; k += 16)
                    umma_bf16(tO, desc_kmajor(duop, C, k), desc_kmajor(sprev, D, k), idCD_k,
                              (CAUSAL || k > 0) ? 1u : 0u);
                // SPLIT: dA is complete here; the epilogue starts on it while
                // the state updates run
                if (SPLIT) umma_commit(da_ready);
                if (CAUSAL) {
                    // S += B^T V, z += B^T 1
#pragma unroll
                    for (int k = 0; k < C; k += 16) {
                        const uint32_t acc = (c > 0 || has_init || k > 0) ? 1u : 0u;
                        umma_bf16(tS, desc_mnmajor(ks, C, k), desc_mnmajor(vs, C, k), idDD, acc);
                        umma_bf16(tZ, desc_mnmajor(ks, C, k), desc_kmajor(eop, 16, k), idD16, acc);
                    }
                }
                if (rec) {
                    // R += A^T dU, r += A^T [dg_hi; dg_lo] (SPLIT: phi(q) comes
                    // on its own barrier)
                    if (SPLIT && !(ok = mbar_wait(&phiq_done[s], (c / NS) & 1, abort_flag))) break;
                    if (SPLIT) tc_fence_after();
#pragma unroll
                    for (int k = 0; k < C; k += 16) {
                        const uint32_t acc = (c > 0 || k > 0) ? 1u : 0u;
                        umma_bf16(tR, desc_mnmajor(qs, C, k), desc_mnmajor(duop, C, k), idDD, acc);
                        umma_bf16(tRZ, desc_mnmajor(qs, C, k), desc_kmajor(dgop, 16, k), idD16, acc);
                    }
                }
                umma_commit(SPLIT ? st_ready : da_ready);
                // SPLIT: k, v, dU and the DG operand are read by now
                if (SPLIT) umma_commit(&empty[s]);
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < 10) {
        // feature map on Q and K (and, with saved statistics, dU and dg)
        const int u = tid - 64;  // 0..255
        if (SAVED) {
            for (int s = 0; s < NS; ++s) {
                __nv_bfloat16* dgt = reinterpret_cast<__nv_bfloat16*>(smem + s * Cfg::STAGE + Cfg::OFF_SDG);
                for (int idx = u; idx < 16 * C; idx += 256)
                    dgt[tile_off(16, idx / C, idx % C) / 2] = __float2bfloat16_rn(0.f);
            }
        }
        // SPLIT, warps 6-9 (one TMEM lane quarter each): after chunk c's
        // products, S -> the bf16 operand of chunk c + 1 and z -> zf (the
        // copy of the other parity)
        auto readout_dq = [&](int c) -> bool {
            if (!named_bar_all(2, 128, mbar_wait(st_ready, c & 1, abort_flag))) return false;
            tc_fence_after();
            const uint32_t lane_base = uint32_t(32 * (warp & 3)) << 16;
            const int frow = acc_row<D>(warp & 3, lane);
            float zv[16];
            tmem_ld16(tmem + lane_base + Cfg::T_Z, zv);
#pragma unroll 1
            for (int v0 = 0; v0 < D; v0 += 32) {
                float sv[32];
                tmem_load<32>(tmem + lane_base + Cfg::T_S + v0, sv);
                store_row16_bf16(smem + Cfg::OFF_SPREV, D, frow, v0, sv);
                store_row16_bf16(smem + Cfg::OFF_SPREV, D, frow, v0 + 16, sv + 16);
            }
            reinterpret_cast<float*>(smem + Cfg::OFF_ZF)[((c + 1) & 1) * D + frow] = zv[0];
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(s_ready);
            return true;
        };
        // the readout warps' share of the initial state's arrival (the
        // epilogue warps write the initial operand)
        if (SPLIT && u >= 128) mbar_arrive(s_ready);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            if (!mbar_wait(&full[s], (c / NS) & 1, abort_flag)) break;
            uint8_t* st = smem + s * Cfg::STAGE;
            const int nvalid = min(C, tok1 - (tok0 + c * C));
            // q -> phi(q); k -> phi(k) - c (the centred key features: see
            // the epilogue's all-ones correction).  SPLIT: q comes later, on
            // its own barrier
            if (u < 128) {
                if (!SPLIT) phi_tile<PHI, C, D, 128>(st, u, nvalid, true);
            } else
                phi_tile<PHI, C, D, 128, true>(st + Cfg::TILE, u - 128, nvalid, true);
            if (SAVED) {
                // dU = dO / g in place, dg = -(dO . O) / g; 256 / C threads per row
                constexpr int TPR = 256 / C;          // threads per row
                constexpr int CHT = (D / 8) / TPR;    // 16-byte chunks per thread
                const int r = u / TPR, part = u % TPR;
                const bool valid = r < nvalid;
                const size_t tok = size_t(head) * prm.N + size_t(tok0 + c * C + r);
                uint8_t* dot_tile = st + 3 * Cfg::TILE;
                uint4 x[CHT], ov[CHT];
#pragma unroll
                for (int j = 0; j < CHT; ++j) {
                    x[j] = *reinterpret_cast<const uint4*>(dot_tile + tile_chunk_off(C, r, part * CHT + j));
                    ov[j] = valid ? __ldg(reinterpret_cast<const uint4*>(prm.o_in + tok * D) + part * CHT + j)
                                  : make_uint4(0u, 0u, 0u, 0u);
                }
                const float g = valid ? prm.gbuf[tok] : 1.f;
                float dotp = 0.f;
#pragma unroll
                for (int j = 0; j < CHT; ++j) {
                    const uint32_t a[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
                    const uint32_t b[4] = {ov[j].x, ov[j].y, ov[j].z, ov[j].w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float2 fa = unpack_bf16(a[t]), fb = unpack_bf16(b[t]);
                        dotp = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, dotp));
                    }
                }
#pragma unroll
                for (int m = 1; m < TPR; m <<= 1) dotp += __shfl_xor_sync(0xffffffffu, dotp, m);
                const float ginv = 1.f / g;
                const float dg = valid ? -dotp * ginv : 0.f;
#pragma unroll
                for (int j = 0; j < CHT; ++j) {
                    uint32_t w[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float2 f = unpack_bf16(w[t]);
                        w[t] = valid ? pack_bf16(f.x * ginv, f.y * ginv) : 0u;
                    }
                    *reinterpret_cast<uint4*>(dot_tile + tile_chunk_off(C, r, part * CHT + j)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
                if (part == 0) {
                    __nv_bfloat16* dgt = reinterpret_cast<__nv_bfloat16*>(st + Cfg::OFF_SDG);
                    const __nv_bfloat16 hi = __float2bfloat16_rn(dg);
                    dgt[tile_off(16, 0, r) / 2] = hi;
                    dgt[tile_off(16, 1, r) / 2] = __float2bfloat16_rn(dg - __bfloat162float(hi));
                    reinterpret_cast<float*>(st + Cfg::OFF_SDGF)[r] = dg;
                    if (valid) prm.dgbuf[tok] = dg;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
            if (SPLIT && u < 128) {
                // phi(q) of chunk c (read by R += A^T dU and the epilogue)
                if (!mbar_wait(&fullq[s], (c / NS) & 1, abort_flag)) break;
                phi_tile<PHI, C, D, 128>(st, u, nvalid, true);
                fence_proxy_async_smem();
                mbar_arrive(&phiq_done[s]);
            }
            // SPLIT: the state readout of the previous chunk, after this
            // chunk's feature map (which the next W waits for)
            if (SPLIT && u >= 128 && c > 0 && !readout_dq(c - 1)) break;
        }
        if (SPLIT && u >= 128 && prm.rec_out && nchunks > 0 &&
            named_bar_all(2, 128, mbar_wait(st_ready, (nchunks - 1) & 1, abort_flag))) {
            // the segment's (R, r) after its last chunk
            tc_fence_after();
            const uint32_t lane_base = uint32_t(32 * (warp & 3)) << 16;
            const int frow = acc_row<D>(warp & 3, lane);
            float* out = prm.rec_out + size_t(blockIdx.x) * (D * D + D);
#pragma unroll 1
            for (int v0 = 0; v0 < D; v0 += 32) {
                float rv[32];
                tmem_load<32>(tmem + lane_base + Cfg::T_R + v0, rv);
                store16_f32(out + size_t(frow) * D + v0, rv);
                store16_f32(out + size_t(frow) * D + v0 + 16, rv + 16);
            }
            float rz[16];
            tmem_ld16(tmem + lane_base + Cfg::T_RZ, rz);
            tmem_wait_ld();
            out[size_t(D) * D + frow] = rz[0] + rz[1];
        }
    } else {
        const int e = tid - 320;
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int irow = acc_row<C>(sp, lane);
        const int frow = acc_row<D>(sp, lane);
        uint8_t* sprev = smem + Cfg::OFF_SPREV;
        uint8_t* zop = smem + Cfg::OFF_ZOP;
        uint8_t* eop = smem + Cfg::OFF_E;
        uint8_t* xop = smem + Cfg::OFF_X;
        uint8_t* duop = smem + Cfg::OFF_DU;
        uint8_t* dgop = smem + Cfg::OFF_DG;
        uint8_t* stg = smem + Cfg::OFF_STG;
        float* zf = reinterpret_cast<float*>(smem + Cfg::OFF_ZF);
        __nv_bfloat16* zop_h = reinterpret_cast<__nv_bfloat16*>(zop);
        __nv_bfloat16* dg_h = reinterpret_cast<__nv_bfloat16*>(dgop);
        float* gb = prm.gbuf + size_t(head) * prm.N;
        float* dgb = prm.dgbuf + size_t(head) * prm.N;

        for (int idx = e; idx < 16 * C; idx += 128) {
            const int r = idx / C, cc = idx % C;
            *reinterpret_cast<__nv_bfloat16*>(eop + tile_off(16, r, cc)) =
                __float2bfloat16_rn(r == 0 ? 1.f : 0.f);
            dg_h[tile_off(16, r, cc) / 2] = __float2bfloat16_rn(0.f);
        }
        for (int idx = e; idx < 16 * D; idx += 128) {
            const int r = idx / D, cc = idx % D;
            zop_h[tile_off(16, r, cc) / 2] = __float2bfloat16_rn(0.f);
        }
        named_bar_sync(1, 128);
        // one read of the record row feeds the operand and the accumulator
        load_record_row<D>(st_in, frow, 1.f, sprev, tmem + lane_base + Cfg::T_S, CAUSAL && st_in);
        const float z0 = (st_in && frow >= 0) ? st_in[size_t(D) * D + frow] : 0.f;
        if (frow >= 0) {
            const __nv_bfloat16 zh = __float2bfloat16_rn(z0);
            zop_h[tile_off(16, 0, frow) / 2] = zh;
            zop_h[tile_off(16, 1, frow) / 2] = __float2bfloat16_rn(z0 - __bfloat162float(zh));
            zf[frow] = z0;
        }
        if (CAUSAL && st_in) {
            float z16[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) z16[t] = t == 0 ? z0 : 0.f;
            tmem_st16(tmem + lane_base + Cfg::T_Z, z16);
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(s_ready);

        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            const uint8_t* qt = smem + s * Cfg::STAGE;
            const uint8_t* dot = qt + 3 * Cfg::TILE;
            const int row0 = tok0 + c * C;
            const int nvalid = min(C, tok1 - row0);
            const bool valid = irow >= 0 && irow < nvalid;
            float dg = 0.f;
            if (SAVED) {
                // dU and dg come with the stage (feature-map warps): wait for them
                if (!named_bar_all(1, 128, mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                dg = irow >= 0 ? reinterpret_cast<const float*>(qt + Cfg::OFF_SDGF)[irow] : 0.f;
            } else {
                float den_intra = 0.f;
                if (CAUSAL) {
                    if (!named_bar_all(1, 128, mbar_wait(p_ready, c & 1, abort_flag))) break;
                    tc_fence_after();
                    if (Cfg::XT) {
                        const uint32_t reg = tmem + lane_base + Cfg::T_P;
    #pragma unroll 1
                        for (int j0 = 0; j0 < C; j0 += 32) {
                            float pv[32];
                            tmem_load<32>(reg + j0, pv);
                            float pk[16];
    #pragma unroll
                            for (int t = 0; t < 16; ++t) {
                                const int j = j0 + 2 * t;
                                const uint32_t w = pack_bf16(j <= irow ? pv[2 * t] : 0.f,
                                                             j + 1 <= irow ? pv[2 * t + 1] : 0.f);
                                const float2 r = unpack_bf16(w);
                                den_intra += r.x + r.y;
                                pk[t] = __uint_as_float(w);
                            }
                            tmem_st16(reg + j0 / 2, pk);
                        }
                        tmem_wait_st();
                    } else {
    #pragma unroll 1
                    for (int j0 = 0; j0 < C; j0 += 32) {
                        float pv[32];
                        tmem_ld16(tmem + lane_base + Cfg::T_P + j0, pv);
                        tmem_ld16(tmem + lane_base + Cfg::T_P + j0 + 16, pv + 16);
                        tmem_wait_ld();
                        if (irow >= 0) {
    #pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint32_t w[4];
    #pragma unroll
                                for (int t = 0; t < 4; ++t) {
                                    const int j = j0 + q * 8 + 2 * t;
                                    w[t] = pack_bf16(j <= irow ? pv[q * 8 + 2 * t] : 0.f,
                                                     j + 1 <= irow ? pv[q * 8 + 2 * t + 1] : 0.f);
                                    const float2 r = unpack_bf16(w[t]);
                                    den_intra += r.x + r.y;
                                }
                                *reinterpret_cast<uint4*>(xop + tile_chunk_off(C, irow, (j0 >> 3) + q)) =
                                    make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                    }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(pt_ready);
                }
                // ---- o, g, du, dg
                if (!named_bar_all(1, 128, mbar_wait(o_ready, c & 1, abort_flag))) break;
                tc_fence_after();
                float oz[16];
                tmem_ld16(tmem + lane_base + Cfg::T_OZ, oz);
                tmem_wait_ld();
                const float g = den_intra + oz[0] + oz[1];
                const float ginv = 1.f / g;
                float dotp = 0.f;
    #pragma unroll 1
                for (int v0 = 0; v0 < D; v0 += 16) {
                    float ov[16];
                    tmem_ld16(tmem + lane_base + Cfg::T_O + v0, ov);
                    tmem_wait_ld();
                    if (irow >= 0) {
                        float d8a[8], d8b[8];
                        load_chunk8(dot, C, irow, v0 >> 3, d8a);
                        load_chunk8(dot, C, irow, (v0 >> 3) + 1, d8b);
                        float du16[16];
    #pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            dotp = fmaf(d8a[t], ov[t] * ginv, dotp);
                            dotp = fmaf(d8b[t], ov[8 + t] * ginv, dotp);
                            du16[t] = valid ? d8a[t] * ginv : 0.f;
                            du16[8 + t] = valid ? d8b[t] * ginv : 0.f;
                        }
                        store_row16_bf16(duop, C, irow, v0, du16);
                    }
                }
                dg = valid ? -dotp * ginv : 0.f;
                if (irow >= 0) {
                    const __nv_bfloat16 h = __float2bfloat16_rn(dg);
                    dg_h[tile_off(16, 0, irow) / 2] = h;
                    dg_h[tile_off(16, 1, irow) / 2] = __float2bfloat16_rn(dg - __bfloat162float(h));
                }
                if (valid) {
                    gb[row0 + irow] = g;
                    dgb[row0 + irow] = dg;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(du_ready);
            }
            if (CAUSAL) {
                // ---- W' = (dU V^T + dg) masked
                if (!named_bar_all(1, 128, mbar_wait(w_ready, c & 1, abort_flag))) break;
                tc_fence_after();
                if (Cfg::XT) {
                    const uint32_t reg = tmem + lane_base + Cfg::T_P;
#pragma unroll 1
                    for (int j0 = 0; j0 < C; j0 += 32) {
                        float wv[32];
                        tmem_load<32>(reg + j0, wv);
                        float pk[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const int j = j0 + 2 * t;
                            pk[t] = __uint_as_float(pack_bf16(j <= irow ? wv[2 * t] + dg : 0.f,
                                                              j + 1 <= irow ? wv[2 * t + 1] + dg : 0.f));
                        }
                        tmem_st16(reg + j0 / 2, pk);
                    }
                    tmem_wait_st();
                } else {
#pragma unroll 1
                for (int j0 = 0; j0 < C; j0 += 32) {
                    float wv[32];
                    tmem_ld16(tmem + lane_base + Cfg::T_P + j0, wv);
                    tmem_ld16(tmem + lane_base + Cfg::T_P + j0 + 16, wv + 16);
                    tmem_wait_ld();
                    if (irow >= 0) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t w[4];
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const int j = j0 + q * 8 + 2 * t;
                                w[t] = pack_bf16(j <= irow ? wv[q * 8 + 2 * t] + dg : 0.f,
                                                 j + 1 <= irow ? wv[q * 8 + 2 * t + 1] + dg : 0.f);
                            }
                            *reinterpret_cast<uint4*>(xop + tile_chunk_off(C, irow, (j0 >> 3) + q)) =
                                make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(wt_ready);
            }
            // ---- dQ = (T + t 1) * phi'(q): T = dA + dg z formed with the
            // centred key features phi(k) - c, which differ from the true dA
            // only along the all-ones vector; that component is restored from
            // <dA_i, a_i> = 0 (t = -(T . a_i) / (1 . a_i)).
            {
                // SPLIT: phi(q) of the chunk has its own barrier
                const bool ok = mbar_wait(da_ready, c & 1, abort_flag) &&
                                (!SPLIT || mbar_wait(&phiq_done[s], (c / NS) & 1, abort_flag));
                if (!named_bar_all(1, 128, ok)) break;
            }
            tc_fence_after();
            if (e == 0) bulk_wait_read0();
            named_bar_sync(1, 128);
            const float* zfc = zf + (SPLIT ? (c & 1) * D : 0);  // z of the chunks before c
            constexpr float kc = phi_center<PHI>();
            float tcoef = 0.f;
            if (kc != 0.f) {
                float dot = 0.f, sa = 0.f;
                // 32 columns per TMEM round trip (two loads, one wait)
#pragma unroll 1
                for (int f0 = 0; f0 < D; f0 += 32) {
                    float av[32];
                    tmem_load<32>(tmem + lane_base + Cfg::T_O + f0, av);
                    if (irow >= 0) {
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            float a8[8];
                            load_chunk8(qt, C, irow, (f0 >> 3) + h, a8);
#pragma unroll
                            for (int t = 0; t < 8; ++t) {
                                dot = fmaf(fmaf(dg, zfc[f0 + 8 * h + t], av[8 * h + t]), a8[t], dot);
                                sa += a8[t];
                            }
                        }
                    }
                }
                tcoef = irow >= 0 ? -kc * dot / sa : 0.f;
            }
#pragma unroll 1
            for (int f0 = 0; f0 < D; f0 += 32) {
                float av[32];
                tmem_load<32>(tmem + lane_base + Cfg::T_O + f0, av);
                if (irow >= 0) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float a8a[8], a8b[8];
                        load_chunk8(qt, C, irow, (f0 >> 3) + 2 * h, a8a);
                        load_chunk8(qt, C, irow, (f0 >> 3) + 2 * h + 1, a8b);
                        float dq16[16];
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            const int f = f0 + 16 * h + t;
                            dq16[t] = (fmaf(dg, zfc[f], av[16 * h + t]) + tcoef) *
                                      dphi_from_phi<PHI>(a8a[t]);
                            dq16[8 + t] = (fmaf(dg, zfc[f + 8], av[16 * h + 8 + t]) + tcoef) *
                                          dphi_from_phi<PHI>(a8b[t]);
                        }
                        store_row16_bf16(stg, C, irow, f0 + 16 * h, dq16);
                    }
                }
            }
            if (SPLIT) {
                // dA read: the next chunk's dA MMAs may overwrite it
                tc_fence_before();
                mbar_arrive(s_ready);
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);  // staging complete; every zf read done
            // SPLIT: the state updates read the stage's tiles too
            if (SPLIT) {
                // R += A^T dU reads q too; k, v, dO go back with the
                // products' own commit
                (void)mbar_wait(st_ready, c & 1, abort_flag);
                mbar_arrive(&emptyq[s]);
            } else {
                mbar_arrive(&empty[s]);  // this thread is done with the stage
            }
            if (e == 0) {
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tma_store_3d(&prm.tm_dq, stg + a * C * 128, a * 64, row0, head);
                bulk_commit();
            }
            if (SPLIT) continue;  // the state readout runs on warps 6-9
            // ---- next state operand; segment (R, r) on the last chunk
            if (CAUSAL) {
                // z rides along with the first S columns' round trip
                float zv[16];
                tmem_ld16(tmem + lane_base + Cfg::T_Z, zv);
#pragma unroll 1
                for (int v0 = 0; v0 < D; v0 += 32) {
                    float sv[32];
                    tmem_load<32>(tmem + lane_base + Cfg::T_S + v0, sv);
                    if (frow >= 0) {
                        store_row16_bf16(sprev, D, frow, v0, sv);
                        store_row16_bf16(sprev, D, frow, v0 + 16, sv + 16);
                    }
                }
                if (frow >= 0) {
                    const __nv_bfloat16 zh = __float2bfloat16_rn(zv[0]);
                    zop_h[tile_off(16, 0, frow) / 2] = zh;
                    zop_h[tile_off(16, 1, frow) / 2] = __float2bfloat16_rn(zv[0] - __bfloat162float(zh));
                    zf[frow] = zv[0];
                }
            }
            if (rec && c == nchunks - 1) {
                float* out = prm.rec_out + size_t(blockIdx.x) * (D * D + D);
#pragma unroll 1
                for (int v0 = 0; v0 < D; v0 += 16) {
                    float rv[16];
                    tmem_ld16(tmem + lane_base + Cfg::T_R + v0, rv);
                    tmem_wait_ld();
                    if (frow >= 0)
                        for (int t = 0; t < 16; ++t) out[size_t(frow) * D + v0 + t] = rv[t];
                }
                float rz[16];
                tmem_ld16(tmem + lane_base + Cfg::T_RZ, rz);
                tmem_wait_ld();
                if (frow >= 0) out[size_t(D) * D + frow] = rz[0] + rz[1];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(s_ready);
        }
        if (e == 0) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::T_COLS);
}

// ======================================================================
// Pass 2: dK, dV (reverse token order).
// ======================================================================
// PART: grouped key/value heads, dK and dV stored as float32 per-query-head
// partials (prm.dk_part, dv_part) instead of the bf16 tiles.
//
// SPLIT (causal, D = 128): the suffix-state readout (R -> the bf16 operand
// of the next, earlier chunk, r -> rf) runs on the key half of the
// feature-map warps (warps 6-9) while the epilogue warps form dV and dK, so
// the two TMEM readouts of a step overlap.
template <int D, int C, int PHI, bool CAUSAL, bool PART = false>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dkdv_kernel(const __grid_constant__ BwdParams prm) {
    using namespace sm100;
    using Cfg = Bwd2Cfg<D, C>;
    constexpr int NS = Cfg::NSTAGE;
    constexpr bool SPLIT = CAUSAL && D == 128 && !Cfg::XT;
    static_assert(!SPLIT || 2 * D * 4 <= 1024, "two copies of r in the rf area");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* phi_done = bars + NS;
    uint64_t* empty = bars + 2 * NS;    // released by the epilogue (count 128)
    uint64_t* x_ready = bars + 3 * NS;  // commit: B A^T, V dU^T
    uint64_t* xt_ready = x_ready + 1;   // 128: X1, X2 written
    uint64_t* d_ready = x_ready + 2;    // commit: dV, dB, R
    uint64_t* r_ready = x_ready + 3;    // 128: R operand for the next (earlier) chunk
    uint64_t* drain = x_ready + 4;
    uint64_t* r_done = x_ready + 5;     // commit (SPLIT): R, r updated
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

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&phi_done[s], 256);
            mbar_init(&empty[s], 128);
        }
        mbar_init(x_ready, 1);
        mbar_init(xt_ready, 128);
        mbar_init(d_ready, 1);
        mbar_init(r_ready, SPLIT ? 256 : 128);
        mbar_init(drain, 1);
        mbar_init(r_done, 1);
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

    // chunk processed at step t (reverse order)
    auto chunk_of = [&](int t) { return nchunks - 1 - t; };

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
                const int row = tok0 + chunk_of(t) * C;
#pragma unroll
                for (int a = 0; a < D / 64; ++a) {
                    tma_load_3d(st + a * C * 128, &prm.tm_q, &full[s], a * 64, row, head);
                    tma_load_3d(st + Cfg::TILE + a * C * 128, &prm.tm_k, &full[s], a * 64, row,
                                kv_head);
                    tma_load_3d(st + 2 * Cfg::TILE + a * C * 128, &prm.tm_v, &full[s], a * 64, row,
                                kv_head);
                    tma_load_3d(st + 3 * Cfg::TILE + a * C * 128, &prm.tm_do, &full[s], a * 64, row,
                                head);
                }
                issued = t + 1;
            }
            for (int t = max(0, issued - NS); t < issued; ++t)
                mbar_wait_drain(&full[t % NS], (t / NS) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t t1 = tmem + Cfg::T_1, t2 = tmem + Cfg::T_2, t3 = tmem + Cfg::T_3;
            const uint32_t t4 = tmem + Cfg::T_4, tR = tmem + Cfg::T_R, tRZ = tmem + Cfg::T_RZ;
            const uint32_t rprev = sbase + Cfg::OFF_RPREV;
            const uint32_t x1 = sbase + Cfg::OFF_X1, x2 = sbase + Cfg::OFF_X2;
            constexpr uint32_t idCC = idesc_bf16(C, C, 0, 0);
            constexpr uint32_t idCD_mn = idesc_bf16(C, D, 0, 1);
            constexpr uint32_t idCD_k = idesc_bf16(C, D, 0, 0);
            constexpr uint32_t idDD = idesc_bf16(D, D, 1, 1);
            constexpr uint32_t idD16 = idesc_bf16(D, 16, 1, 0);
            const bool has_init = st_in != nullptr;
            bool ok = true;
            for (int t = 0; ok && t < nchunks; ++t) {
                const int s = t % NS;
                const uint32_t qs = sbase + s * Cfg::STAGE, ks = qs + Cfg::TILE;
                const uint32_t vs = qs + 2 * Cfg::TILE, dus = qs + 3 * Cfg::TILE;
                const uint32_t dgs = qs + Cfg::OFF_DGT;
                if (!(ok = mbar_wait(&phi_done[s], (t / NS) & 1, abort_flag))) break;
                if (!(ok = mbar_wait(r_ready, t & 1, abort_flag))) break;
                tc_fence_after();
                if (CAUSAL) {
#pragma unroll
                    for (int k = 0; k < D; k += 16) {
                        // B A^T and V dU^T
                        umma_bf16(t1, desc_kmajor(ks, C, k), desc_kmajor(qs, C, k), idCC, k > 0);
                        umma_bf16(t2, desc_kmajor(vs, C, k), desc_kmajor(dus, C, k), idCC, k > 0);
                    }
                    umma_commit(x_ready);
                    if (!(ok = mbar_wait(xt_ready, t & 1, abort_flag))) break;
                    tc_fence_after();
                    if (Cfg::XT) {
#pragma unroll
                        for (int k = 0; k < C; k += 16) {
                            umma_bf16_ts(t3, t1 + k / 2, desc_mnmajor(dus, C, k), idCD_mn, k > 0);
                            umma_bf16_ts(t4, t2 + k / 2, desc_mnmajor(qs, C, k), idCD_mn, k > 0);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < C; k += 16) {
                            umma_bf16(t3, desc_kmajor(x1, C, k), desc_mnmajor(dus, C, k), idCD_mn,
                                      k > 0);
                            umma_bf16(t4, desc_kmajor(x2, C, k), desc_mnmajor(qs, C, k), idCD_mn,
                                      k > 0);
                        }
                    }
                }
#pragma unroll
                for (int k = 0; k < D; k += 16) {
                    // dV += B R, dB += V R^T
                    umma_bf16(t3, desc_kmajor(ks, C, k), desc_mnmajor(rprev, D, k), idCD_mn,
                              (CAUSAL || k > 0) ? 1u : 0u);
                    umma_bf16(t4, desc_kmajor(vs, C, k), desc_kmajor(rprev, D, k), idCD_k,
                              (CAUSAL || k > 0) ? 1u : 0u);
                }
                // SPLIT: dV, dB are complete here; the epilogue starts on
                // them while the suffix state updates
                if (SPLIT) umma_commit(d_ready);
                if (CAUSAL) {
#pragma unroll
                    for (int k = 0; k < C; k += 16) {
                        const uint32_t acc = (t > 0 || has_init || k > 0) ? 1u : 0u;
                        umma_bf16(tR, desc_mnmajor(qs, C, k), desc_mnmajor(dus, C, k), idDD, acc);
                        umma_bf16(tRZ, desc_mnmajor(qs, C, k), desc_kmajor(dgs, 16, k), idD16, acc);
                    }
                }
                umma_commit(SPLIT ? r_done : d_ready);
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < 10) {
        // phi on Q and K, dU = dO / g, DG rows = (dg_hi, dg_lo); 8 warps
        const int u = tid - 64;  // 0..255
        for (int s = 0; s < NS; ++s) {
            __nv_bfloat16* dgt = reinterpret_cast<__nv_bfloat16*>(smem + s * Cfg::STAGE + Cfg::OFF_DGT);
            for (int idx = u; idx < 16 * C; idx += 256) {
                const int r = idx / C, cc = idx % C;
                dgt[tile_off(16, r, cc) / 2] = __float2bfloat16_rn(0.f);
            }
        }
        const float* gb = prm.gbuf + size_t(head) * prm.N;
        const float* dgb = prm.dgbuf + size_t(head) * prm.N;
        // SPLIT, warps 6-9 (one TMEM lane quarter each): after step t's
        // products, R -> the bf16 operand of step t + 1 and r -> rf (the
        // copy of the other parity)
        auto readout_dkdv = [&](int t) {
            if (!named_bar_all(2, 128, mbar_wait(r_done, t & 1, abort_flag))) return;
            tc_fence_after();
            const uint32_t lane_base = uint32_t(32 * (warp & 3)) << 16;
            const int frow = acc_row<D>(warp & 3, lane);
            float rz[16];
            tmem_ld16(tmem + lane_base + Cfg::T_RZ, rz);
#pragma unroll 1
            for (int v0 = 0; v0 < D; v0 += 32) {
                float rv[32];
                tmem_load<32>(tmem + lane_base + Cfg::T_R + v0, rv);
                store_row16_bf16(smem + Cfg::OFF_RPREV, D, frow, v0, rv);
                store_row16_bf16(smem + Cfg::OFF_RPREV, D, frow, v0 + 16, rv + 16);
            }
            reinterpret_cast<float*>(smem + Cfg::OFF_RF)[((t + 1) & 1) * D + frow] = rz[0] + rz[1];
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(r_ready);
        };
        // the readout warps' share of the initial state's arrival
        if (SPLIT && u >= 128) mbar_arrive(r_ready);
        for (int t = 0; t < nchunks; ++t) {
            const int s = t % NS;
            if (!mbar_wait(&full[s], (t / NS) & 1, abort_flag)) break;
            uint8_t* st = smem + s * Cfg::STAGE;
            const int row0 = tok0 + chunk_of(t) * C;
            const int nvalid = min(C, tok1 - row0);
            __nv_bfloat16* dgt = reinterpret_cast<__nv_bfloat16*>(st + Cfg::OFF_DGT);
            float* dgf = reinterpret_cast<float*>(st + Cfg::OFF_DGF);
            float* rinv = reinterpret_cast<float*>(st + Cfg::OFF_RINV);
            if (u < C) {
                const bool valid = u < nvalid;
                const float dg = valid ? dgb[row0 + u] : 0.f;
                rinv[u] = valid ? 1.f / gb[row0 + u] : 0.f;
                const __nv_bfloat16 h = __float2bfloat16_rn(dg);
                dgt[tile_off(16, 0, u) / 2] = h;
                dgt[tile_off(16, 1, u) / 2] = __float2bfloat16_rn(dg - __bfloat162float(h));
                dgf[u] = dg;
            }
            named_bar_sync(3, 256);  // rinv ready
            if (u < 128)
                phi_tile<PHI, C, D, 128>(st, u, nvalid, true);
            else
                phi_tile<PHI, C, D, 128>(st + Cfg::TILE, u - 128, nvalid, true);
            scale_tile_rows<C, D, 256>(st + 3 * Cfg::TILE, u, nvalid, rinv);
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
            // SPLIT: the suffix-state readout of the previous step, after
            // this step's feature map (which this step's products wait for).
            // A failed wait skips it but stays in the loop, so the
            // 256-thread barrier above keeps its members.
            if (SPLIT && u >= 128 && t > 0) readout_dkdv(t - 1);
        }
    } else {
        const int e = tid - 320;
        const int sp = warp & 3;
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int jrow = acc_row<C>(sp, lane);
        const int frow = acc_row<D>(sp, lane);
        uint8_t* rprev = smem + Cfg::OFF_RPREV;
        float* rf = reinterpret_cast<float*>(smem + Cfg::OFF_RF);
        uint8_t* x1 = smem + Cfg::OFF_X1;
        uint8_t* x2 = smem + Cfg::OFF_X2;
        uint8_t* stgv = smem + Cfg::OFF_STGV;
        uint8_t* stgk = smem + Cfg::OFF_STGK;

        // one read of the record row feeds the operand and the accumulator
        load_record_row<D>(st_in, frow, 1.f, rprev, tmem + lane_base + Cfg::T_R, CAUSAL && st_in);
        const float r0 = (st_in && frow >= 0) ? st_in[size_t(D) * D + frow] : 0.f;
        if (frow >= 0) rf[frow] = r0;
        if (CAUSAL && st_in) {
            float z16[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) z16[t] = t == 0 ? r0 : 0.f;
            tmem_st16(tmem + lane_base + Cfg::T_RZ, z16);
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(r_ready);

        for (int t = 0; t < nchunks; ++t) {
            const int s = t % NS;
            const uint8_t* st = smem + s * Cfg::STAGE;
            const uint8_t* kt = st + Cfg::TILE;
            const float* dgf = reinterpret_cast<const float*>(st + Cfg::OFF_DGF);
            const int row0 = tok0 + chunk_of(t) * C;
            if (CAUSAL) {
                if (!named_bar_all(1, 128, mbar_wait(x_ready, t & 1, abort_flag))) break;
                tc_fence_after();
                if (Cfg::XT) {
                    // mask and pack X1, X2 in place in TMEM (block i0 is read
                    // before columns i0/2.. are overwritten)
                    const uint32_t r1 = tmem + lane_base + Cfg::T_1;
                    const uint32_t r2 = tmem + lane_base + Cfg::T_2;
#pragma unroll 1
                    for (int i0 = 0; i0 < C; i0 += 32) {
                        float pv[32], wv[32];
                        tmem_load<32>(r1 + i0, pv);
                        tmem_load<32>(r2 + i0, wv);
                        float a16[16], b16[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int i = i0 + 2 * k;
                            a16[k] = __uint_as_float(pack_bf16(i >= jrow ? pv[2 * k] : 0.f,
                                                               i + 1 >= jrow ? pv[2 * k + 1] : 0.f));
                            b16[k] = __uint_as_float(
                                pack_bf16(i >= jrow ? wv[2 * k] + dgf[i] : 0.f,
                                          i + 1 >= jrow ? wv[2 * k + 1] + dgf[i + 1] : 0.f));
                        }
                        tmem_st16(r1 + i0 / 2, a16);
                        tmem_st16(r2 + i0 / 2, b16);
                    }
                    tmem_wait_st();
                } else {
                if (Cfg::STG_ALIAS) {
                    if (e == 0) bulk_wait_read0();
                    named_bar_sync(1, 128);
                }
                // 32 columns of each product per TMEM round trip
#pragma unroll 1
                for (int i0 = 0; i0 < C; i0 += 32) {
                    float pv[32], wv[32];
                    sm100::tmem_ld16(tmem + lane_base + Cfg::T_1 + i0, pv);
                    sm100::tmem_ld16(tmem + lane_base + Cfg::T_1 + i0 + 16, pv + 16);
                    sm100::tmem_ld16(tmem + lane_base + Cfg::T_2 + i0, wv);
                    sm100::tmem_ld16(tmem + lane_base + Cfg::T_2 + i0 + 16, wv + 16);
                    tmem_wait_ld();
                    if (jrow >= 0) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            float a16[16], b16[16];
#pragma unroll
                            for (int k = 0; k < 16; ++k) {
                                const int i = i0 + 16 * h + k;
                                a16[k] = i >= jrow ? pv[16 * h + k] : 0.f;
                                b16[k] = i >= jrow ? wv[16 * h + k] + dgf[i] : 0.f;
                            }
                            store_row16_bf16(x1, C, jrow, i0 + 16 * h, a16);
                            store_row16_bf16(x2, C, jrow, i0 + 16 * h, b16);
                        }
                    }
                }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(xt_ready);
            }
            if (!named_bar_all(1, 128, mbar_wait(d_ready, t & 1, abort_flag))) break;
            tc_fence_after();
            if (Cfg::XT || !Cfg::STG_ALIAS || !CAUSAL) {
                if (e == 0) bulk_wait_read0();
                named_bar_sync(1, 128);
            }
            const float* rfc = rf + (SPLIT ? (t & 1) * D : 0);  // r of the later chunks
            // SPLIT: 32 columns of dV and of dB per TMEM round trip
            constexpr int NCOL = SPLIT ? 32 : 16;
#pragma unroll 1
            for (int c00 = 0; c00 < D; c00 += NCOL) {
                float dvw[NCOL], dbw[NCOL];
#pragma unroll
                for (int h = 0; h < NCOL / 16; ++h) {
                    tmem_ld16(tmem + lane_base + Cfg::T_3 + c00 + 16 * h, dvw + 16 * h);
                    tmem_ld16(tmem + lane_base + Cfg::T_4 + c00 + 16 * h, dbw + 16 * h);
                }
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < NCOL / 16; ++h) {
                    const int c0 = c00 + 16 * h;
                    const float* dv16 = dvw + 16 * h;
                    const float* db16 = dbw + 16 * h;
                    if (jrow >= 0) {
                        float b8a[8], b8b[8];
                        load_chunk8(kt, C, jrow, c0 >> 3, b8a);
                        load_chunk8(kt, C, jrow, (c0 >> 3) + 1, b8b);
                        float dk16[16];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            dk16[k] = (db16[k] + rfc[c0 + k]) * dphi_from_phi<PHI>(b8a[k]);
                            dk16[8 + k] = (db16[8 + k] + rfc[c0 + 8 + k]) * dphi_from_phi<PHI>(b8b[k]);
                        }
                        if constexpr (PART) {
                            if (row0 + jrow < prm.N) {
                                const size_t off = (size_t(head) * prm.N + row0 + jrow) * D + c0;
                                store16_f32(prm.dv_part + off, dv16);
                                store16_f32(prm.dk_part + off, dk16);
                            }
                        } else {
                            store_row16_bf16(stgv, C, jrow, c0, dv16);
                            store_row16_bf16(stgk, C, jrow, c0, dk16);
                        }
                    }
                }
            }
            if (SPLIT) {
                // dV, dB read: the next step's products may overwrite them
                tc_fence_before();
                mbar_arrive(r_ready);
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 128);  // staging complete; every rf read done
            // SPLIT: the suffix-state update reads the stage's tiles too
            if (SPLIT) (void)mbar_wait(r_done, t & 1, abort_flag);
            mbar_arrive(&empty[s]);
            if (e == 0 && !PART) {
#pragma unroll
                for (int a = 0; a < D / 64; ++a) {
                    tma_store_3d(&prm.tm_dv, stgv + a * C * 128, a * 64, row0, head);
                    tma_store_3d(&prm.tm_dk, stgk + a * C * 128, a * 64, row0, head);
                }
                bulk_commit();
            }
            if (SPLIT) continue;  // the suffix-state readout runs on warps 6-9
            if (CAUSAL) {
                // r rides along with the first R columns' round trip
                float rz[16];
                tmem_ld16(tmem + lane_base + Cfg::T_RZ, rz);
#pragma unroll 1
                for (int v0 = 0; v0 < D; v0 += 32) {
                    float rv[32];
                    tmem_load<32>(tmem + lane_base + Cfg::T_R + v0, rv);
                    if (frow >= 0) {
                        store_row16_bf16(rprev, D, frow, v0, rv);
                        store_row16_bf16(rprev, D, frow, v0 + 16, rv + 16);
                    }
                }
                if (frow >= 0) rf[frow] = rz[0] + rz[1];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(r_ready);
        }
        if (e == 0) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, Cfg::T_COLS);
}

}  // namespace la
