// la_chunk_fwd.cuh — chunked linear-attention forward on sm_100a tensor cores.
//
// One kernel template, three modes, one thread block per (head, segment):
//
//  CAUSAL  the causal forward over a run of C-token chunks.  Per chunk c,
//          with A = phi(Q_c), B = phi(K_c) and the state S (D x D) and z (D)
//          of every earlier token:
//              P   = A B^T                     (C x C, tensor cores)
//              num = (P . tril) V_c + A S      (tensor cores)
//              den = rowsum(P . tril) + A z    (rowsum on CUDA cores, A z on
//                                               tensor cores with z split into
//                                               two bf16 terms)
//              O_c = num / den
//              S  += B^T V_c,  z += B^T 1      (tensor cores, fp32 in TMEM)
//          Inside a chunk this is the quadratic form, across chunks the
//          associativity reorder (QK^T)V = Q(K^T V) of "Efficient Transformers
//          Survey", Proposition "Linear Attention via Kernel Decomposition"
//          (Intuition), with S and z carried chunk to chunk as in its "Why It
//          Matters" paragraph.
//  REDUCE  only S += B^T V, z += B^T 1 over the segment; writes the segment's
//          (S, z) to global memory (non-causal totals, causal segment sums).
//  QUERY   O = A S / (A z) against a fixed (S, z) read from global memory
//          (the non-causal query pass: "each attention output costs O(md)").
//
// Data flow: a producer warp streams Q/K/V chunk tiles with TMA (128-byte
// swizzle) into an NSTAGE-deep ring; a feature-map warpgroup applies phi in
// place; one thread issues tcgen05.mma with fp32 accumulators in TMEM; an
// epilogue warpgroup masks P, forms O = num/den, stores O with TMA and
// converts the updated state to the bf16 operand of the next chunk.  All
// handshakes are mbarriers with bounded waits.
#pragma once

#include "la_common.cuh"
#include "la_sm100.cuh"

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
};

template <int D, int C>
struct ChunkCfg {
    static constexpr int NSTAGE = 3;
    static constexpr int TILE_QKV = C * D * 2;  // bytes of one [C][D] bf16 tile
    static constexpr int STAGE = 3 * TILE_QKV;
    static constexpr int OFF_STAGES = 0;
    static constexpr int OFF_SPREV = NSTAGE * STAGE;
    static constexpr int OFF_ZOP = OFF_SPREV + D * D * 2;
    static constexpr int OFF_E = OFF_ZOP + 16 * D * 2;
    static constexpr int OFF_PT = OFF_E + 16 * C * 2;
    static constexpr int OFF_OST = OFF_PT + C * C * 2;
    static constexpr int OFF_BAR = OFF_OST + C * D * 2;
    static constexpr int NBAR = 3 * NSTAGE + 5;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
    // TMEM columns
    static constexpr int T_P = 0;
    static constexpr int T_O = C;
    static constexpr int T_OZ = C + D;
    static constexpr int T_S = C + D + 16;
    static constexpr int T_Z = C + 2 * D + 16;
    static constexpr int T_COLS = 512;
    static_assert(T_Z + 16 <= T_COLS, "TMEM budget");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(C == 64 || C == 128, "chunk");
    static_assert(D == 64 || D == 128, "head size");
};

constexpr int kChunkThreads = 320;  // producer, MMA, 4 phi warps, 4 epilogue warps

template <int D, int C, int PHI, int MODE>
__global__ void __launch_bounds__(kChunkThreads, 1)
chunk_fwd_kernel(const __grid_constant__ ChunkParams prm) {
    using namespace sm100;
    using Cfg = ChunkCfg<D, C>;
    constexpr int NS = Cfg::NSTAGE;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
    uint64_t* full = bars;                 // TMA landed             (count 1 + tx)
    uint64_t* phi_done = bars + NS;        // phi applied            (count 128)
    uint64_t* empty = bars + 2 * NS;       // MMAs done with stage   (commit)
    uint64_t* p_ready = bars + 3 * NS;     // P, A S, A z in TMEM    (commit)
    uint64_t* pt_ready = p_ready + 1;      // masked P in smem       (count 128)
    uint64_t* o_ready = p_ready + 2;       // O, state in TMEM       (commit)
    uint64_t* s_ready = p_ready + 3;       // state operand ready    (count 128)
    uint64_t* drain = p_ready + 4;         // every MMA finished     (commit)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x / prm.nseg;
    const int seg = blockIdx.x % prm.nseg;
    const int tok0 = seg * prm.seg_len;
    const int tok1 = min(prm.N, tok0 + prm.seg_len);
    const int nchunks = (tok1 - tok0 + C - 1) / C;
    const float* st_in = prm.state_in
                             ? prm.state_in + size_t(prm.in_per_head ? head : blockIdx.x) *
                                                  size_t(D * D + D)
                             : nullptr;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&phi_done[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(p_ready, 1);
        mbar_init(pt_ready, 128);
        mbar_init(o_ready, 1);
        mbar_init(s_ready, 128);
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
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            if (kQ) tma_prefetch_desc(&prm.tm_q);
            if (kKV) {
                tma_prefetch_desc(&prm.tm_k);
                tma_prefetch_desc(&prm.tm_v);
            }
            constexpr uint32_t bytes = Cfg::TILE_QKV * ((kQ ? 1 : 0) + (kKV ? 2 : 0));
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % NS;
                if (c >= NS && !mbar_wait(&empty[s], ((c / NS) - 1) & 1, abort_flag)) break;
                uint8_t* st = smem + Cfg::OFF_STAGES + s * Cfg::STAGE;
                mbar_arrive_expect_tx(&full[s], bytes);
                const int row = tok0 + c * C;
#pragma unroll
                for (int a = 0; a < D / 64; ++a) {
                    if (kQ) tma_load_3d(st + a * C * 128, &prm.tm_q, &full[s], a * 64, row, head);
                    if (kKV) {
                        tma_load_3d(st + Cfg::TILE_QKV + a * C * 128, &prm.tm_k, &full[s], a * 64,
                                    row, head);
                        tma_load_3d(st + 2 * Cfg::TILE_QKV + a * C * 128, &prm.tm_v, &full[s],
                                    a * 64, row, head);
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
            const uint32_t tP = tmem + Cfg::T_P, tO = tmem + Cfg::T_O, tOZ = tmem + Cfg::T_OZ;
            const uint32_t tS = tmem + Cfg::T_S, tZ = tmem + Cfg::T_Z;
            const uint32_t sprev = sbase + Cfg::OFF_SPREV, zop = sbase + Cfg::OFF_ZOP;
            const uint32_t eop = sbase + Cfg::OFF_E, pt = sbase + Cfg::OFF_PT;
            constexpr uint32_t idP = idesc_bf16(C, C, 0, 0);    // A B^T
            constexpr uint32_t idO = idesc_bf16(C, D, 0, 1);    // A S
            constexpr uint32_t idOZ = idesc_bf16(C, 16, 0, 0);  // A [z_hi z_lo]^T
            constexpr uint32_t idPV = idesc_bf16(C, D, 0, 1);   // (P.tril) V
            constexpr uint32_t idS = idesc_bf16(D, D, 1, 1);    // B^T V
            constexpr uint32_t idSZ = idesc_bf16(D, 16, 1, 0);  // B^T [1 0 ...]
            const bool has_init = st_in != nullptr;
            bool ok = mbar_wait(s_ready, 0, abort_flag);
            for (int c = 0; ok && c < nchunks; ++c) {
                const int s = c % NS;
                const uint32_t qs = sbase + Cfg::OFF_STAGES + s * Cfg::STAGE;
                const uint32_t ks = qs + Cfg::TILE_QKV, vs = qs + 2 * Cfg::TILE_QKV;
                if (!(ok = mbar_wait(&phi_done[s], (c / NS) & 1, abort_flag))) break;
                if (MODE != MODE_REDUCE && c > 0 &&
                    !(ok = mbar_wait(s_ready, c & 1, abort_flag)))
                    break;
                tc_fence_after();
                if (MODE == MODE_CAUSAL) {
#pragma unroll
                    for (int k = 0; k < D; k += 16)
                        umma_bf16(tP, desc_kmajor(qs, C, k), desc_kmajor(ks, C, k), idP, k > 0);
                }
                if (MODE != MODE_REDUCE) {
#pragma unroll
                    for (int k = 0; k < D; k += 16) {
                        umma_bf16(tO, desc_kmajor(qs, C, k), desc_mnmajor(sprev, D, k), idO, k > 0);
                        umma_bf16(tOZ, desc_kmajor(qs, C, k), desc_kmajor(zop, 16, k), idOZ, k > 0);
                    }
                }
                if (MODE == MODE_CAUSAL) {
                    umma_commit(p_ready);
                    if (!(ok = mbar_wait(pt_ready, c & 1, abort_flag))) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < C; k += 16)
                        umma_bf16(tO, desc_kmajor(pt, C, k), desc_mnmajor(vs, C, k), idPV, 1);
                }
                if (MODE != MODE_QUERY) {
#pragma unroll
                    for (int k = 0; k < C; k += 16) {
                        const uint32_t acc = (c > 0 || has_init || k > 0) ? 1u : 0u;
                        umma_bf16(tS, desc_mnmajor(ks, C, k), desc_mnmajor(vs, C, k), idS, acc);
                        umma_bf16(tZ, desc_mnmajor(ks, C, k), desc_kmajor(eop, 16, k), idSZ, acc);
                    }
                }
                if (MODE != MODE_REDUCE) umma_commit(o_ready);
                umma_commit(&empty[s]);
            }
            if (MODE == MODE_REDUCE) umma_commit(o_ready);
            // every MMA issued above completes before TMEM is released
            umma_commit(drain);
            mbar_wait_drain(drain, 0);
        }
    } else if (warp < 6) {
        // ------------------------------------------- feature-map warpgroup
        const int u = tid - 64;  // 0..127
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            if (!mbar_wait(&full[s], (c / NS) & 1, abort_flag)) break;
            uint8_t* st = smem + Cfg::OFF_STAGES + s * Cfg::STAGE;
            const int nvalid = min(C, tok1 - (tok0 + c * C));
            constexpr int first = kQ ? 0 : C;
            constexpr int last = kKV ? 2 * C : C;
            for (int r = first + u; r < last; r += 128) {
                const bool isk = r >= C;
                const int row = isk ? r - C : r;
                uint8_t* tile = st + (isk ? Cfg::TILE_QKV : 0);
                const bool zero = isk && row >= nvalid;
#pragma unroll
                for (int q = 0; q < D / 8; ++q) {
                    uint4* p = reinterpret_cast<uint4*>(tile + tile_chunk_off(C, row, q));
                    uint4 x = *p;
                    uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float2 f = unpack_bf16(w[t]);
                        w[t] = zero ? 0u : pack_bf16(phi_fast<PHI>(f.x), phi_fast<PHI>(f.y));
                    }
                    *p = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&phi_done[s]);
        }
    } else {
        // ------------------------------------------------ epilogue warpgroup
        const int e = tid - 192;      // 0..127
        const int sp = warp & 3;      // TMEM sub-partition of this warp
        const uint32_t lane_base = uint32_t(32 * sp) << 16;
        const int irow = acc_row<C>(sp, lane);  // token row of this thread (or -1)
        const int frow = acc_row<D>(sp, lane);  // state row of this thread (or -1)
        uint8_t* sprev = smem + Cfg::OFF_SPREV;
        uint8_t* zop = smem + Cfg::OFF_ZOP;
        uint8_t* eop = smem + Cfg::OFF_E;
        uint8_t* pt = smem + Cfg::OFF_PT;
        uint8_t* ost = smem + Cfg::OFF_OST;
        __nv_bfloat16* zop_h = reinterpret_cast<__nv_bfloat16*>(zop);

        // ---- constant operand E (row 0 = ones) and the zero rows of Zop
        for (int idx = e; idx < 16 * C; idx += 128) {
            const int r = idx / C, cc = idx % C;
            *reinterpret_cast<__nv_bfloat16*>(eop + tile_off(16, r, cc)) =
                __float2bfloat16_rn(r == 0 ? 1.f : 0.f);
        }
        for (int idx = e; idx < 16 * D; idx += 128) {
            const int r = idx / D, cc = idx % D;
            zop_h[tile_off(16, r, cc) / 2] = __float2bfloat16_rn(0.f);
        }
        named_bar_sync(1, 128);  // zero rows written before row 0/1 of Zop below
        // ---- initial state: bf16 operand (+ TMEM accumulator in CAUSAL mode)
        if (MODE != MODE_REDUCE) {
            if (frow >= 0) {
                for (int q = 0; q < D / 8; ++q) {
                    float v8[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t)
                        v8[t] = st_in ? st_in[size_t(frow) * D + q * 8 + t] : 0.f;
                    *reinterpret_cast<uint4*>(sprev + tile_chunk_off(D, frow, q)) =
                        make_uint4(pack_bf16(v8[0], v8[1]), pack_bf16(v8[2], v8[3]),
                                   pack_bf16(v8[4], v8[5]), pack_bf16(v8[6], v8[7]));
                }
                const float zf = st_in ? st_in[size_t(D) * D + frow] : 0.f;
                const __nv_bfloat16 zh = __float2bfloat16_rn(zf);
                zop_h[tile_off(16, 0, frow) / 2] = zh;
                zop_h[tile_off(16, 1, frow) / 2] = __float2bfloat16_rn(zf - __bfloat162float(zh));
            }
        }
        if (MODE == MODE_CAUSAL && st_in) {
            // TMEM accumulator starts at the initial state (all lanes execute)
            for (int cc = 0; cc < D; cc += 16) {
                float v16[16];
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    v16[t] = frow >= 0 ? st_in[size_t(frow) * D + cc + t] : 0.f;
                tmem_st16(tmem + lane_base + Cfg::T_S + cc, v16);
            }
            float z16[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) z16[t] = (t == 0 && frow >= 0) ? st_in[size_t(D) * D + frow] : 0.f;
            tmem_st16(tmem + lane_base + Cfg::T_Z, z16);
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(s_ready);

        if (MODE == MODE_REDUCE) {
            if (mbar_wait(o_ready, 0, abort_flag)) {
                tc_fence_after();
                const size_t idx = blockIdx.x;
                for (int cc = 0; cc < D; cc += 16) {
                    float v16[16];
                    tmem_ld16(tmem + lane_base + Cfg::T_S + cc, v16);
                    tmem_wait_ld();
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
                tmem_ld16(tmem + lane_base + Cfg::T_Z, z16);
                tmem_wait_ld();
                if (frow >= 0) prm.z_out[idx * prm.stride_z + frow] = z16[0];
            }
        } else {
            for (int c = 0; c < nchunks; ++c) {
                const int row0 = tok0 + c * C;
                float den_intra = 0.f;
                if (MODE == MODE_CAUSAL) {
                    // ---- P -> masked bf16 P in smem, intra-chunk row sums
                    if (!named_bar_all(1, 128, mbar_wait(p_ready, c & 1, abort_flag))) break;
                    tc_fence_after();
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
                                    const float a = j <= irow ? pv[q * 8 + 2 * t] : 0.f;
                                    const float b = j + 1 <= irow ? pv[q * 8 + 2 * t + 1] : 0.f;
                                    w[t] = pack_bf16(a, b);
                                    const float2 r = unpack_bf16(w[t]);
                                    den_intra += r.x + r.y;
                                }
                                *reinterpret_cast<uint4*>(
                                    pt + tile_chunk_off(C, irow, (j0 >> 3) + q)) =
                                    make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(pt_ready);
                }
                // ---- O = num / den -> smem -> TMA store
                if (!named_bar_all(1, 128, mbar_wait(o_ready, c & 1, abort_flag))) break;
                tc_fence_after();
                if (e == 0) bulk_wait_read0();
                named_bar_sync(1, 128);
                float oz[16];
                tmem_ld16(tmem + lane_base + Cfg::T_OZ, oz);
                tmem_wait_ld();
                const float inv = 1.f / (den_intra + oz[0] + oz[1]);
#pragma unroll 1
                for (int v0 = 0; v0 < D; v0 += 32) {
                    float ov[32];
                    tmem_ld16(tmem + lane_base + Cfg::T_O + v0, ov);
                    tmem_ld16(tmem + lane_base + Cfg::T_O + v0 + 16, ov + 16);
                    tmem_wait_ld();
                    if (irow >= 0) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float* x = ov + q * 8;
                            *reinterpret_cast<uint4*>(ost + tile_chunk_off(C, irow, (v0 >> 3) + q)) =
                                make_uint4(pack_bf16(x[0] * inv, x[1] * inv),
                                           pack_bf16(x[2] * inv, x[3] * inv),
                                           pack_bf16(x[4] * inv, x[5] * inv),
                                           pack_bf16(x[6] * inv, x[7] * inv));
                        }
                    }
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (e == 0) {
#pragma unroll
                    for (int a = 0; a < D / 64; ++a)
                        tma_store_3d(&prm.tm_o, ost + a * C * 128, a * 64, row0, head);
                    bulk_commit();
                }
                // ---- state S_{<=c} -> bf16 operand for the next chunk
                if (MODE == MODE_CAUSAL) {
                    const bool last = c == nchunks - 1;
                    const bool write_final = last && seg == prm.nseg - 1;
#pragma unroll 1
                    for (int v0 = 0; v0 < D; v0 += 16) {
                        float sv[16];
                        tmem_ld16(tmem + lane_base + Cfg::T_S + v0, sv);
                        tmem_wait_ld();
                        if (frow >= 0) {
                            *reinterpret_cast<uint4*>(sprev + tile_chunk_off(D, frow, v0 >> 3)) =
                                make_uint4(pack_bf16(sv[0], sv[1]), pack_bf16(sv[2], sv[3]),
                                           pack_bf16(sv[4], sv[5]), pack_bf16(sv[6], sv[7]));
                            *reinterpret_cast<uint4*>(
                                sprev + tile_chunk_off(D, frow, (v0 >> 3) + 1)) =
                                make_uint4(pack_bf16(sv[8], sv[9]), pack_bf16(sv[10], sv[11]),
                                           pack_bf16(sv[12], sv[13]), pack_bf16(sv[14], sv[15]));
                            if (write_final && prm.S_out)
                                for (int t = 0; t < 16; ++t)
                                    prm.S_out[size_t(head) * prm.stride_S + size_t(frow) * D +
                                              v0 + t] = sv[t];
                        }
                    }
                    float zv[16];
                    tmem_ld16(tmem + lane_base + Cfg::T_Z, zv);
                    tmem_wait_ld();
                    if (frow >= 0) {
                        const __nv_bfloat16 zh = __float2bfloat16_rn(zv[0]);
                        zop_h[tile_off(16, 0, frow) / 2] = zh;
                        zop_h[tile_off(16, 1, frow) / 2] =
                            __float2bfloat16_rn(zv[0] - __bfloat162float(zh));
                        if (write_final && prm.z_out)
                            prm.z_out[size_t(head) * prm.stride_z + frow] = zv[0];
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(s_ready);
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
