// la_api.cu — the C ABI of liblinattn (declared in include/la_api.h):
// argument validation, workspace sizing and kernel dispatch.
//
// Every entry point validates all of its arguments before it launches
// anything, maps CUDA launch failures to LA_ERR_CUDA, never throws and never
// synchronises (except la_get_device_error, which exists to do so).
#include "la_api.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <type_traits>

#include "la_chunk_bwd.cuh"
#include "la_favor.cuh"
#include "la_pad.cuh"
#include "la_reduce.cuh"
#include "la_chunk_bwd64.cuh"
#include "la_chunk_fwd.cuh"
#include "la_chunk_fwd64.cuh"
#include "la_common.cuh"
#include "la_decode.cuh"
#include "la_generic.cuh"
#include "la_phi_map.cuh"
#include "la_runtime.cuh"
#include "la_sm100.cuh"
#include "la_state.cuh"

namespace {

using la::PHI_ELU1;
using la::PHI_RELU_EPS;

constexpr int64_t kMaxElems = int64_t(1) << 62;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_d(int64_t D) { return D == 16 || D == 32 || D == 64 || D == 128; }

la_status check_sizes(int64_t B, int64_t H, int64_t N, int64_t D) {
    if (B < 0 || H < 0 || N < 0 || D <= 0) return LA_ERR_INVALID_ARG;
    if (!supported_d(D)) return LA_ERR_UNSUPPORTED;
    if (N >= (int64_t(1) << 31) || B * H >= (int64_t(1) << 31)) return LA_ERR_UNSUPPORTED;
    // B*H*N*D < 2^62 without overflowing on the way
    if (B != 0 && H != 0 && N != 0) {
        const int64_t bh = B * H;
        if (bh > kMaxElems / N || bh * N > kMaxElems / D) return LA_ERR_UNSUPPORTED;
    }
    return LA_OK;
}

la_status check_enums(la_dtype dt, la_phi phi) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (phi != LA_PHI_ELU1 && phi != LA_PHI_RELU_EPS && phi != LA_PHI_IDENTITY)
        return LA_ERR_INVALID_ARG;
    return LA_OK;
}

// Key/value heads: at least one, and a divisor of the query heads.
la_status check_group(int64_t H, int64_t Hkv) {
    if (H == 0 && Hkv == 0) return LA_OK;  // no heads: nothing to launch
    if (Hkv < 1 || H < 0 || H % Hkv != 0) return LA_ERR_INVALID_ARG;
    return LA_OK;
}

la_status check_ptr(const void* p) {
    if (p == nullptr || !aligned16(p)) return LA_ERR_INVALID_ARG;
    return LA_OK;
}

thread_local char g_last_error[160] = "";

la_status cuda_fail(const char* where, cudaError_t e) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorName(e));
    return LA_ERR_CUDA;
}

// Make the calling thread's current device context current at the driver
// level too: the runtime binds it lazily, and the tensor-map encoder (a
// driver call) needs it.  The current device is left unchanged.
la_status bind_context() {
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return cuda_fail("cudaGetDevice", e);
    if (cudaError_t e = cudaSetDevice(dev)) return cuda_fail("cudaSetDevice", e);
    return LA_OK;
}

la_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LA_OK : cuda_fail("kernel launch", e);
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------ workspace plan
// Backward: g and dg, float32 [B, H, N] each; with grouped key/value heads
// also float32 dK, dV per query head [B, H, N, D] each.
struct BwdWorkspace {
    size_t g_off = 0, dg_off = 0, part_off = 0, bytes = 0;
};

BwdWorkspace plan_bwd(int64_t B, int64_t H, int64_t N, int64_t D = 0, int G = 1) {
    BwdWorkspace w;
    const size_t tok = size_t(B) * size_t(H) * size_t(N) * sizeof(float);
    w.g_off = 0;
    w.dg_off = round_up(tok, 256);
    w.bytes = w.dg_off + round_up(tok, 256);
    if (G > 1) {
        // float32 dK, dV per query head, summed per key/value group afterwards
        w.part_off = w.bytes;
        w.bytes += 2 * round_up(size_t(B) * size_t(H) * size_t(N) * size_t(D) * 4, 256);
    }
    return w;
}


// ------------------------------------------------------------ tensor maps
// cuTensorMapEncodeTiled, fetched through the runtime so the library does
// not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [heads][N][D] bf16 viewed as a 3-D tensor (D, N, heads); box (64, C, 1),
// 128-byte swizzle.  Rows past N read as zero and are clipped on store.
bool make_qkv_map(CUtensorMap* m, const void* base, int64_t heads, int64_t N, int64_t D, int C) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(N), cuuint64_t(heads)};
    cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(N) * cuuint64_t(D) * 2};
    cuuint32_t box[3] = {64, cuuint32_t(C), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        snprintf(g_last_error, sizeof(g_last_error),
                 "cuTensorMapEncodeTiled: CUresult %d (map at %p, base %p)", int(r),
                 static_cast<void*>(m), base);
    return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------ chunked path
// Streaming multiprocessors of the current device (queried once per device
// and cached; 148, the B200's count, where no device answers, so that sizing
// calls made without a GPU still plan like the launches will).
constexpr int kDefaultSMs = 148;
int num_sms() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return kDefaultSMs;
    }
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return kDefaultSMs;
    }
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

bool fast_path(la_dtype dt, int64_t D) { return dt == LA_BF16 && (D == 64 || D == 128); }
int chunk_len(int64_t D) { return D == 64 ? 128 : 64; }

// Segments per head.  Each chunked kernel holds one block per SM (its shared
// memory), so a launch of heads * s blocks takes ceil(heads * s / SMs) waves
// of ceil(nchunks / s) chunks each, plus a few chunks' worth of pipeline fill
// per block; splitting (s > 1) also adds the segment-state pass, which reads
// k and v again (about 0.3 of a chunk each).  Pick the s with the smallest
// modelled makespan; 120 or more heads stay unsplit (one wave or close).
int pick_nseg(int64_t heads, int64_t nchunks) {
    const int kNumSM = num_sms();
    if (heads >= kNumSM * 120 / 148 || nchunks < 4) return 1;
    constexpr double kFill = 3.0, kStatePass = 0.3;
    int best = 1;
    double best_cost = double((heads + kNumSM - 1) / kNumSM) * (double(nchunks) + kFill);
    for (int64_t sg = 2; sg <= nchunks / 2; ++sg) {
        const int64_t per = (nchunks + sg - 1) / sg;
        const int64_t used = (nchunks + per - 1) / per;  // segments that are not empty
        if (used != sg) continue;
        const double waves = double((heads * sg + kNumSM - 1) / kNumSM);
        const double cost = waves * ((1.0 + kStatePass) * double(per) + kFill);
        if (cost < best_cost) {
            best_cost = cost;
            best = int(sg);
        }
    }
    return best;
}

struct SegSplit {
    int nseg = 1, seg_len = 0;
};
SegSplit split(int64_t N, int C, int nseg) {
    SegSplit s;
    const int64_t per = (N + nseg - 1) / nseg;
    s.seg_len = int((per + C - 1) / C * C);
    s.nseg = int((N + s.seg_len - 1) / s.seg_len);
    return s;
}

// Reduce split for the starts of a causal pass cut into segments: only the
// tokens before the last segment are summed (its own state is never a
// start), each segment as `ratio` equal sub-segments (ratio dividing its
// chunks) chosen so that the reduce blocks fill the SMs: the smallest
// modelled makespan waves x (chunks per block + fill).  A wave holds two
// blocks per SM at head size 128 (the compact reduce block), one otherwise.
struct StartSplit {
    int ratio = 1, nsub = 0, sub_len = 0;
};
StartSplit start_split(int64_t heads, const SegSplit& seg, int C, int64_t D) {
    StartSplit r;
    if (seg.nseg <= 1) return r;
    const int seg_chunks = seg.seg_len / C;
    const int kNumSM = num_sms() * (D == 128 ? 2 : 1);
    constexpr double kFill = 3.0;
    double best = 0.0;
    for (int q = 1; q <= std::min(seg_chunks, 16); ++q) {
        if (seg_chunks % q) continue;
        const int64_t blocks = heads * (seg.nseg - 1) * q;
        const double cost =
            double((blocks + kNumSM - 1) / kNumSM) * (double(seg_chunks / q) + kFill);
        if (q == 1 || cost < best - 1e-9) {
            best = cost;
            r.ratio = q;
        }
    }
    r.sub_len = seg.seg_len / r.ratio;
    r.nsub = (seg.nseg - 1) * r.ratio;
    return r;
}

struct FwdPlan {
    bool fast = false;
    int C = 0;
    SegSplit seg, qseg;
    StartSplit ss;  // causal, split heads: the reduce pass for the segment starts
    size_t rec_off = 0, tot_off = 0, sub_off = 0, bytes = 0;
};

FwdPlan plan_fwd(int64_t B, int64_t H, int64_t N, int64_t D, int causal, la_dtype dt) {
    FwdPlan p;
    if (!fast_path(dt, D) || N == 0 || B * H == 0) return p;
    p.fast = true;
    p.C = chunk_len(D);
    const int64_t heads = B * H;
    const int64_t nch = (N + p.C - 1) / p.C;
    const int kNumSM = num_sms();
    p.seg = split(N, p.C, pick_nseg(heads, nch));
    const size_t R = size_t(D) * D + D;
    if (causal) {
        // rec: the segment starts (or, decayed, the per-segment records
        // scanned in place); sub: the start reduce's records
        p.rec_off = 0;
        p.bytes = 0;
        if (p.seg.nseg > 1) {
            p.ss = start_split(heads, p.seg, p.C, D);
            p.sub_off = round_up(size_t(heads) * p.seg.nseg * R * sizeof(float), 256);
            p.bytes = p.sub_off + size_t(heads) * p.ss.nsub * R * sizeof(float);
        }
    } else {
        const int64_t want = heads >= 2 * kNumSM ? 1 : (2 * kNumSM + heads - 1) / heads;
        p.qseg = split(N, p.C, int(std::max<int64_t>(1, std::min<int64_t>(want, nch))));
        p.rec_off = 0;
        p.tot_off = round_up(size_t(heads) * p.seg.nseg * R * sizeof(float), 256);
        p.bytes = p.tot_off + round_up(size_t(heads) * R * sizeof(float), 256);
    }
    return p;
}

template <int D, int C, int PHI, int MODE, bool DECAY = false>
la_status launch_chunk(const la::ChunkParams& prm, int64_t grid, cudaStream_t st,
                       const char* name) {
    auto go = [&](auto kern, int smem, int threads) -> la_status {
        if (cudaError_t e =
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))
            return cuda_fail("cudaFuncSetAttribute", e);
        la::LaunchScope scope(name, st);
        kern<<<unsigned(grid), threads, smem, st>>>(prm);
        return launch_status();
    };
    if constexpr (D == 64)
        return go(la::chunk_fwd64_kernel<PHI, MODE, DECAY>, la::Chunk64Cfg::SMEM,
                  la::kChunk64Threads);
    else
        return go(la::chunk_fwd_kernel<D, C, PHI, MODE, DECAY>, la::ChunkCfg<D, C>::SMEM,
                  la::kChunkThreads);
}

const la::DecayArg kNoDecay{};  // H = 0: no decay

// Smallest decay factor the chunked kernels take with C-token chunks: their
// chunk-local factors reach gamma^(-C) (an unmasked product), kept <= 2^64.
float chunk_gamma_min(int C) { return exp2f(-64.f / float(C)); }

la_status launch_state_kernel(int which, float* rec, float* out, float* S, float* z,
                              int64_t heads, int nseg, int64_t D, cudaStream_t st,
                              int rec_step = 1, const la::DecayArg& dec = kNoDecay,
                              int seg_len = 0, const float* init = nullptr) {
    const int R = int(D * D + D);
    const int bph = (R + la::kStateThreads - 1) / la::kStateThreads;
    const unsigned grid = unsigned(heads * bph);
    // the sums and scans run over float4 columns (R is a multiple of 4)
    const int R4 = R / 4;
    const int bph4 = (R4 + la::kStateThreads - 1) / la::kStateThreads;
    const unsigned grid4 = unsigned(heads * bph4);
    if (which == 0) {
        la::LaunchScope scope("state_scan", st);
        la::state_exclusive_scan_kernel<<<grid4, la::kStateThreads, 0, st>>>(rec, nseg, R4, bph4,
                                                                             dec, seg_len, init);
    } else if (which == 3) {
        la::LaunchScope scope("state_rscan", st);
        la::state_exclusive_rscan_kernel<<<grid4, la::kStateThreads, 0, st>>>(rec, nseg, R4,
                                                                              bph4, init);
    } else if (which == 1) {
        la::LaunchScope scope("state_sum", st);
        la::state_sum_kernel<<<grid4, la::kStateThreads, 0, st>>>(rec, out, nseg, R4, bph4);
    } else {
        la::LaunchScope scope("state_unpack", st);
        la::state_unpack_kernel<<<grid, la::kStateThreads, 0, st>>>(out, S, z, int(D), bph,
                                                                     rec_step);
    }
    return launch_status();
}

// The REDUCE pass (state record of each block's token range, no decay):
// for head size 128 the compact reduce block (two per SM), otherwise the
// chunked kernel's REDUCE mode.
template <int D, int C, int PHI>
la_status launch_reduce(const la::ChunkParams& r, int64_t grid, cudaStream_t st) {
    if constexpr (D == 128) {
        auto kern = la::reduce128_kernel<PHI>;
        if (cudaError_t e = cudaFuncSetAttribute(
                kern, cudaFuncAttributeMaxDynamicSharedMemorySize, la::Reduce128Cfg::SMEM))
            return cuda_fail("cudaFuncSetAttribute", e);
        la::LaunchScope scope("reduce128", st);
        kern<<<unsigned(grid), la::kReduce128Threads, la::Reduce128Cfg::SMEM, st>>>(r);
        return launch_status();
    } else {
        return launch_chunk<D, C, PHI, la::MODE_REDUCE>(r, grid, st, "chunk_reduce");
    }
}

// Starts of the segments of a causal pass (no decay): the REDUCE pass of
// `red` (its k, v maps, N, kv_group and centring) over the sub-segments of
// the tokens before the last segment into `sub`, then starts[h][p] =
// init[h] + the sub-segment records before segment p.
template <int D, int C, int PHI>
la_status run_segment_starts(const la::ChunkParams& red, int64_t heads, const SegSplit& seg,
                             const StartSplit& ss, float* sub, float* starts, const float* init,
                             cudaStream_t st) {
    const int64_t R = int64_t(D) * D + D;
    la::ChunkParams r = red;
    r.state_in = nullptr;
    r.g_out = nullptr;
    r.store_phi = 0;
    r.seg_len = ss.sub_len;
    r.nseg = ss.nsub;
    r.S_out = sub;
    r.z_out = sub + D * D;
    r.stride_S = r.stride_z = R;
    la_status s = launch_reduce<D, C, PHI>(r, heads * ss.nsub, st);
    if (s != LA_OK) return s;
    const int R4 = int(R / 4);
    const int bph = (R4 + la::kStateThreads - 1) / la::kStateThreads;
    la::LaunchScope scope("state_starts", st);
    la::state_segment_starts_kernel<<<unsigned(heads * bph), la::kStateThreads, 0, st>>>(
        sub, starts, seg.nseg, ss.ratio, R4, bph, init);
    return launch_status();
}

template <int D, int PHI>
la_status run_fwd_chunked(const void* q, const void* k, const void* v, void* o, float* S_out,
                          float* z_out, float* g_out, void* pq, void* pk, int64_t heads, int64_t N,
                          int causal, const FwdPlan& p, char* ws, cudaStream_t st, int G,
                          const la::DecayArg& dec) {
    constexpr int C = D == 64 ? 128 : 64;
    const int64_t kv_heads = heads / G;
    const bool decay = dec.H > 0;  // causal only (checked by the caller)
    la::ChunkParams prm;
    memset(&prm, 0, sizeof(prm));
    if (!make_qkv_map(&prm.tm_q, q, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_k, k, kv_heads, N, D, C) ||
        !make_qkv_map(&prm.tm_v, v, kv_heads, N, D, C) || !make_qkv_map(&prm.tm_o, o, heads, N, D, C))
        return LA_ERR_CUDA;
    prm.N = int(N);
    prm.g_out = g_out;
    prm.kv_group = G;
    prm.dec = dec;
    const int64_t R = int64_t(D) * D + D;
    float* rec = reinterpret_cast<float*>(ws + p.rec_off);
    la_status s;
    if (causal) {
        if (p.seg.nseg > 1 && decay) {
            // decayed: every segment's record, scanned with the decay factors
            la::ChunkParams r = prm;
            r.seg_len = p.seg.seg_len;
            r.nseg = p.seg.nseg;
            r.S_out = rec;
            r.z_out = rec + D * D;
            r.stride_S = r.stride_z = R;
            if ((s = launch_chunk<D, C, PHI, la::MODE_REDUCE, true>(r, heads * p.seg.nseg, st,
                                                                    "chunk_reduce")) != LA_OK)
                return s;
            if ((s = launch_state_kernel(0, rec, nullptr, nullptr, nullptr, heads, p.seg.nseg, D,
                                         st, 1, dec, p.seg.seg_len)) != LA_OK)
                return s;
        } else if (p.seg.nseg > 1) {
            float* sub = reinterpret_cast<float*>(ws + p.sub_off);
            if ((s = run_segment_starts<D, C, PHI>(prm, heads, p.seg, p.ss, sub, rec, nullptr,
                                                   st)) != LA_OK)
                return s;
        }
        if (p.seg.nseg > 1) {
            prm.state_in = rec;
            prm.in_per_head = 0;
        }
        prm.seg_len = p.seg.seg_len;
        prm.nseg = p.seg.nseg;
        prm.S_out = S_out;
        prm.z_out = z_out;
        prm.stride_S = int64_t(D) * D;
        prm.stride_z = D;
        if (D == 64 && pq) {
            // the D = 64 causal kernel stores its phi(q), phi(k) tiles itself
            if (!make_qkv_map(&prm.tm_pq, pq, heads, N, D, C) ||
                !make_qkv_map(&prm.tm_pk, pk, heads, N, D, C))
                return LA_ERR_CUDA;
            prm.store_phi = 1;
        }
        if (decay)
            return launch_chunk<D, C, PHI, la::MODE_CAUSAL, true>(prm, heads * p.seg.nseg, st,
                                                                  "chunk_causal");
        return launch_chunk<D, C, PHI, la::MODE_CAUSAL>(prm, heads * p.seg.nseg, st, "chunk_causal");
    }
    // non-causal: segment sums -> totals -> query pass
    float* tot = reinterpret_cast<float*>(ws + p.tot_off);
    la::ChunkParams r = prm;
    r.seg_len = p.seg.seg_len;
    r.nseg = p.seg.nseg;
    r.S_out = rec;
    r.z_out = rec + D * D;
    r.stride_S = r.stride_z = R;
    if ((s = launch_reduce<D, C, PHI>(r, heads * p.seg.nseg, st)) != LA_OK) return s;
    if ((s = launch_state_kernel(1, rec, tot, nullptr, nullptr, heads, p.seg.nseg, D, st)) != LA_OK)
        return s;
    // the state of each key/value head: the record of its group's first query head
    if ((S_out || z_out) &&
        (s = launch_state_kernel(2, nullptr, tot, S_out, z_out, kv_heads, 1, D, st, G)) != LA_OK)
        return s;
    prm.seg_len = p.qseg.seg_len;
    prm.nseg = p.qseg.nseg;
    prm.state_in = tot;
    prm.in_per_head = 1;
    return launch_chunk<D, C, PHI, la::MODE_QUERY>(prm, heads * p.qseg.nseg, st, "chunk_query");
}

template <int PHI>
la_status run_fwd_chunked_d(const void* q, const void* k, const void* v, void* o, float* S_out,
                            float* z_out, float* g_out, void* pq, void* pk, int64_t heads,
                            int64_t N, int64_t D, int causal, const FwdPlan& p, char* ws,
                            cudaStream_t st, int G, const la::DecayArg& dec = kNoDecay) {
    if (D == 64)
        return run_fwd_chunked<64, PHI>(q, k, v, o, S_out, z_out, g_out, pq, pk, heads, N, causal,
                                        p, ws, st, G, dec);
    return run_fwd_chunked<128, PHI>(q, k, v, o, S_out, z_out, g_out, pq, pk, heads, N, causal, p,
                                     ws, st, G, dec);
}


// ------------------------------------------------------------ chunked backward
struct BwdPlan {
    bool fast = false;
    int C = 0;
    SegSplit seg;   // causal: segments of both passes; non-causal: reduce split
    SegSplit qseg;  // non-causal: split of the two gradient passes
    size_t g_off = 0, dg_off = 0, srec_off = 0, stot_off = 0, rrec_off = 0, rtot_off = 0;
    // without the forward's o and g, la_backward first runs the forward into
    // o (o_off) and g (g_off) with the forward's own workspace at fwd_off
    size_t o_off = 0, fwd_off = 0;
    // grouped key/value heads (G > 1): dK, dV per query head, summed per group
    size_t part_off = 0;
    // causal, split heads: the reduce pass for the dQ pass's segment starts
    StartSplit ss;
    size_t sub_off = 0;
    size_t bytes = 0;
};

BwdPlan plan_bwd_fast(int64_t B, int64_t H, int64_t N, int64_t D, int causal, la_dtype dt,
                      int G = 1) {
    BwdPlan p;
    if (!fast_path(dt, D) || N == 0 || B * H == 0) return p;
    p.fast = true;
    p.C = chunk_len(D);
    const int64_t heads = B * H;
    const int64_t nch = (N + p.C - 1) / p.C;
    const int kNumSM = num_sms();
    const size_t R = size_t(D) * D + D;
    const size_t tok = size_t(heads) * size_t(N) * sizeof(float);
    size_t off = 0;
    p.g_off = off;
    off += round_up(tok, 256);
    p.dg_off = off;
    off += round_up(tok, 256);
    p.seg = split(N, p.C, pick_nseg(heads, nch));
    if (causal) {
        p.qseg = p.seg;
        if (p.seg.nseg > 1) {
            p.ss = start_split(heads, p.seg, p.C, D);
            p.srec_off = off;
            off += round_up(size_t(heads) * p.seg.nseg * R * 4, 256);
            p.rrec_off = off;
            off += round_up(size_t(heads) * p.seg.nseg * R * 4, 256);
            p.sub_off = off;
            off += round_up(size_t(heads) * p.ss.nsub * R * 4, 256);
        }
    } else {
        const int64_t want = heads >= 2 * kNumSM ? 1 : (2 * kNumSM + heads - 1) / heads;
        p.qseg = split(N, p.C, int(std::max<int64_t>(1, std::min<int64_t>(want, nch))));
        p.srec_off = off;
        off += round_up(size_t(heads) * p.seg.nseg * R * 4, 256);
        p.stot_off = off;
        off += round_up(size_t(heads) * R * 4, 256);
        p.rrec_off = off;
        off += round_up(size_t(heads) * p.qseg.nseg * R * 4, 256);
        p.rtot_off = off;
        off += round_up(size_t(heads) * R * 4, 256);
    }
    p.o_off = off;
    off += round_up(size_t(heads) * size_t(N) * size_t(D) * 2, 256);
    p.fwd_off = off;
    off += round_up(plan_fwd(B, H, N, D, causal, dt).bytes, 256);
    if (G > 1) {
        p.part_off = off;
        off += 2 * round_up(size_t(heads) * size_t(N) * size_t(D) * 4, 256);
    }
    p.bytes = off;
    return p;
}

template <typename Kern>
la_status launch_bwd_kernel(Kern kern, int smem, const la::BwdParams& prm, int64_t grid,
                            cudaStream_t st, const char* name, int threads = la::kBwdThreads) {
    if (cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))
        return cuda_fail("cudaFuncSetAttribute", e);
    la::LaunchScope scope(name, st);
    kern<<<unsigned(grid), threads, smem, st>>>(prm);
    return launch_status();
}

template <int D, int PHI>
la_status run_bwd_chunked(const void* q, const void* k, const void* v, const void* dO,
                          const void* o_saved, const float* g_saved, const void* pq,
                          const void* pk, void* dq, void* dk, void* dv, int64_t heads,
                          int64_t N, int causal, const BwdPlan& p, char* ws, cudaStream_t st,
                          int G, float* dk_part, float* dv_part,
                          const la::DecayArg& dec = kNoDecay) {
    constexpr int C = D == 64 ? 128 : 64;
    const int64_t kv_heads = heads / G;
    // with grouped key/value heads the kernels store float32 partials per
    // query head; the bf16 dK, dV maps (never stored through then) span the
    // caller's key/value heads
    const int64_t dkv_heads = G > 1 ? kv_heads : heads;
    la::BwdParams prm;
    memset(&prm, 0, sizeof(prm));
    if (!make_qkv_map(&prm.tm_q, q, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_k, k, kv_heads, N, D, C) ||
        !make_qkv_map(&prm.tm_v, v, kv_heads, N, D, C) ||
        !make_qkv_map(&prm.tm_do, dO, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_dq, dq, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_dk, dk, dkv_heads, N, D, C) ||
        !make_qkv_map(&prm.tm_dv, dv, dkv_heads, N, D, C))
        return LA_ERR_CUDA;
    prm.kv_group = G;
    prm.dk_part = G > 1 ? dk_part : nullptr;
    prm.dv_part = G > 1 ? dv_part : nullptr;
    prm.dec = dec;
    prm.N = int(N);
    // the forward's o and g: the caller's, or computed into the workspace
    // by la_backward before this runs
    if (o_saved == nullptr || g_saved == nullptr) return LA_ERR_INVALID_ARG;
    prm.gbuf = const_cast<float*>(g_saved);
    prm.dgbuf = reinterpret_cast<float*>(ws + p.dg_off);
    prm.o_in = static_cast<const __nv_bfloat16*>(o_saved);
    // the D = 64 pipelined passes read phi(q), phi(k) through the q, k maps
    // when the forward's feature maps are given
    const bool pin = pq != nullptr;
    CUtensorMap tm_pq, tm_pk;
    if (pin && (!make_qkv_map(&tm_pq, pq, heads, N, D, C) || !make_qkv_map(&tm_pk, pk, heads, N, D, C)))
        return LA_ERR_CUDA;
    auto with_phi = [&](la::BwdParams b) {
        if (pin) {
            b.tm_q = tm_pq;
            b.tm_k = tm_pk;
        }
        return b;
    };
    const int64_t R = int64_t(D) * D + D;
    float* srec = reinterpret_cast<float*>(ws + p.srec_off);
    float* rrec = reinterpret_cast<float*>(ws + p.rrec_off);
    constexpr int smem1 = la::Bwd1Cfg<D, C>::SMEM;
    constexpr int smem2 = la::Bwd2Cfg<D, C>::SMEM;
    la_status s;

    // (S, z) of earlier segments / the whole sequence
    la::ChunkParams red;
    memset(&red, 0, sizeof(red));
    red.tm_k = prm.tm_k;
    red.tm_v = prm.tm_v;
    red.N = int(N);
    red.seg_len = p.seg.seg_len;
    red.nseg = p.seg.nseg;
    red.S_out = srec;
    red.z_out = srec + D * D;
    red.stride_S = red.stride_z = R;
    // the dQ products use the centred key features phi(k) - c, and so do
    // the states they start from
    red.center = 1;
    red.kv_group = G;

    if (causal) {
        la::BwdParams p1 = prm, p2 = prm;
        p1.seg_len = p2.seg_len = p.seg.seg_len;
        p1.nseg = p2.nseg = p.seg.nseg;
        if (p.seg.nseg > 1) {
            float* sub = reinterpret_cast<float*>(ws + p.sub_off);
            if ((s = run_segment_starts<D, C, PHI>(red, heads, p.seg, p.ss, sub, srec, nullptr,
                                                   st)) != LA_OK)
                return s;
            p1.state_in = srec;
            p1.rec_out = rrec;
        }
        if constexpr (D == 64) {
            // decayed recurrence: the pipelined passes with chunk-local decay
            // factors (the caller takes this path with one segment per head,
            // no saved feature maps and no grouping)
            if (dec.H > 0) {
                if (p.seg.nseg != 1 || pin || G != 1) return LA_ERR_INVALID_ARG;
                la_status s1 = launch_bwd_kernel(la::bwd_dq64_kernel<PHI, false, true>,
                                                 la::Bwd1x64Cfg::SMEM, p1, heads, st, "bwd_dq",
                                                 la::kBwd64Threads);
                if (s1 != LA_OK) return s1;
                return launch_bwd_kernel(la::bwd_dkdv64_kernel<PHI, false, false, true>,
                                         la::Bwd2x64Cfg::SMEM, p2, heads, st, "bwd_dkdv",
                                         la::kBwd64Threads);
            }
            // one segment per head: the pipelined passes (pass 1 reads the
            // forward's phi(q) when given, and k itself: it centres phi(k))
            if (p.seg.nseg == 1) {
                la::BwdParams q1 = p1;
                if (pin) q1.tm_q = tm_pq;
                if ((s = pin ? launch_bwd_kernel(la::bwd_dq64_kernel<PHI, true>, la::Bwd1x64Cfg::SMEM,
                                                 q1, heads, st, "bwd_dq", la::kBwd64Threads)
                             : launch_bwd_kernel(la::bwd_dq64_kernel<PHI, false>, la::Bwd1x64Cfg::SMEM,
                                                 q1, heads, st, "bwd_dq", la::kBwd64Threads)) != LA_OK)
                    return s;
                if (pin)
                    return launch_bwd_kernel(la::bwd_dkdv64_kernel<PHI, true>, la::Bwd2x64Cfg::SMEM,
                                             with_phi(p2), heads, st, "bwd_dkdv", la::kBwd64Threads);
                return p2.dk_part
                           ? launch_bwd_kernel(la::bwd_dkdv64_kernel<PHI, false, true>,
                                               la::Bwd2x64Cfg::SMEM, p2, heads, st, "bwd_dkdv",
                                               la::kBwd64Threads)
                           : launch_bwd_kernel(la::bwd_dkdv64_kernel<PHI, false>, la::Bwd2x64Cfg::SMEM,
                                               p2, heads, st, "bwd_dkdv", la::kBwd64Threads);
            }
        }
        if ((s = launch_bwd_kernel(la::bwd_dq_kernel<D, C, PHI, true, true>, smem1, p1,
                                   heads * p.seg.nseg, st, "bwd_dq")) != LA_OK)
            return s;
        if (p.seg.nseg > 1) {
            if ((s = launch_state_kernel(3, rrec, nullptr, nullptr, nullptr, heads, p.seg.nseg, D,
                                         st)) != LA_OK)
                return s;
            p2.state_in = rrec;
        }
        if constexpr (D == 64) {
            if (pin)
                return launch_bwd_kernel(la::bwd_dkdv64_kernel<PHI, true>, la::Bwd2x64Cfg::SMEM,
                                         with_phi(p2), heads * p.seg.nseg, st, "bwd_dkdv",
                                         la::kBwd64Threads);
            return p2.dk_part
                       ? launch_bwd_kernel(la::bwd_dkdv64_kernel<PHI, false, true>,
                                           la::Bwd2x64Cfg::SMEM, p2, heads * p.seg.nseg, st,
                                           "bwd_dkdv", la::kBwd64Threads)
                       : launch_bwd_kernel(la::bwd_dkdv64_kernel<PHI, false>, la::Bwd2x64Cfg::SMEM,
                                           p2, heads * p.seg.nseg, st, "bwd_dkdv",
                                           la::kBwd64Threads);
        } else {
            return p2.dk_part
                       ? launch_bwd_kernel(la::bwd_dkdv_kernel<D, C, PHI, true, true>, smem2, p2,
                                           heads * p.seg.nseg, st, "bwd_dkdv")
                       : launch_bwd_kernel(la::bwd_dkdv_kernel<D, C, PHI, true>, smem2, p2,
                                           heads * p.seg.nseg, st, "bwd_dkdv");
        }
    }
    float* stot = reinterpret_cast<float*>(ws + p.stot_off);
    float* rtot = reinterpret_cast<float*>(ws + p.rtot_off);
    if ((s = launch_reduce<D, C, PHI>(red, heads * p.seg.nseg, st)) != LA_OK) return s;
    if ((s = launch_state_kernel(1, srec, stot, nullptr, nullptr, heads, p.seg.nseg, D, st)) !=
        LA_OK)
        return s;
    la::BwdParams p1 = prm, p2 = prm;
    p1.seg_len = p2.seg_len = p.qseg.seg_len;
    p1.nseg = p2.nseg = p.qseg.nseg;
    p1.state_in = stot;
    p1.in_per_head = 1;
    p1.rec_out = rrec;
    if ((s = launch_bwd_kernel(la::bwd_dq_kernel<D, C, PHI, false, true>, smem1, p1,
                               heads * p.qseg.nseg, st, "bwd_dq")) != LA_OK)
        return s;
    if ((s = launch_state_kernel(1, rrec, rtot, nullptr, nullptr, heads, p.qseg.nseg, D, st)) !=
        LA_OK)
        return s;
    p2.state_in = rtot;
    p2.in_per_head = 1;
    return p2.dk_part ? launch_bwd_kernel(la::bwd_dkdv_kernel<D, C, PHI, false, true>, smem2, p2,
                                          heads * p.qseg.nseg, st, "bwd_dkdv")
                      : launch_bwd_kernel(la::bwd_dkdv_kernel<D, C, PHI, false>, smem2, p2,
                                          heads * p.qseg.nseg, st, "bwd_dkdv");
}

// dK or dV of each key/value head <- the sum of its group's float32
// per-query-head partials (n = N*D elements per head, a multiple of 4).
template <typename T>
la_status launch_group_sum(const float* part, void* out, int64_t kv_heads, int64_t n, int G,
                           cudaStream_t st) {
    const int64_t total4 = kv_heads * n / 4;
    const int64_t blocks = std::min<int64_t>((total4 + 255) / 256, int64_t(num_sms()) * 16);
    la::LaunchScope scope("group_sum", st);
    la::group_sum_kernel<T><<<unsigned(std::max<int64_t>(blocks, 1)), 256, 0, st>>>(
        part, static_cast<T*>(out), n, G, total4);
    return launch_status();
}

template <int PHI>
la_status run_bwd_chunked_d(const void* q, const void* k, const void* v, const void* dO,
                            const void* o_saved, const float* g_saved, const void* pq,
                            const void* pk, void* dq, void* dk, void* dv, int64_t heads,
                            int64_t N, int64_t D, int causal, const BwdPlan& p, char* ws,
                            cudaStream_t st, int G, const la::DecayArg& dec = kNoDecay) {
    // with grouped key/value heads each query head's dK, dV go to the
    // workspace first, in float32, and are summed per group after the passes
    const size_t part_bytes = round_up(size_t(heads) * size_t(N) * size_t(D) * 4, 256);
    float* dk_p = G > 1 ? reinterpret_cast<float*>(ws + p.part_off) : nullptr;
    float* dv_p = G > 1 ? reinterpret_cast<float*>(ws + p.part_off + part_bytes) : nullptr;
    la_status s;
    if (D == 64)
        s = run_bwd_chunked<64, PHI>(q, k, v, dO, o_saved, g_saved, pq, pk, dq, dk, dv, heads,
                                     N, causal, p, ws, st, G, dk_p, dv_p, dec);
    else if (dec.H > 0)  // the decayed backward runs chunked for D = 64 only
        return LA_ERR_INVALID_ARG;
    else  // the D = 128 kernels evaluate the feature map themselves
        s = run_bwd_chunked<128, PHI>(q, k, v, dO, o_saved, g_saved, nullptr, nullptr, dq, dk,
                                      dv, heads, N, causal, p, ws, st, G, dk_p, dv_p);
    if (s != LA_OK || G == 1) return s;
    if ((s = launch_group_sum<__nv_bfloat16>(dk_p, dk, heads / G, N * D, G, st)) != LA_OK) return s;
    return launch_group_sum<__nv_bfloat16>(dv_p, dv, heads / G, N * D, G, st);
}

// ------------------------------------------------------------ FAVOR+ features
template <int D, int M, bool BWD>
la_status launch_favor(const void* x, const void* omega, const void* dphi, void* out,
                       int64_t heads, int64_t N, cudaStream_t st) {
    using Cfg = la::FavorCfg<D, M, BWD>;
    la::FavorParams prm;
    memset(&prm, 0, sizeof(prm));
    if (!make_qkv_map(&prm.tm_x, x, heads, N, D, Cfg::R) ||
        !make_qkv_map(&prm.tm_w, omega, 1, M, D, M))
        return LA_ERR_CUDA;
    if (!BWD && !make_qkv_map(&prm.tm_phi, out, heads, N, M, Cfg::R)) return LA_ERR_CUDA;
    if (BWD && (!make_qkv_map(&prm.tm_dphi, dphi, heads, N, M, Cfg::R) ||
                !make_qkv_map(&prm.tm_dx, out, heads, N, D, Cfg::R)))
        return LA_ERR_CUDA;
    const int64_t tph = (N + Cfg::R - 1) / Cfg::R;
    if (heads * tph >= (int64_t(1) << 31)) return LA_ERR_UNSUPPORTED;
    prm.tiles_per_head = int(tph);
    prm.ntiles = int(heads * tph);
    prm.log_scale = -0.5f * logf(float(M));
    auto kern = la::favor_kernel<D, M, BWD>;
    if (cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg::SMEM))
        return cuda_fail("cudaFuncSetAttribute", e);
    const unsigned grid = unsigned(std::min<int64_t>(prm.ntiles, num_sms()));
    la::LaunchScope scope(BWD ? "favor_bwd" : "favor_fwd", st);
    kern<<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(prm);
    return launch_status();
}

// Head size D and m features, each 64 or 128.
template <bool BWD>
la_status launch_favor_dm(int64_t D, int64_t m, const void* x, const void* omega,
                          const void* dphi, void* out, int64_t heads, int64_t N,
                          cudaStream_t st) {
    if (D == 64)
        return m == 64 ? launch_favor<64, 64, BWD>(x, omega, dphi, out, heads, N, st)
                       : launch_favor<64, 128, BWD>(x, omega, dphi, out, heads, N, st);
    return m == 64 ? launch_favor<128, 64, BWD>(x, omega, dphi, out, heads, N, st)
                   : launch_favor<128, 128, BWD>(x, omega, dphi, out, heads, N, st);
}

// Rows of `ws` bf16 elements -> rows of `wd` (zero-filled past ws, or cut).
la_status copy_cols(const void* src, void* dst, int64_t rows, int64_t ws, int64_t wd,
                    cudaStream_t st) {
    const int64_t total = rows * (wd / 8);
    if (total == 0) return LA_OK;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, int64_t(num_sms()) * 16);
    la::LaunchScope scope("copy_cols", st);
    la::copy_cols_kernel<<<unsigned(blocks), 256, 0, st>>>(static_cast<const uint4*>(src),
                                                           static_cast<uint4*>(dst), rows,
                                                           int(ws / 8), int(wd / 8));
    return launch_status();
}

// Attention with m = Dk features and head size Dv != Dk: workspace layout.
// D = max(Dk, Dv); the narrower side's tensors are widened to D (`npad`
// tensors of heads x N x D bf16 each), then the inner call's own workspace.
struct MvPlan {
    int64_t D = 0;
    int npad = 0;
    size_t tile = 0, inner_off = 0, inner = 0, bytes = 0;
};
MvPlan plan_mv(la_op op, int64_t B, int64_t H, int64_t N, int64_t Dk, int64_t Dv, int causal) {
    MvPlan p;
    p.D = std::max(Dk, Dv);
    const int64_t heads = B * H;
    p.tile = round_up(size_t(heads) * size_t(N) * size_t(p.D) * 2, 256);
    if (Dk != Dv) p.npad = op == LA_OP_FORWARD ? 2 : 4;  // (v, o) | (q, k); bwd: + dO, o, dv | dq, dk
    p.inner_off = size_t(p.npad) * p.tile;
    p.inner = la_workspace_size(op, B, H, N, p.D, causal, LA_BF16);
    p.bytes = p.inner_off + p.inner;
    return p;
}

// ------------------------------------------------------------ generic path
template <typename T, int PHI>
la_status run_fwd_generic(const void* q, const void* k, const void* v, void* o, float* S_out,
                          float* z_out, float* g_out, int64_t heads, int64_t N, int64_t D,
                          int causal, cudaStream_t st, int G, const la::DecayArg& dec) {
    auto kern = la::fwd_generic_kernel<T, PHI>;
    const size_t smem = la::generic_smem_bytes(int(D));
    if (cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem)))
        return cuda_fail("cudaFuncSetAttribute", e);
    la::LaunchScope scope("fwd_generic", st);
    kern<<<unsigned(heads), la::kGenericThreads, smem, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
        static_cast<T*>(o), S_out, z_out, g_out, int(N), int(D), causal, G, dec);
    return launch_status();
}

template <typename T, int PHI>
la_status run_bwd_generic(const void* q, const void* k, const void* v, const void* dO, void* dq,
                          void* dk, void* dv, int64_t heads, int64_t N, int64_t D, int causal,
                          float* gbuf, float* dgbuf, cudaStream_t st, int G, char* part,
                          const la::DecayArg& dec) {
    // with grouped key/value heads each query head's dK, dV go to `part`
    // first, in float32, and are summed per group afterwards
    const size_t part_bytes = round_up(size_t(heads) * size_t(N) * size_t(D) * 4, 256);
    float* dk_p = reinterpret_cast<float*>(part);
    float* dv_p = reinterpret_cast<float*>(part + part_bytes);
    const size_t smem = la::generic_smem_bytes(int(D)) + size_t(D) * sizeof(float);
    if (G > 1) {
        auto kern = la::bwd_generic_kernel<T, PHI, float>;
        if (cudaError_t e = cudaFuncSetAttribute(
                kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)))
            return cuda_fail("cudaFuncSetAttribute", e);
        la::LaunchScope scope("bwd_generic", st);
        kern<<<unsigned(heads), la::kGenericThreads, smem, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
            static_cast<const T*>(dO), static_cast<T*>(dq), dk_p, dv_p, gbuf, dgbuf, int(N),
            int(D), causal, G, dec);
        la_status s = launch_status();
        if (s != LA_OK) return s;
        if ((s = launch_group_sum<T>(dk_p, dk, heads / G, N * D, G, st)) != LA_OK) return s;
        return launch_group_sum<T>(dv_p, dv, heads / G, N * D, G, st);
    }
    auto kern = la::bwd_generic_kernel<T, PHI>;
    if (cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem)))
        return cuda_fail("cudaFuncSetAttribute", e);
    la::LaunchScope scope("bwd_generic", st);
    kern<<<unsigned(heads), la::kGenericThreads, smem, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
        static_cast<const T*>(dO), static_cast<T*>(dq), static_cast<T*>(dk), static_cast<T*>(dv),
        gbuf, dgbuf, int(N), int(D), causal, 1, dec);
    return launch_status();
}

template <typename T, int PHI>
la_status run_decode(float* S, float* z, const void* q, const void* k, const void* v, void* o,
                     int64_t heads, int64_t D, cudaStream_t st, int G,
                     const la::DecayArg& dec) {
    const T* qq = static_cast<const T*>(q);
    const T* kk = static_cast<const T*>(k);
    const T* vv = static_cast<const T*>(v);
    T* oo = static_cast<T*>(o);
    if (G > 1) {
        // one block per key/value head: its state read once for the group
        const unsigned grid = unsigned(heads / G);
        la::LaunchScope scope("decode_step_gqa", st);
        switch (D) {
            case 16: la::decode_step_gqa_kernel<T, PHI, 16><<<grid, 32, 0, st>>>(S, z, qq, kk, vv, oo, G); break;
            case 32: la::decode_step_gqa_kernel<T, PHI, 32><<<grid, 64, 0, st>>>(S, z, qq, kk, vv, oo, G); break;
            case 64: la::decode_step_gqa_kernel<T, PHI, 64><<<grid, 128, 0, st>>>(S, z, qq, kk, vv, oo, G); break;
            case 128: la::decode_step_gqa_kernel<T, PHI, 128><<<grid, 256, 0, st>>>(S, z, qq, kk, vv, oo, G); break;
            default: return LA_ERR_UNSUPPORTED;
        }
        return launch_status();
    }
    const unsigned grid = unsigned(heads);
    la::LaunchScope scope("decode_step", st);
    switch (D) {
        case 16: la::decode_step_kernel<T, PHI, 16><<<grid, 32, 0, st>>>(S, z, qq, kk, vv, oo, dec); break;
        case 32: la::decode_step_kernel<T, PHI, 32><<<grid, 64, 0, st>>>(S, z, qq, kk, vv, oo, dec); break;
        case 64: la::decode_step_kernel<T, PHI, 64><<<grid, 128, 0, st>>>(S, z, qq, kk, vv, oo, dec); break;
        case 128: la::decode_step_kernel<T, PHI, 128><<<grid, 256, 0, st>>>(S, z, qq, kk, vv, oo, dec); break;
        default: return LA_ERR_UNSUPPORTED;
    }
    return launch_status();
}

// fn(std::integral_constant<int, PHI>) for the call's feature map
template <typename Fn>
la_status with_phi_map(la_phi phi, Fn&& fn) {
    if (phi == LA_PHI_ELU1) return fn(std::integral_constant<int, PHI_ELU1>{});
    if (phi == LA_PHI_RELU_EPS) return fn(std::integral_constant<int, PHI_RELU_EPS>{});
    return fn(std::integral_constant<int, la::PHI_IDENTITY>{});
}

// dtype x phi dispatch helper
template <template <typename, int> class F, typename... Args>
la_status dispatch(la_dtype dt, la_phi phi, Args... args) {
    if (dt == LA_F32) {
        return phi == LA_PHI_ELU1       ? F<float, PHI_ELU1>::run(args...)
               : phi == LA_PHI_RELU_EPS ? F<float, PHI_RELU_EPS>::run(args...)
                                        : F<float, la::PHI_IDENTITY>::run(args...);
    }
    return phi == LA_PHI_ELU1       ? F<__nv_bfloat16, PHI_ELU1>::run(args...)
           : phi == LA_PHI_RELU_EPS ? F<__nv_bfloat16, PHI_RELU_EPS>::run(args...)
                                    : F<__nv_bfloat16, la::PHI_IDENTITY>::run(args...);
}

template <typename T, int PHI>
struct FwdOp {
    static la_status run(const void* q, const void* k, const void* v, void* o, float* S_out,
                         float* z_out, float* g_out, int64_t heads, int64_t N, int64_t D,
                         int causal, cudaStream_t st, int G, const la::DecayArg* dec) {
        return run_fwd_generic<T, PHI>(q, k, v, o, S_out, z_out, g_out, heads, N, D, causal, st,
                                       G, *dec);
    }
};

template <typename T, int PHI>
struct BwdOp {
    static la_status run(const void* q, const void* k, const void* v, const void* dO, void* dq,
                         void* dk, void* dv, int64_t heads, int64_t N, int64_t D, int causal,
                         float* gbuf, float* dgbuf, cudaStream_t st, int G, char* part,
                         const la::DecayArg* dec) {
        return run_bwd_generic<T, PHI>(q, k, v, dO, dq, dk, dv, heads, N, D, causal, gbuf, dgbuf,
                                       st, G, part, *dec);
    }
};

template <typename T, int PHI>
struct PhiMapOp {
    static la_status run(const void* q, const void* k, void* pq, void* pk, int64_t n,
                         cudaStream_t st) {
        la::LaunchScope scope("phi_map", st);
        const int64_t blocks = std::min<int64_t>((n + 255) / 256, int64_t(num_sms()) * 16);
        la::phi_map_kernel<T, PHI><<<unsigned(blocks), 256, 0, st>>>(
            static_cast<const T*>(q), static_cast<const T*>(k), static_cast<T*>(pq),
            static_cast<T*>(pk), n);
        return launch_status();
    }
};

template <typename T, int PHI>
struct DecodeOp {
    static la_status run(float* S, float* z, const void* q, const void* k, const void* v,
                         void* o, int64_t heads, int64_t D, cudaStream_t st, int G,
                         const la::DecayArg* dec) {
        return run_decode<T, PHI>(S, z, q, k, v, o, heads, D, st, G, *dec);
    }
};

}  // namespace

// ------------------------------------------------------------ static scratch
// Scratch for la_backward_noalloc: a fixed array in device memory, reserved
// when the library's device code is loaded on a GPU.  Host code must not use
// the symbol as an address; the device address comes from
// cudaGetSymbolAddress, resolved once per device.
static __device__ __align__(256) unsigned char g_static_scratch[LA_NOALLOC_MAX_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device (resolved on
// the first call for that device).
la_status static_scratch(void** out) {
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "la_backward_noalloc: device index %d beyond the %d devices it tracks", dev,
                 kMaxDevices);
        return LA_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> g(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch))
            return cuda_fail("cudaGetSymbolAddress", e);
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LA_OK;
}

}  // namespace

extern "C" {

int la_version(void) { return LA_API_VERSION; }

const char* la_last_error(void) { return g_last_error; }

const char* la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "ok";
        case LA_ERR_INVALID_ARG: return "invalid argument";
        case LA_ERR_UNSUPPORTED: return "unsupported configuration";
        case LA_ERR_CUDA: return "CUDA error";
        case LA_ERR_WORKSPACE: return "workspace missing or too small";
        case LA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
    }
    return "unknown status";
}

size_t la_workspace_size_gqa(la_op op, int64_t B, int64_t H, int64_t Hkv, int64_t N, int64_t D,
                             int causal, la_dtype dt) {
    if (check_sizes(B, H, N, D) != LA_OK || check_group(H, Hkv) != LA_OK) return 0;
    if (dt != LA_F32 && dt != LA_BF16) return 0;
    if (B == 0 || H == 0 || N == 0) return 0;
    const int G = int(H / Hkv);
    if (op == LA_OP_FORWARD) return plan_fwd(B, H, N, D, causal, dt).bytes;
    if (op == LA_OP_BACKWARD) {
        const BwdPlan bp = plan_bwd_fast(B, H, N, D, causal, dt, G);
        return bp.fast ? bp.bytes : plan_bwd(B, H, N, D, G).bytes;
    }
    return 0;
}

size_t la_workspace_size(la_op op, int64_t B, int64_t H, int64_t N, int64_t D, int causal,
                         la_dtype dt) {
    return la_workspace_size_gqa(op, B, H, H, N, D, causal, dt);
}

size_t la_workspace_size_decay(la_op op, int64_t B, int64_t H, int64_t N, int64_t D,
                               la_dtype dt) {
    if (check_sizes(B, H, N, D) != LA_OK) return 0;
    if (dt != LA_F32 && dt != LA_BF16) return 0;
    if (B == 0 || H == 0 || N == 0) return 0;
    // enough for either path (the decay factors choose it)
    if (op == LA_OP_FORWARD) return plan_fwd(B, H, N, D, 1, dt).bytes;
    if (op == LA_OP_BACKWARD)
        return std::max(plan_bwd_fast(B, H, N, D, 1, dt, 1).bytes, plan_bwd(B, H, N, D, 1).bytes);
    return 0;
}

namespace {

// Per-head decay factors from a host array: finite, in [0, 1], at most
// kMaxDecayHeads heads.
la_status make_decay(const float* gamma, int64_t H, la::DecayArg* out) {
    if (gamma == nullptr) return LA_ERR_INVALID_ARG;
    if (H > la::kMaxDecayHeads) return LA_ERR_UNSUPPORTED;
    memset(out, 0, sizeof(*out));
    for (int64_t h = 0; h < H; ++h) {
        const float g = gamma[h];
        if (!(g >= 0.f && g <= 1.f)) return LA_ERR_INVALID_ARG;  // NaN fails too
        out->gamma[h] = g;
    }
    out->H = int(H);
    return LA_OK;
}

la_status forward_impl(const void* q, const void* k, const void* v, void* o, float* S_out,
                       float* z_out, float* g_out, void* phi_q_out, void* phi_k_out, int64_t B,
                       int64_t H, int64_t Hkv, int64_t N, int64_t D, la_dtype dt, int causal,
                       la_phi phi, void* workspace, size_t workspace_bytes, la_stream_t stream,
                       const la::DecayArg& dec) {
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if ((s = check_sizes(B, H, N, D)) != LA_OK) return s;
    if ((s = check_group(H, Hkv)) != LA_OK) return s;
    if ((S_out && !aligned16(S_out)) || (z_out && !aligned16(z_out)) ||
        (g_out && !aligned16(g_out)))
        return LA_ERR_INVALID_ARG;
    // feature-map outputs: both or neither, and one key map per query head
    if ((phi_q_out == nullptr) != (phi_k_out == nullptr)) return LA_ERR_INVALID_ARG;
    if (phi_q_out && Hkv != H) return LA_ERR_UNSUPPORTED;
    if (workspace && !aligned16(workspace)) return LA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t heads = B * H;
    const int G = int(H == 0 ? 1 : H / Hkv);
    if (heads == 0) return LA_OK;
    if (N == 0) {
        // nothing to attend over; a requested final state is all zero
        const int64_t kv_heads = B * Hkv;
        if (S_out && cudaMemsetAsync(S_out, 0, size_t(kv_heads * D * D) * 4, st) != cudaSuccess)
            return LA_ERR_CUDA;
        if (z_out && cudaMemsetAsync(z_out, 0, size_t(kv_heads * D) * 4, st) != cudaSuccess)
            return LA_ERR_CUDA;
        return LA_OK;
    }
    if ((s = check_ptr(q)) || (s = check_ptr(k)) || (s = check_ptr(v)) || (s = check_ptr(o)))
        return s;
    if (phi_q_out && ((s = check_ptr(phi_q_out)) || (s = check_ptr(phi_k_out)))) return s;
    // decayed calls run the chunked kernels when every factor is within
    // their range, the token-sequential ones otherwise
    bool chunked = true;
    for (int h = 0; h < dec.H; ++h)
        chunked = chunked && dec.gamma[h] >= chunk_gamma_min(chunk_len(D));
    const FwdPlan plan = chunked ? plan_fwd(B, H, N, D, causal ? 1 : 0, dt) : FwdPlan{};
    if (plan.bytes > 0 && (workspace == nullptr || workspace_bytes < plan.bytes))
        return LA_ERR_WORKSPACE;
    if ((s = bind_context()) != LA_OK) return s;
    // the D = 64 causal kernel stores phi(q), phi(k) from its own tiles;
    // every other path writes them with one elementwise pass
    const bool phi_fused = plan.fast && D == 64 && causal;
    if (plan.fast) {
        char* ws = static_cast<char*>(workspace);
        void* pq = phi_fused ? phi_q_out : nullptr;
        void* pk = phi_fused ? phi_k_out : nullptr;
        s = with_phi_map(phi, [&](auto P) {
            return run_fwd_chunked_d<decltype(P)::value>(q, k, v, o, S_out, z_out, g_out, pq, pk,
                                                         heads, N, D, causal ? 1 : 0, plan, ws,
                                                         st, G, dec);
        });
    } else {
        s = dispatch<FwdOp>(dt, phi, q, k, v, o, S_out, z_out, g_out, heads, N, D,
                            causal ? 1 : 0, st, G, &dec);
    }
    if (s != LA_OK || phi_q_out == nullptr || phi_fused) return s;
    return dispatch<PhiMapOp>(dt, phi, q, k, phi_q_out, phi_k_out, heads * N * D, st);
}

}  // namespace

la_status la_forward_gqa(const void* q, const void* k, const void* v, void* o, float* S_out,
                         float* z_out, float* g_out, void* phi_q_out, void* phi_k_out, int64_t B,
                         int64_t H, int64_t Hkv, int64_t N, int64_t D, la_dtype dt, int causal,
                         la_phi phi, void* workspace, size_t workspace_bytes, la_stream_t stream) {
    return forward_impl(q, k, v, o, S_out, z_out, g_out, phi_q_out, phi_k_out, B, H, Hkv, N, D,
                        dt, causal, phi, workspace, workspace_bytes, stream, kNoDecay);
}

la_status la_forward_decay(const void* q, const void* k, const void* v, void* o, float* S_out,
                           float* z_out, float* g_out, const float* gamma, int64_t B, int64_t H,
                           int64_t N, int64_t D, la_dtype dt, la_phi phi, void* workspace,
                           size_t workspace_bytes, la_stream_t stream) {
    la::DecayArg dec;
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if ((s = check_sizes(B, H, N, D)) != LA_OK) return s;
    if ((s = make_decay(gamma, H, &dec)) != LA_OK) return s;
    return forward_impl(q, k, v, o, S_out, z_out, g_out, nullptr, nullptr, B, H, H, N, D, dt, 1,
                        phi, workspace, workspace_bytes, stream, dec);
}

la_status la_forward(const void* q, const void* k, const void* v, void* o, float* S_out,
                     float* z_out, float* g_out, void* phi_q_out, void* phi_k_out, int64_t B,
                     int64_t H, int64_t N, int64_t D, la_dtype dt, int causal, la_phi phi,
                     void* workspace, size_t workspace_bytes, la_stream_t stream) {
    return la_forward_gqa(q, k, v, o, S_out, z_out, g_out, phi_q_out, phi_k_out, B, H, H, N, D,
                          dt, causal, phi, workspace, workspace_bytes, stream);
}

namespace {

la_status backward_impl(const void* q, const void* k, const void* v, const void* dO,
                        const void* o, const float* g, const void* phi_q, const void* phi_k,
                        void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Hkv,
                        int64_t N, int64_t D, la_dtype dt, int causal, la_phi phi,
                        void* workspace, size_t workspace_bytes, la_stream_t stream,
                        const la::DecayArg& dec) {
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if ((s = check_sizes(B, H, N, D)) != LA_OK) return s;
    if ((s = check_group(H, Hkv)) != LA_OK) return s;
    if (workspace && !aligned16(workspace)) return LA_ERR_INVALID_ARG;
    const int64_t heads = B * H;
    if (heads == 0 || N == 0) return LA_OK;
    const int G = int(H / Hkv);
    if ((s = check_ptr(q)) || (s = check_ptr(k)) || (s = check_ptr(v)) || (s = check_ptr(dO)) ||
        (s = check_ptr(dq)) || (s = check_ptr(dk)) || (s = check_ptr(dv)))
        return s;
    // saved forward statistics: both or neither
    if ((o == nullptr) != (g == nullptr)) return LA_ERR_INVALID_ARG;
    if (o && ((s = check_ptr(o)) || (s = check_ptr(g)))) return s;
    // saved feature maps: both or neither, and only with o and g
    if ((phi_q == nullptr) != (phi_k == nullptr) || (phi_q && !o)) return LA_ERR_INVALID_ARG;
    if (phi_q && G != 1) return LA_ERR_UNSUPPORTED;
    if (phi_q && ((s = check_ptr(phi_q)) || (s = check_ptr(phi_k)))) return s;
    // decayed calls run the chunked passes for head size 64 when every factor
    // is within their range and the plan keeps one segment per head, the
    // token-sequential kernels otherwise
    BwdPlan bp = plan_bwd_fast(B, H, N, D, causal ? 1 : 0, dt, G);
    if (dec.H > 0) {
        bool chunked = bp.fast && D == 64 && causal && G == 1 && bp.seg.nseg == 1;
        for (int h = 0; h < dec.H; ++h)
            chunked = chunked && dec.gamma[h] >= chunk_gamma_min(chunk_len(D));
        if (!chunked) bp = BwdPlan{};
    }
    const size_t need = bp.fast ? bp.bytes : plan_bwd(B, H, N, D, G).bytes;
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return LA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((s = bind_context()) != LA_OK) return s;
    if (bp.fast) {
        char* wsp = static_cast<char*>(workspace);
        if (o == nullptr) {
            // the chunked backward reads the forward's o and g: compute them
            // here (into the workspace) when the caller has not kept them
            const FwdPlan fp = plan_fwd(B, H, N, D, causal ? 1 : 0, dt);
            void* o_ws = wsp + bp.o_off;
            float* g_ws = reinterpret_cast<float*>(wsp + bp.g_off);
            s = with_phi_map(phi, [&](auto P) {
                return run_fwd_chunked_d<decltype(P)::value>(
                    q, k, v, o_ws, nullptr, nullptr, g_ws, nullptr, nullptr, heads, N, D,
                    causal ? 1 : 0, fp, wsp + bp.fwd_off, st, G, dec);
            });
            if (s != LA_OK) return s;
            o = o_ws;
            g = g_ws;
        }
        return with_phi_map(phi, [&](auto P) {
            return run_bwd_chunked_d<decltype(P)::value>(q, k, v, dO, o, g, phi_q, phi_k, dq, dk,
                                                         dv, heads, N, D, causal ? 1 : 0, bp, wsp,
                                                         st, G, dec);
        });
    }
    const BwdWorkspace w = plan_bwd(B, H, N, D, G);
    char* ws = static_cast<char*>(workspace);
    float* gbuf = reinterpret_cast<float*>(ws + w.g_off);
    float* dgbuf = reinterpret_cast<float*>(ws + w.dg_off);
    return dispatch<BwdOp>(dt, phi, q, k, v, dO, dq, dk, dv, heads, N, D, causal ? 1 : 0, gbuf,
                           dgbuf, st, G, ws + w.part_off, &dec);
}

}  // namespace

la_status la_backward_gqa(const void* q, const void* k, const void* v, const void* dO,
                          const void* o, const float* g, const void* phi_q, const void* phi_k,
                          void* dq, void* dk, void* dv, int64_t B, int64_t H, int64_t Hkv,
                          int64_t N, int64_t D, la_dtype dt, int causal, la_phi phi,
                          void* workspace, size_t workspace_bytes, la_stream_t stream) {
    return backward_impl(q, k, v, dO, o, g, phi_q, phi_k, dq, dk, dv, B, H, Hkv, N, D, dt, causal,
                         phi, workspace, workspace_bytes, stream, kNoDecay);
}

la_status la_backward_decay(const void* q, const void* k, const void* v, const void* dO,
                            const void* o, const float* g, void* dq, void* dk, void* dv,
                            const float* gamma, int64_t B, int64_t H, int64_t N, int64_t D,
                            la_dtype dt, la_phi phi, void* workspace, size_t workspace_bytes,
                            la_stream_t stream) {
    la::DecayArg dec;
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if ((s = check_sizes(B, H, N, D)) != LA_OK) return s;
    if ((s = make_decay(gamma, H, &dec)) != LA_OK) return s;
    return backward_impl(q, k, v, dO, o, g, nullptr, nullptr, dq, dk, dv, B, H, H, N, D, dt, 1,
                         phi, workspace, workspace_bytes, stream, dec);
}

la_status la_backward(const void* q, const void* k, const void* v, const void* dO,
                      const void* o, const float* g, const void* phi_q, const void* phi_k,
                      void* dq, void* dk, void* dv, int64_t B,
                      int64_t H, int64_t N, int64_t D, la_dtype dt, int causal, la_phi phi,
                      void* workspace, size_t workspace_bytes, la_stream_t stream) {
    return la_backward_gqa(q, k, v, dO, o, g, phi_q, phi_k, dq, dk, dv, B, H, H, N, D, dt, causal,
                           phi, workspace, workspace_bytes, stream);
}

la_status la_backward_noalloc(const void* q, const void* k, const void* v, const void* dO,
                              const void* o, const float* g, const void* phi_q,
                              const void* phi_k, void* dq, void* dk, void* dv,
                              int64_t B, int64_t H, int64_t N, int64_t D, la_dtype dt, int causal,
                              la_phi phi, la_stream_t stream) {
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if ((s = check_sizes(B, H, N, D)) != LA_OK) return s;
    const size_t need = la_workspace_size(LA_OP_BACKWARD, B, H, N, D, causal, dt);
    if (need > size_t(LA_NOALLOC_MAX_BYTES)) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "la_backward_noalloc: needs %zu bytes of scratch, limit %u", need,
                 unsigned(LA_NOALLOC_MAX_BYTES));
        return LA_ERR_WORKSPACE;
    }
    if ((s = bind_context()) != LA_OK) return s;
    void* scratch = nullptr;
    if ((s = static_scratch(&scratch)) != LA_OK) return s;
    return la_backward(q, k, v, dO, o, g, phi_q, phi_k, dq, dk, dv, B, H, N, D, dt, causal, phi,
                       scratch, size_t(LA_NOALLOC_MAX_BYTES), stream);
}

// ------------------------------------------------------------ sequence split across ranks
// The tokens of every head split into consecutive shards, one per rank.
// States are sums over tokens ("Efficient Transformers Survey", Proposition
// "Linear Attention via Kernel Decomposition", Statement), so a rank's
// causal outputs need only the sum of the states of the shards before it
// (non-causal: of every shard), and the backward's suffix state of the
// shards after it: one exchange of one record per head each way.
}  // extern "C"

namespace {

// seg: the causal passes and the local reduce; qseg: the non-causal query
// and gradient passes (one block each).  Backward workspace: dg [heads][N],
// the centred prefix records of a split head (srec) and one (R, r) record
// per pass-1 block (rrec), which the dK/dV call reads back.
struct SpPlan {
    bool fast = false;
    int C = 0;
    SegSplit seg, qseg;
    StartSplit ss;  // causal, split heads: the reduce pass for the segment starts
    size_t fwd_sub_off = 0, fwd_bytes = 0;
    size_t dg_off = 0, srec_off = 0, rrec_off = 0, sub_off = 0, bwd_bytes = 0;
};

SpPlan plan_sp(int64_t B, int64_t H, int64_t N, int64_t D, int causal, la_dtype dt) {
    SpPlan p;
    if (!fast_path(dt, D) || N == 0 || B * H == 0) return p;
    p.fast = true;
    p.C = chunk_len(D);
    const int64_t heads = B * H;
    const int64_t nch = (N + p.C - 1) / p.C;
    const int kNumSM = num_sms();
    p.seg = split(N, p.C, pick_nseg(heads, nch));
    const int64_t want = heads >= 2 * kNumSM ? 1 : (2 * kNumSM + heads - 1) / heads;
    p.qseg = causal ? p.seg
                    : split(N, p.C, int(std::max<int64_t>(1, std::min<int64_t>(want, nch))));
    const size_t R4 = size_t(D * D + D) * sizeof(float);
    p.ss = start_split(heads, p.seg, p.C, D);
    // forward: per-segment records (la_state_local) or starts, then the
    // start reduce's sub-segment records
    p.fwd_sub_off = p.seg.nseg > 1 ? round_up(size_t(heads) * p.seg.nseg * R4, 256) : 0;
    p.fwd_bytes = p.fwd_sub_off + round_up(size_t(heads) * p.ss.nsub * R4, 256);
    size_t off = 0;
    p.dg_off = off;
    off += round_up(size_t(heads) * size_t(N) * sizeof(float), 256);
    p.srec_off = off;
    if (causal && p.seg.nseg > 1) off += round_up(size_t(heads) * p.seg.nseg * R4, 256);
    p.rrec_off = off;
    off += round_up(size_t(heads) * p.qseg.nseg * R4, 256);
    p.sub_off = off;
    if (causal) off += round_up(size_t(heads) * p.ss.nsub * R4, 256);
    p.bwd_bytes = std::max(off, p.fwd_bytes);
    return p;
}

template <int D, int PHI>
la_status run_state_local(const void* k, const void* v, float* out, int64_t heads, int64_t N,
                          int centred, const SpPlan& p, char* ws, cudaStream_t st) {
    constexpr int C = D == 64 ? 128 : 64;
    const int64_t R = int64_t(D) * D + D;
    la::ChunkParams r;
    memset(&r, 0, sizeof(r));
    if (!make_qkv_map(&r.tm_k, k, heads, N, D, C) || !make_qkv_map(&r.tm_v, v, heads, N, D, C))
        return LA_ERR_CUDA;
    r.N = int(N);
    r.seg_len = p.seg.seg_len;
    r.nseg = p.seg.nseg;
    r.center = centred;
    r.kv_group = 1;
    float* dst = p.seg.nseg > 1 ? reinterpret_cast<float*>(ws) : out;
    r.S_out = dst;
    r.z_out = dst + D * D;
    r.stride_S = r.stride_z = R;
    la_status s = launch_reduce<D, C, PHI>(r, heads * p.seg.nseg, st);
    if (s != LA_OK || p.seg.nseg == 1) return s;
    return launch_state_kernel(1, dst, out, nullptr, nullptr, heads, p.seg.nseg, D, st);
}

template <int D, int PHI>
la_status run_fwd_sp(const void* q, const void* k, const void* v, void* o, const float* state_in,
                     float* state_out, float* g_out, int64_t heads, int64_t N, int causal,
                     const SpPlan& p, char* ws, cudaStream_t st) {
    constexpr int C = D == 64 ? 128 : 64;
    const int64_t R = int64_t(D) * D + D;
    la::ChunkParams prm;
    memset(&prm, 0, sizeof(prm));
    if (!make_qkv_map(&prm.tm_q, q, heads, N, D, C) || !make_qkv_map(&prm.tm_k, k, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_v, v, heads, N, D, C) || !make_qkv_map(&prm.tm_o, o, heads, N, D, C))
        return LA_ERR_CUDA;
    prm.N = int(N);
    prm.g_out = g_out;
    prm.kv_group = 1;
    la_status s;
    if (!causal) {
        prm.seg_len = p.qseg.seg_len;
        prm.nseg = p.qseg.nseg;
        prm.state_in = state_in;
        prm.in_per_head = 1;
        return launch_chunk<D, C, PHI, la::MODE_QUERY>(prm, heads * p.qseg.nseg, st,
                                                       "chunk_query");
    }
    prm.state_in = state_in;
    prm.in_per_head = 1;
    if (p.seg.nseg > 1) {
        // segment starts: the incoming state plus the segments before
        float* starts = reinterpret_cast<float*>(ws);
        float* sub = reinterpret_cast<float*>(ws + p.fwd_sub_off);
        if ((s = run_segment_starts<D, C, PHI>(prm, heads, p.seg, p.ss, sub, starts, state_in,
                                               st)) != LA_OK)
            return s;
        prm.state_in = starts;
        prm.in_per_head = 0;
    }
    prm.seg_len = p.seg.seg_len;
    prm.nseg = p.seg.nseg;
    prm.S_out = state_out;
    prm.z_out = state_out ? state_out + D * D : nullptr;
    prm.stride_S = prm.stride_z = R;
    return launch_chunk<D, C, PHI, la::MODE_CAUSAL>(prm, heads * p.seg.nseg, st, "chunk_causal");
}

template <int D, int PHI>
la_status run_bwd_sp_dq(const void* q, const void* k, const void* v, const void* dO,
                        const void* o, const float* g, const float* state_in, void* dq,
                        float* state_out, int64_t heads, int64_t N, int causal, const SpPlan& p,
                        char* ws, cudaStream_t st) {
    constexpr int C = D == 64 ? 128 : 64;
    constexpr int smem1 = la::Bwd1Cfg<D, C>::SMEM;
    la::BwdParams prm;
    memset(&prm, 0, sizeof(prm));
    if (!make_qkv_map(&prm.tm_q, q, heads, N, D, C) || !make_qkv_map(&prm.tm_k, k, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_v, v, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_do, dO, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_dq, dq, heads, N, D, C))
        return LA_ERR_CUDA;
    prm.kv_group = 1;
    prm.N = int(N);
    prm.gbuf = const_cast<float*>(g);
    prm.dgbuf = reinterpret_cast<float*>(ws + p.dg_off);
    prm.o_in = static_cast<const __nv_bfloat16*>(o);
    float* rrec = reinterpret_cast<float*>(ws + p.rrec_off);
    prm.rec_out = rrec;
    prm.state_in = state_in;
    prm.in_per_head = 1;
    const SegSplit& sg = causal ? p.seg : p.qseg;
    prm.seg_len = sg.seg_len;
    prm.nseg = sg.nseg;
    la_status s;
    if (causal && p.seg.nseg > 1) {
        // segment starts: the incoming centred state plus the centred
        // states of the segments before (the dQ products' key features)
        float* srec = reinterpret_cast<float*>(ws + p.srec_off);
        float* sub = reinterpret_cast<float*>(ws + p.sub_off);
        la::ChunkParams red;
        memset(&red, 0, sizeof(red));
        red.tm_k = prm.tm_k;
        red.tm_v = prm.tm_v;
        red.N = int(N);
        red.center = 1;
        red.kv_group = 1;
        if ((s = run_segment_starts<D, C, PHI>(red, heads, p.seg, p.ss, sub, srec, state_in,
                                               st)) != LA_OK)
            return s;
        prm.state_in = srec;
        prm.in_per_head = 0;
    }
    s = causal ? launch_bwd_kernel(la::bwd_dq_kernel<D, C, PHI, true, true>, smem1, prm,
                                   heads * sg.nseg, st, "bwd_dq")
               : launch_bwd_kernel(la::bwd_dq_kernel<D, C, PHI, false, true>, smem1, prm,
                                   heads * sg.nseg, st, "bwd_dq");
    if (s != LA_OK) return s;
    // this rank's (R, r): the sum of its blocks' records (which stay in the
    // workspace for the dK/dV call)
    return launch_state_kernel(1, rrec, state_out, nullptr, nullptr, heads, sg.nseg, D, st);
}

template <int D, int PHI>
la_status run_bwd_sp_dkdv(const void* q, const void* k, const void* v, const void* dO,
                          const float* g, const float* state_in, void* dk, void* dv,
                          int64_t heads, int64_t N, int causal, const SpPlan& p, char* ws,
                          cudaStream_t st) {
    constexpr int C = D == 64 ? 128 : 64;
    constexpr int smem2 = la::Bwd2Cfg<D, C>::SMEM;
    la::BwdParams prm;
    memset(&prm, 0, sizeof(prm));
    if (!make_qkv_map(&prm.tm_q, q, heads, N, D, C) || !make_qkv_map(&prm.tm_k, k, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_v, v, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_do, dO, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_dk, dk, heads, N, D, C) ||
        !make_qkv_map(&prm.tm_dv, dv, heads, N, D, C))
        return LA_ERR_CUDA;
    prm.kv_group = 1;
    prm.N = int(N);
    prm.gbuf = const_cast<float*>(g);
    prm.dgbuf = reinterpret_cast<float*>(ws + p.dg_off);
    if (!causal) {
        prm.seg_len = p.qseg.seg_len;
        prm.nseg = p.qseg.nseg;
        prm.state_in = state_in;
        prm.in_per_head = 1;
        return launch_bwd_kernel(la::bwd_dkdv_kernel<D, C, PHI, false>, smem2, prm,
                                 heads * p.qseg.nseg, st, "bwd_dkdv");
    }
    // block starts of the reverse walk: the incoming suffix state plus the
    // records of the blocks after (left in the workspace by the dQ call)
    float* rrec = reinterpret_cast<float*>(ws + p.rrec_off);
    la_status s = launch_state_kernel(3, rrec, nullptr, nullptr, nullptr, heads, p.seg.nseg, D,
                                      st, 1, kNoDecay, 0, state_in);
    if (s != LA_OK) return s;
    prm.seg_len = p.seg.seg_len;
    prm.nseg = p.seg.nseg;
    prm.state_in = rrec;
    prm.in_per_head = 0;
    if constexpr (D == 64)
        return launch_bwd_kernel(la::bwd_dkdv64_kernel<PHI, false>, la::Bwd2x64Cfg::SMEM, prm,
                                 heads * p.seg.nseg, st, "bwd_dkdv", la::kBwd64Threads);
    else
        return launch_bwd_kernel(la::bwd_dkdv_kernel<D, C, PHI, true>, smem2, prm,
                                 heads * p.seg.nseg, st, "bwd_dkdv");
}

// Shared checks of the sequence-parallel calls: the tensor-core path only
// (bf16, D = 64 or 128, one key/value head per query head).
la_status check_sp(int64_t B, int64_t H, int64_t N, int64_t D, la_dtype dt, la_phi phi,
                   const void* workspace) {
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if ((s = check_sizes(B, H, N, D)) != LA_OK) return s;
    if (!fast_path(dt, D)) return LA_ERR_UNSUPPORTED;
    if (workspace && !aligned16(workspace)) return LA_ERR_INVALID_ARG;
    return LA_OK;
}

la_status check_ws(const void* workspace, size_t have, size_t need) {
    if (need > 0 && (workspace == nullptr || have < need)) return LA_ERR_WORKSPACE;
    return LA_OK;
}

template <typename Fn>
la_status with_head_size(int64_t D, Fn&& fn) {
    if (D == 64) return fn(std::integral_constant<int, 64>{});
    return fn(std::integral_constant<int, 128>{});
}

}  // namespace

extern "C" {

size_t la_workspace_size_sp(la_op op, int64_t B, int64_t H, int64_t N, int64_t D, int causal,
                            la_dtype dt) {
    if (check_sizes(B, H, N, D) != LA_OK || !fast_path(dt, D)) return 0;
    const SpPlan p = plan_sp(B, H, N, D, causal ? 1 : 0, dt);
    if (!p.fast) return 0;
    if (op == LA_OP_FORWARD) return p.fwd_bytes;
    if (op == LA_OP_BACKWARD) return p.bwd_bytes;
    return 0;
}

la_status la_state_local(const void* k, const void* v, float* state_out, int64_t B, int64_t H,
                         int64_t N, int64_t D, la_dtype dt, la_phi phi, int centred,
                         void* workspace, size_t workspace_bytes, la_stream_t stream) {
    la_status s;
    if ((s = check_sp(B, H, N, D, dt, phi, workspace)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0) return LA_OK;
    if ((s = check_ptr(state_out)) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        if (cudaError_t e = cudaMemsetAsync(state_out, 0, size_t(heads * (D * D + D)) * 4, st))
            return cuda_fail("cudaMemsetAsync", e);
        return LA_OK;
    }
    if ((s = check_ptr(k)) || (s = check_ptr(v))) return s;
    const SpPlan p = plan_sp(B, H, N, D, 1, dt);
    if ((s = check_ws(workspace, workspace_bytes, p.fwd_bytes)) != LA_OK) return s;
    if ((s = bind_context()) != LA_OK) return s;
    char* ws = static_cast<char*>(workspace);
    return with_phi_map(phi, [&](auto P) {
        return with_head_size(D, [&](auto Dc) {
            return run_state_local<decltype(Dc)::value, decltype(P)::value>(
                k, v, state_out, heads, N, centred ? 1 : 0, p, ws, st);
        });
    });
}

la_status la_state_range_sum(const float* states, int64_t P, int64_t lo, int64_t hi,
                             float* out, int64_t B, int64_t H, int64_t D, la_stream_t stream) {
    la_status s;
    if (B < 0 || H < 0 || D <= 0 || P < 0 || lo < 0 || hi < lo || hi > P)
        return LA_ERR_INVALID_ARG;
    if (!supported_d(D)) return LA_ERR_UNSUPPORTED;
    const int64_t heads = B * H;
    if (heads == 0) return LA_OK;
    if (heads >= (int64_t(1) << 31) || P >= (int64_t(1) << 20)) return LA_ERR_UNSUPPORTED;
    if ((s = check_ptr(out)) != LA_OK) return s;
    if (hi > lo && (s = check_ptr(states)) != LA_OK) return s;
    if ((s = bind_context()) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int R4 = int(D * D + D) / 4;  // float4 columns (R is a multiple of 4)
    const int bph = (R4 + la::kStateThreads - 1) / la::kStateThreads;
    la::LaunchScope scope("state_range_sum", st);
    la::state_range_sum_kernel<<<unsigned(heads * bph), la::kStateThreads, 0, st>>>(
        states, out, int(lo), int(hi), heads, R4, bph);
    return launch_status();
}

la_status la_forward_sp(const void* q, const void* k, const void* v, void* o,
                        const float* state_in, float* state_out, float* g_out, int64_t B,
                        int64_t H, int64_t N, int64_t D, la_dtype dt, int causal, la_phi phi,
                        void* workspace, size_t workspace_bytes, la_stream_t stream) {
    la_status s;
    if ((s = check_sp(B, H, N, D, dt, phi, workspace)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0) return LA_OK;
    if ((s = check_ptr(state_in)) != LA_OK) return s;
    if (state_out && !causal) return LA_ERR_INVALID_ARG;
    if ((state_out && !aligned16(state_out)) || (g_out && !aligned16(g_out)))
        return LA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        // no tokens here: the state passes through unchanged
        if (state_out) {
            if (cudaError_t e = cudaMemcpyAsync(state_out, state_in,
                                                size_t(heads * (D * D + D)) * 4,
                                                cudaMemcpyDeviceToDevice, st))
                return cuda_fail("cudaMemcpyAsync", e);
        }
        return LA_OK;
    }
    if ((s = check_ptr(q)) || (s = check_ptr(k)) || (s = check_ptr(v)) || (s = check_ptr(o)))
        return s;
    const SpPlan p = plan_sp(B, H, N, D, causal ? 1 : 0, dt);
    if ((s = check_ws(workspace, workspace_bytes, p.fwd_bytes)) != LA_OK) return s;
    if ((s = bind_context()) != LA_OK) return s;
    char* ws = static_cast<char*>(workspace);
    return with_phi_map(phi, [&](auto P) {
        return with_head_size(D, [&](auto Dc) {
            return run_fwd_sp<decltype(Dc)::value, decltype(P)::value>(
                q, k, v, o, state_in, state_out, g_out, heads, N, causal ? 1 : 0, p, ws, st);
        });
    });
}

la_status la_backward_sp_dq(const void* q, const void* k, const void* v, const void* dO,
                            const void* o, const float* g, const float* state_in, void* dq,
                            float* state_out, int64_t B, int64_t H, int64_t N, int64_t D,
                            la_dtype dt, int causal, la_phi phi, void* workspace,
                            size_t workspace_bytes, la_stream_t stream) {
    la_status s;
    if ((s = check_sp(B, H, N, D, dt, phi, workspace)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0) return LA_OK;
    if ((s = check_ptr(state_in)) || (s = check_ptr(state_out))) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {
        if (cudaError_t e = cudaMemsetAsync(state_out, 0, size_t(heads * (D * D + D)) * 4, st))
            return cuda_fail("cudaMemsetAsync", e);
        return LA_OK;
    }
    if ((s = check_ptr(q)) || (s = check_ptr(k)) || (s = check_ptr(v)) || (s = check_ptr(dO)) ||
        (s = check_ptr(o)) || (s = check_ptr(g)) || (s = check_ptr(dq)))
        return s;
    const SpPlan p = plan_sp(B, H, N, D, causal ? 1 : 0, dt);
    if ((s = check_ws(workspace, workspace_bytes, p.bwd_bytes)) != LA_OK) return s;
    if ((s = bind_context()) != LA_OK) return s;
    char* ws = static_cast<char*>(workspace);
    return with_phi_map(phi, [&](auto P) {
        return with_head_size(D, [&](auto Dc) {
            return run_bwd_sp_dq<decltype(Dc)::value, decltype(P)::value>(
                q, k, v, dO, o, g, state_in, dq, state_out, heads, N, causal ? 1 : 0, p, ws, st);
        });
    });
}

la_status la_backward_sp_dkdv(const void* q, const void* k, const void* v, const void* dO,
                              const float* g, const float* state_in, void* dk, void* dv,
                              int64_t B, int64_t H, int64_t N, int64_t D, la_dtype dt, int causal,
                              la_phi phi, void* workspace, size_t workspace_bytes,
                              la_stream_t stream) {
    la_status s;
    if ((s = check_sp(B, H, N, D, dt, phi, workspace)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0 || N == 0) return LA_OK;
    if ((s = check_ptr(state_in)) != LA_OK) return s;
    if ((s = check_ptr(q)) || (s = check_ptr(k)) || (s = check_ptr(v)) || (s = check_ptr(dO)) ||
        (s = check_ptr(g)) || (s = check_ptr(dk)) || (s = check_ptr(dv)))
        return s;
    const SpPlan p = plan_sp(B, H, N, D, causal ? 1 : 0, dt);
    if ((s = check_ws(workspace, workspace_bytes, p.bwd_bytes)) != LA_OK) return s;
    if ((s = bind_context()) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    return with_phi_map(phi, [&](auto P) {
        return with_head_size(D, [&](auto Dc) {
            return run_bwd_sp_dkdv<decltype(Dc)::value, decltype(P)::value>(
                q, k, v, dO, g, state_in, dk, dv, heads, N, causal ? 1 : 0, p, ws, st);
        });
    });
}

size_t la_workspace_size_mv(la_op op, int64_t B, int64_t H, int64_t N, int64_t Dk, int64_t Dv,
                            int causal, la_dtype dt) {
    if (dt != LA_BF16 || (Dk != 64 && Dk != 128) || (Dv != 64 && Dv != 128)) return 0;
    if (check_sizes(B, H, N, std::max(Dk, Dv)) != LA_OK || B * H == 0 || N == 0) return 0;
    if (op != LA_OP_FORWARD && op != LA_OP_BACKWARD) return 0;
    return plan_mv(op, B, H, N, Dk, Dv, causal ? 1 : 0).bytes;
}

namespace {

// Shared checks of la_forward_mv / la_backward_mv.
la_status check_mv(int64_t B, int64_t H, int64_t N, int64_t Dk, int64_t Dv, la_dtype dt,
                   la_phi phi) {
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if (Dk <= 0 || Dv <= 0) return LA_ERR_INVALID_ARG;
    if (dt != LA_BF16 || (Dk != 64 && Dk != 128) || (Dv != 64 && Dv != 128))
        return LA_ERR_UNSUPPORTED;
    // zero feature columns add nothing only when the features are given
    if (Dk < Dv && phi != LA_PHI_IDENTITY) return LA_ERR_UNSUPPORTED;
    return check_sizes(B, H, N, std::max(Dk, Dv));
}

}  // namespace

la_status la_forward_mv(const void* q, const void* k, const void* v, void* o, float* g_out,
                        int64_t B, int64_t H, int64_t N, int64_t Dk, int64_t Dv, la_dtype dt,
                        int causal, la_phi phi, void* workspace, size_t workspace_bytes,
                        la_stream_t stream) {
    la_status s;
    if ((s = check_mv(B, H, N, Dk, Dv, dt, phi)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0 || N == 0) return LA_OK;
    if ((s = check_ptr(q)) || (s = check_ptr(k)) || (s = check_ptr(v)) || (s = check_ptr(o)))
        return s;
    if ((g_out && !aligned16(g_out)) || (workspace && !aligned16(workspace)))
        return LA_ERR_INVALID_ARG;
    const MvPlan p = plan_mv(LA_OP_FORWARD, B, H, N, Dk, Dv, causal);
    if (p.bytes > 0 && (workspace == nullptr || workspace_bytes < p.bytes))
        return LA_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    char* inner = p.inner > 0 ? ws + p.inner_off : nullptr;
    if (Dk == Dv)
        return la_forward(q, k, v, o, nullptr, nullptr, g_out, nullptr, nullptr, B, H, N, Dk, dt,
                          causal, phi, inner, p.inner, stream);
    if ((s = bind_context()) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t rows = heads * N, D = p.D;
    void* t0 = ws;
    void* t1 = ws + p.tile;
    if (Dv < Dk) {
        // values widened with zero columns; the output's first Dv columns
        if ((s = copy_cols(v, t0, rows, Dv, D, st)) != LA_OK) return s;
        if ((s = la_forward(q, k, t0, t1, nullptr, nullptr, g_out, nullptr, nullptr, B, H, N, D,
                            dt, causal, phi, inner, p.inner, stream)) != LA_OK)
            return s;
        return copy_cols(t1, o, rows, D, Dv, st);
    }
    // features widened with zero columns (identity map)
    if ((s = copy_cols(q, t0, rows, Dk, D, st)) != LA_OK) return s;
    if ((s = copy_cols(k, t1, rows, Dk, D, st)) != LA_OK) return s;
    return la_forward(t0, t1, v, o, nullptr, nullptr, g_out, nullptr, nullptr, B, H, N, D, dt,
                      causal, phi, inner, p.inner, stream);
}

la_status la_backward_mv(const void* q, const void* k, const void* v, const void* dO,
                         const void* o, const float* g, void* dq, void* dk, void* dv, int64_t B,
                         int64_t H, int64_t N, int64_t Dk, int64_t Dv, la_dtype dt, int causal,
                         la_phi phi, void* workspace, size_t workspace_bytes,
                         la_stream_t stream) {
    la_status s;
    if ((s = check_mv(B, H, N, Dk, Dv, dt, phi)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0 || N == 0) return LA_OK;
    if ((s = check_ptr(q)) || (s = check_ptr(k)) || (s = check_ptr(v)) || (s = check_ptr(dO)) ||
        (s = check_ptr(dq)) || (s = check_ptr(dk)) || (s = check_ptr(dv)))
        return s;
    if ((o == nullptr) != (g == nullptr)) return LA_ERR_INVALID_ARG;
    if (o && ((s = check_ptr(o)) || (s = check_ptr(g)))) return s;
    if (workspace && !aligned16(workspace)) return LA_ERR_INVALID_ARG;
    const MvPlan p = plan_mv(LA_OP_BACKWARD, B, H, N, Dk, Dv, causal);
    if (p.bytes > 0 && (workspace == nullptr || workspace_bytes < p.bytes))
        return LA_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    char* inner = p.inner > 0 ? ws + p.inner_off : nullptr;
    if (Dk == Dv)
        return la_backward(q, k, v, dO, o, g, nullptr, nullptr, dq, dk, dv, B, H, N, Dk, dt,
                           causal, phi, inner, p.inner, stream);
    if ((s = bind_context()) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t rows = heads * N, D = p.D;
    void* t[4] = {ws, ws + p.tile, ws + 2 * p.tile, ws + 3 * p.tile};
    if (Dv < Dk) {
        // v, dO (and o) widened; dV is the first Dv columns of the wide dV
        if ((s = copy_cols(v, t[0], rows, Dv, D, st)) != LA_OK) return s;
        if ((s = copy_cols(dO, t[1], rows, Dv, D, st)) != LA_OK) return s;
        if (o && (s = copy_cols(o, t[2], rows, Dv, D, st)) != LA_OK) return s;
        if ((s = la_backward(q, k, t[0], t[1], o ? t[2] : nullptr, g, nullptr, nullptr, dq, dk,
                             t[3], B, H, N, D, dt, causal, phi, inner, p.inner, stream)) != LA_OK)
            return s;
        return copy_cols(t[3], dv, rows, D, Dv, st);
    }
    // features widened (identity map); dQ, dK are the first Dk columns
    if ((s = copy_cols(q, t[0], rows, Dk, D, st)) != LA_OK) return s;
    if ((s = copy_cols(k, t[1], rows, Dk, D, st)) != LA_OK) return s;
    if ((s = la_backward(t[0], t[1], v, dO, o, g, nullptr, nullptr, t[2], t[3], dv, B, H, N, D,
                         dt, causal, phi, inner, p.inner, stream)) != LA_OK)
        return s;
    if ((s = copy_cols(t[2], dq, rows, D, Dk, st)) != LA_OK) return s;
    return copy_cols(t[3], dk, rows, D, Dk, st);
}

namespace {

la_status decode_impl(float* S, float* z, const void* q, const void* k, const void* v, void* o,
                      int64_t B, int64_t H, int64_t Hkv, int64_t D, la_dtype dt, la_phi phi,
                      la_stream_t stream, const la::DecayArg& dec) {
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if ((s = check_sizes(B, H, 1, D)) != LA_OK) return s;
    if ((s = check_group(H, Hkv)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0) return LA_OK;
    if ((s = check_ptr(S)) || (s = check_ptr(z)) || (s = check_ptr(q)) || (s = check_ptr(k)) ||
        (s = check_ptr(v)) || (s = check_ptr(o)))
        return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return dispatch<DecodeOp>(dt, phi, S, z, q, k, v, o, heads, D, st, int(H / Hkv), &dec);
}

}  // namespace

la_status la_decode_step_gqa(float* S, float* z, const void* q, const void* k, const void* v,
                             void* o, int64_t B, int64_t H, int64_t Hkv, int64_t D, la_dtype dt,
                             la_phi phi, la_stream_t stream) {
    return decode_impl(S, z, q, k, v, o, B, H, Hkv, D, dt, phi, stream, kNoDecay);
}

la_status la_decode_step_decay(float* S, float* z, const void* q, const void* k, const void* v,
                               void* o, const float* gamma, int64_t B, int64_t H, int64_t D,
                               la_dtype dt, la_phi phi, la_stream_t stream) {
    la::DecayArg dec;
    la_status s;
    if ((s = check_enums(dt, phi)) != LA_OK) return s;
    if ((s = check_sizes(B, H, 1, D)) != LA_OK) return s;
    if ((s = make_decay(gamma, H, &dec)) != LA_OK) return s;
    return decode_impl(S, z, q, k, v, o, B, H, H, D, dt, phi, stream, dec);
}

la_status la_decode_step(float* S, float* z, const void* q, const void* k, const void* v,
                         void* o, int64_t B, int64_t H, int64_t D, la_dtype dt, la_phi phi,
                         la_stream_t stream) {
    return la_decode_step_gqa(S, z, q, k, v, o, B, H, H, D, dt, phi, stream);
}

namespace {

// FAVOR+ sizes: bf16, D and m each 64 or 128
la_status check_favor(int64_t B, int64_t H, int64_t N, int64_t D, int64_t m, la_dtype dt) {
    if (B < 0 || H < 0 || N < 0 || D <= 0 || m <= 0) return LA_ERR_INVALID_ARG;
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (dt != LA_BF16 || (D != 64 && D != 128) || (m != 64 && m != 128))
        return LA_ERR_UNSUPPORTED;
    la_status s = check_sizes(B, H, N, D);
    return s != LA_OK ? s : check_sizes(B, H, N, m);
}


}  // namespace

la_status la_favor_features(const void* x, const void* omega, void* phi, int64_t B, int64_t H,
                            int64_t N, int64_t D, int64_t m, la_dtype dt, la_stream_t stream) {
    la_status s;
    if ((s = check_favor(B, H, N, D, m, dt)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0 || N == 0) return LA_OK;
    if ((s = check_ptr(x)) || (s = check_ptr(omega)) || (s = check_ptr(phi))) return s;
    if ((s = bind_context()) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return launch_favor_dm<false>(D, m, x, omega, nullptr, phi, heads, N, st);
}

la_status la_favor_features_backward(const void* x, const void* omega, const void* dphi,
                                     void* dx, int64_t B, int64_t H, int64_t N, int64_t D,
                                     int64_t m, la_dtype dt, la_stream_t stream) {
    la_status s;
    if ((s = check_favor(B, H, N, D, m, dt)) != LA_OK) return s;
    const int64_t heads = B * H;
    if (heads == 0 || N == 0) return LA_OK;
    if ((s = check_ptr(x)) || (s = check_ptr(omega)) || (s = check_ptr(dphi)) ||
        (s = check_ptr(dx)))
        return s;
    if ((s = bind_context()) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return launch_favor_dm<true>(D, m, x, omega, dphi, dx, heads, N, st);
}

uint64_t la_launch_count(void) { return la::profiler().launches.load(); }

void la_profile_enable(int on) { la::profiler().on.store(on != 0); }

int la_profile_collect(la_profile_entry* out, int max_entries) {
    la::Profiler& p = la::profiler();
    std::lock_guard<std::mutex> g(p.mu);
    struct Agg {
        const char* name;
        int64_t n;
        double ms;
    };
    std::vector<Agg> agg;
    for (auto& r : p.records) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.stop) == cudaSuccess &&
            cudaEventElapsedTime(&ms, r.start, r.stop) == cudaSuccess) {
            bool found = false;
            for (auto& a : agg)
                if (strcmp(a.name, r.name) == 0) {
                    a.n += 1;
                    a.ms += ms;
                    found = true;
                    break;
                }
            if (!found) agg.push_back({r.name, 1, double(ms)});
        }
        p.pool.push_back(r.start);
        p.pool.push_back(r.stop);
    }
    p.records.clear();
    for (int i = 0; i < int(agg.size()) && i < max_entries && out; ++i) {
        memset(out[i].name, 0, sizeof(out[i].name));
        strncpy(out[i].name, agg[i].name, sizeof(out[i].name) - 1);
        out[i].launches = agg[i].n;
        out[i].total_ms = agg[i].ms;
    }
    return int(agg.size());
}

la_status la_selftest_wait_timeout(int nthreads, la_stream_t stream) {
    if (nthreads < 1 || nthreads > 1024) return LA_ERR_INVALID_ARG;
    la_status s;
    if ((s = bind_context()) != LA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    la::LaunchScope scope("wait_timeout_selftest", st);
    la::wait_timeout_selftest_kernel<<<1, unsigned(nthreads), 0, st>>>();
    return launch_status();
}

la_status la_get_device_error(la_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LA_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, la::g_device_error, sizeof(word)) != cudaSuccess)
        return LA_ERR_CUDA;
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(la::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
            return LA_ERR_CUDA;
        return LA_ERR_DEVICE_TIMEOUT;
    }
    return LA_OK;
}

}  // extern "C"
