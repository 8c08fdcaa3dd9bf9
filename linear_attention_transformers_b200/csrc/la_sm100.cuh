// la_sm100.cuh — thin wrappers over the sm_100a instructions the chunked
// kernels use: mbarriers (with bounded waits), TMA tensor copies, the
// tcgen05 tensor-core MMA with TMEM accumulators, and the shared-memory
// matrix / instruction descriptors those MMAs read.
//
// Conventions used by every kernel in this library:
//  * A "row tile" is a bf16 matrix R[rows][cols] in shared memory stored as
//    cols/64 "atoms" of [rows][64] (128 bytes per row), atom a at byte
//    a*rows*128, with the 128-byte swizzle: the 16-byte chunk j of row r sits
//    at position j ^ (r % 8).  This is exactly what a TMA load with
//    CU_TENSOR_MAP_SWIZZLE_128B and a 64-column box writes, and atoms start on
//    1024-byte boundaries.
//  * Used as a K-major MMA operand (rows = M or N, cols = K) the descriptor
//    starts at atom k/64, byte 32*((k%64)/16) of the row, SBO = 1024.
//  * Used as an MN-major operand (rows = K, cols = M or N) the descriptor
//    starts at row k (byte 128*k), LBO = rows*128 (next 64 columns),
//    SBO = 1024 (next 8 rows).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "la_common.cuh"

namespace la {
namespace sm100 {

// Give up a wait after this long; the kernel then records an error and
// finishes instead of hanging.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
// One try_wait without a suspend-time hint: returns at once when the phase
// has completed (about 14 cycles on B200; with a hint it costs ~46), else
// after the hardware's own short suspension.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Slow path of mbar_wait: keeps trying until the phase completes, gives up
// after kWaitLimitNs (or at once if another thread of the block already gave
// up), records the failure in g_device_error and in *abort, returns false.
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort) {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 7u) == 0) {
            if (*abort) return false;
            if (global_ns() - t0 > kWaitLimitNs) {
                *abort = 1;
                atomicOr(&g_device_error, 1u);
                return false;
            }
        }
    }
}

// Wait for phase `parity` of `bar` to complete (bounded, see mbar_wait_slow).
// The completed case stays inline: a call costs ~150 cycles on this path.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, abort);
}

// Wait used on the way out of a kernel (drains copies / MMAs in flight): it
// ignores the abort flag but still gives up after kWaitLimitNs.
__device__ __noinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 7u) == 7u && global_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_device_error, 1u);
            return false;
        }
    }
}

// Wait of a whole thread group (a named barrier `id` of `nthreads`) for a
// phase: only `leader` polls the mbarrier; the others park on the named
// barrier (parked warps issue nothing, so the group's wait does not take
// issue slots from the warps that are working), then every thread takes the
// completed phase with one try_wait (its acquire).  Returns false for every
// thread when the leader's wait gave up.
__device__ __forceinline__ bool group_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                           int id, int nthreads, bool leader);

// ----------------------------------------------------------------- proxies
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also ANDs a predicate over the participating threads,
// so a group leaves a loop together when any member's wait gave up.
__device__ __forceinline__ bool named_bar_all(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(uint32_t(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ bool group_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                           int id, int nthreads, bool leader) {
    bool ok = true;
    if (leader) ok = mbar_wait(bar, parity, abort);
    ok = named_bar_all(id, nthreads, ok);
    if (ok) (void)mbar_try_wait(bar, parity);
    return ok;
}

// --------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// 3-D tiled load into this CTA's shared memory; completes a transaction on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::
                     "l"(map),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05
// TMEM addresses: bits 31..16 lane, bits 15..0 column.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]: A is K-major in TMEM, row m in lane m,
// bf16 pairs (k even in the low half) one per 32-bit column, so the K-step at
// element k starts at column a_tmem + k/2.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns: thread t of the warp receives
// lane (warp's sub-partition base + t), columns col..col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// --------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;  // descriptor version for sm_100
    d |= uint64_t(2) << 61;  // SWIZZLE_128B
    return d;
}

// Row tile used as a K-major operand: k-step at element k (multiple of 16).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int rows, int k) {
    const uint32_t addr = tile + uint32_t(k / 64) * uint32_t(rows) * 128u + uint32_t(k % 64) * 2u;
    return sdesc_sw128(addr, 16, 1024);
}
// Row tile used as an MN-major operand (rows = K): k-step at row k.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int rows, int k) {
    return sdesc_sw128(tile + uint32_t(k) * 128u, uint32_t(rows) * 128u, 1024);
}

// Base descriptors (k = 0) and the constant offsets that step them along K:
// adding kstep_*() to a base descriptor moves its start address field.
__device__ __forceinline__ uint64_t desc_k_base(uint32_t tile) { return sdesc_sw128(tile, 16, 1024); }
__device__ __forceinline__ uint64_t desc_mn_base(uint32_t tile, int rows) {
    return sdesc_sw128(tile, uint32_t(rows) * 128u, 1024);
}
__host__ __device__ constexpr uint64_t kstep_k(int rows, int k) {
    return uint64_t(((k / 64) * rows * 128 + (k % 64) * 2) >> 4);
}
__host__ __device__ constexpr uint64_t kstep_mn(int k) { return uint64_t((k * 128) >> 4); }

// Instruction descriptor: kind::f16 with bf16 A/B, fp32 D, dense.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn_major) << 15) |
           (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Byte offset of element (r, c) of a bf16 row tile with `rows` rows.
__device__ __forceinline__ uint32_t tile_off(int rows, int r, int c) {
    const int atom = c >> 6, cc = c & 63;
    const int chunk = (cc >> 3) ^ (r & 7);
    return uint32_t(atom) * uint32_t(rows) * 128u + uint32_t(r) * 128u + uint32_t(chunk) * 16u +
           uint32_t(cc & 7) * 2u;
}
// Byte offset of the 16-byte chunk holding columns 8q..8q+7 of row r.
__device__ __forceinline__ uint32_t tile_chunk_off(int rows, int r, int q) {
    const int atom = q >> 3;
    const int chunk = (q & 7) ^ (r & 7);
    return uint32_t(atom) * uint32_t(rows) * 128u + uint32_t(r) * 128u + uint32_t(chunk) * 16u;
}

// Accumulator row -> (sub-partition, lane) for an M-row cta_group::1 MMA:
// M = 128 uses every lane; M = 64 uses lanes 0-15 of each sub-partition.
template <int M>
__device__ __forceinline__ int acc_row(int subpart, int lane) {
    if (M == 128) return 32 * subpart + lane;
    return lane < 16 ? 16 * subpart + lane : -1;
}

// bf16 packing helpers
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(h);
}

}  // namespace sm100

// One block whose threads wait on an mbarrier that nothing arrives at (the
// bounded wait of the chunked kernels gives up, records the error and the
// kernel returns).
__global__ void wait_timeout_selftest_kernel() {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    (void)sm100::mbar_wait(&bar, 0, &abort_flag);
    __syncthreads();
}

}  // namespace la
