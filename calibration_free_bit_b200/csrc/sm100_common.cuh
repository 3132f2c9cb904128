// sm100_common.cuh -- small sm_100a building blocks shared by liboq's GEMM kernels:
// shared-memory addressing, bounded mbarrier waits, TMA tile loads and stores, tcgen05
// descriptors, MMA issue/commit, TMEM loads and stores, the output epilogue chunk.  Inline PTX;
// every tile load writes only the issuing CTA's shared memory.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cstdint>

namespace oq {

// Host side (k2_linear.cu): the driver's tensor-map encoder, looked up once through the
// runtime (nullptr if unavailable), and the output map of y [T, N] row-major with 128-byte
// swizzle: fp32 in 32 x 32 boxes (the layout store_chunk writes) or bf16 in 32-row x
// 64-column boxes (store_chunk_bf16).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
bool make_out_map(CUtensorMap *map, void *y, int T, int N, bool bf16);

namespace sm100 {

// A bounded wait gives up after this many SM clock cycles (about 2 s at the B200's 1.9 GHz
// boost clock, longer at lower clocks).
constexpr long long kWaitLimitCycles = 4000000000ll;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// A waiting thread may sleep in try_wait up to this long (it wakes when the phase completes),
// so warps parked on a barrier do not take issue slots from the warps doing the work.
constexpr unsigned kSuspendHintNs = 200000;

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done) : "r"(bar), "r"(parity), "n"(kSuspendHintNs) : "memory");
    return done != 0;
}

// Wait for the phase with the given parity to complete; false after `limit` SM cycles
// (kWaitLimitCycles by default).  The first test costs no clock read (most waits in a running
// pipeline are already satisfied).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          long long limit = kWaitLimitCycles) {
    if (mbar_try(bar, parity))
        return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try(bar, parity))
            return true;
        if (clock64() - t0 > limit)
            return false;
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// K-major operand in the canonical 128-byte-swizzled layout (8-row atoms of 1024 bytes).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu)     // start address
           | ((uint64_t)1 << 16)                  // leading byte offset (unused for SW128 K)
           | ((uint64_t)(1024 >> 4) << 32)        // stride byte offset: next 8-row atom
           | ((uint64_t)1 << 46)                  // descriptor version (sm_100)
           | ((uint64_t)2 << 61);                 // swizzle mode: 128B
}

// Instruction descriptor, kind::f16: A = B = fp16, K-major; D = fp32; shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
    return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T
__device__ __forceinline__ void mma_ss(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(tmem_d), "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// 32 consecutive TMEM columns of this thread's lane -> registers (warp-collective).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// registers -> 32 consecutive TMEM columns of this thread's lane (warp-collective); the
// caller waits with tmem_st_wait() before signalling the consumer.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
          "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
          "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// registers -> 16 consecutive TMEM columns of this thread's lane (warp-collective).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- TMA tensor stores (shared -> global), bulk-group completion ----
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// At most N of this thread's committed bulk groups may still be reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// All of this thread's committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Epilogue chunk: this warp's 32 accumulator rows (acc = this thread's row) x 32 columns,
// scaled by srow * rn32[j], written to global memory by one TMA tensor store at (x, y) from
// `stage` (4 KB, 1024-byte aligned; 128-byte swizzle: 16-byte piece k of row r sits at piece
// k ^ (r % 8), so the eight v4 stores of a warp hit all 32 banks).  rn32: 32 floats in shared
// memory.  The caller guarantees that no earlier store still reads `stage`; lane 0 issues and
// commits the store as one bulk group.
__device__ __forceinline__ void store_chunk(const CUtensorMap *map, unsigned char *stage_ptr,
                                            uint32_t stage, const uint32_t (&acc)[32],
                                            float srow, const float *rn32, int lane, int x,
                                            int y) {
    float4 *rowp = reinterpret_cast<float4 *>(stage_ptr + lane * 128);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float4 rn4 = reinterpret_cast<const float4 *>(rn32)[k];
        float4 o;
        o.x = __uint_as_float(acc[4 * k + 0]) * srow * rn4.x;
        o.y = __uint_as_float(acc[4 * k + 1]) * srow * rn4.y;
        o.z = __uint_as_float(acc[4 * k + 2]) * srow * rn4.z;
        o.w = __uint_as_float(acc[4 * k + 3]) * srow * rn4.w;
        rowp[k ^ (lane & 7)] = o;
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(map, stage, x, y);
        bulk_commit();
    }
}

// bf16 variant: 32 rows x 64 columns (two 32-column accumulator loads acc0, acc1), each
// value scaled by srow * rn64[j] in fp32 and rounded to nearest-even bf16; same staging
// layout (a row is 64 bf16 = 128 bytes) and issue rules as store_chunk.
__device__ __forceinline__ void store_chunk_bf16(const CUtensorMap *map, unsigned char *stage_ptr,
                                                 uint32_t stage, const uint32_t (&acc0)[32],
                                                 const uint32_t (&acc1)[32], float srow,
                                                 const float *rn64, int lane, int x, int y) {
    uint4 *rowp = reinterpret_cast<uint4 *>(stage_ptr + lane * 128);
#pragma unroll
    for (int k = 0; k < 8; ++k) {                       // 16-byte piece k = columns 8k .. 8k+7
        const float4 ra = reinterpret_cast<const float4 *>(rn64)[2 * k];
        const float4 rb = reinterpret_cast<const float4 *>(rn64)[2 * k + 1];
        const uint32_t *a = (k < 4) ? &acc0[8 * k] : &acc1[8 * (k - 4)];
        auto pk = [&](uint32_t u0, float r0, uint32_t u1, float r1) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(u0) * srow * r0,
                                                          __uint_as_float(u1) * srow * r1);
            return *reinterpret_cast<const uint32_t *>(&h);
        };
        uint4 o;
        o.x = pk(a[0], ra.x, a[1], ra.y);
        o.y = pk(a[2], ra.z, a[3], ra.w);
        o.z = pk(a[4], rb.x, a[5], rb.y);
        o.w = pk(a[6], rb.z, a[7], rb.w);
        rowp[k ^ (lane & 7)] = o;
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(map, stage, x, y);
        bulk_commit();
    }
}

// ---- CTA pairs (cluster of 2, tcgen05 .cta_group::2) ----
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// The shared::cluster address of the variable at shared::cta address `addr` in CTA `rank` of
// this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Every thread of both CTAs: arrive (release) and wait (acquire) on the cluster barrier.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (possibly the peer CTA's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
                 ::"r"(cluster_bar) : "memory");
}

// The same arrive with the instruction's default semantics (release at CTA scope): for a
// producer whose data the peer's tensor core reads through the async proxy, after
// fence.proxy.async has ordered the data writes before it.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// Pair TMA load: this CTA's tile lands in its own shared memory; the transaction bytes count
// on the mbarrier at `cluster_bar` (the leader CTA's); the data lands in this CTA only.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x,
                                                 int y, uint32_t cluster_bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(cluster_bar)
        : "memory");
}

// Pair MMA, issued by the leader CTA: D[tmem] (+)= A * B^T with A split by rows (M) and B by
// rows (N) across the two CTAs' shared memory at the same offsets; each CTA's tensor memory
// receives its own M/2 rows of D.
__device__ __forceinline__ void mma_ss_pair(uint32_t tmem_d, uint64_t da, uint64_t db,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
        : "memory");
}

// When the pair's MMAs issued so far complete, arrive once on the mbarrier at this shared
// offset in every CTA of `cta_mask`.
__device__ __forceinline__ void mma_commit_pair_mc(uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar), "h"(cta_mask) : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

}  // namespace sm100
}  // namespace oq
