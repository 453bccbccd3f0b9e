// Shared device helpers for the sm_100a kernels: error words, mbarriers with
// bounded waits, TMA / bulk copies, tcgen05 (TMEM alloc, MMA, commit, loads)
// and programmatic-dependent-launch controls. Inline PTX only; no library code.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

#define MOE_DEV __device__ __forceinline__

namespace moe {

// ---------------------------------------------------------------- error word
// The first 256 bytes of every workspace: word 0 = status code of the first
// device-detected error, word 1 = detail (an index or a wait-site id).
struct DevError {
    int code;
    int detail;
};
constexpr size_t kErrBytes = 256;

MOE_DEV void report_error(DevError* e, int code, int detail) {
    if (e && atomicCAS(&e->code, 0, code) == 0) atomicExch(&e->detail, detail);
}

// Default upper bound for any single wait, in SM clock cycles (~1 s at 2 GHz). Pipeline
// waits take the launch's own limit (GemmArgs::wait_limit, this by default); the waits that
// let copies and MMAs in flight finish after an abort always take this one.
constexpr long long kWaitLimitCycles = 2000000000LL;

// ---------------------------------------------------------------- PDL
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MOE_DEV void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- smem addr
MOE_DEV uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
MOE_DEV void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
MOE_DEV void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
MOE_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
MOE_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
MOE_DEV bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits until the phase with the given parity has completed. Gives up after `limit`
// cycles or when *abort becomes non-zero; returns false then.
MOE_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, long long limit = kWaitLimitCycles) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(a, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit) return false;
    }
}

// ---------------------------------------------------------------- fences
MOE_DEV void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
MOE_DEV void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
MOE_DEV void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
MOE_DEV void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}
// The same two loads with an L2 cache policy (a createpolicy value; see l2_policy).
MOE_DEV void tma_load_2d_hint(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
MOE_DEV void tma_load_3d_hint(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y, int z, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
// L2 cache policies: 0 = none (plain loads), 1 = evict first (data read once), 2 = evict last
// (data many CTAs re-read). Returns 0 for "none", which no createpolicy value equals.
MOE_DEV uint64_t l2_policy(int kind) {
    uint64_t p = 0;
    if (kind == 1) asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, %1;" : "=l"(p) : "f"(1.0f));
    else if (kind == 2) asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, %1;" : "=l"(p) : "f"(1.0f));
    return p;
}
MOE_DEV void tma_load_2d_p(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y, uint64_t pol) {
    if (pol) tma_load_2d_hint(dst, m, bar, x, y, pol);
    else tma_load_2d(dst, m, bar, x, y);
}
MOE_DEV void tma_load_3d_p(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y, int z, uint64_t pol) {
    if (pol) tma_load_3d_hint(dst, m, bar, x, y, z, pol);
    else tma_load_3d(dst, m, bar, x, y, z);
}
// Untiled bulk copy global -> shared; both addresses 16-byte aligned, bytes % 16 == 0.
MOE_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
MOE_DEV void bulk_load_p(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
    if (pol)
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
                smem_u32(dst)),
            "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
            : "memory");
    else
        bulk_load(dst, src, bytes, bar);
}

// 16 bytes global -> shared through L2 (cp.async, LSU path); src_bytes < 16 zero-fills the rest.
MOE_DEV void cp_async16(uint32_t dst_smem, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src), "r"(src_bytes)
                 : "memory");
}
// The same with an L2 cache policy (from l2_policy; 0 = none).
MOE_DEV void cp_async16_p(uint32_t dst_smem, const void* src, uint32_t src_bytes, uint64_t pol) {
    if (pol)
        asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst_smem), "l"(src),
                     "r"(src_bytes), "l"(pol)
                     : "memory");
    else
        cp_async16(dst_smem, src, src_bytes);
}
// Arrive on an mbarrier (counted in its expected arrivals) once this thread's cp.asyncs land.
MOE_DEV void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// ---------------------------------------------------------------- tcgen05
MOE_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
MOE_DEV void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
MOE_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
MOE_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 or f16 inputs, fp32 accumulate).
MOE_DEV void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Same, with A read from tensor memory: a_tmem addresses row 0 (lane 0) of a 128-row
// operand whose row m sits in lane m, two 16-bit values per 32-bit column along K.
MOE_DEV void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on an mbarrier once every previously issued tcgen05.mma of this thread completes.
MOE_DEV void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored with the 128-byte
// swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart. Bits: start address
// >>4 [0,14), leading offset >>4 [16,30) (unused for this layout), stride offset
// >>4 [32,46), version 1 [46,48), layout 2 = SWIZZLE_128B [61,64).
MOE_DEV uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, both operands K-major.
// in_fmt: 0 = f16, 1 = bf16. M = 128 rows of A, N = columns of B.
__host__ __device__ constexpr uint32_t idesc_f16(int in_fmt, int M, int N) {
    return (1u << 4) | ((uint32_t)in_fmt << 7) | ((uint32_t)in_fmt << 10) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- block-scaled FP4 MMA
// D[tmem] (+)= (A * SFA) * (B * SFB)^T with A, B packed e2m1 (two values per byte, the
// even K index in the low nibble) in K-major 128-byte-swizzled smem, one fp8-e4m3
// scale per 16 K values for every row of A and of B, read from tensor memory; fp32
// accumulate; K = 64 per instruction (32 bytes of each row).
MOE_DEV void mma_nvf4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// Instruction descriptor of that MMA: A and B e2m1 (format 1 at bits [7,10) and
// [10,13)), N >> 3 at [17,23), scale format 0 = ue4m3 at bit 23, M >> 4 at [24,29),
// scale-factor ids 0, dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// D[tmem] (+)= (A * SFA) * (B * SFB)^T with A e2m1 held one value per byte in smem (the
// 4-bit tensor map's 16-byte-aligned form), B e4m3, one e8m0 scale per 32 K values for
// every row of A and of B; K = 32 per instruction. The scale of this instruction is byte
// `id` of the 32-bit TMEM word at sfa/sfb; the id goes in the descriptor and in bits
// 30-31 of both scale addresses.
MOE_DEV void mma_mx8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                        uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// Its instruction descriptor: B scale id at [4,6), A e2m1 (5) at [7,10), B e4m3 (0) at
// [10,13), N >> 3 at [17,23), scale format 1 = ue8m0 at bit 23, M >> 4 at [24,29),
// A scale id at [29,31), dense K = 32.
__host__ __device__ constexpr uint32_t idesc_mx8(int M, int N, uint32_t id) {
    return (id << 4) | (5u << 7) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24) |
           (id << 29);
}
// Copies 32 rows x 16 bytes of shared memory (rows 16 bytes apart) into tensor-memory
// lanes 0..31, columns taddr..taddr+3 (bytes 4c..4c+3 of a row in column c), and the
// same data into the other three lane quarters. Ordered with the MMAs this thread issues.
MOE_DEV void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t src_desc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc) : "memory");
}
// Shared-memory descriptor of a scale-factor block for that copy: no swizzle, 8-row
// core matrices of 16-byte rows, consecutive 8-row groups 128 bytes apart.
MOE_DEV uint64_t sf_block_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
    d |= (uint64_t)(128 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// 32 lanes x 32-bit, 16 consecutive columns per thread.
MOE_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
MOE_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32-bit stores: 32 (x32) or 16 (x16) consecutive columns per thread.
MOE_DEV void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0],"
        " {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
MOE_DEV void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
        " {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
MOE_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- CTA pairs (cta_group::2)
// A cluster of two CTAs on two SMs runs one MMA stream: the CTA of rank 0 (the leader) issues
// tcgen05.mma.cta_group::2, whose A operand is 128 rows from each CTA's shared memory, whose B
// operand is N/2 rows from each, and whose accumulator is 128 rows x N columns in each CTA's
// tensor memory (its own A rows). Both CTAs allocate tensor memory together; every tcgen05
// instruction of such a kernel takes cta_group::2.
MOE_DEV uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of both CTAs: release what this thread wrote, wait for all, acquire.
MOE_DEV void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// The address of the same shared-memory location in the CTA of cluster rank `rank`.
MOE_DEV uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// Arrive on an mbarrier given by its cluster address (mapa), with cluster-scope release.
MOE_DEV void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
MOE_DEV bool mbar_try_wait_cluster(uint32_t bar_addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return ok != 0;
}
// mbar_wait for a barrier that the other CTA of the pair arrives on (cluster-scope acquire).
MOE_DEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort, long long limit) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_cluster(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_cluster(a, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit) return false;
    }
}
// TMA loads of a CTA pair: the destination is this CTA's shared memory, the mbarrier may be
// in either CTA of the pair (a cluster address, e.g. the leader's from mapa).
MOE_DEV void tma_load_2d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
MOE_DEV void tma_load_3d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(bar_cluster)
        : "memory");
}

// Tensor memory of the pair: the same warp of both CTAs, the same destination slot.
MOE_DEV void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
MOE_DEV void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
MOE_DEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A * B^T over the pair (M = 256: 128 rows of A per CTA; B: N/2 rows per CTA).
MOE_DEV void mma_f16_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on the mbarrier at this offset in each CTA of `mask` when the pair MMAs this
// thread issued so far complete.
MOE_DEV void mma_commit_pair(uint64_t* bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(mask)
        : "memory");
}

// ---------------------------------------------------------------- e4m3 / MX staging
// fp32 -> e4m3 (round to nearest even, saturating at +-448) and back.
MOE_DEV uint8_t cvt_e4m3(float x) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return (uint8_t)(r & 0xFF);
}
MOE_DEV float e4m3_to_f32(uint8_t c) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)c));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}
// Exponent e of the e8m0 scale 2^e of a 32-value block with largest magnitude amax, for the
// MXFP4 GEMM's activations: two terms (hi/lo staging of bf16): the smallest e with
// amax <= 448 * 2^e; one term (MXFP8, the OCP MX v1.0 rule): floor(log2 amax) - 8. A zero
// block takes -127. Clamped to e8m0's [-127, 127].
MOE_DEV int mx8_block_exp(float amax, bool two) {
    if (!(amax > 0.0f)) return -127;
    int ex;
    const float m = frexpf(amax, &ex);  // amax = m * 2^ex, m in [0.5, 1)
    // hi/lo: 448 * 2^(ex-9) = 0.875 * 2^ex; one term: floor(log2 amax) - 8 = ex - 9
    const int e = (two && m > 0.875f) ? ex - 8 : ex - 9;
    return max(-127, min(127, e));
}
// 2^-e as a normal float for the e of mx8_block_exp (finite inputs give e <= 120).
MOE_DEV float mx8_inv_scale(int e) {
    return __int_as_float((127 - max(e, -126)) << 23) * (e < -126 ? 2.0f : 1.0f);
}

// ---------------------------------------------------------------- misc
MOE_DEV int warp_id() { return threadIdx.x >> 5; }
MOE_DEV int lane_id() { return threadIdx.x & 31; }

MOE_DEV float silu_f(float g) { return g / (1.0f + expf(-g)); }

MOE_DEV float act_apply(int act, float g, float u, float a, float b) {
    if (act == MOE_ACT_SITU) {
        const float sig = 1.0f / (1.0f + expf(-g));
        return a * tanhf(g / a) * sig * (b * tanhf(u / b));
    }
    return silu_f(g) * u;
}

// The same activations for the GEMM epilogue, from the exponential intrinsic and
// approximate division (relative error ~1e-6, far below the 16-bit output rounding):
// sigmoid(x) = 1/(1+e^-x), tanh(y) = 1 - 2/(1+e^(2y)) (exact limits +-1 as e^(2y) -> inf / 0).
MOE_DEV float fast_sigmoid(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
MOE_DEV float fast_tanh(float y) { return 1.0f - __fdividef(2.0f, 1.0f + __expf(2.0f * y)); }
MOE_DEV float act_apply_fast(int act, float g, float u, float a, float b, float inv_a, float inv_b) {
    if (act == MOE_ACT_SITU) return a * fast_tanh(g * inv_a) * fast_sigmoid(g) * (b * fast_tanh(u * inv_b));
    return g * fast_sigmoid(g) * u;
}
// SWIGLUOAI (the GPT-OSS gated activation): g = min(gate, lim), u = clamp(up, -lim, lim),
// g * sigmoid(alpha * g) * (u + beta); lim = +inf is no clamp.
MOE_DEV float swigluoai_fast(float g, float u, float alpha, float beta, float lim) {
    const float gc = fminf(g, lim);
    const float uc = fminf(fmaxf(u, -lim), lim);
    return gc * fast_sigmoid(alpha * gc) * (uc + beta);
}

}  // namespace moe
