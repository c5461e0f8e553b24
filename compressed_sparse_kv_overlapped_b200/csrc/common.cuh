// common.cuh -- shared device helpers of the CSA/HCA library (sm_100a only).
//
// Thin inline-PTX wrappers for mbarriers, cp.async, tcgen05 (TMEM allocation, UMMA issue and
// commit, TMEM loads/stores) and the shared-memory matrix descriptors that tcgen05.mma reads,
// plus the device status word through which kernels report bad indices and wait timeouts
// without trapping.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/csa.h"

namespace csa {

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------------------------------------
// Device status word: the first error recorded wins; read and cleared by csa_sync_status().
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void report(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Wall-clock limit of every spin wait (nanoseconds).  A wait that runs out records
// CSA_ERR_TIMEOUT and returns false; the kernel then winds down without touching more data.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One test of the phase (the hardware may briefly suspend the thread; no explicit time hint, since a
// long hint was measured to delay the wake-up after the phase completes by about a microsecond).
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns false (and records a
// timeout) if it does not complete within `limit_ns` (kWaitLimitNs unless a kernel was given a
// shorter limit), or if *abort becomes non-zero.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0u) {
            if (abort && *abort) return false;
            if (globaltimer() - t0 > limit_ns) {
                report(status, CSA_ERR_TIMEOUT);
                if (abort) *abort = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Bulk copy (no tensor map) of `bytes` (a multiple of 16, both addresses 16-byte aligned) from
// global memory into this CTA's shared memory; completes `bytes` of transaction count on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst_smem),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Barrier of every thread of every CTA in the thread-block cluster; orders all earlier memory
// accesses (shared, distributed shared and global) before all later ones at cluster scope.
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Distributed shared memory of the thread-block cluster: this CTA's rank, and loads of the word /
// 16 bytes at the location `p` (an address in this CTA's shared memory) in the CTA of rank `rank`.
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// (not volatile: several of these loads may be in flight at once; they read data that a cluster
// barrier, which orders memory, made visible)
__device__ __forceinline__ float ld_cluster_f32(const void* p, uint32_t rank) {
    uint32_t a, v;
    asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    asm("ld.shared::cluster.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return __uint_as_float(v);
}
__device__ __forceinline__ float4 ld_cluster_f32x4(const void* p, uint32_t rank) {
    uint32_t a;
    float4 v;
    asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    asm("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}

// ---------------------------------------------------------------------------------------------
// cp.async (16-byte, L2-only); src_bytes = 0 writes zeros without reading.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// One more pending arrival on `bar`, resolved when every cp.async this thread has issued so far has
// completed; it does not count toward the expected arrivals, so the thread still arrives itself.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 16-byte store to shared memory (a shared-window address).
__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Make generic-proxy writes to shared memory visible to the async proxy (tensor-core reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------------------------
// Shared-memory layout of tcgen05 operands: 128-byte swizzle.  A tile is stored as "blocks" of
// R rows x 128 bytes (64 bf16); inside a block, row r lives at r*128 and its 16-byte chunk c at
// chunk position c ^ (r % 8).  Block bases are 1024-byte aligned.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// Shared-memory matrix descriptor (tcgen05 format): start address, leading/stride byte offsets,
// descriptor version 1, layout type 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// K-major operand: rows of 128 bytes, 8-row groups 1024 bytes apart (LBO unused -> 16 bytes).
__device__ __forceinline__ uint64_t sdesc_kmajor(uint32_t saddr) { return make_sdesc(saddr, 16u, 1024u); }

// MN-major operand: 64-element MN groups `mn_stride` bytes apart, 8-row K groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_mnmajor(uint32_t saddr, uint32_t mn_stride) {
    return make_sdesc(saddr, mn_stride, 1024u);
}

// Instruction descriptor of kind::f16 with bf16 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------------------------
// tcgen05
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// The tcgen05.mma / tcgen05.commit wrappers below are called by a whole converged warp with
// warp-uniform operands; elect.sync inside each instruction lets one lane (the lowest, so always the
// same one) issue it.  Keeping the issuing loop warp-uniform lets the compiler hold the operands in
// uniform registers: measured on this part, 32 M64 N64 products issued this way take about 1,000
// clocks against 2,600 when one lane runs the loop alone.

// D[tmem] (+)= A[smem desc] * B[smem desc].
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    const uint32_t zero = 0;  // disable-output-lane mask: every lane enabled
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b32 l;\n\t"
        "elect.sync l|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(zero)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]; A (K-major, 2 bf16 per 32-bit column) must sit in the same
// lanes as D.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b32 l;\n\t"
        "elect.sync l|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on the mbarrier when all previously issued tcgen05.mma of the issuing lane complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 l;\n\t"
        "elect.sync l|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 16 consecutive columns: thread i of the warp gets lane (base_lane + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// 16 lanes x 256 bits, 8 repetitions along the columns (64 columns).  Thread t of the warp gets,
// for repetition k, rows (base_lane + t/4) and (base_lane + t/4 + 8) at columns 8k + 2*(t%4) and
// 8k + 2*(t%4) + 1, in the order (row, col), (row, col+1), (row+8, col), (row+8, col+1).
__device__ __forceinline__ void tmem_ld_16x256_x8(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Store counterpart of tmem_ld_16x256_x8 (same thread / register layout).
__device__ __forceinline__ void tmem_st_16x256_x8(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Programmatic dependent launch: wait for the preceding grid in the stream (and its memory), and
// allow the next grid to start its prologue.  Both are no-ops for a normally launched grid.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// A flag word between two grids that run at the same time (a producer and the grid it launched
// early): the producer publishes with a release store after its results, the consumer polls with
// acquire loads, after which the producer's results are visible to it.
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Bounded wait for *word >= target, same contract as mbar_wait.  Polls with a short sleep between
// reads, so that many waiting warps leave the memory system to the grid they wait for.
__device__ __forceinline__ bool count_wait(const uint32_t* word, uint32_t target, int* status, volatile int* abort,
                                           uint64_t limit_ns = kWaitLimitNs) {
    if (ld_acquire_gpu(word) >= target) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(32);
        if (ld_acquire_gpu(word) >= target) return true;
        if ((it & 15u) == 0u) {
            if (abort && *abort) return false;
            if (globaltimer() - t0 > limit_ns) {
                report(status, CSA_ERR_TIMEOUT);
                if (abort) *abort = 1;
                return false;
            }
        }
    }
}

// 2^x with the hardware approximation (relative error about 2^-22; subnormal results flush to 0).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------------------------------------
// Small numeric helpers
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Eight bf16 values (one 16-byte vector) to fp32.
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
    f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
    f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// 8-bit block-scaled keys: the 8 bf16 channels `kb` one lane holds of a 32-channel block that four
// consecutive lanes of `mask` hold together -> 8 E4M3 bytes (the block's elements x / 2^e rounded to
// nearest even) and, in *scale_byte, e + 127, where 2^e is the smallest power of two with
// amax <= 448 * 2^e (amax = 0: e = -127).  All four lanes must call it.
__device__ __forceinline__ uint2 quant_mx8(const uint4& kb, unsigned mask, uint32_t* scale_byte) {
    float f[8];
    unpack8(kb, f);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(mask, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(mask, amax, 2));
    int e = -127;
    if (amax > 0.f) {
        int ex;
        frexpf(amax, &ex);  // amax in [2^(ex-1), 2^ex)
        e = ex - 9;
        while (amax > ldexpf(448.f, e)) ++e;
        while (e > -127 && amax <= ldexpf(448.f, e - 1)) --e;
    }
    *scale_byte = (uint32_t)(e + 127);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint16_t two;
        // the first operand goes to the high byte: element 2i + 1 high, 2i low
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(ldexpf(f[2 * i + 1], -e)), "f"(ldexpf(f[2 * i], -e)));
        w[i] = two;
    }
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// The 4-bit form for the FP4 entry cache: eight bf16 values (four lanes per 32-channel block, `mask`
// those lanes) to E2M1 codes (sign, two exponent bits with bias 1, one mantissa bit; the hardware
// conversion rounds to nearest, ties to even) with the block's scale 2^e, e the smallest integer
// such that amax <= 6 * 2^e (e >= -127).  Returns the eight codes, the even channel in the low nibble
// of each byte; *scale_byte = e + 127.
__device__ __forceinline__ uint32_t quant_mx4(const uint4& kb, unsigned mask, uint32_t* scale_byte) {
    float f[8];
    unpack8(kb, f);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(mask, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(mask, amax, 2));
    int e = -127;
    if (amax > 0.f) {
        int ex;
        frexpf(amax, &ex);  // amax in [2^(ex-1), 2^ex)
        e = ex - 3;
        while (amax > ldexpf(6.f, e)) ++e;
        while (e > -127 && amax <= ldexpf(6.f, e - 1)) --e;
    }
    *scale_byte = (uint32_t)(e + 127);
    uint32_t w = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t two;
        // the first operand goes to the high nibble: element 2i + 1 high, 2i low
        asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
            : "=r"(two) : "f"(ldexpf(f[2 * i + 1], -e)), "f"(ldexpf(f[2 * i], -e)));
        w |= (two & 0xFFu) << (8 * i);
    }
    return w;
}

// Eight E2M1 codes (a word, the even channel in the low nibble of each byte) with the block scale
// byte s to eight bf16 values: code value * 2^(s - 127), exact (two significant bits times a power of
// two; the product is formed in fp32, subnormals included).
__device__ __forceinline__ uint4 mx4_to_bf16x8(uint32_t w, uint32_t s) {
    const float f = s ? __uint_as_float(s << 23) : __uint_as_float(0x00400000u);  // 2^(s - 127)
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t h2;
        asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "r"((w >> (8 * i)) & 0xFFu));
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&h2));
        const __nv_bfloat162 b = __floats2bfloat162_rn(v.x * f, v.y * f);
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Order-preserving map of fp32 onto uint32 (larger float -> larger key; -0 < +0).
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

// Host side: run a set-up step (function attributes such as the dynamic shared-memory opt-in)
// once per device, with that device current.  Function attributes belong to a device, so a
// process that launches on several devices needs the step on each; concurrent first calls on one
// device are serialized, and a step that fails is retried by the next call.
class PerDeviceOnce {
   public:
    template <typename F>
    cudaError_t run(F&& step) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lock(mu_);
        if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        e = step();
        if (e == cudaSuccess) done_[dev].store(true, std::memory_order_release);
        return e;
    }

   private:
    static constexpr int kMaxDevices = 64;
    std::mutex mu_;
    std::atomic<bool> done_[kMaxDevices] = {};
};

// Launch `kernel` with an optional programmatic-dependent-launch attribute: the grid may start
// while the previous kernel in the stream finishes; it must call grid_dep_wait() before it reads
// anything that kernel writes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// The same with a thread-block cluster shape.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                         cudaStream_t stream, bool pdl, dim3 cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster.x;
    attr[0].val.clusterDim.y = cluster.y;
    attr[0].val.clusterDim.z = cluster.z;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace csa
