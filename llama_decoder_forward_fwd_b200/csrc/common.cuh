// Shared device helpers: PTX wrappers for sm_100a (mbarrier, TMA, tcgen05,
// mma.sync, ldmatrix, programmatic dependent launch) and small numeric helpers.
// Every spin on an mbarrier is bounded by wall time (%globaltimer); when it
// runs out the kernel records a code in the caller's device error word and
// the wait reports failure so the kernel can wind down instead of hanging.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "errors.cuh"

#define DEVI __device__ __forceinline__

namespace lfw {

// Bounds-checking build (-DLLM_BOUNDS_CHECK): LFW_CHECK(cond, err, site) records
// a failed index check in the error word (first one wins) and yields false, so
// the caller skips the access. In the normal build it is `true`, and the
// condition is not evaluated.
#ifdef LLM_BOUNDS_CHECK
#define LFW_CHECK(cond, err, site) ::lfw::bounds_check((cond), (err), (site))
#else
#define LFW_CHECK(cond, err, site) true
#endif

// 4 seconds: far longer than any legitimate wait for one pipeline stage.
constexpr uint64_t kWaitLimitNs = 4000000000ull;

DEVI bool bounds_check(bool ok, uint32_t* err, uint32_t site) {
    if (!ok && err) atomicCAS(err, 0u, (uint32_t)DERR_BOUNDS | site);
    return ok;
}

DEVI uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

DEVI uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- programmatic dependent launch ------------------------------------
// pdl_wait(): block until the preceding kernel in the stream has completed and
// its writes are visible. Every kernel calls it before touching activations.
DEVI void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// pdl_trigger(): allow the next kernel in the stream to start launching.
DEVI void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Barrier over the first `count` threads of the CTA (id 1..15; 0 is __syncthreads).
DEVI void named_bar_sync(int id, int count) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory"); }

// ---- mbarrier ---------------------------------------------------------
DEVI void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
DEVI void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
DEVI void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
DEVI void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
DEVI void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
DEVI bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase with the given parity to complete. Returns false
// (after recording `code` in *err) if it did not complete within limit_ns
// (kWaitLimitNs unless a caller asks for another bound).
DEVI bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err, uint32_t code, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) {
            if (err) atomicCAS(err, 0u, code);
            return false;
        }
    }
}

// Release increment: every write that happens before it (this thread's, and the
// writes of other threads ordered before it by a CTA or warp barrier) is visible
// to a thread that observes the new count with an acquire load. It orders only
// what a publish needs, unlike a full fence followed by an atomic.
DEVI void red_release_add(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Acquire-release increment returning the previous count: publishes this
// thread's earlier writes (and those ordered before it by a barrier) and, for the
// thread that sees the final count, makes every earlier publisher's writes
// visible to what follows it.
DEVI unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

DEVI unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier of a cooperative launch, entered by the first `nthreads`
// threads of every CTA (the CTA's other warps do not take part). Barrier number
// `index` (0, 1, 2, ...) of the launch waits until every CTA has arrived
// `index + 1` times (*count is zero at launch). Writes made before the barrier
// by any CTA are visible to every thread after it (CTA barrier, release
// arrival, acquire polling, CTA barrier). The wait is bounded: on timeout it records
// `code` in *err and returns false; it also returns false as soon as *err
// holds another CTA's error, so all CTAs leave promptly.
DEVI bool grid_barrier(unsigned* count, unsigned index, int nthreads, uint32_t* err, uint32_t code,
                       uint64_t limit_ns = kWaitLimitNs) {
    __shared__ int gb_ok;
    named_bar_sync(1, nthreads);
    if (threadIdx.x == 0) {
        red_release_add(count, 1u);
        const unsigned target = (index + 1) * gridDim.x;
        int ok = 1;
        if (ld_acquire_gpu(count) < target) {
            const uint64_t t0 = globaltimer();
            while (ld_acquire_gpu(count) < target) {
                __nanosleep(32);
                // leave at once if another CTA has already recorded an error
                if (*reinterpret_cast<volatile uint32_t*>(err) != 0u) {
                    ok = 0;
                    break;
                }
                if (globaltimer() - t0 > limit_ns) {
                    atomicCAS(err, 0u, code);
                    ok = 0;
                    break;
                }
            }
        }
        __threadfence();
        gb_ok = ok;
    }
    named_bar_sync(1, nthreads);
    return gb_ok != 0;
}

// ---- TMA --------------------------------------------------------------
DEVI void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 2-D tiled load of box at (x = inner element index, y = row) into shared memory,
// completing `bytes` of transaction on bar. x * element size must be a multiple
// of 16 bytes (callers only pass multiples of 64 bf16 elements).
DEVI void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// ---- tcgen05 (5th-generation tensor cores, accumulators in TMEM) ------
DEVI void tc_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
DEVI void tc_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
DEVI void tc_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
DEVI void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
DEVI void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Arrive once on bar when every tcgen05.mma issued so far by this thread has completed.
DEVI void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
DEVI void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
DEVI void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Each thread of the warp reads 32 consecutive 32-bit columns of its own TMEM lane.
DEVI void tc_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

DEVI void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Each thread of the warp writes 32 consecutive 32-bit columns of its own TMEM lane.
DEVI void tc_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored as rows of
// 128 bytes (64 bf16) with the 128-byte swizzle TMA produces: 8-row groups are
// 1024 bytes apart (stride byte offset), version 1, layout SWIZZLE_128B.
DEVI uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);          // start address
    d |= (uint64_t)(16 >> 4) << 16;                  // leading byte offset (unused here)
    d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset
    d |= (uint64_t)1 << 46;                          // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                          // SWIZZLE_128B
    return d;
}
// Descriptor for an MN-major operand (the N index contiguous) stored as blocks of
// [K rows][64 bf16] with the 128-byte swizzle: K rows 128 bytes apart, 8-row
// groups 1024 bytes apart (stride byte offset), the next 64-wide block of N
// `mn_block_bytes` further on (leading byte offset).
DEVI uint64_t smem_desc_sw128_mn(uint32_t saddr, uint32_t mn_block_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((mn_block_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// Instruction descriptor, kind::f16: fp32 D, bf16 A and B, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// The same with B MN-major (bit 16: B transposed).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) { return idesc_bf16_f32(M, N) | (1u << 16); }

// ---- legacy warp-level tensor core path (decode GEMV, flash attention) ----
DEVI void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
DEVI void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
DEVI void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// ---- numeric helpers --------------------------------------------------
DEVI float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
DEVI float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
DEVI uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
DEVI float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
DEVI float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
DEVI float silu(float z) { return z / (1.0f + __expf(-z)); }

template <typename T> DEVI float to_f(T v);
template <> DEVI float to_f<float>(float v) { return v; }
template <> DEVI float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> DEVI T from_f(float v);
template <> DEVI float from_f<float>(float v) { return v; }
template <> DEVI __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

}  // namespace lfw
