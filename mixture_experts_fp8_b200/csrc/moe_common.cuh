// moe_common.cuh -- device helpers shared by the kernels of libmoefp8.so (sm_100a only):
// launch/status plumbing, warp reductions, E4M3 / UE8M0 conversion, mbarrier, TMA and
// tcgen05 (5th-generation tensor core + tensor memory) wrappers written as inline PTX.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moefp8.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libmoefp8 targets sm_100a (B200) only"
#endif

namespace moe {

// Bounded waits: a wait that has not finished after this long gives up, records
// MOE_ERR_TIMEOUT in the status word and lets the kernel leave (no trap, no hang).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Debug builds (MOE_FAULT_INJECTION): true for the one producer step that an armed
// MOE_FAULT_SKIP_STAGE drops (CTA 0, first K stage).  Compiled out of the release library.
__device__ __forceinline__ bool fault_skip_stage(int fault, uint32_t it) {
#ifdef MOE_FAULT_INJECTION
    return fault == MOE_FAULT_SKIP_STAGE && blockIdx.x == 0 && it == 0;
#else
    (void)fault;
    (void)it;
    return false;
#endif
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
    if (status) atomicCAS(reinterpret_cast<int*>(status), MOE_OK, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Loads from a 32-bit shared-memory address (the data is written by the async proxy and made
// visible by an mbarrier wait, so the loads must not be hoisted above it: volatile + memory).
__device__ __forceinline__ float ld_shared_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float4 ld_shared_f32x4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a)
                 : "memory");
    return v;
}

// ------------------------------------------------------------------------------ warp helpers
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ------------------------------------------------------------------------------ FP8 codes
// E4M3 (OCP "fn" variant): round to nearest even, saturating to +-448.  Two values per
// instruction; `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}"
        : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    return e4m3x2(a, b) | (e4m3x2(c, d) << 16);
}

// Smallest e with amax <= 448 * 2^e, from the fp32 bits of amax (exact); 0 for amax == 0.
// amax = m * 2^E with m in [1,2): e = E - 8, plus one when m > 1.75.  Clamped to [-127, 127].
__device__ __forceinline__ int mx_exponent(float amax) {
    if (!(amax > 0.0f)) return 0;
    uint32_t b = __float_as_uint(amax);
    int biased = (b >> 23) & 0xFF;
    int e;
    if (biased == 0) {
        e = -127;                                       // subnormal amax: below 448 * 2^-127
    } else {
        e = (biased - 127) - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    }
    return max(-127, min(127, e));
}

// 2^n as fp32 for integer n (exact, subnormal results included).
__device__ __forceinline__ float exp2_int(int n) {
    if (n >= -126 && n <= 127) return __uint_as_float(static_cast<uint32_t>(n + 127) << 23);
    return ldexpf(1.0f, n);
}

// ------------------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done) : "r"(bar_addr), "r"(parity) : "memory");
    return done != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Gives up (returning false)
// when *abort is set by another role, or after kWaitLimitNs, in which case it sets *abort and
// records MOE_ERR_TIMEOUT.  kSleepNs > 0 makes a thread that has to wait sleep that long between
// polls: for roles that wait on slower ones (a producer on its consumers), so that polling does
// not take issue slots from the warps doing the work on the same scheduler.
template <uint32_t kSleepNs = 0>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* status) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    unsigned long long t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (kSleepNs) __nanosleep(kSleepNs);
        if (mbar_try_wait(a, parity)) return true;
        if (kSleepNs || (i & 255u) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort = 1;
                set_status(status, MOE_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// The same two calls on 32-bit shared-memory addresses (the barrier's and the abort flag's), for
// code that is short of registers: one 32-bit base stands in for several 64-bit pointers.
__device__ __forceinline__ void mbar_arrive_at(uint32_t bar_addr) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar_addr) : "memory");
}

// One arrival from lane 0 of the warp, predicated inside the asm (no divergent branch).  For use
// after warp-collective operations (tcgen05.wait::ld, or loads whose values the whole warp has
// consumed), which every lane has completed when lane 0 gets here.
__device__ __forceinline__ void mbar_arrive_lane0(uint32_t bar_addr, int lane) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.s32 p, %1, 0;\n\t@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(
            bar_addr),
        "r"(lane)
        : "memory");
}

template <uint32_t kSleepNs = 0>
__device__ __forceinline__ bool mbar_wait_at(uint32_t bar_addr, uint32_t parity, uint32_t abort_addr,
                                             int32_t* status) {
    if (mbar_try_wait(bar_addr, parity)) return true;
    unsigned long long t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (kSleepNs) __nanosleep(kSleepNs);
        if (mbar_try_wait(bar_addr, parity)) return true;
        if (kSleepNs || (i & 255u) == 0) {
            uint32_t ab;
            asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(ab) : "r"(abort_addr) : "memory");
            if (ab) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(abort_addr), "r"(1u) : "memory");
                set_status(status, MOE_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// ------------------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 prefetch of one tensor-map box (a hint: no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* holder_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(holder_smem)), "r"(ncols) : "memory");
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

// Shared-memory matrix descriptor for a K-major operand tile stored as TMA writes it with
// 128-byte swizzling: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);   // start address
    d |= static_cast<uint64_t>(1) << 16;                       // leading byte offset (unused)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;               // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                       // descriptor version
    d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f8f6f4, A and B E4M3, fp32 accumulate, both K-major.
__host__ __device__ constexpr uint32_t f8_idesc(int M, int N) {
    return (1u << 4)                                   // D format: f32
           | (0u << 7) | (0u << 10)                    // A, B: E4M3
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp gets lane (quadrant + i).
#define MOE_TMEM_LD32(taddr, v)                                                                 \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                     \
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"                     \
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"    \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),     \
                   "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),   \
                   "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),            \
                   "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),            \
                   "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]),            \
                   "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])             \
                 : "r"(taddr))

// 32 lanes x 16 consecutive fp32 columns.
#define MOE_TMEM_LD16(taddr, v)                                                                 \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "                                     \
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"             \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),     \
                   "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),   \
                   "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])                          \
                 : "r"(taddr))

#define MOE_TMEM_WAIT_LD16(v)                                                                   \
    asm volatile("tcgen05.wait::ld.sync.aligned;"                                              \
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),     \
                   "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),   \
                   "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])                          \
                 :: "memory")

// Wait for this thread's outstanding tcgen05.ld; the loaded registers are passed through so the
// compiler cannot read them before the wait.
#define MOE_TMEM_WAIT_LD(v)                                                                     \
    asm volatile("tcgen05.wait::ld.sync.aligned;"                                              \
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),     \
                   "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),   \
                   "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]),            \
                   "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),            \
                   "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]),            \
                   "+r"(v[27]), "+r"(v[28]), "+r"(v[29]), "+r"(v[30]), "+r"(v[31])             \
                 :: "memory")

// Programmatic dependent launch: wait until the preceding kernel in the stream has finished and
// its writes are visible, then allow the next kernel to start launching.  A dependent launches
// only after every block of this kernel has passed this point (or exited), so its waiting
// blocks never take an SM that one of ours still needs.
__device__ __forceinline__ void pdl_wait_then_release() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Launch with programmatic stream serialization (the kernel calls pdl_wait_then_release()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace moe
