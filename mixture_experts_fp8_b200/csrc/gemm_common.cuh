// gemm_common.cuh -- pieces shared by the two grouped FP8 GEMM kernels (gemm.cu, gemm_narrow.cu).
#pragma once

#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

constexpr unsigned long long kDrainLimitNs = 100000000ull;

// Bounded wait used only while leaving after an abort: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(a, parity)) {
        __nanosleep(128);
        if (globaltimer_ns() - t0 > kDrainLimitNs) break;
    }
}

// ------------------------------------------------------------------ weight prefetch before the wait
// Before its wait on the preceding kernel, a GEMM CTA hints the weight tiles of its first work
// unit into L2: the weights do not come from that kernel, so their fetch can overlap it.  The
// unit's expert is found from the permutation's outputs (offsets, tile_start), read from L2 by
// one warp.  The permutation completed before the preceding kernel started its work, and a stale
// value could only make the hint miss: the real loads use the values read after the wait.
constexpr int kPrefetchStages = 6;

// Narrow kernels: expert e owns nblk * ceil(rows_e / NT) units, weight block by weight block
// (a warp scan of the per-expert unit counts).
template <int NT>
__device__ __forceinline__ bool early_unit_rows(const int* offsets, int E, int nblk, int u, int lane, int& e_out,
                                                int& blk_out) {
    int base = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        int n = 0;
        if (e < E) n = nblk * ((__ldcg(offsets + e + 1) - __ldcg(offsets + e) + NT - 1) / NT);
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int excl = base + incl - n;
        const unsigned m = __ballot_sync(0xffffffffu, n > 0 && u >= excl && u < excl + n);
        if (m) {
            const int src = __ffs(m) - 1;
            const int ex = __shfl_sync(0xffffffffu, excl, src), nn = __shfl_sync(0xffffffffu, n, src);
            e_out = e0 + src;
            blk_out = (u - ex) / (nn / nblk);
            return true;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    return false;
}

// Wide kernels: expert e owns units [nt * tile_start[e], nt * tile_start[e+1]), column block by
// column block; the expert is the last one whose first unit is <= u.
__device__ __forceinline__ bool early_unit_tiles(const int* tile_start, int E, int nt, int u, int lane, int& e_out,
                                                 int& blk_out) {
    if (u >= nt * __ldcg(tile_start + E)) return false;
    int cnt = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        cnt += __popc(__ballot_sync(0xffffffffu, e < E && nt * __ldcg(tile_start + e) <= u));
    }
    const int e = cnt - 1;
    const int t0 = __ldcg(tile_start + e), mt = __ldcg(tile_start + e + 1) - t0;
    if (e < 0 || mt <= 0) return false;
    e_out = e;
    blk_out = (u - nt * t0) / mt;
    return true;
}

// One thread: the first n K stages of the weight box at row `row` toward L2.
__device__ __forceinline__ void prefetch_weight_stages(const CUtensorMap* map, int row, int K) {
    const int n = min(kPrefetchStages, K / kTileK);
    for (int kb = 0; kb < n; ++kb) tma_prefetch_2d(map, kb * kTileK, row);
}

// Poll intervals of the single-thread roles, which mostly wait on the epilogue warps (the
// producer for a free stage, the MMA issuer for a free accumulator): sleeping between polls keeps
// them from taking issue slots on the schedulers they share with epilogue warps.
constexpr uint32_t kProducerSleepNs = 256;
constexpr uint32_t kIssuerSleepNs = 0;

// silu(z) = z / (1 + e^-z), with the hardware exponential and a fast reciprocal division
// (every GEMM kernel uses this same function, so their outputs agree bit for bit).  For z below
// about -87 the divisor exceeds 2^126 and the quotient is 0, where the exact value is under 1e-36.
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// Add 8 bf16 bias values (one 16-byte word) to acc[0..7].
__device__ __forceinline__ void add_bias8(float* acc, uint4 w) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        acc[2 * q] += __uint_as_float(ww[q] << 16);
        acc[2 * q + 1] += __uint_as_float(ww[q] & 0xFFFF0000u);
    }
}

// A 16-byte read-only load kept in program order (volatile), so the compiler does not hoist all of
// an epilogue's bias loads at once and run out of registers.
__device__ __forceinline__ uint4 ld_nc_u4(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// One 32-byte store of eight fp32 values (p 32-byte aligned): a whole L2 sector per lane, half
// as many store instructions and write requests as two 16-byte stores.
__device__ __forceinline__ void st_global_f32x8(float* p, const float* a) {
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(a[0]), "f"(a[1]),
                 "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7])
                 : "memory");
}

// Add 32 bf16 bias values (16-byte aligned) to acc[0..31].
__device__ __forceinline__ void add_bias32(float* acc, const __nv_bfloat16* bias) {
    const uint4* b4 = reinterpret_cast<const uint4*>(bias);
#pragma unroll
    for (int v = 0; v < 4; ++v) add_bias8(acc + 8 * v, ld_nc_u4(b4 + v));
}

// ------------------------------------------------------------------ block-scaled (MX) MMA pieces
// Instruction descriptor, kind::mxf8f6f4 block-scaled, UE8M0 scale factors, both operands
// K-major: afmt / bfmt 0 = E4M3, 5 = E2M1; the scale-factor ids pick byte k of the 32-bit scale
// words (the k-th 32-deep block of a 128-deep stage).
__device__ __forceinline__ uint32_t mx_block_idesc(uint32_t k, uint32_t afmt, uint32_t bfmt, int M, int N) {
    return (k << 4)                                       // B scale-factor id
           | (afmt << 7) | (bfmt << 10)                   // A, B element formats
           | (static_cast<uint32_t>(N >> 3) << 17)        // N / 8
           | (1u << 23)                                   // scale format: UE8M0
           | (static_cast<uint32_t>(M >> 4) << 24)        // M / 16
           | (k << 29);                                   // A scale-factor id
}

__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// Shared-memory descriptor of one scale-factor atom: 32 rows of 16 bytes, contiguous, no swizzle
// (8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(128 >> 4) << 32;   // stride between 8-row core matrices
    d |= static_cast<uint64_t>(1) << 46;           // descriptor version
    return d;                                       // layout type 0: no swizzle
}

// Copy one scale-factor atom (32 rows x 16 bytes) into 4 TMEM columns of every lane quadrant:
// row i's word c lands in lane i, column c.  The MMA reads the scale of row r from lane r % 32,
// column r / 32, byte = its scale-factor id.
__device__ __forceinline__ void sf_copy(uint32_t tmem_col_addr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem_col_addr), "l"(sdesc) : "memory");
}

// ------------------------------------------------------------------ clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA in the cluster: writes to shared memory before it are visible to
// the cluster's loads after it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace moe
