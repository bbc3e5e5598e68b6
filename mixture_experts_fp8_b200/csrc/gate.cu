// gate.cu -- the gate in front of the router ("mlx_native ops/moe_gate.rs": per token, RMS-Norm
// of the bf16 hidden state, the router matmul, then top-K + softmax + per-expert scale):
//   xn[h]     = x[h] / sqrt( mean_h x[h]^2 + eps ) * norm_w[h]
//   logit[e]  = sum_h xn[h] * router_w[e, h]
// computed as  logit[e] = r * sum_h x[h] * w'[e, h],  w'[e, h] = fl32(norm_w[h] * router_w[e, h]),
// r = 1/sqrt(mean x^2 + eps): the norm's per-token factor leaves the sum and its per-column
// weight is folded into the router rows once (k_gate_split, moe_transform_gate_weights).
//
// The router matmul runs on the tensor core: tcgen05.mma kind::f16 with bf16 operands and fp32
// accumulation in TMEM.  x is bf16 already.  w' is split into three bf16 parts hi + mid + lo that
// carry its 24 significant bits; the three products x * part are exact and accumulate into the
// same fp32 accumulator, so the sum keeps fp32 precision.
//
// k_gate_mma: tiles of 128 tokens x 64 experts.  The K range (H/64 steps of 64 columns) is split
// over a cluster of 8 CTAs, each accumulating a contiguous share in TMEM; the 8 partial tiles are
// added through distributed shared memory in rank order.  The split and the order depend on H
// alone: a token's logits do not depend on T or on the other tokens.  The router kernel then
// scales each row by r (the same per-token sum of squares as before) and routes it.
#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kGM = 128;                  // tokens per tile (the MMA's M)
constexpr int kGN = 64;                   // experts per tile (the MMA's N)
constexpr int kGK = 64;                   // bf16 columns per stage: one 128-byte swizzled row
constexpr int kGSplit = 8;                // CTAs per cluster = shares of K
constexpr int kGThreads = 128;
constexpr int kGParts = 3;                // hi, mid, lo
constexpr uint32_t kGABytes = kGM * kGK * 2;                       // 16 KB of x
constexpr uint32_t kGBBytes = kGN * kGK * 2;                       // 8 KB per part of w'
constexpr uint32_t kGStageBytes = kGABytes + kGParts * kGBBytes;   // 40 KB
constexpr int kGPitch = kGN + 1;          // row pitch (floats) of the partial tile in shared memory
constexpr uint32_t kGTmemCols = 64;

// Shared memory: the stages, whose space holds the partial tile once the MMAs are done, then
// the barriers.  Four stages (one CTA per SM) when the grid fits on the SMs at once; otherwise
// two stages, so that two CTAs share an SM and one's prologue and reduction overlap the other's
// loads (measured: two CTAs of two stages beat one CTA of five stages by 1.4x at 4096 tokens).
template <int STAGES>
struct GL {
    static constexpr uint32_t part = 0;
    static constexpr uint32_t bars = STAGES * kGStageBytes;
    static constexpr uint32_t nbars = 2 * STAGES + 1;                // full, empty, done
    static constexpr uint32_t misc = bars + nbars * 8;               // tmem holder, abort flag
    static constexpr uint32_t total = misc + 16;
    static constexpr size_t smem = total + 1024;                     // + alignment slack
    static_assert(kGM * kGPitch * 4 <= bars, "the partial tile fits in the stages");
    static_assert(smem <= 232448, "gate shared memory");
};

// Instruction descriptor: kind::f16, A and B bf16, fp32 accumulate, both K-major.
__host__ __device__ constexpr uint32_t bf16_idesc(int M, int N) {
    return (1u << 4)                                   // D format: f32
           | (1u << 7) | (1u << 10)                    // A, B: bf16
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// The address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

}  // namespace

// w'[e, h] = fl32(norm_w[h] * router_w[e, h]) split into bf16 parts: out[0] = hi = rn(w'),
// out[1] = mid = rn(w' - hi), out[2] = lo = rn(w' - hi - mid), each part [E, H].  Both
// subtractions are exact (the operands are within a factor of two of each other).
__global__ void __launch_bounds__(256) k_gate_split(const float* __restrict__ norm_w, const float* __restrict__ router_w,
                                                    __nv_bfloat16* __restrict__ out, int E, int H) {
    const size_t n = static_cast<size_t>(E) * H;
    for (size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x * 4) {
        const int h = static_cast<int>(i % H);
        const float4 w = *reinterpret_cast<const float4*>(router_w + i);
        const float4 g = *reinterpret_cast<const float4*>(norm_w + h);
        const float v[4] = {__fmul_rn(g.x, w.x), __fmul_rn(g.y, w.y), __fmul_rn(g.z, w.z), __fmul_rn(g.w, w.w)};
        __nv_bfloat16 p[3][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            p[0][j] = __float2bfloat16_rn(v[j]);
            const float r1 = __fsub_rn(v[j], __bfloat162float(p[0][j]));
            p[1][j] = __float2bfloat16_rn(r1);
            const float r2 = __fsub_rn(r1, __bfloat162float(p[1][j]));
            p[2][j] = __float2bfloat16_rn(r2);
        }
#pragma unroll
        for (int q = 0; q < 3; ++q) *reinterpret_cast<uint2*>(out + q * n + i) = *reinterpret_cast<const uint2*>(p[q]);
    }
}

template <int kGStages>
__global__ void __launch_bounds__(kGThreads, 1)
    k_gate_mma(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, GateArgs g) {
    using L = GL<kGStages>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::bars);
    uint64_t* empty = full + kGStages;
    uint64_t* done = empty + kGStages;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 4);
    float* part = reinterpret_cast<float*>(smem + L::part);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int e0 = static_cast<int>(blockIdx.x / kGSplit) * kGN, t0 = static_cast<int>(blockIdx.y) * kGM;
    const int nsteps = g.H / kGK;
    const int s_lo = static_cast<int>(rank) * nsteps / kGSplit;
    const int n = (static_cast<int>(rank) + 1) * nsteps / kGSplit - s_lo;   // this CTA's steps (may be 0)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
    }
    if (warp == 0) tmem_alloc(tmem_holder, kGTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    pdl_wait_then_release();

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------------------- TMA producer
        int i = 0;
        bool ok = true;
        for (; i < n; ++i) {
            const int s = i % kGStages;
            if (i >= kGStages && !mbar_wait(&empty[s], ((i / kGStages) - 1) & 1, abort_flag, nullptr)) {
                ok = false;
                break;
            }
            uint8_t* st = smem + s * kGStageBytes;
            const int kx = (s_lo + i) * kGK * 2;   // byte column of this step
            mbar_arrive_expect_tx(&full[s], kGStageBytes);
            tma_load_2d(st, &tmX, kx, t0, &full[s]);
#pragma unroll
            for (int q = 0; q < kGParts; ++q)
                tma_load_2d(st + kGABytes + q * kGBBytes, &tmW, kx, q * g.E + e0, &full[s]);
        }
        if (!ok) {   // leave no copy in flight: wait out the stages issued and not yet consumed
            for (int j = i > kGStages ? i - kGStages : 0; j < i; ++j) drain_wait(&full[j % kGStages], (j / kGStages) & 1);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------------------------------------------------------------- MMA issuer
        const uint32_t idesc = bf16_idesc(kGM, kGN);
        for (int i = 0; i < n; ++i) {
            const int s = i % kGStages;
            if (!mbar_wait(&full[s], (i / kGStages) & 1, abort_flag, nullptr)) break;
            tc_fence_after();
            const uint32_t a = smem_u32(smem + s * kGStageBytes);
#pragma unroll
            for (int kk = 0; kk < kGK / 16; ++kk)
#pragma unroll
                for (int q = 0; q < kGParts; ++q)
                    mma_bf16(tmem, sw128_kmajor_desc(a + kk * 32),
                             sw128_kmajor_desc(a + kGABytes + q * kGBBytes + kk * 32), idesc,
                             (i | kk | q) != 0 ? 1u : 0u);
            mma_commit(&empty[s]);
        }
        mma_commit(done);   // arrives once every MMA issued above has completed
    }
    __syncwarp();
    __syncthreads();   // the roles are over: no copy in flight (the producer drained after an abort)

    // -------------------------------------------------------------------------- partial tile
    // warp w reads TMEM lanes 32w .. 32w+31 (tile rows) into the stages' space, free once every
    // MMA has completed; NaN marks a tile that timed out.
    const int row = warp * 32 + lane;
    float* prow = part + row * kGPitch;
    bool have = false;
    if (n > 0) {
        const bool got = mbar_wait(done, 0, abort_flag, nullptr);
        have = __all_sync(0xffffffffu, got && *abort_flag == 0);
    }
    if (have) {
        tc_fence_after();
        uint32_t v[32];
        const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            MOE_TMEM_LD32(taddr + h * 32, v);
            MOE_TMEM_WAIT_LD(v);
#pragma unroll
            for (int c = 0; c < 32; ++c) prow[h * 32 + c] = __uint_as_float(v[c]);
        }
    } else {
        const float z = n > 0 ? __int_as_float(0x7fc00000) : 0.0f;
#pragma unroll 8
        for (int c = 0; c < kGN; ++c) prow[c] = z;
    }
    tc_fence_before();
    cluster_sync_all();

    // -------------------------------------------------------------------------- K reduction
    // CTA `rank` sums rows 16*rank .. +15 of the 8 partial tiles, in rank order.
    const uint32_t part_addr = smem_u32(part);
    uint32_t src[kGSplit];
#pragma unroll
    for (int q = 0; q < kGSplit; ++q) src[q] = cluster_map(part_addr, static_cast<uint32_t>(q));
    const int col = threadIdx.x % kGN, e = e0 + col;
#pragma unroll
    for (int j = 0; j < kGM / kGSplit / 2; ++j) {
        const int r = static_cast<int>(rank) * (kGM / kGSplit) + j * 2 + threadIdx.x / kGN;
        const uint32_t off = static_cast<uint32_t>(r * kGPitch + col) * 4u;
        float acc = ld_cluster_f32(src[0] + off);
#pragma unroll
        for (int q = 1; q < kGSplit; ++q) acc += ld_cluster_f32(src[q] + off);
        const int t = t0 + r;
        if (t < g.T && e < g.E) g.logits[static_cast<size_t>(t) * g.E + e] = acc;
    }
    cluster_sync_all();   // no CTA leaves while another still reads its partial tile
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kGTmemCols);
    }
}

cudaError_t launch_gate_split(const float* norm_w, const float* router_w, void* out, int E, int H, cudaStream_t s) {
    const size_t n4 = static_cast<size_t>(E) * H / 4;
    const size_t want = (n4 + 255) / 256;
    const int blocks = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
    k_gate_split<<<blocks, 256, 0, s>>>(norm_w, router_w, static_cast<__nv_bfloat16*>(out), E, H);
    return cudaGetLastError();
}

uint32_t gate_token_box() { return kGM; }
uint32_t gate_weight_box() { return kGN; }

template <int STAGES>
static cudaError_t launch_gate_mma(const CUtensorMap& tmX, const CUtensorMap& tmW, const GateArgs& g,
                                   cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_gate_mma<STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(GL<STAGES>::smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kGSplit * ((g.E + kGN - 1) / kGN), (g.T + kGM - 1) / kGM);
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = GL<STAGES>::smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kGSplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k_gate_mma<STAGES>, tmX, tmW, g);
}

cudaError_t launch_gate(const CUtensorMap& tmX, const CUtensorMap& tmW, const GateArgs& g, const RouteArgs& ra,
                        cudaStream_t s) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long ctas = 1LL * kGSplit * ((g.E + kGN - 1) / kGN) * ((g.T + kGM - 1) / kGM);
    const cudaError_t e = ctas > sms ? launch_gate_mma<2>(tmX, tmW, g, s) : launch_gate_mma<4>(tmX, tmW, g, s);
    if (e != cudaSuccess) return e;
    return launch_route(ra, s);
}

}  // namespace moe
