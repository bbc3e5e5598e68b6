// gemm.cu -- grouped FP8 GEMM with fp32 block scales on the 5th-generation tensor cores
// (tcgen05), for both expert projections of the layer (recipe 0; MXFP8 runs gemm_mx.cu).
//
//   mode 0 (gate+up): h[r, n] = sum_g a_s[r,g] * w_s[e,g,n] * sum_{k in g} xq[r,k] * w13[e,n,k]
//                     (+ b13), then act = silu(h_gate) * h_up, requantized per (row, g)
//   mode 1 (down):    o[r, n] = sum_g ... act_q[r,k] * w2[e,n,k] (+ b2), stored fp32
// for every permuted row r of expert e.  "metrale_model_layers fp8_grouped_tc_w8a8.rs",
// run_fp8_grouped_w8a8: the FP8 weights go into E4M3 tensor-core MMAs undecoded, gate+up writes
// quantized SiLU products, then the down projection; "MATE Mega MoE", API: swiglu;
// "MindIE-SD Fused MoE", parameter table: w13_bias / w2_bias.
//
// Design (one persistent CTA per SM, 640 threads = five warpgroups):
//   warp 0   TMA producer: per 128-deep K stage, a 128x128 A tile and a 256x128 B tile (both
//            K-major, 128-byte swizzle), the 256 weight scales of the stage and the tile rows'
//            activation scales (bulk copies).
//   warp 1   MMA issuer (one thread): tcgen05.mma.kind::f8f6f4, M=128 N=256 K=32.  Each 128-deep
//            scale group is accumulated alone into one of two 256-column fp32 TMEM buffers.
//   warps 2-3 idle.  Warpgroup 0 gives registers back (setmaxnreg.dec to 32).
//   warps 4-19 epilogue (setmaxnreg.inc to 112): warp w reads TMEM lanes 32*(w%4) .. +31 (tile
//            rows) and one quarter of the columns; every group partial is multiplied by
//            a_s * w_s and added into fp32 registers (the "promotion"), then the tile's epilogue
//            runs from registers.  Four warps per lane quadrant keep the TMEM reads, which are
//            the critical path of the promotion, in parallel.
// Work unit = (expert, 256-column block, 128-row block), enumerated expert by expert, column
// block, then row block; CTA c takes units c, c + grid, ...  Rows past an expert's end are
// computed on whatever the tile holds and never stored.  Every wait is bounded.
#include <math.h>

#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kStages = 4;
constexpr int kThreads = 640;
constexpr int kFirstEpiWarp = 4;
constexpr int kEpiWarps = 16;
constexpr int kCols = kTileN / 4;                  // columns per epilogue thread
// Registers: 640 threads launch with 96 each (5 warps per SM sub-partition); warpgroup 0 keeps
// 32, the four epilogue warpgroups take 112: 128 * 32 + 512 * 112 = 640 * 96.
constexpr int kRegsLaunch = 96, kRegsLow = 32, kRegsHigh = 112;
static_assert(128 * kRegsLow + 512 * kRegsHigh == kThreads * kRegsLaunch, "register split");
constexpr uint32_t kABytes = kTileM * kTileK;      // 16 KB
constexpr uint32_t kBBytes = kTileN * kTileK;      // 32 KB
constexpr uint32_t kWsBytes = kTileN * 4;          // weight scales: fp32 or 4 x UE8M0 per column
constexpr uint32_t kSaWords = kTileM + 4;          // activation scales of the tile's rows (+ 16-byte alignment)
constexpr uint32_t kSaBytes = kSaWords * 4;
constexpr uint32_t kScaleSlot = 2048;              // per stage: [weight scales | activation scales]
constexpr uint32_t kTmemCols = 2 * kTileN;         // two fp32 accumulators

struct L {
    static constexpr uint32_t a = 0;
    static constexpr uint32_t b = a + kStages * kABytes;
    static constexpr uint32_t sc = b + kStages * kBBytes;
    static constexpr uint32_t bars = sc + kStages * kScaleSlot;
    static constexpr uint32_t nbars = 2 * kStages + 7;   // full, empty, tfull[2], tempty[2], drain, amax[2]
    static constexpr uint32_t misc = bars + nbars * 8;   // tmem holder, abort flag
    static constexpr uint32_t amax = misc + 16;          // float [2 buffers][4 quarters][128 rows]
    static constexpr uint32_t tstart = amax + 2 * 4 * 128 * 4;
    static constexpr uint32_t off = tstart + (MOE_MAX_EXPERTS + 1) * 4;
    static constexpr uint32_t end = off + (MOE_MAX_EXPERTS + 1) * 4;
};
constexpr uint32_t kSmemBytes = L::end + 1024;   // + slack to align the base to 1024 bytes
static_assert(kSmemBytes <= 232448, "shared memory");

// Unit u -> (expert e, column block nb, row block mb).  Expert e owns units
// [nt * tstart[e], nt * tstart[e+1]); empty experts own none.
__device__ __forceinline__ void decode_unit(int u, int nt, const int* tstart, int E, int& e, int& nb,
                                            int& mb) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (nt * tstart[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    e = lo;
    const int local = u - nt * tstart[e];
    const int mt = tstart[e + 1] - tstart[e];
    nb = local / mt;
    mb = local - nb * mt;
}

// acc[j] += P[j] * (sa * ws[j]) over 16 columns [c0, c0 + 16) already loaded into v; packed
// fp32x2 multiply and FMA (each lane rounds as the scalar operations would).
__device__ __forceinline__ void fma_chunk16(float2 (&acc)[kCols / 2], const uint32_t (&v)[16], const float* ws,
                                            int c0, float2 sa2) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(ws + c0 + j);
        const float2 s0 = __fmul2_rn(make_float2(w4.x, w4.y), sa2);
        const float2 s1 = __fmul2_rn(make_float2(w4.z, w4.w), sa2);
        acc[(c0 + j) / 2] = __ffma2_rn(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])), s0,
                                       acc[(c0 + j) / 2]);
        acc[(c0 + j) / 2 + 1] = __ffma2_rn(make_float2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])), s1,
                                           acc[(c0 + j) / 2 + 1]);
    }
}

// The promotion of one scale group over this thread's 64 columns, software-pipelined in
// 16-column chunks: the next chunk's TMEM load is in flight while the current one is multiplied in.
__device__ __forceinline__ void promote_fp32(float2 (&acc)[kCols / 2], uint32_t taddr, const float* ws, float sa) {
    const float2 sa2 = make_float2(sa, sa);
    uint32_t a[16], b[16];
    MOE_TMEM_LD16(taddr, a);
    MOE_TMEM_WAIT_LD16(a);
    MOE_TMEM_LD16(taddr + 16, b);
    fma_chunk16(acc, a, ws, 0, sa2);
    MOE_TMEM_WAIT_LD16(b);
    MOE_TMEM_LD16(taddr + 32, a);
    fma_chunk16(acc, b, ws, 16, sa2);
    MOE_TMEM_WAIT_LD16(a);
    MOE_TMEM_LD16(taddr + 48, b);
    fma_chunk16(acc, a, ws, 32, sa2);
    MOE_TMEM_WAIT_LD16(b);
    fma_chunk16(acc, b, ws, 48, sa2);
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    const int nt = (p.N + kTileN - 1) / kTileN;

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::bars);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* amax_bar = drain + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 4);
    float* s_amax = reinterpret_cast<float*>(smem + L::amax);
    int* s_tstart = reinterpret_cast<int*>(smem + L::tstart);
    int* s_off = reinterpret_cast<int*>(smem + L::off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + kEpiWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
            mbar_init(&amax_bar[b], kEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);
    // everything above overlaps the previous kernel; its outputs are read only from here on
    pdl_wait_then_release();
    for (int i = threadIdx.x; i <= p.E; i += kThreads) {
        s_tstart[i] = p.tile_start[i];
        s_off[i] = p.offsets[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int total_units = s_tstart[p.E] * nt;
    const int KB = p.K / kTileK;                 // pipeline stages per unit
    constexpr int GPS = 1;                       // scale groups per stage
    constexpr int MPG = 4;                       // K=32 MMAs per scale group

    if (warp < kFirstEpiWarp) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
        if (warp == 0 && lane == 0) {
            // -------------------------------------------------------------- TMA producer
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                int e, nb, mb;
                decode_unit(u, nt, s_tstart, p.E, e, nb, mb);
                const int row0 = s_off[e] + mb * kTileM;
                const int brow0 = e * p.N + nb * kTileN;
                const uint32_t ws_bytes = static_cast<uint32_t>(min(kTileN, p.N - nb * kTileN)) * 4u;
                const uint8_t* ws_src = static_cast<const uint8_t*>(p.w_scale) +
                                        (static_cast<size_t>(e) * KB * p.N + static_cast<size_t>(nb) * kTileN) * 4;
                // activation scales are stored [K/128][a_pad]: one 16-byte-aligned run per stage
                const uint8_t* sa_src = static_cast<const uint8_t*>(p.a_scale) + static_cast<size_t>(row0 & ~3) * 4;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], kABytes + kBBytes + ws_bytes + kSaBytes);
                    tma_load_2d(smem + L::a + s * kABytes, &tmA, kb * kTileK, row0, &full[s]);
                    tma_load_2d(smem + L::b + s * kBBytes, &tmB, kb * kTileK, brow0, &full[s]);
                    bulk_load(smem + L::sc + s * kScaleSlot, ws_src + static_cast<size_t>(kb) * p.N * 4, ws_bytes,
                              &full[s]);
                    bulk_load(smem + L::sc + s * kScaleSlot + kWsBytes,
                              sa_src + static_cast<size_t>(kb) * p.a_pad * 4, kSaBytes, &full[s]);
                }
            }
            if (!ok) {   // let the copies already issued land before the CTA leaves
                const uint32_t n = it < static_cast<uint32_t>(kStages) ? it : kStages;
                for (uint32_t i = it - n; i < it; ++i) drain_wait(&full[i % kStages], (i / kStages) & 1);
            }
        } else if (warp == 1 && lane == 0) {
            // -------------------------------------------------------------- MMA issuer
            const uint32_t idesc = f8_idesc(kTileM, kTileN);
            uint32_t it = 0, kg = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                for (int kb = 0; kb < KB && ok; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(&full[s], (it / kStages) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + L::a + s * kABytes);
                    const uint32_t b_addr = smem_u32(smem + L::b + s * kBBytes);
                    for (int g = 0; g < GPS; ++g, ++kg) {
                        const int b = kg & 1;
                        if (!mbar_wait(&tempty[b], ((kg >> 1) & 1) ^ 1, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem_base + static_cast<uint32_t>(b * kTileN);
                        for (int m = 0; m < MPG; ++m) {
                            const uint32_t koff = static_cast<uint32_t>((g * MPG + m) * 32);
                            mma_f8(d, sw128_kmajor_desc(a_addr + koff), sw128_kmajor_desc(b_addr + koff), idesc,
                                   m > 0 ? 1u : 0u);
                        }
                        mma_commit(&tfull[b]);
                    }
                    if (ok) mma_commit(&empty[s]);
                }
            }
            mma_commit(drain);          // all MMAs issued by this thread have finished
            drain_wait(drain, 0);
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
        // ------------------------------------------------------------------ epilogue
        const int ew = warp - kFirstEpiWarp;
        const int quad = warp & 3;                // TMEM lanes 32*quad .. 32*quad+31
        const int qtr = ew >> 2;                  // columns qtr*64 .. qtr*64+63 of the tile
        const int row_in_tile = quad * 32 + lane;
        uint32_t it = 0, kg = 0, tile = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++tile) {
            int e, nb, mb;
            decode_unit(u, nt, s_tstart, p.E, e, nb, mb);
            const int row0 = s_off[e] + mb * kTileM;
            const int cnt = min(kTileM, s_off[e + 1] - row0);
            const bool warp_active = quad * 32 < cnt;
            const bool row_ok = row_in_tile < cnt;
            const int r = row0 + row_in_tile;

            float2 acc2[kCols / 2];
#pragma unroll
            for (int i = 0; i < kCols / 2; ++i) acc2[i] = make_float2(0.0f, 0.0f);
            float* acc = reinterpret_cast<float*>(acc2);

            for (int kb = 0; kb < KB && ok; ++kb, ++it) {
                const int s = it % kStages;
                // acquire the stage (its scales were written by the bulk copies)
                if (!mbar_wait(&full[s], (it / kStages) & 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                const uint8_t* ws_stage = smem + L::sc + s * kScaleSlot + qtr * kCols * 4;
                const uint32_t saw = reinterpret_cast<const uint32_t*>(smem + L::sc + s * kScaleSlot + kWsBytes)
                    [(row0 & 3) + row_in_tile];
                for (int g = 0; g < GPS; ++g, ++kg) {
                    const int b = kg & 1;
                    if (!mbar_wait(&tfull[b], (kg >> 1) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (warp_active) {
                        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                               static_cast<uint32_t>(b * kTileN + qtr * kCols);
                        promote_fp32(acc2, taddr, reinterpret_cast<const float*>(ws_stage), __uint_as_float(saw));
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[b]);
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;

            if (MODE == 0) {
                // ---- SwiGLU + requantization.  This quarter holds acc[0:32] gate and acc[32:64] up
                // of act columns c0 .. c0+31 (the transform's 32-column interleave).
                const int I = p.N >> 1;
                const int c0 = nb * 128 + qtr * 32;
                if (warp_active) {
                    if (p.bias) {
                        add_bias32(acc, p.bias + static_cast<size_t>(e) * p.N + c0);
                        add_bias32(acc + 32, p.bias + static_cast<size_t>(e) * p.N + I + c0);
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        acc[i] = silu(acc[i]) * acc[32 + i];
                    }
                }
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(acc[i]));
                // one 128-column group per row: combine the four quarters' maxima
                const int buf = tile & 1;
                s_amax[(buf * 4 + qtr) * 128 + row_in_tile] = amax;
                __syncwarp();
                if (lane == 0) mbar_arrive(&amax_bar[buf]);
                if (!mbar_wait(&amax_bar[buf], (tile >> 1) & 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) amax = fmaxf(amax, s_amax[(buf * 4 + q) * 128 + row_in_tile]);
                const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                if (warp_active && row_ok) {
                    uint4* dst = reinterpret_cast<uint4*>(p.act_q + static_cast<size_t>(r) * I + c0);
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        uint4 q;
                        q.x = e4m3x4(__fdiv_rn(acc[16 * w + 0], sc), __fdiv_rn(acc[16 * w + 1], sc),
                                     __fdiv_rn(acc[16 * w + 2], sc), __fdiv_rn(acc[16 * w + 3], sc));
                        q.y = e4m3x4(__fdiv_rn(acc[16 * w + 4], sc), __fdiv_rn(acc[16 * w + 5], sc),
                                     __fdiv_rn(acc[16 * w + 6], sc), __fdiv_rn(acc[16 * w + 7], sc));
                        q.z = e4m3x4(__fdiv_rn(acc[16 * w + 8], sc), __fdiv_rn(acc[16 * w + 9], sc),
                                     __fdiv_rn(acc[16 * w + 10], sc), __fdiv_rn(acc[16 * w + 11], sc));
                        q.w = e4m3x4(__fdiv_rn(acc[16 * w + 12], sc), __fdiv_rn(acc[16 * w + 13], sc),
                                     __fdiv_rn(acc[16 * w + 14], sc), __fdiv_rn(acc[16 * w + 15], sc));
                        dst[w] = q;
                    }
                    if (qtr == 0) static_cast<float*>(p.act_s)[static_cast<size_t>(nb) * p.a_pad + r] = sc;
                }
            } else {
                // ---- down projection: + bias, fp32 rows
                const int c0 = nb * kTileN + qtr * kCols;
                if (warp_active && row_ok && c0 < p.N) {
                    if (p.bias) {
                        add_bias32(acc, p.bias + static_cast<size_t>(e) * p.N + c0);
                        add_bias32(acc + 32, p.bias + static_cast<size_t>(e) * p.N + c0 + 32);
                    }
                    float4* dst = reinterpret_cast<float4*>(p.out + static_cast<size_t>(r) * p.N + c0);
#pragma unroll
                    for (int c = 0; c < kCols; c += 4)
                        dst[c >> 2] = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int MODE>
static cudaError_t launch_gemm_t(const GemmArgs& a, const CUtensorMap& tmA, const CUtensorMap& tmB, int num_sms,
                                 cudaStream_t s) {
    // The register split above must fit what the block is launched with, or setmaxnreg.inc
    // would wait forever: refuse to launch otherwise.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, k_grouped_gemm<MODE>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * kThreads < kRegsLow * 128 + kRegsHigh * 512) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(k_grouped_gemm<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    return launch_pdl(k_grouped_gemm<MODE>, dim3(num_sms), dim3(kThreads), kSmemBytes, s, tmA, tmB, a);
}

cudaError_t launch_gemm(const GemmArgs& a, const CUtensorMap& tmA, const CUtensorMap& tmB, int num_sms,
                        cudaStream_t s) {
    if (a.recipe != 0) return cudaErrorInvalidValue;   // MXFP8 runs gemm_mx.cu
    return a.mode == 0 ? launch_gemm_t<0>(a, tmA, tmB, num_sms, s) : launch_gemm_t<1>(a, tmA, tmB, num_sms, s);
}

}  // namespace moe
