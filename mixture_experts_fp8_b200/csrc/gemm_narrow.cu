// gemm_narrow.cu -- the grouped FP8 GEMMs with fp32 block scales (recipe 0) for problems with few
// routed rows per expert (decode), in the swap-AB orientation: the expert's weights are the MMA's
// M=128 operand and its routed rows (tokens) the N=16 operand.
//
// Same arithmetic as gemm.cu, term for term ("metrale_model_layers fp8_grouped_tc_w8a8.rs",
// run_fp8_grouped_w8a8; "MATE Mega MoE", API: swiglu):
//   mode 0: h = sum_g a_s[r,g] * w_s[n,g] * P_g (+ b13), act = silu(h_gate) * h_up, requantized
//   mode 1: o = sum_g ... (+ b2), fp32
// Each 128-deep group partial P_g comes from the tensor core; it is multiplied by
// (w_s * a_s) and added with one fma, the same operations in the same order as the wide kernel,
// so a row's result does not depend on which of the two kernels computed it.
//
// Why a second kernel: the wide kernel's accumulator is 128 rows x 256 columns per group, and
// reading it back from TMEM for the per-group scale promotion dominates when an expert has only a
// few rows.  Here the accumulator is 128 weight rows x 16 tokens, so each group's read-back is
// 4 KB per TMEM lane quadrant, and the kernel streams weights at HBM speed.
//
// Tile = (expert e, weight block wb, token block tb):
//   mode 0: 256 consecutive rows of the transformed w13, 128 gate rows and the 128 matching up
//           rows -> accumulators D0 (gate), D1 (up): lane j of both holds act column wb*128 + j,
//           so SwiGLU stays in-thread.
//   mode 1: 256 consecutive rows of w2 -> D0 (rows 0..127), D1 (rows 128..255).
// Threads: warp 0 TMA producer, warp 1 MMA issuer (one thread), warps 4-7 epilogue (warp w reads
// TMEM lanes 32*(w%4) .. +31), warps 2-3 idle.  Four TMEM accumulator pairs; every wait bounded.
#include <math.h>

#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kNT = 16;                           // tokens per tile (MMA N)
constexpr int kNStages = 5;
constexpr int kNThreads = 256;
constexpr int kNFirstEpi = 4;
constexpr int kNEpiWarps = 4;
constexpr int kNBuf = 4;                          // TMEM accumulator pairs
constexpr uint32_t kNTmemCols = 128;              // >= kNBuf * 2 * kNT, a power of two
constexpr uint32_t kWBytes = 256 * kTileK;        // 32 KB of weights per stage
constexpr uint32_t kTBytes = kNT * kTileK;        // 2 KB of token rows per stage
constexpr uint32_t kWsBytes = 256 * 4;            // weight scales of the 256 rows
constexpr uint32_t kNSaWords = kNT + 4;           // token scales (+ 16-byte alignment)
constexpr uint32_t kNSaBytes = kNSaWords * 4;
constexpr uint32_t kStageBytes = 36864;           // [W 32 KB | T 2 KB | ws 1 KB | sa | pad], 1024-aligned

struct NL {
    static constexpr uint32_t t = kWBytes;
    static constexpr uint32_t ws = t + kTBytes;
    static constexpr uint32_t sa = ws + kWsBytes;
    static constexpr uint32_t bars = kNStages * kStageBytes;
    static constexpr uint32_t nbars = 2 * kNStages + 2 * kNBuf + 5;  // full, empty, tfull, tempty, drain, amax[2], free[2]
    static constexpr uint32_t misc = bars + nbars * 8;               // tmem holder, abort flag
    static constexpr uint32_t amax = misc + 16;                      // float [2][4 quads][kNT]
    static constexpr uint32_t ustart = amax + 2 * 4 * kNT * 4;       // int [E + 1] unit prefix
    static constexpr uint32_t off = ustart + (MOE_MAX_EXPERTS + 2) * 4;   // experts + a shared one, + 1
    static constexpr uint32_t end = off + (MOE_MAX_EXPERTS + 2) * 4;   // experts + a shared one, + 1
};
static_assert(NL::sa + kNSaBytes <= kStageBytes, "stage layout");
static_assert(kStageBytes % 1024 == 0, "stage alignment");
constexpr uint32_t kNSmemBytes = NL::end + 1024;
static_assert(kNSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ void decode_unit_narrow(int u, const int* ustart, const int* off, int E, int& e, int& wb,
                                                   int& tb) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ustart[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    e = lo;
    const int ntb = (off[e + 1] - off[e] + kNT - 1) / kNT;
    const int local = u - ustart[e];
    wb = local / ntb;
    tb = local - wb * ntb;
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kNThreads, 1)
    k_grouped_gemm_narrow(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmT,
                          const GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    const int nwb = MODE == 0 ? p.N / 256 : (p.N + 255) / 256;   // weight blocks per expert

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NL::bars);
    uint64_t* empty = full + kNStages;
    uint64_t* tfull = empty + kNStages;
    uint64_t* tempty = tfull + kNBuf;
    uint64_t* drain = tempty + kNBuf;
    uint64_t* amax_bar = drain + 1;
    uint64_t* amax_free = amax_bar + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + NL::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + NL::misc + 4);
    float* s_amax = reinterpret_cast<float*>(smem + NL::amax);
    int* s_ustart = reinterpret_cast<int*>(smem + NL::ustart);
    int* s_off = reinterpret_cast<int*>(smem + NL::off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kNStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + kNEpiWarps);
        }
        for (int b = 0; b < kNBuf; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kNEpiWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&amax_bar[b], kNEpiWarps);
            mbar_init(&amax_free[b], kNEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmW);
        prefetch_tmap(&tmT);
    }
    if (warp == 1) tmem_alloc(tmem_holder, kNTmemCols);
    if (warp == 0) {   // the first unit's weight tiles toward L2 while the preceding kernel runs
        int e, wb;
        if (early_unit_rows<kNT>(p.offsets, p.E, nwb, blockIdx.x, lane, e, wb) && lane == 0)
            prefetch_weight_stages(&tmW, e * p.N + wb * 256, p.K);
    }
    pdl_wait_then_release();
    for (int i = threadIdx.x; i <= p.E; i += kNThreads) s_off[i] = p.offsets[i];
    __syncthreads();
    if (threadIdx.x == 0) {   // unit prefix: expert e owns nwb * ceil(rows / kNT) units
        int acc = 0;
        for (int e = 0; e < p.E; ++e) {
            s_ustart[e] = acc;
            acc += nwb * ((s_off[e + 1] - s_off[e] + kNT - 1) / kNT);
        }
        s_ustart[p.E] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int total_units = s_ustart[p.E];
    const int KB = p.K / kTileK;
    constexpr int GPS = 1;                       // one 128-deep scale group per stage
    constexpr int MPG = 4;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------------ TMA producer
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                int e, wb, tb;
                decode_unit_narrow(u, s_ustart, s_off, p.E, e, wb, tb);
                const int row0 = s_off[e] + tb * kNT;
                const int wrow0 = e * p.N + wb * 256;
                const uint32_t ws_bytes = static_cast<uint32_t>(min(256, p.N - wb * 256)) * 4u;
                const uint8_t* ws_src = static_cast<const uint8_t*>(p.w_scale) +
                                        (static_cast<size_t>(e) * KB * p.N + static_cast<size_t>(wb) * 256) * 4;
                const uint8_t* sa_src = static_cast<const uint8_t*>(p.a_scale) + static_cast<size_t>(row0 & ~3) * 4;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % kNStages;
                    if (!mbar_wait<kProducerSleepNs>(&empty[s], ((it / kNStages) & 1) ^ 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    if (fault_skip_stage(p.fault, it)) continue;   // debug builds: an injected fault
                    uint8_t* st = smem + s * kStageBytes;
                    mbar_arrive_expect_tx(&full[s], kWBytes + kTBytes + ws_bytes + kNSaBytes);
                    // mode 0: the 128 gate rows, then the 128 up rows of act columns wb*128 .. +127
                    tma_load_2d(st, &tmW, kb * kTileK, wrow0, &full[s]);
                    tma_load_2d(st + NL::t, &tmT, kb * kTileK, row0, &full[s]);
                    bulk_load(st + NL::ws, ws_src + static_cast<size_t>(kb) * p.N * 4, ws_bytes, &full[s]);
                    bulk_load(st + NL::sa, sa_src + static_cast<size_t>(kb) * p.a_pad * 4, kNSaBytes, &full[s]);
                }
            }
            if (!ok) {
                const uint32_t n = it < static_cast<uint32_t>(kNStages) ? it : kNStages;
                for (uint32_t i = it - n; i < it; ++i) drain_wait(&full[i % kNStages], (i / kNStages) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------------ MMA issuer
            const uint32_t idesc = f8_idesc(128, kNT);
            uint32_t it = 0, kg = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                for (int kb = 0; kb < KB && ok; ++kb, ++it) {
                    const int s = it % kNStages;
                    if (!mbar_wait<kIssuerSleepNs>(&full[s], (it / kNStages) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t w_addr = smem_u32(smem + s * kStageBytes);
                    const uint32_t t_addr = w_addr + NL::t;
                    for (int g = 0; g < GPS; ++g, ++kg) {
                        const int b = kg % kNBuf;
                        if (!mbar_wait<kIssuerSleepNs>(&tempty[b], ((kg / kNBuf) & 1) ^ 1, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem_base + static_cast<uint32_t>(b * 2 * kNT);
                        for (int m = 0; m < MPG; ++m) {
                            const uint32_t koff = static_cast<uint32_t>((g * MPG + m) * 32);
                            const uint64_t tdesc = sw128_kmajor_desc(t_addr + koff);
                            mma_f8(d, sw128_kmajor_desc(w_addr + koff), tdesc, idesc, m > 0 ? 1u : 0u);
                            mma_f8(d + kNT, sw128_kmajor_desc(w_addr + 16384 + koff), tdesc, idesc, m > 0 ? 1u : 0u);
                        }
                        mma_commit(&tfull[b]);
                    }
                    if (ok) mma_commit(&empty[s]);
                }
            }
            mma_commit(drain);
            drain_wait(drain, 0);
        }
    } else if (warp >= kNFirstEpi) {
        // ---------------------------------------------------------------------- epilogue
        const int quad = warp & 3;
        const int j = quad * 32 + lane;           // TMEM lane = weight row within each half
        uint32_t it = 0, kg = 0, tile = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++tile) {
            int e, wb, tb;
            decode_unit_narrow(u, s_ustart, s_off, p.E, e, wb, tb);
            const int row0 = s_off[e] + tb * kNT;
            const int cnt = min(kNT, s_off[e + 1] - row0);
            float acc0[kNT], acc1[kNT];
#pragma unroll
            for (int t = 0; t < kNT; ++t) acc0[t] = acc1[t] = 0.0f;

            for (int kb = 0; kb < KB && ok; ++kb, ++it) {
                const int s = it % kNStages;
                if (!mbar_wait(&full[s], (it / kNStages) & 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                const uint8_t* st = smem + s * kStageBytes;
                const uint32_t* wsw = reinterpret_cast<const uint32_t*>(st + NL::ws);
                // this thread's two weight rows j and 128 + j: gate and up of act column j in mode 0
                const uint32_t w0 = wsw[j];
                const uint32_t w1 = wsw[128 + j];
                const uint32_t* saw = reinterpret_cast<const uint32_t*>(st + NL::sa) + (row0 & 3);
                for (int g = 0; g < GPS; ++g, ++kg) {
                    const int b = kg % kNBuf;
                    if (!mbar_wait(&tfull[b], (kg / kNBuf) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                           static_cast<uint32_t>(b * 2 * kNT);
                    uint32_t v0[16], v1[16];
                    MOE_TMEM_LD16(taddr, v0);
                    MOE_TMEM_LD16(taddr + kNT, v1);
                    MOE_TMEM_WAIT_LD16(v0);
                    MOE_TMEM_WAIT_LD16(v1);
                    const float ws0 = __uint_as_float(w0), ws1 = __uint_as_float(w1);
#pragma unroll
                    for (int t = 0; t < kNT; ++t) {
                        const float sa = __uint_as_float(saw[t]);
                        acc0[t] = fmaf(__uint_as_float(v0[t]), ws0 * sa, acc0[t]);
                        acc1[t] = fmaf(__uint_as_float(v1[t]), ws1 * sa, acc1[t]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[b]);
                }
                if (!ok) break;
                // The stage's scales were read through the generic proxy; the producer's next bulk
                // copy into this stage is an async-proxy write.  Order the reads before it.
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;

            if (MODE == 0) {
                const int I = p.N >> 1;
                const int c = wb * 128 + j;       // act column of this thread
                if (p.bias) {
                    const float bg = __bfloat162float(p.bias[static_cast<size_t>(e) * p.N + c]);
                    const float bu = __bfloat162float(p.bias[static_cast<size_t>(e) * p.N + I + c]);
#pragma unroll
                    for (int t = 0; t < kNT; ++t) {
                        acc0[t] += bg;
                        acc1[t] += bu;
                    }
                }
#pragma unroll
                for (int t = 0; t < kNT; ++t) acc0[t] = silu(acc0[t]) * acc1[t];
                // per token, the maximum over the 128 act columns of this tile (four warps)
                const int buf = tile & 1;
                if (tile >= 2 && !mbar_wait(&amax_free[buf], ((tile >> 1) + 1) & 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int t = 0; t < kNT; ++t) {
                    const float m = warp_max(fabsf(acc0[t]));
                    if (lane == t) s_amax[(buf * 4 + quad) * kNT + t] = m;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&amax_bar[buf]);
                if (!mbar_wait(&amax_bar[buf], (tile >> 1) & 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                float sc[kNT];
#pragma unroll
                for (int t = 0; t < kNT; ++t) {
                    float m = s_amax[(buf * 4 + 0) * kNT + t];
#pragma unroll
                    for (int q = 1; q < 4; ++q) m = fmaxf(m, s_amax[(buf * 4 + q) * kNT + t]);
                    sc[t] = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&amax_free[buf]);
#pragma unroll
                for (int t = 0; t < kNT; ++t) {
                    if (t < cnt) {
                        const size_t r = static_cast<size_t>(row0 + t);
                        p.act_q[r * I + c] = static_cast<uint8_t>(e4m3x2(__fdiv_rn(acc0[t], sc[t]), 0.0f) & 0xFFu);
                        if (quad == 0 && lane == 0)
                            static_cast<float*>(p.act_s)[static_cast<size_t>(wb) * p.a_pad + r] = sc[t];
                    }
                }
            } else {
                const int n0 = wb * 256 + j, n1 = n0 + 128;
                float b0 = 0.0f, b1 = 0.0f;
                if (p.bias) {
                    if (n0 < p.N) b0 = __bfloat162float(p.bias[static_cast<size_t>(e) * p.N + n0]);
                    if (n1 < p.N) b1 = __bfloat162float(p.bias[static_cast<size_t>(e) * p.N + n1]);
                }
#pragma unroll
                for (int t = 0; t < kNT; ++t) {
                    if (t < cnt) {
                        float* orow = p.out + static_cast<size_t>(row0 + t) * p.N;
                        if (n0 < p.N) orow[n0] = p.bias ? acc0[t] + b0 : acc0[t];
                        if (n1 < p.N) orow[n1] = p.bias ? acc1[t] + b1 : acc1[t];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kNTmemCols);
    }
}

template <int MODE>
static cudaError_t launch_narrow_t(const GemmArgs& a, const CUtensorMap& tmW, const CUtensorMap& tmT, int num_sms,
                                   cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm_narrow<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kNSmemBytes));
    if (e != cudaSuccess) return e;
    return launch_pdl(k_grouped_gemm_narrow<MODE>, dim3(num_sms), dim3(kNThreads), kNSmemBytes, s, tmW,
                      tmT, a);
}

cudaError_t launch_gemm_narrow(const GemmArgs& a, const CUtensorMap& tmW, const CUtensorMap& tmT, int num_sms,
                               cudaStream_t s) {
    if (a.recipe != 0) return cudaErrorInvalidValue;   // MXFP8 runs gemm_mx.cu
    return a.mode == 0 ? launch_narrow_t<0>(a, tmW, tmT, num_sms, s) : launch_narrow_t<1>(a, tmW, tmT, num_sms, s);
}

}  // namespace moe
