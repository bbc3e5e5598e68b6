// gemm_mx_narrow.cu -- the block-scaled grouped GEMMs (MXFP8, and W4A8 with E2M1 weights) for
// problems with few routed rows per expert (decode), in the swap-AB orientation: 128 rows of the
// expert's transformed weights are the MMA's M operand and up to 32 of its routed rows (tokens)
// the N operand, so a tile computes no padding rows when an expert has only a few tokens
// ("DeepGEMM PR #371", Changes: UE8M0 scale factors, W4A8 e2m1 weights; "MindIE-SD Fused MoE",
// W8A8_MXFP8; "metrale_model_layers fp8_grouped_tc_w8a8.rs", run_fp8_grouped_w8a8).
//
// tcgen05.mma.kind::mxf8f6f4.block_scale, M = 128 (weights: E4M3, or E2M1 spread by the tensor
// map over 16-byte slots), N = 32 (tokens, E4M3), K = 32; the scale factors ride in TMEM:
//   A (weights): the transformed 512-byte atoms, one per 128 rows and 128-deep stage, copied by
//                tcgen05.cp (lane i, column c, byte k = scale of row 32c + i, block k);
//   B (tokens):  an atom built per stage by one warp: row i's first word = the four UE8M0 bytes of
//                token i for the stage's four 32-deep blocks (the MMA reads column 0 for N = 32).
// The whole K accumulates in TMEM (the tensor core applies 2^(ea + ew) per 32-deep block), so the
// epilogue runs once per tile:
//   mode 0: the 128 transformed rows are [gate 32 | up 32 | gate 32 | up 32] (32-column blocks of
//           the transform); the up quadrants hand their values to the gate quadrants through
//           shared memory, which apply silu(gate) * up (+ b13) and requantize per (token, 32 act
//           columns) with a UE8M0 power of two, as the wide MXFP8 kernel does.
//   mode 1: o[token, n] (+ b2), fp32, one row of 32 consecutive columns per warp and token.
// Threads: warp 0 TMA producer, warp 1 MMA issuer, warp 2 token scale atoms, warp 3 idle,
// warps 4-7 epilogue (warp w: TMEM lane quadrant w % 4).  Four TMEM accumulators; every wait
// bounded.
#include <math.h>

#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kQT = 32;                            // tokens per tile (MMA N)
constexpr int kQStages = 8;
constexpr int kQThreads = 256;
constexpr int kQBuf = 4;                           // TMEM accumulators
constexpr uint32_t kQA = kTileM * kTileK;          // 16 KB of weights in shared memory per stage
constexpr uint32_t kQB = kQT * kTileK;             // 4 KB of token rows per stage
constexpr uint32_t kQSf = 512;
constexpr uint32_t kQStage = 22528;                // [A 16 KB | B 4 KB | SFA | SFB | pad], 1024-aligned
constexpr uint32_t kQSfCol0 = kQBuf * kQT;         // scale factors after the accumulators: 8 columns a stage
constexpr uint32_t kQTmemCols = 256;
static_assert(kQSfCol0 + kQStages * 8 <= kQTmemCols, "TMEM");

struct QL {
    static constexpr uint32_t b = kQA;
    static constexpr uint32_t sfa = kQA + kQB;
    static constexpr uint32_t sfb = sfa + kQSf;
    static constexpr uint32_t bars = kQStages * kQStage;
    // barriers: full, sfready, empty [kQStages]; tfull, tempty [kQBuf]; drain; xfull, xfree [2]
    static constexpr uint32_t nbars = 3 * kQStages + 2 * kQBuf + 1 + 4;
    static constexpr uint32_t misc = bars + nbars * 8;                // tmem holder, abort flag
    static constexpr uint32_t xch = misc + 16;                        // float [2 bufs][2 pairs][32 lanes][kQT + 1]
    static constexpr uint32_t ustart = xch + 2 * 2 * 32 * (kQT + 1) * 4;
    static constexpr uint32_t off = ustart + (MOE_MAX_EXPERTS + 2) * 4;   // experts + a shared one, + 1
    static constexpr uint32_t end = off + (MOE_MAX_EXPERTS + 2) * 4;
};
static_assert(QL::sfb + kQSf <= kQStage, "stage layout");
static_assert(kQStage % 1024 == 0, "stage alignment");
constexpr uint32_t kQSmemBytes = QL::end + 1024;
static_assert(kQSmemBytes <= 232448, "shared memory");

// Unit u -> (expert e, 128-row weight block nb, token block tb); expert e owns
// nt * ceil(rows / kQT) units from ustart[e], weight block by weight block.
__device__ __forceinline__ void decode_unit_q(int u, const int* ustart, const int* off, int E, int& e, int& nb,
                                              int& tb) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ustart[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    e = lo;
    const int ntb = (off[e + 1] - off[e] + kQT - 1) / kQT;
    const int local = u - ustart[e];
    nb = local / ntb;
    tb = local - nb * ntb;
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kQThreads, 1)
    k_grouped_gemm_mx_narrow(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmT,
                             const GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    const int nt = p.N / kTileM;                   // 128-row weight blocks per expert

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + QL::bars);
    uint64_t* sfready = full + kQStages;
    uint64_t* empty = sfready + kQStages;
    uint64_t* tfull = empty + kQStages;
    uint64_t* tempty = tfull + kQBuf;
    uint64_t* drain = tempty + kQBuf;
    uint64_t* xfull = drain + 1;                   // mode 0: the up quadrants' values are in s_xch
    uint64_t* xfree = xfull + 2;                   // mode 0: the gate quadrants have read them
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + QL::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + QL::misc + 4);
    float* s_xch = reinterpret_cast<float*>(smem + QL::xch);
    int* s_ustart = reinterpret_cast<int*>(smem + QL::ustart);
    int* s_off = reinterpret_cast<int*>(smem + QL::off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sfready[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < kQBuf; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(drain, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&xfull[b], 2);
            mbar_init(&xfree[b], 2);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmW);
        prefetch_tmap(&tmT);
    }
    if (warp == 1) tmem_alloc(tmem_holder, kQTmemCols);
    if (warp == 0) {   // the first unit's weight tiles toward L2 while the preceding kernel runs
        int e, nb;
        if (early_unit_rows<kQT>(p.offsets, p.E, nt, blockIdx.x, lane, e, nb) && lane == 0)
            prefetch_weight_stages(&tmW, e * p.N + nb * kTileM, p.K);
    }
    pdl_wait_then_release();
    for (int i = threadIdx.x; i <= p.E; i += kQThreads) s_off[i] = p.offsets[i];
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int e = 0; e < p.E; ++e) {
            s_ustart[e] = acc;
            acc += nt * ((s_off[e + 1] - s_off[e] + kQT - 1) / kQT);
        }
        s_ustart[p.E] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int total_units = s_ustart[p.E];
    const int KB = p.K / kTileK;
    const bool fp4 = p.recipe == 2;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------------ TMA producer
            const uint32_t a_bytes = fp4 ? kQA / 2 : kQA;   // E2M1 weights arrive packed
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                int e, nb, tb;
                decode_unit_q(u, s_ustart, s_off, p.E, e, nb, tb);
                const int row0 = s_off[e] + tb * kQT;
                const int wrow0 = e * p.N + nb * kTileM;
                const uint8_t* sfa_src = static_cast<const uint8_t*>(p.w_scale) +
                                         (static_cast<size_t>(e) * nt + nb) * KB * kQSf;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % kQStages;
                    if (!mbar_wait<kProducerSleepNs>(&empty[s], ((it / kQStages) & 1) ^ 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    if (fault_skip_stage(p.fault, it)) continue;   // debug builds: an injected fault
                    uint8_t* st = smem + s * kQStage;
                    mbar_arrive_expect_tx(&full[s], a_bytes + kQB + kQSf);
                    tma_load_2d(st, &tmW, kb * kTileK, wrow0, &full[s]);
                    tma_load_2d(st + QL::b, &tmT, kb * kTileK, row0, &full[s]);
                    bulk_load(st + QL::sfa, sfa_src + static_cast<size_t>(kb) * kQSf, kQSf, &full[s]);
                }
            }
            if (!ok) {
                const uint32_t n = it < static_cast<uint32_t>(kQStages) ? it : kQStages;
                for (uint32_t i = it - n; i < it; ++i) drain_wait(&full[i % kQStages], (i / kQStages) & 1);
            }
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------------------- token scale atoms
        // lane i writes row i of the stage's B atom: token row0 + i's four UE8M0 bytes (one word).
        // Words are gathered two stages ahead by an iterator that decodes each unit once.
        constexpr int kAhead = 2;
        const int my_units = total_units > static_cast<int>(blockIdx.x)
                                 ? (total_units - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                                 : 0;
        const int n_stages = my_units * KB;
        int gu = static_cast<int>(blockIdx.x), gkb = 0, grow0 = 0;
        if (gu < total_units) {
            int e, nb, tb;
            decode_unit_q(gu, s_ustart, s_off, p.E, e, nb, tb);
            grow0 = s_off[e] + tb * kQT;
        }
        auto gather = [&]() {
            uint32_t w = 0u;
            if (gu < total_units) {
                w = __ldg(static_cast<const uint32_t*>(p.a_scale) + static_cast<size_t>(gkb) * p.a_pad + grow0 + lane);
                if (++gkb == KB) {
                    gkb = 0;
                    gu += static_cast<int>(gridDim.x);
                    if (gu < total_units) {
                        int e, nb, tb;
                        decode_unit_q(gu, s_ustart, s_off, p.E, e, nb, tb);
                        grow0 = s_off[e] + tb * kQT;
                    }
                }
            }
            return w;
        };
        uint32_t ring[kAhead];
#pragma unroll
        for (int d = 0; d < kAhead; ++d) ring[d] = gather();
        bool ok = true;
        for (int base = 0; base < n_stages && ok; base += kAhead) {
#pragma unroll
            for (int d = 0; d < kAhead; ++d) {
                const int it = base + d;
                if (it >= n_stages) break;
                const uint32_t w = ring[d];
                ring[d] = gather();
                const int s = it % kQStages;
                if (!mbar_wait<kProducerSleepNs>(&empty[s], ((it / kQStages) & 1) ^ 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                *reinterpret_cast<uint32_t*>(smem + s * kQStage + QL::sfb + 16 * lane) = w;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to tcgen05.cp
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfready[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------------ MMA issuer
            const uint32_t afmt = fp4 ? 5u : 0u;
            uint32_t it = 0, tile = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++tile) {
                const int b = tile % kQBuf;
                if (!mbar_wait<kIssuerSleepNs>(&tempty[b], ((tile / kQBuf) & 1) ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(b * kQT);
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % kQStages;
                    if (!mbar_wait<kIssuerSleepNs>(&full[s], (it / kQStages) & 1, abort_flag, p.status) ||
                        !mbar_wait<kIssuerSleepNs>(&sfready[s], (it / kQStages) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * kQStage);
                    const uint32_t sfa_t = tmem_base + kQSfCol0 + static_cast<uint32_t>(s * 8);
                    const uint32_t sfb_t = sfa_t + 4;
                    sf_copy(sfa_t, sf_atom_desc(st + QL::sfa));
                    sf_copy(sfb_t, sf_atom_desc(st + QL::sfb));
#pragma unroll
                    for (uint32_t k = 0; k < 4; ++k)
                        mma_mx(d, sw128_kmajor_desc(st + k * 32), sw128_kmajor_desc(st + QL::b + k * 32),
                               mx_block_idesc(k, afmt, 0u, kTileM, kQT), sfa_t, sfb_t, (kb > 0 || k > 0) ? 1u : 0u);
                    mma_commit(&empty[s]);
                }
                if (!ok) break;
                mma_commit(&tfull[b]);
            }
            mma_commit(drain);
            drain_wait(drain, 0);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------------- epilogue
        const int quad = warp & 3;                // TMEM lanes 32*quad .. +31 = weight rows of the tile
        uint32_t tile = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++tile) {
            int e, nb, tb;
            decode_unit_q(u, s_ustart, s_off, p.E, e, nb, tb);
            const int row0 = s_off[e] + tb * kQT;
            const int cnt = min(kQT, s_off[e + 1] - row0);
            const int b = tile % kQBuf;
            if (!mbar_wait(&tfull[b], (tile / kQBuf) & 1, abort_flag, p.status)) break;
            tc_fence_after();
            uint32_t v[32];
            MOE_TMEM_LD32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(b * kQT), v);
            MOE_TMEM_WAIT_LD(v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);     // the accumulator may be refilled now

            if (MODE == 0) {
                // lanes of quadrants 0 / 2: gate rows of act columns c0 + lane; 1 / 3: the matching up rows
                const int I = p.N >> 1;
                const int pair = quad >> 1;
                const int c = (nb >> 1) * 128 + (nb & 1) * 64 + pair * 32 + lane;
                const int xb = tile & 1;
                float* x = s_xch + ((xb * 2 + pair) * 32 + lane) * (kQT + 1);
                if (quad & 1) {
                    // hand the up values over (once the gate quadrants have read this buffer's last use)
                    if (tile >= 2 && !mbar_wait(&xfree[xb], ((tile >> 1) + 1) & 1, abort_flag, p.status)) break;
#pragma unroll
                    for (int t = 0; t < kQT; ++t) x[t] = __uint_as_float(v[t]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&xfull[xb]);
                } else {
                    if (!mbar_wait(&xfull[xb], (tile >> 1) & 1, abort_flag, p.status)) break;
                    float bg = 0.0f, bu = 0.0f;
                    if (p.bias) {
                        bg = __bfloat162float(p.bias[static_cast<size_t>(e) * p.N + c]);
                        bu = __bfloat162float(p.bias[static_cast<size_t>(e) * p.N + I + c]);
                    }
                    uint8_t* act_s = static_cast<uint8_t*>(p.act_s);
#pragma unroll
                    for (int t = 0; t < kQT; ++t) {
                        float g = __uint_as_float(v[t]), up = x[t];
                        if (p.bias) {
                            g += bg;
                            up += bu;
                        }
                        const float a = silu(g) * up;
                        const float amax = warp_max(fabsf(a));     // the token's 32 act columns
                        if (t < cnt) {
                            const int ex = mx_exponent(amax);
                            const size_t r = static_cast<size_t>(row0 + t);
                            p.act_q[r * I + c] = static_cast<uint8_t>(e4m3x2(a * exp2_int(-ex), 0.0f) & 0xFFu);
                            if (lane == 0)
                                act_s[(static_cast<size_t>(c >> 7) * p.a_pad + r) * 4 + ((c & 127) >> 5)] =
                                    static_cast<uint8_t>(ex + 127);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&xfree[xb]);   // this buffer may be rewritten
                }
            } else {
                const int n = nb * kTileM + quad * 32 + lane;
                const float bn = p.bias ? __bfloat162float(p.bias[static_cast<size_t>(e) * p.N + n]) : 0.0f;
#pragma unroll
                for (int t = 0; t < kQT; ++t)
                    if (t < cnt) p.out[static_cast<size_t>(row0 + t) * p.N + n] = __uint_as_float(v[t]) + bn;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kQTmemCols);
    }
}

template <int MODE>
static cudaError_t launch_mxq_t(const GemmArgs& a, const CUtensorMap& tmW, const CUtensorMap& tmT, int num_sms,
                                cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm_mx_narrow<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kQSmemBytes));
    if (e != cudaSuccess) return e;
    return launch_pdl(k_grouped_gemm_mx_narrow<MODE>, dim3(num_sms), dim3(kQThreads), kQSmemBytes, s, tmW, tmT, a);
}

// Token rows per tile of the swap-AB block-scaled kernels (the token tensor map's box).
uint32_t gemm_mx_narrow_tokens() { return static_cast<uint32_t>(kQT); }

cudaError_t launch_gemm_mx_narrow(const GemmArgs& a, const CUtensorMap& tmW, const CUtensorMap& tmT, int num_sms,
                                  cudaStream_t s) {
    if (a.recipe == 0 || a.N % kTileM != 0) return cudaErrorInvalidValue;
    return a.mode == 0 ? launch_mxq_t<0>(a, tmW, tmT, num_sms, s) : launch_mxq_t<1>(a, tmW, tmT, num_sms, s);
}

}  // namespace moe
