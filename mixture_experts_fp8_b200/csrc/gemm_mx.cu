// gemm_mx.cu -- grouped MXFP8 GEMMs on the block-scaled tensor core instruction
// (tcgen05.mma.kind::mxf8f6f4.block_scale): E4M3 operands with one UE8M0 power-of-two scale per
// 32 K-elements, for rows and for weight columns ("DeepGEMM PR #371", Changes: UE8M0 scale
// factors, 4 packed per 32-bit word, scale-factor tensors moved by TMA; "MindIE-SD Fused MoE",
// W8A8_MXFP8).  The W4A8 recipe runs the same kernel with E2M1 weights: the weight tensor map
// reads them packed two per byte from HBM and spreads each 16 codes over a 16-byte slot of
// shared memory (the layout the instruction takes for 4-bit operands), the instruction
// descriptor names E2M1 for B, and the stage expects half the weight bytes.  The tensor core applies 2^(ea + ew) to every 32-deep product block itself and
// accumulates the whole K in TMEM, so there is no per-group promotion:
//   mode 0: h = sum_k dec(a) 2^ea dec(w) 2^ew (+ b13); act = silu(h_gate) * h_up, requantized
//           to E4M3 with a UE8M0 scale per 32 act columns
//   mode 1: o = sum_k ... (+ b2), fp32 rows
//
// Scale factors in TMEM (per 128 rows and one 128-deep stage: 4 columns x 128 lanes): the
// 512-byte atom byte[16*i + 4*c + k] = scale of row (32*c + i) for the stage's K-block k is copied
// by tcgen05.cp.32x128b.warpx4, which puts its 32 rows of 16 bytes into every lane quadrant; the
// MMA for K-block k selects byte k (the instruction descriptor's scale-factor id).
//   weights: atoms prepared once by moe_transform_weights, [E][N/128][K/128][512 B];
//   rows:    gathered per stage by one warp from the K-block-major scale words ([K/128][a_pad],
//            word = the row's four scale bytes for that stage), since an expert's rows start at
//            any offset.
// Threads (384): warp 0 TMA producer, warp 1 MMA issuer, warp 2 row-scale atoms, warp 3 idle,
// warps 4-11 epilogue (warp w: TMEM lanes 32*(w%4).., half of the 128 columns).  Tile 128 x 128,
// two TMEM accumulators so a tile's epilogue overlaps the next tile's MMAs.  Every wait bounded.
#include <math.h>

#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kXStages = 6;
constexpr int kXThreads = 384;
constexpr int kXEpiWarps = 8;
constexpr int kXN = 128;                          // tile columns
constexpr uint32_t kXA = kTileM * kTileK;         // 16 KB
constexpr uint32_t kXB = kXN * kTileK;            // 16 KB
constexpr uint32_t kXSf = 512;                    // one scale-factor atom
constexpr uint32_t kXStage = kXA + kXB + 2 * kXSf + 1024;   // [A | B | SFA atom | SFB atom | pad]
constexpr uint32_t kXAccCols = 2 * kXN;           // two fp32 accumulators
constexpr uint32_t kXSfCol0 = kXAccCols;          // scale factors after them: 8 columns per stage
constexpr uint32_t kXTmemCols = 512;
static_assert(kXSfCol0 + kXStages * 8 <= kXTmemCols, "TMEM");

struct XL {
    static constexpr uint32_t b = kXA;
    static constexpr uint32_t sfa = kXA + kXB;
    static constexpr uint32_t sfb = sfa + kXSf;
    static constexpr uint32_t bars = kXStages * kXStage;
    static constexpr uint32_t nbars = 3 * kXStages + 5;   // full, sfready, empty, tfull[2], tempty[2], drain
    static constexpr uint32_t misc = bars + nbars * 8;
    static constexpr uint32_t tstart = misc + 16;
    static constexpr uint32_t off = tstart + (MOE_MAX_EXPERTS + 2) * 4;   // experts + a shared one, + 1
    static constexpr uint32_t end = off + (MOE_MAX_EXPERTS + 2) * 4;   // experts + a shared one, + 1
};
static_assert(kXStage % 1024 == 0, "stage alignment");
constexpr uint32_t kXSmemBytes = XL::end + 1024;
static_assert(kXSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ void decode_unit_x(int u, int nt, const int* tstart, int E, int& e, int& nb, int& mb) {
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

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kXThreads, 1)
    k_grouped_gemm_mx(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    const int nt = p.N / kXN;

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + XL::bars);
    uint64_t* sfready = full + kXStages;
    uint64_t* empty = sfready + kXStages;
    uint64_t* tfull = empty + kXStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + XL::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + XL::misc + 4);
    int* s_tstart = reinterpret_cast<int*>(smem + XL::tstart);
    int* s_off = reinterpret_cast<int*>(smem + XL::off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kXStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sfready[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kXEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) tmem_alloc(tmem_holder, kXTmemCols);
    if (warp == 0) {   // the first unit's weight tiles toward L2 while the preceding kernel runs
        int e, nb;
        if (early_unit_tiles(p.tile_start, p.E, nt, blockIdx.x, lane, e, nb) && lane == 0)
            prefetch_weight_stages(&tmB, e * p.N + nb * kXN, p.K);
    }
    pdl_wait_then_release();
    for (int i = threadIdx.x; i <= p.E; i += kXThreads) {
        s_tstart[i] = p.tile_start[i];
        s_off[i] = p.offsets[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int total_units = s_tstart[p.E] * nt;
    const int KB = p.K / kTileK;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------------ TMA producer
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                int e, nb, mb;
                decode_unit_x(u, nt, s_tstart, p.E, e, nb, mb);
                const int row0 = s_off[e] + mb * kTileM;
                const int brow0 = e * p.N + nb * kXN;
                const uint8_t* sfb_src = static_cast<const uint8_t*>(p.w_scale) +
                                         (static_cast<size_t>(e) * nt + nb) * KB * kXSf;
                // E2M1 weights arrive packed: the copy moves (and signals) half the bytes
                const uint32_t b_bytes = p.recipe == 2 ? kXB / 2 : kXB;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % kXStages;
                    if (!mbar_wait<kProducerSleepNs>(&empty[s], ((it / kXStages) & 1) ^ 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    if (fault_skip_stage(p.fault, it)) continue;   // debug builds: an injected fault
                    uint8_t* st = smem + s * kXStage;
                    mbar_arrive_expect_tx(&full[s], kXA + b_bytes + kXSf);
                    tma_load_2d(st, &tmA, kb * kTileK, row0, &full[s]);
                    tma_load_2d(st + XL::b, &tmB, kb * kTileK, brow0, &full[s]);
                    bulk_load(st + XL::sfb, sfb_src + static_cast<size_t>(kb) * kXSf, kXSf, &full[s]);
                }
            }
            if (!ok) {
                const uint32_t n = it < static_cast<uint32_t>(kXStages) ? it : kXStages;
                for (uint32_t i = it - n; i < it; ++i) drain_wait(&full[i % kXStages], (i / kXStages) & 1);
            }
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------------------- row-scale atoms
        // lane i writes the atom's row i: the scale words of tile rows i, 32+i, 64+i, 96+i.  The
        // words are gathered kSfAhead stages ahead of the stage being written (a register ring)
        // by an iterator that decodes each unit once, so the gather's global-load latency is not
        // paid once per stage.
        constexpr int kSfAhead = 2;
        const int my_units = total_units > static_cast<int>(blockIdx.x)
                                 ? (total_units - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                                 : 0;
        const int n_stages = my_units * KB;           // stages this CTA runs, in order
        // the gather's own position (unit, stage, first row), advanced one stage per call
        int gu = static_cast<int>(blockIdx.x), gkb = 0, grow0 = 0;
        if (gu < total_units) {
            int e, nb, mb;
            decode_unit_x(gu, nt, s_tstart, p.E, e, nb, mb);
            grow0 = s_off[e] + mb * kTileM;
        }
        auto gather = [&]() {                         // the next stage's scale words (zeros past the end)
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (gu < total_units) {
                const uint32_t* src = static_cast<const uint32_t*>(p.a_scale) + static_cast<size_t>(gkb) * p.a_pad + grow0;
                w = make_uint4(__ldg(src + lane), __ldg(src + 32 + lane), __ldg(src + 64 + lane), __ldg(src + 96 + lane));
                if (++gkb == KB) {
                    gkb = 0;
                    gu += static_cast<int>(gridDim.x);
                    if (gu < total_units) {
                        int e, nb, mb;
                        decode_unit_x(gu, nt, s_tstart, p.E, e, nb, mb);
                        grow0 = s_off[e] + mb * kTileM;
                    }
                }
            }
            return w;
        };
        uint4 ring[kSfAhead];
#pragma unroll
        for (int d = 0; d < kSfAhead; ++d) ring[d] = gather();
        bool ok = true;
        for (int base = 0; base < n_stages && ok; base += kSfAhead) {
#pragma unroll
            for (int d = 0; d < kSfAhead; ++d) {
                const int it = base + d;
                if (it >= n_stages) break;
                const uint4 w = ring[d];
                ring[d] = gather();
                const int s = it % kXStages;
                if (!mbar_wait<kProducerSleepNs>(&empty[s], ((it / kXStages) & 1) ^ 1, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                *reinterpret_cast<uint4*>(smem + s * kXStage + XL::sfa + 16 * lane) = w;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to tcgen05.cp
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfready[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------------ MMA issuer
            uint32_t it = 0, tile = 0;
            bool ok = true;
            const uint32_t bfmt = p.recipe == 2 ? 5u : 0u;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++tile) {
                const int b = tile & 1;
                if (!mbar_wait<kIssuerSleepNs>(&tempty[b], ((tile >> 1) & 1) ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(b * kXN);
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % kXStages;
                    if (!mbar_wait<kIssuerSleepNs>(&full[s], (it / kXStages) & 1, abort_flag, p.status) ||
                        !mbar_wait<kIssuerSleepNs>(&sfready[s], (it / kXStages) & 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * kXStage);
                    const uint32_t sfa_t = tmem_base + kXSfCol0 + static_cast<uint32_t>(s * 8);
                    const uint32_t sfb_t = sfa_t + 4;
                    sf_copy(sfa_t, sf_atom_desc(st + XL::sfa));
                    sf_copy(sfb_t, sf_atom_desc(st + XL::sfb));
#pragma unroll
                    for (uint32_t k = 0; k < 4; ++k)
                        mma_mx(d, sw128_kmajor_desc(st + k * 32), sw128_kmajor_desc(st + XL::b + k * 32), mx_block_idesc(k, 0u, bfmt, kTileM, kXN),
                               sfa_t, sfb_t, (kb > 0 || k > 0) ? 1u : 0u);
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
        const int quad = warp & 3;
        const int h = (warp - 4) >> 2;            // columns h*64 .. h*64+63 of the tile
        const int row_in_tile = quad * 32 + lane;
        uint32_t tile = 0;
        for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++tile) {
            int e, nb, mb;
            decode_unit_x(u, nt, s_tstart, p.E, e, nb, mb);
            const int row0 = s_off[e] + mb * kTileM;
            const int cnt = min(kTileM, s_off[e + 1] - row0);
            const bool warp_active = quad * 32 < cnt;
            const bool row_ok = row_in_tile < cnt;
            const int r = row0 + row_in_tile;
            const int b = tile & 1;
            if (!mbar_wait(&tfull[b], (tile >> 1) & 1, abort_flag, p.status)) break;
            tc_fence_after();
            float acc[64];
            if (warp_active) {
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                       static_cast<uint32_t>(b * kXN + h * 64);
                uint32_t v[32], w[32];
                MOE_TMEM_LD32(taddr, v);
                MOE_TMEM_LD32(taddr + 32, w);
                MOE_TMEM_WAIT_LD(v);
                MOE_TMEM_WAIT_LD(w);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    acc[i] = __uint_as_float(v[i]);
                    acc[32 + i] = __uint_as_float(w[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);     // the accumulator may be refilled now
            if (!warp_active || !row_ok) continue;

            if (MODE == 0) {
                // tile columns h*64 .. +63 = [gate 32 | up 32] of act columns c0 .. c0+31
                const int I = p.N >> 1;
                const int c0 = (nb >> 1) * 128 + (nb & 1) * 64 + h * 32;
                if (p.bias) {
                    add_bias32(acc, p.bias + static_cast<size_t>(e) * p.N + c0);
                    add_bias32(acc + 32, p.bias + static_cast<size_t>(e) * p.N + I + c0);
                }
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    acc[i] = silu(acc[i]) * acc[32 + i];
                    amax = fmaxf(amax, fabsf(acc[i]));
                }
                const int ex = mx_exponent(amax);
                const float inv = exp2_int(-ex);
                uint32_t q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    q[i] = e4m3x4(acc[4 * i] * inv, acc[4 * i + 1] * inv, acc[4 * i + 2] * inv, acc[4 * i + 3] * inv);
                uint4* d4 = reinterpret_cast<uint4*>(p.act_q + static_cast<size_t>(r) * I + c0);
                d4[0] = make_uint4(q[0], q[1], q[2], q[3]);
                d4[1] = make_uint4(q[4], q[5], q[6], q[7]);
                static_cast<uint8_t*>(p.act_s)[(static_cast<size_t>(nb >> 1) * p.a_pad + r) * 4 + (nb & 1) * 2 + h] =
                    static_cast<uint8_t>(ex + 127);
            } else {
                const int c0 = nb * kXN + h * 64;
                if (p.bias) {
                    add_bias32(acc, p.bias + static_cast<size_t>(e) * p.N + c0);
                    add_bias32(acc + 32, p.bias + static_cast<size_t>(e) * p.N + c0 + 32);
                }
                float* dst = p.out + static_cast<size_t>(r) * p.N + c0;
#pragma unroll
                for (int c = 0; c < 64; c += 8) st_global_f32x8(dst + c, acc + c);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kXTmemCols);
    }
}

template <int MODE>
static cudaError_t launch_mx_t(const GemmArgs& a, const CUtensorMap& tmA, const CUtensorMap& tmB, int num_sms,
                               cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm_mx<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kXSmemBytes));
    if (e != cudaSuccess) return e;
    return launch_pdl(k_grouped_gemm_mx<MODE>, dim3(num_sms), dim3(kXThreads), kXSmemBytes, s, tmA, tmB, a);
}

cudaError_t launch_gemm_mx(const GemmArgs& a, const CUtensorMap& tmA, const CUtensorMap& tmB, int num_sms,
                           cudaStream_t s) {
    return a.mode == 0 ? launch_mx_t<0>(a, tmA, tmB, num_sms, s) : launch_mx_t<1>(a, tmA, tmB, num_sms, s);
}

}  // namespace moe
