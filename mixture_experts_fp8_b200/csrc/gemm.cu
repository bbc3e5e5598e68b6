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
// What bounds it: the scales vary with the row, the column and the 128-deep group, so every group
// partial leaves the tensor core and is multiplied in, acc += P * (a_s * w_s): two fp32
// operations per output element per group, as much FP32-pipe time as the MMAs themselves.  The
// epilogue therefore keeps its per-group bookkeeping to a few instructions: one predicated barrier
// arrival per warp (no divergent branches), no per-row predicates in the group loop, stage and
// phase counters carried incrementally, 32-bit shared-memory addresses.
//
// Design (one persistent CTA per SM, 640 threads = five warpgroups):
//   warp 0   TMA producer: per 128-deep K stage, a 128x128 A tile and a 256x128 B tile (both
//            K-major, 128-byte swizzle), the 256 weight scales of the stage and the tile rows'
//            activation scales (bulk copies).
//   warp 1   MMA issuer (one thread): tcgen05.mma.kind::f8f6f4, M=128 N=256 K=32.  Each 128-deep
//            scale group is accumulated alone into one of two 256-column fp32 TMEM buffers.
//   warps 2-3 idle.  Warpgroup 0 gives registers back (setmaxnreg.dec to 32).
//   warps 4-19 epilogue (setmaxnreg.inc to 112): warp w reads TMEM lanes 32*(w%4) .. +31 (tile
//            rows) and columns 32q .. +31 and 128 + 32q .. +31 of the tile, q = (w-4)/4; with
//            w13's gate and up columns in 128-column blocks these are the gate and the up
//            projections of the same 32 act columns.  Every group partial is multiplied by
//            a_s * w_s and added into 64 fp32 registers (the "promotion"), then the tile's
//            epilogue runs from registers.
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
constexpr int kCols = kTileN / 4;                  // columns per epilogue thread (32 per half)
constexpr int kHalf = kTileN / 2;
// Registers: 640 threads launch with 96 each (5 warps per SM sub-partition); warpgroup 0 keeps
// 32, the four epilogue warpgroups take 112: 128 * 32 + 512 * 112 = 640 * 96.
constexpr int kRegsLaunch = 96, kRegsLow = 32, kRegsHigh = 112;
static_assert(128 * kRegsLow + 512 * kRegsHigh == kThreads * kRegsLaunch, "register split");
constexpr uint32_t kABytes = kTileM * kTileK;      // 16 KB
constexpr uint32_t kBBytes = kTileN * kTileK;      // 32 KB
constexpr uint32_t kWsBytes = kTileN * 4;          // weight scales of the 256 columns
constexpr uint32_t kSaWords = kTileM + 4;          // activation scales of the tile's rows (+ 16-byte alignment)
constexpr uint32_t kSaBytes = kSaWords * 4;
constexpr uint32_t kScaleSlot = 2048;              // per stage: [weight scales | activation scales]
constexpr uint32_t kTmemCols = 2 * kTileN;         // two fp32 accumulators

struct L {
    static constexpr uint32_t a = 0;
    static constexpr uint32_t b = a + kStages * kABytes;
    static constexpr uint32_t sc = b + kStages * kBBytes;
    // barriers: full[kStages], empty[kStages], tfull[2], tempty[2], drain, amax[2]
    static constexpr uint32_t full = sc + kStages * kScaleSlot;
    static constexpr uint32_t empty = full + 8 * kStages;
    static constexpr uint32_t tfull = empty + 8 * kStages;
    static constexpr uint32_t tempty = tfull + 16;
    static constexpr uint32_t drain = tempty + 16;
    static constexpr uint32_t amax_bar = drain + 8;
    static constexpr uint32_t misc = amax_bar + 16;      // tmem holder, abort flag
    static constexpr uint32_t amax = misc + 16;          // float [2 buffers][4 quarters][128 rows]
    static constexpr uint32_t tstart = amax + 2 * 4 * 128 * 4;
    static constexpr uint32_t off = tstart + (MOE_MAX_EXPERTS + 2) * 4;   // experts + a shared one, + 1
    static constexpr uint32_t end = off + (MOE_MAX_EXPERTS + 2) * 4;   // experts + a shared one, + 1
};
static_assert(kWsBytes + kSaBytes <= kScaleSlot, "scale slot");
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

// acc[a0 + j] += P[j] * (sa * ws[j]) for j < 16, with P in v and ws[] at shared address ws; packed
// fp32x2 multiply and FMA (each lane rounds as the scalar operations would).
__device__ __forceinline__ void fma_chunk16(float2 (&acc)[kCols / 2], const uint32_t (&v)[16], uint32_t ws,
                                            int a0, float2 sa2) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const float4 w4 = ld_shared_f32x4(ws + 4 * j);
        const float2 s0 = __fmul2_rn(make_float2(w4.x, w4.y), sa2);
        const float2 s1 = __fmul2_rn(make_float2(w4.z, w4.w), sa2);
        acc[(a0 + j) / 2] = __ffma2_rn(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])), s0,
                                       acc[(a0 + j) / 2]);
        acc[(a0 + j) / 2 + 1] = __ffma2_rn(make_float2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])), s1,
                                           acc[(a0 + j) / 2 + 1]);
    }
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
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::full);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::empty);
    uint64_t* tfull = reinterpret_cast<uint64_t*>(smem + L::tfull);
    uint64_t* tempty = reinterpret_cast<uint64_t*>(smem + L::tempty);
    uint64_t* drain = reinterpret_cast<uint64_t*>(smem + L::drain);
    uint64_t* amax_bar = reinterpret_cast<uint64_t*>(smem + L::amax_bar);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc + 4);
    float* s_amax = reinterpret_cast<float*>(smem + L::amax);
    int* s_tstart = reinterpret_cast<int*>(smem + L::tstart);
    int* s_off = reinterpret_cast<int*>(smem + L::off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + kEpiWarps);   // the MMA commit + one arrival per epilogue warp
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
    if (warp == 0) {   // the first unit's weight tiles toward L2 while the preceding kernel runs
        int e, nb;
        if (early_unit_tiles(p.tile_start, p.E, nt, blockIdx.x, lane, e, nb) && lane == 0)
            prefetch_weight_stages(&tmB, e * p.N + nb * kTileN, p.K);
    }
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
    const int KB = p.K / kTileK;                 // pipeline stages = scale groups per unit
    constexpr int MPG = kTileK / 32;             // K=32 MMAs per scale group

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
                    if (!mbar_wait<kProducerSleepNs>(&empty[s], ((it / kStages) & 1) ^ 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    if (fault_skip_stage(p.fault, it)) continue;   // debug builds: an injected fault
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
            // descriptors of stage 0; a stage or a K step moves the start address field (bits
            // 0..13, address / 16) by a fixed amount that never carries out of it
            const uint64_t a_desc0 = sw128_kmajor_desc(smem_u32(smem + L::a));
            const uint64_t b_desc0 = sw128_kmajor_desc(smem_u32(smem + L::b));
            uint32_t s = 0, ph = 0, buf = 0, bph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait<kIssuerSleepNs>(&full[s], ph, abort_flag, p.status) ||
                        !mbar_wait<kIssuerSleepNs>(&tempty[buf], bph ^ 1, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = a_desc0 + s * (kABytes >> 4), bd = b_desc0 + s * (kBBytes >> 4);
                    const uint32_t d = tmem_base + buf * static_cast<uint32_t>(kTileN);
#pragma unroll
                    for (int m = 0; m < MPG; ++m) mma_f8(d, ad + 2 * m, bd + 2 * m, idesc, m > 0 ? 1u : 0u);
                    mma_commit(&tfull[buf]);
                    mma_commit(&empty[s]);
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1;
                    }
                    buf ^= 1;
                    bph ^= buf ^ 1;   // flips after both buffers were used
                }
            }
            mma_commit(drain);          // all MMAs issued by this thread have finished
            drain_wait(drain, 0);
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
        // ------------------------------------------------------------------ epilogue
        const int quad = warp & 3;                // TMEM lanes 32*quad .. 32*quad+31
        const int qtr = (warp - kFirstEpiWarp) >> 2;
        const int row_in_tile = quad * 32 + lane;
        // TMEM address of this thread's columns 32q.. (half 0) in buffer 0; its half-1 columns
        // are 128 further.  Shared-memory addresses of its weight scales and of the activation-
        // scale run in stage 0.
        const uint32_t t_warp = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(32 * qtr);
        const uint32_t ws0 = smem_u32(smem + L::sc) + static_cast<uint32_t>(32 * qtr * 4);
        const uint32_t sa0 = smem_u32(smem + L::sc + kWsBytes) + static_cast<uint32_t>(row_in_tile * 4);
        const uint32_t full0 = smem_u32(full), empty0 = smem_u32(empty);
        const uint32_t tfull0 = smem_u32(tfull), tempty0 = smem_u32(tempty);
        const uint32_t abort_at = smem_u32(smem + L::misc + 4);
        uint32_t s = 0, ph = 0, buf = 0, bph = 0, tile = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++tile) {
            uint32_t sa_addr;
            {
                int e, nb, mb;
                decode_unit(u, nt, s_tstart, p.E, e, nb, mb);
                sa_addr = sa0 + static_cast<uint32_t>(((s_off[e] + mb * kTileM) & 3) * 4);
            }

            float2 acc2[kCols / 2];
#pragma unroll
            for (int i = 0; i < kCols / 2; ++i) acc2[i] = make_float2(0.0f, 0.0f);
            float* acc = reinterpret_cast<float*>(acc2);

            for (int kb = 0; kb < KB; ++kb) {
                // the stage's scales (bulk copies), then the group partial in TMEM buffer buf
                if (!mbar_wait_at(full0 + 8 * s, ph, abort_at, p.status) ||
                    !mbar_wait_at(tfull0 + 8 * buf, bph, abort_at, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t so = s * kScaleSlot;
                const float sa = ld_shared_f32(sa_addr + so);
                const float2 sa2 = make_float2(sa, sa);
                const uint32_t ws = ws0 + so;
                const uint32_t taddr = t_warp + buf * static_cast<uint32_t>(kTileN);
                // four 16-column chunks; each chunk's read overlaps the previous chunk's arithmetic
                uint32_t va[16], vb[16];
                MOE_TMEM_LD16(taddr, va);
                MOE_TMEM_WAIT_LD16(va);
                MOE_TMEM_LD16(taddr + 16, vb);
                fma_chunk16(acc2, va, ws, 0, sa2);
                MOE_TMEM_WAIT_LD16(vb);
                MOE_TMEM_LD16(taddr + kHalf, va);
                fma_chunk16(acc2, vb, ws + 64, 16, sa2);
                MOE_TMEM_WAIT_LD16(va);
                MOE_TMEM_LD16(taddr + kHalf + 16, vb);
                fma_chunk16(acc2, va, ws + 4 * kHalf, 32, sa2);
                MOE_TMEM_WAIT_LD16(vb);
                // every read of buffer buf by this warp is complete: hand it back
                tc_fence_before();
                mbar_arrive_lane0(tempty0 + 8 * buf, lane);
                fma_chunk16(acc2, vb, ws + 4 * kHalf + 64, 48, sa2);
                // the scales were read through the generic proxy; the producer's next bulk copy
                // into this stage is an async-proxy write: order the reads before it
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive_lane0(empty0 + 8 * s, lane);   // done with the stage's scales
                if (++s == kStages) {
                    s = 0;
                    ph ^= 1;
                }
                buf ^= 1;
                bph ^= buf ^ 1;
            }
            if (!ok) break;

            int e, nb, mb;
            decode_unit(u, nt, s_tstart, p.E, e, nb, mb);
            const int row0 = s_off[e] + mb * kTileM;
            const int cnt = min(kTileM, s_off[e + 1] - row0);
            const bool row_ok = row_in_tile < cnt;
            const int r = row0 + row_in_tile;
            if (MODE == 0) {
                // ---- SwiGLU + requantization: acc[0:32] gate (half 0) and acc[32:64] up (half 1)
                // of act columns c0 .. c0+31.
                const int I = p.N >> 1;
                const int c0 = nb * 128 + qtr * 32;
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
                // one 128-column group per row: combine the four quarters' maxima
                const int ab = tile & 1;
                s_amax[(ab * 4 + qtr) * 128 + row_in_tile] = amax;
                const uint32_t amax_at = smem_u32(&amax_bar[ab]);
                __syncwarp();                          // every lane's s_amax store before the arrival
                mbar_arrive_lane0(amax_at, lane);
                if (!mbar_wait_at(amax_at, (tile >> 1) & 1, abort_at, p.status)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) amax = fmaxf(amax, s_amax[(ab * 4 + q) * 128 + row_in_tile]);
                const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                if (row_ok) {
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
                // ---- down projection: + bias, fp32 rows; acc[32h : 32h+32] are columns
                // nb*256 + 128h + 32q .. +31
                if (row_ok) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int c0 = nb * kTileN + h * kHalf + qtr * 32;
                        if (c0 < p.N) {
                            float* dst = p.out + static_cast<size_t>(r) * p.N + c0;
                            const uint4* b4 =
                                p.bias ? reinterpret_cast<const uint4*>(p.bias + static_cast<size_t>(e) * p.N + c0)
                                       : nullptr;
#pragma unroll
                            for (int c = 0; c < 32; c += 8) {   // 8 columns: one bias load, one 32-byte store
                                float* a = acc + 32 * h + c;
                                if (b4) add_bias8(a, ld_nc_u4(b4 + (c >> 3)));
                                st_global_f32x8(dst + c, a);
                            }
                        }
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

// Rows of the weight tensor-map box the wide kernel loads per stage (both modes).
uint32_t gemm_weight_box(int) { return static_cast<uint32_t>(kTileN); }

cudaError_t launch_gemm(const GemmArgs& a, const CUtensorMap& tmA, const CUtensorMap& tmB, int num_sms,
                        cudaStream_t s) {
    if (a.recipe != 0) return cudaErrorInvalidValue;   // MXFP8 runs gemm_mx.cu
    return a.mode == 0 ? launch_gemm_t<0>(a, tmA, tmB, num_sms, s) : launch_gemm_t<1>(a, tmA, tmB, num_sms, s);
}

}  // namespace moe
