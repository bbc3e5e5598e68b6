// quant_combine.cu -- the two HBM-bound ends of the layer.
//
// k_quant (dispatch side): dynamic E4M3 quantization of the layer input, scattered straight
// into expert-contiguous order.  "metrale_model_layers fp8_grouped_tc_w8a8.rs", module doc:
// the layer input is quantized to E4M3 per (row, 128 group); "DeepGEMM PR #371", Changes:
// UE8M0 scale factors per 32 elements.  Each token is quantized once and its codes are
// written to the k permuted rows it was routed to (the codes do not depend on the expert).
//   recipe 0: s = amax / 448 (IEEE division), q = e4m3_rn_satfinite(x / s); amax 0 -> s = 1
//   recipe 1: s = 2^e, e the smallest with amax <= 448 * 2^e; byte e + 127; q = e4m3(x * 2^-e)
//
// k_combine: y[t] = bf16_rn( sum_j w[t,j] * o[row_of[t,j]] ), fp32, fixed slot order (the
// shared expert's slot, if any, last with weight 1), no
// atomics ("MindIE-SD Fused MoE", execution flow: combine; "MATE Mega MoE", Current Limits:
// contiguous bf16 output).
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

// One warp per (token, 512 columns): two 256-column chunks, both loads issued before any
// arithmetic so that more bytes are in flight per warp.  In a chunk, lane l owns columns
// 8l .. 8l+7 (one 16-byte load, one 8-byte code store per destination row): a 128-column group
// is 16 lanes, a 32-column group 4 lanes.  H need only be a multiple of 128: lanes past the end
// of the row take part in the shuffles but load and store nothing.
constexpr int kQuantChunks = 2;

__device__ __forceinline__ void quant_chunk(const QuantArgs& a, int t, int c, uint4 raw, bool in_row, int r_lane,
                                            bool lane_row_ok) {
    const int lane = threadIdx.x & 31;
    float v[8];
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        v[2 * i] = __low2float(b);
        v[2 * i + 1] = __high2float(b);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    uint2 q;
    float s32 = 1.0f;
    uint8_t e8 = 127;
    if (a.recipe == 0) {
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        s32 = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        q.x = e4m3x4(__fdiv_rn(v[0], s32), __fdiv_rn(v[1], s32), __fdiv_rn(v[2], s32), __fdiv_rn(v[3], s32));
        q.y = e4m3x4(__fdiv_rn(v[4], s32), __fdiv_rn(v[5], s32), __fdiv_rn(v[6], s32), __fdiv_rn(v[7], s32));
    } else {
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const int e = mx_exponent(amax);
        const float inv = exp2_int(-e);                 // x * 2^-e == x / 2^e exactly
        q.x = e4m3x4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
        q.y = e4m3x4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
        e8 = static_cast<uint8_t>(e + 127);
    }
    const int A = a.T * a.K;
    const int32_t* rows = a.row_of + static_cast<size_t>(t) * a.K;
    const int col = c * 256 + 8 * lane;                // this lane's first column
    const int g128 = col >> 7;                         // its 128-column block
    for (int j = 0; j < a.K; ++j) {
        const int r = j < 32 ? __shfl_sync(0xffffffffu, r_lane, j) : __ldg(rows + j);
        if (r < 0 || r >= A) continue;                 // reported once per token by the caller
        if (in_row) {
            *reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(r) * a.H + col) = q;
            if (a.recipe != 0 && (lane & 3) == 0)
                static_cast<uint8_t*>(a.xs)[(static_cast<size_t>(g128) * a.a_pad + r) * 4 + ((col >> 5) & 3)] = e8;
        }
    }
    // fp32 scales, one per 128-column block: lane j stores block h's scale for the token's row j
    if (a.recipe == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float sh = __shfl_sync(0xffffffffu, s32, 16 * h);
            const int gb = c * 2 + h;
            if ((gb << 7) >= a.H) break;
            if (lane < a.K && lane_row_ok) static_cast<float*>(a.xs)[static_cast<size_t>(gb) * a.a_pad + r_lane] = sh;
            for (int j = 32 + lane; j < a.K; j += 32) {
                const int r = __ldg(rows + j);
                if (r >= 0 && r < A) static_cast<float*>(a.xs)[static_cast<size_t>(gb) * a.a_pad + r] = sh;
            }
        }
    }
}

__global__ void __launch_bounds__(256) k_quant(QuantArgs a) {
    pdl_wait_then_release();
    const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int nchunks = (a.H + 255) >> 8;
    const int nw = (nchunks + kQuantChunks - 1) / kQuantChunks;   // warps per token
    if (gw >= a.T * nw) return;
    const int t = gw / nw, c0 = (gw - t * nw) * kQuantChunks;
    uint4 raw[kQuantChunks];
    bool in_row[kQuantChunks];
#pragma unroll
    for (int i = 0; i < kQuantChunks; ++i) {
        const int col = (c0 + i) * 256 + 8 * lane;
        in_row[i] = c0 + i < nchunks && col < a.H;
        raw[i] = in_row[i] ? __ldg(reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.H + col))
                           : make_uint4(0, 0, 0, 0);
    }
    // the token's destination rows: lane j holds row_of[t, j] (slots past 32 are read in the loop)
    const int A = a.T * a.K;
    const int32_t* rows = a.row_of + static_cast<size_t>(t) * a.K;
    const int r_lane = lane < a.K ? __ldg(rows + lane) : -1;
    const bool lane_row_ok = r_lane >= 0 && r_lane < A;
    if (c0 == 0) {                                     // report a bad destination once per token
        if (lane < a.K && !lane_row_ok) set_status(a.status, MOE_ERR_BOUNDS);
        for (int j = 32 + lane; j < a.K; j += 32) {
            const int r = __ldg(rows + j);
            if (r < 0 || r >= A) set_status(a.status, MOE_ERR_BOUNDS);
        }
    }
#pragma unroll
    for (int i = 0; i < kQuantChunks; ++i)
        if (c0 + i < nchunks) quant_chunk(a, t, c0 + i, raw[i], in_row[i], r_lane, lane_row_ok);
}

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t s) {
    const int nchunks = (a.H + 255) >> 8;
    const int warps = a.T * ((nchunks + kQuantChunks - 1) / kQuantChunks);
    return launch_pdl(k_quant, dim3((warps + 7) / 8), dim3(256), 0, s, a);
}

// Grid (token, column block): thread i of block (t, cb) handles float4 column cb * 256 + i, so
// every routed row's loads are in flight at once.
__global__ void __launch_bounds__(256) k_combine(CombineArgs a) {
    __shared__ int s_row[MOE_MAX_EXPERTS + 1];
    __shared__ float s_w[MOE_MAX_EXPERTS + 1];
    pdl_wait_then_release();
    const int t = blockIdx.x;
    for (int j = threadIdx.x; j < a.K; j += blockDim.x) {
        const int r = a.row_of[static_cast<size_t>(t) * a.K + j];
        const bool ok = r >= 0 && r < a.rows;
        if (!ok && blockIdx.y == 0) set_status(a.status, MOE_ERR_BOUNDS);
        s_row[j] = ok ? r : -1;
        s_w[j] = j < a.k ? a.w[static_cast<size_t>(t) * a.k + j] : 1.0f;   // shared expert: weight 1
    }
    __syncthreads();
    const int c = blockIdx.y * blockDim.x + threadIdx.x;
    if (c >= (a.H >> 2)) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < a.K; ++j) {
        if (s_row[j] < 0) continue;                  // a position out of range adds nothing
        const float4 v = __ldg(reinterpret_cast<const float4*>(a.o + static_cast<size_t>(s_row[j]) * a.H) + c);
        const float w = s_w[j];
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 out;
    out.x = *reinterpret_cast<uint32_t*>(&lo);
    out.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(a.y + static_cast<size_t>(t) * a.H)[c] = out;
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
    const int cblocks = ((a.H >> 2) + 255) / 256;
    return launch_pdl(k_combine, dim3(a.T, cblocks), dim3(256), 0, s, a);
}

// ------------------------------------------------------------------------------------------
// Weight transform (offline): E4M3 codes [E, K, N] -> K-major [E, N', K], with w13's gate and up
// columns interleaved in blocks (moe::w13_interleaved_row, moe::w13_block), and the block scales
// re-laid to match:
//   recipe 0: fp32 [E, K/128, N] -> [E, K/128, N'] (columns permuted like the codes)
//   recipe 1: UE8M0 [E, K/32, N] -> 512-byte scale-factor atoms [E, N/128, K/128] for the
//             block-scaled tensor core (see gemm_mx.cu)
//   recipe 2 (W4A8): E2M1 codes packed two per byte along N, [E, K, N/2] -> packed two per
//             byte along K, [E, N', K/2] (the lower K in the low nibble; k_transpose_nibbles),
//             scales as recipe 1
// ("MATE Mega MoE", transform_weights_for_mega_moe; "DeepGEMM PR #371", 4-packed UE8M0.)
__global__ void __launch_bounds__(256) k_transpose_codes(const uint8_t* src, uint8_t* dst, int K,
                                                        int N, int interleave_I, int blk) {
    __shared__ uint8_t tile[64][65];
    const int e = blockIdx.z;
    const int k0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const uint8_t* s = src + static_cast<size_t>(e) * K * N;
    uint8_t* d = dst + static_cast<size_t>(e) * K * N;
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
        const int kk = i / 64, nn = i % 64;
        if (k0 + kk < K && n0 + nn < N) tile[kk][nn] = s[static_cast<size_t>(k0 + kk) * N + n0 + nn];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 64 * 64; i += 256) {
        const int nn = i / 64, kk = i % 64;
        const int n = n0 + nn, k = k0 + kk;
        if (n < N && k < K) {
            const int row = interleave_I ? w13_interleaved_row(n, interleave_I, blk) : n;
            d[static_cast<size_t>(row) * K + k] = tile[kk][nn];
        }
    }
}

// E2M1 codes: a 64 x 64 tile of [K, N] codes (N packed in pairs) is unpacked into shared
// memory, then written back K-major with K packed in pairs.
__global__ void __launch_bounds__(256) k_transpose_nibbles(const uint8_t* src, uint8_t* dst, int K,
                                                          int N, int interleave_I, int blk) {
    __shared__ uint8_t tile[64][65];
    const int e = blockIdx.z;
    const int k0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const uint8_t* s = src + static_cast<size_t>(e) * K * (N / 2);
    uint8_t* d = dst + static_cast<size_t>(e) * N * (K / 2);
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {          // 64 rows x 32 bytes
        const int kk = i / 32, jj = i % 32;
        if (k0 + kk < K && n0 + 2 * jj < N) {
            const uint8_t b = s[static_cast<size_t>(k0 + kk) * (N / 2) + n0 / 2 + jj];
            tile[kk][2 * jj] = b & 15;
            tile[kk][2 * jj + 1] = b >> 4;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {          // 64 columns x 32 bytes
        const int nn = i / 32, jj = i % 32;
        const int n = n0 + nn, k = k0 + 2 * jj;
        if (n < N && k < K) {
            const int row = interleave_I ? w13_interleaved_row(n, interleave_I, blk) : n;
            d[static_cast<size_t>(row) * (K / 2) + k / 2] =
                static_cast<uint8_t>(tile[2 * jj][nn] | (tile[2 * jj + 1][nn] << 4));
        }
    }
}

__global__ void k_transform_scales(const void* src, void* dst, int E, int K, int N, int recipe,
                                   int interleave_I) {
    const int blk = w13_block(recipe);
    if (recipe == 0) {
        // fp32 [E, K/128, N] -> [E, K/128, N'] (columns permuted like the codes)
        const size_t total = static_cast<size_t>(E) * (K / 128) * N;
        for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
             i += static_cast<size_t>(gridDim.x) * blockDim.x) {
            const int n = static_cast<int>(i % N);
            const size_t ek = i / N;                    // e * (K/128) + kb
            const int row = interleave_I ? w13_interleaved_row(n, interleave_I, blk) : n;
            static_cast<float*>(dst)[ek * N + row] = static_cast<const float*>(src)[ek * N + n];
        }
        return;
    }
    // UE8M0 [E, K/32, N] -> scale-factor atoms [E, N/128, K/128][512 B]: in the atom of column block
    // nb and stage kb, byte 16*i + 4*c + k is the scale of transformed row nb*128 + 32*c + i for the
    // 32-deep block kb*4 + k.
    const int NB = N / 128, KB = K / 128;
    const size_t total = static_cast<size_t>(E) * NB * KB * 512;
    const uint8_t* s = static_cast<const uint8_t*>(src);
    uint8_t* d = static_cast<uint8_t*>(dst);
    for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int byte = static_cast<int>(idx & 511);
        const size_t atom = idx >> 9;                   // (e * NB + nb) * KB + kb
        const int kb = static_cast<int>(atom % KB);
        const size_t enb = atom / KB;
        const int nb = static_cast<int>(enb % NB);
        const size_t e = enb / NB;
        const int i = byte >> 4, c = (byte >> 2) & 3, k = byte & 3;
        const int row = nb * 128 + 32 * c + i;
        const int col = interleave_I ? w13_original_col(row, interleave_I, blk) : row;
        d[idx] = s[(e * (K / 32) + kb * 4 + k) * N + col];
    }
}

cudaError_t launch_transform(const TransformArgs& a, cudaStream_t s) {
    const int H = a.H, I = a.I, E = a.E;
    auto codes = a.recipe == 2 ? k_transpose_nibbles : k_transpose_codes;
    codes<<<dim3((2 * I + 63) / 64, (H + 63) / 64, E), 256, 0, s>>>(a.w13, a.w13_t, H, 2 * I, I, w13_block(a.recipe));
    codes<<<dim3((H + 63) / 64, (I + 63) / 64, E), 256, 0, s>>>(a.w2, a.w2_t, I, H, 0, 1);
    k_transform_scales<<<1024, 256, 0, s>>>(a.w13s, a.w13s_t, E, H, 2 * I, a.recipe, I);
    k_transform_scales<<<1024, 256, 0, s>>>(a.w2s, a.w2s_t, E, I, H, a.recipe, 0);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Failure-detection self test: wait on an mbarrier that nothing completes, bounded by
// timeout_us, then record MOE_ERR_TIMEOUT and return.
__global__ void k_selftest_wait(int32_t* status, uint32_t timeout_us) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t a = smem_u32(&bar);
        const unsigned long long t0 = globaltimer_ns();
        bool done = false;
        while (!(done = mbar_try_wait(a, 0))) {
            if (globaltimer_ns() - t0 > 1000ull * timeout_us) break;
        }
        *status = done ? MOE_OK : MOE_ERR_TIMEOUT;
    }
}

cudaError_t launch_selftest_wait(int32_t* status, uint32_t timeout_us, cudaStream_t s) {
    k_selftest_wait<<<1, 32, 0, s>>>(status, timeout_us);
    return cudaGetLastError();
}

}  // namespace moe
