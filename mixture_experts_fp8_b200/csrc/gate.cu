// gate.cu -- the gate in front of the router: RMS-Norm of the bf16 hidden state, the router matmul
// against fp32 router weights, then the router's top-k ("mlx_native ops/moe_gate.rs": per token,
// RMS-Norm, router matmul, then top-K + softmax + per-expert scale):
//   xn[h]     = x[h] / sqrt( mean_h x[h]^2 + eps ) * norm_w[h]
//   logit[e]  = sum_h xn[h] * router_w[e, h]
// computed as  logit[e] = r * sum_h (x[h] * norm_w[h]) * router_w[e, h],  r = 1/sqrt(mean x^2 + eps)
// (the norm's per-token factor taken out of the sum).
//
// Two launches: k_gate_logits, a tiled fp32 SIMT matmul over (token tile, expert tile) blocks,
// then the router kernel (k_route) on the logits.  Every logit is summed by one thread in
// ascending h, and every token's sum of squares by one warp in a fixed lane order, whatever the
// tile shape: a token's logits do not depend on the other tokens or on the batch size.  The
// tile shape follows the batch: 64 x 64 (4 x 4 outputs per thread) when that gives the SMs enough
// blocks, else 16 x 16 (one output per thread).  H is a multiple of 128; chunks are 64 deep.
#include "route_device.cuh"

namespace moe {

namespace {

constexpr int kGateThreads = 256;

// Butterfly sum over the warp: every lane gets the same total, in the same order.
__device__ __forceinline__ float warp_sum_xor(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace

// TM tokens x TN experts per block; thread (ty, tx) owns MI consecutive tokens ty*MI .. and NJ
// consecutive experts tx*NJ .., (TM/MI) * (TN/NJ) = 256 threads.  K advances in chunks of KC: the
// next chunk is loaded into registers while the current one is multiplied out of shared memory.
template <int TM, int TN, int MI, int NJ, int KC>
__global__ void __launch_bounds__(kGateThreads) k_gate_logits(GateArgs g) {
    constexpr int kGateK = KC;
    constexpr int RY = TM / MI, RX = TN / NJ;
    static_assert(RY * RX == kGateThreads, "thread tile");
    constexpr int XP = TM * kGateK / 8, WP = TN * kGateK / 4;           // pieces per chunk
    constexpr int XL = (XP + kGateThreads - 1) / kGateThreads;          // x pieces (8 bf16) per thread
    constexpr int WL = (WP + kGateThreads - 1) / kGateThreads;          // router pieces (4 fp32) per thread
    __shared__ __align__(16) float xs[kGateK][TM];          // x * norm_w, k-major
    __shared__ __align__(16) float ws[kGateK][TN];          // router rows, k-major
    __shared__ float rs[TM];                                // 1 / sqrt(mean x^2 + eps) per token

    pdl_wait_then_release();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.y * TM, e0 = blockIdx.x * TN;
    const int H = g.H;

    // ---- per-token norm factor: one warp per token, lane-strided partial sums, then a butterfly
    for (int m = warp; m < TM; m += kGateThreads / 32) {
        const int t = t0 + m;
        float ss = 0.0f;
        if (t < g.T) {
            const __nv_bfloat16* xr = g.x + static_cast<size_t>(t) * H;
            for (int h = lane * 8; h < H; h += 256) {
                const uint4 raw = *reinterpret_cast<const uint4*>(xr + h);
                const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(p2[i]);
                    ss = fmaf(f.x, f.x, ss);
                    ss = fmaf(f.y, f.y, ss);
                }
            }
        }
        ss = warp_sum_xor(ss);
        if (lane == 0) rs[m] = 1.0f / sqrtf(ss / static_cast<float>(H) + g.eps);
    }

    // ---- chunk loaders: x piece i = (row, 8 columns), router piece = (row, 4 columns)
    uint4 xr[XL];
    float4 wr[WL];
    auto load = [&](int k0) {
#pragma unroll
        for (int l = 0; l < XL; ++l) {
            const int i = threadIdx.x + l * kGateThreads;
            const int m = i / (kGateK / 8), c = (i % (kGateK / 8)) * 8, t = t0 + m;
            xr[l] = i < XP && t < g.T && k0 + c < H ? *reinterpret_cast<const uint4*>(g.x + static_cast<size_t>(t) * H + k0 + c)
                            : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int l = 0; l < WL; ++l) {
            const int i = threadIdx.x + l * kGateThreads;
            const int n = i / (kGateK / 4), c = (i % (kGateK / 4)) * 4, e = e0 + n;
            wr[l] = i < WP && e < g.E && k0 + c < H ? __ldg(reinterpret_cast<const float4*>(g.router_w + static_cast<size_t>(e) * H + k0 + c))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto store = [&](int k0) {
#pragma unroll
        for (int l = 0; l < XL; ++l) {
            const int i = threadIdx.x + l * kGateThreads;
            if (XP % kGateThreads != 0 && i >= XP) break;
            const int m = i / (kGateK / 8), c = (i % (kGateK / 8)) * 8;
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&xr[l]);
            const bool in = k0 + c < H;                      // a chunk may run past H (KC > 128)
            const float4 n0 = in ? *reinterpret_cast<const float4*>(g.norm_w + k0 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 n1 = in ? *reinterpret_cast<const float4*>(g.norm_w + k0 + c + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float nw[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __bfloat1622float2(p2[q]);
                xs[c + 2 * q][m] = f.x * nw[2 * q];
                xs[c + 2 * q + 1][m] = f.y * nw[2 * q + 1];
            }
        }
#pragma unroll
        for (int l = 0; l < WL; ++l) {
            const int i = threadIdx.x + l * kGateThreads;
            if (WP % kGateThreads != 0 && i >= WP) break;
            const int n = i / (kGateK / 4), c = (i % (kGateK / 4)) * 4;
            ws[c][n] = wr[l].x;
            ws[c + 1][n] = wr[l].y;
            ws[c + 2][n] = wr[l].z;
            ws[c + 3][n] = wr[l].w;
        }
    };

    const int ty = threadIdx.x / RX, tx = threadIdx.x % RX;
    float acc[MI][NJ];
#pragma unroll
    for (int i = 0; i < MI; ++i)
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[i][j] = 0.0f;

    load(0);
    for (int k0 = 0; k0 < H; k0 += kGateK) {
        __syncthreads();                      // the previous chunk is consumed (and rs is written)
        store(k0);
        __syncthreads();
        if (k0 + kGateK < H) load(k0 + kGateK);
        const int kn = min(kGateK, H - k0);   // columns of this chunk inside H (the sum stops at H)
#pragma unroll 16
        for (int k = 0; k < kn; ++k) {
            float a[MI], b[NJ];
            if constexpr (MI == 4) {
                const float4 v = *reinterpret_cast<const float4*>(&xs[k][ty * 4]);
                a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
            } else {
#pragma unroll
                for (int i = 0; i < MI; ++i) a[i] = xs[k][ty * MI + i];
            }
            if constexpr (NJ == 4) {
                const float4 v = *reinterpret_cast<const float4*>(&ws[k][tx * 4]);
                b[0] = v.x; b[1] = v.y; b[2] = v.z; b[3] = v.w;
            } else {
#pragma unroll
                for (int j = 0; j < NJ; ++j) b[j] = ws[k][tx * NJ + j];
            }
#pragma unroll
            for (int i = 0; i < MI; ++i)
#pragma unroll
                for (int j = 0; j < NJ; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
    }

#pragma unroll
    for (int i = 0; i < MI; ++i) {
        const int m = ty * MI + i, t = t0 + m;
        if (t >= g.T) continue;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int e = e0 + tx * NJ + j;
            if (e < g.E) g.logits[static_cast<size_t>(t) * g.E + e] = acc[i][j] * rs[m];
        }
    }
}

size_t gate_smem_bytes(int) { return 0; }

cudaError_t launch_gate(const GateArgs& g, const RouteArgs& ra, cudaStream_t s) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long big_blocks = 1LL * ((g.T + 63) / 64) * ((g.E + 63) / 64);
    cudaError_t e;
    if (big_blocks >= sms)
        e = launch_pdl(k_gate_logits<64, 64, 4, 4, 64>, dim3((g.E + 63) / 64, (g.T + 63) / 64), dim3(kGateThreads), 0, s,
                       g);
    else
        e = launch_pdl(k_gate_logits<16, 16, 1, 1, 64>, dim3((g.E + 15) / 16, (g.T + 15) / 16), dim3(kGateThreads), 0, s,
                       g);
    if (e != cudaSuccess) return e;
    return launch_route(ra, s);
}

}  // namespace moe
