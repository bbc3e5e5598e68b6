// gate.cu -- the gate in front of the router, fused with it: RMS-Norm of the bf16 hidden state,
// the router matmul against fp32 router weights, then the router's top-k ("mlx_native
// ops/moe_gate.rs": one pass per token does the norm, the matmul and top-K + softmax +
// per-expert scale):
//   xn[h]     = x[h] / sqrt( mean_h x[h]^2 + eps ) * norm_w[h]
//   logit[e]  = sum_h xn[h] * router_w[e, h]
// One block of 8 warps takes kGateTokens tokens: a warp per token normalizes it into shared
// memory (fp32); then every warp takes every 8th expert, streams its router row once for all
// of the block's tokens (coalesced float4 loads) and reduces the dot products across lanes in a
// fixed butterfly order; then a warp per token runs route_token on the logits.  Sums are fp32
// in a fixed order, so a token's logits do not depend on the other tokens.
#include "route_device.cuh"

namespace moe {

namespace {

constexpr int kGateTokens = 4;
constexpr int kGateWarps = 8;

// Butterfly sum over the warp: every lane gets the same total, in the same order.
__device__ __forceinline__ float warp_sum_xor(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace

__global__ void __launch_bounds__(kGateWarps * 32) k_gate(GateArgs g, RouteArgs ra) {
    extern __shared__ float xn[];                      // [kGateTokens][H]
    __shared__ float s_score[kGateTokens][256];
    __shared__ float s_gscore[kGateTokens][256];
    __shared__ int s_sel[kGateTokens][256];
    __shared__ unsigned char s_elig[kGateTokens][256];

    pdl_wait_then_release();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = g.H, E = g.E;
    const int t0 = blockIdx.x * kGateTokens;
    const int nt = min(kGateTokens, g.T - t0);

    // ---- RMS-Norm: warp w normalizes token t0 + w (8 bf16 per lane per step)
    if (warp < kGateTokens) {
        float* xw = xn + static_cast<size_t>(warp) * H;
        if (warp < nt) {
            const __nv_bfloat16* xr = g.x + static_cast<size_t>(t0 + warp) * H;
            float ss = 0.0f;
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
            ss = warp_sum_xor(ss);
            const float r = 1.0f / sqrtf(ss / static_cast<float>(H) + g.eps);
            for (int h = lane * 8; h < H; h += 256) {
                const uint4 raw = *reinterpret_cast<const uint4*>(xr + h);
                const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(p2[i]);
                    xw[h + 2 * i] = f.x * r * g.norm_w[h + 2 * i];
                    xw[h + 2 * i + 1] = f.y * r * g.norm_w[h + 2 * i + 1];
                }
            }
        } else {
            for (int h = lane; h < H; h += 32) xw[h] = 0.0f;   // rows of absent tokens
        }
    }
    __syncthreads();

    // ---- router matmul: warp w takes experts w, w + 8, ...; one pass over the row for all tokens
    for (int e = warp; e < E; e += kGateWarps) {
        const float* wr = g.router_w + static_cast<size_t>(e) * H;
        float acc[kGateTokens];
#pragma unroll
        for (int j = 0; j < kGateTokens; ++j) acc[j] = 0.0f;
        for (int h = lane * 4; h < H; h += 128) {
            const float4 wv = __ldg(reinterpret_cast<const float4*>(wr + h));
#pragma unroll
            for (int j = 0; j < kGateTokens; ++j) {
                const float4 xv = *reinterpret_cast<const float4*>(xn + static_cast<size_t>(j) * H + h);
                acc[j] = fmaf(xv.x, wv.x, acc[j]);
                acc[j] = fmaf(xv.y, wv.y, acc[j]);
                acc[j] = fmaf(xv.z, wv.z, acc[j]);
                acc[j] = fmaf(xv.w, wv.w, acc[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kGateTokens; ++j) acc[j] = warp_sum_xor(acc[j]);
        if (lane == 0)
            for (int j = 0; j < nt; ++j) g.logits[static_cast<size_t>(t0 + j) * E + e] = acc[j];
    }
    __syncthreads();                                   // the block's logits are written

    // ---- the router on those logits: a warp per token
    if (warp < nt) route_token(ra, t0 + warp, lane, s_score[warp], s_gscore[warp], s_sel[warp], s_elig[warp], nullptr);
}

size_t gate_smem_bytes(int H) { return static_cast<size_t>(kGateTokens) * H * sizeof(float); }

cudaError_t launch_gate(const GateArgs& g, const RouteArgs& ra, cudaStream_t s) {
    const size_t smem = gate_smem_bytes(g.H);
    cudaError_t e = cudaFuncSetAttribute(k_gate, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int blocks = (g.T + kGateTokens - 1) / kGateTokens;
    return launch_pdl(k_gate, dim3(blocks), dim3(kGateWarps * 32), smem, s, g, ra);
}

}  // namespace moe
