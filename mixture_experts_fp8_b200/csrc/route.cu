// route.cu -- the router top-k kernel (moe_route, the first stage of large batches, and the
// second launch of the gate): one warp per token; the per-token work is route_token() in
// route_device.cuh.
#include "route_device.cuh"

namespace moe {

constexpr int kRouteWarps = 4;

__global__ void __launch_bounds__(kRouteWarps * 32) k_route(RouteArgs a) {
    __shared__ float s_score[kRouteWarps][256];
    __shared__ float s_gscore[kRouteWarps][256];
    __shared__ int s_sel[kRouteWarps][256];
    __shared__ unsigned char s_elig[kRouteWarps][256];

    pdl_wait_then_release();
    if (a.status && blockIdx.x == 0 && threadIdx.x == 0) *a.status = MOE_OK;   // first kernel of a forward
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kRouteWarps + warp;
    if (t >= a.T) return;
    if (a.gate_x) {
        // Gate mode: the token's RMS-Norm factor from lane-strided partial sums of x^2 (8 columns
        // per load) and a butterfly over the warp, then its row of matmul sums scaled in place.
        const __nv_bfloat16* xr = a.gate_x + static_cast<size_t>(t) * a.gate_H;
        float ss = 0.0f;
        for (int h = lane * 8; h < a.gate_H; h += 256) {
            const uint4 raw = *reinterpret_cast<const uint4*>(xr + h);
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(p2[i]);
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
            }
        }
        ss = warp_sum(ss);
        const float r = 1.0f / sqrtf(ss / static_cast<float>(a.gate_H) + a.gate_eps);
        float* l = const_cast<float*>(a.logits) + static_cast<size_t>(t) * a.E;   // the gate's own buffer
        for (int e = lane; e < a.E; e += 32) l[e] *= r;
        __syncwarp();
    }
    route_token(a, t, lane, s_score[warp], s_gscore[warp], s_sel[warp], s_elig[warp], nullptr);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
    const int blocks = (a.T + kRouteWarps - 1) / kRouteWarps;
    return launch_pdl(k_route, dim3(blocks), dim3(kRouteWarps * 32), 0, s, a);
}

}  // namespace moe
