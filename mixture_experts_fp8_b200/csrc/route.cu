// route.cu -- the router top-k kernel (moe_route, and the first stage of large batches):
// one warp per token; the per-token work is route_token() in route_device.cuh.
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
    route_token(a, t, lane, s_score[warp], s_gscore[warp], s_sel[warp], s_elig[warp], nullptr);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
    const int blocks = (a.T + kRouteWarps - 1) / kRouteWarps;
    return launch_pdl(k_route, dim3(blocks), dim3(kRouteWarps * 32), 0, s, a);
}

}  // namespace moe
