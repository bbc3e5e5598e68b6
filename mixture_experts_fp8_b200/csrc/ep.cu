// ep.cu -- expert parallelism over R ranks of one node (the dispatch/combine around the grouped
// GEMMs: "MindIE-SD Fused MoE", execution flow (dispatch, mlp, combine) and the dynamic
// dispatcher's all-to-all; "MATE Mega MoE", Typical Flow: intranode ranks).  Rank r owns experts
// r*E/R .. (r+1)*E/R - 1.  The kernels here are the device steps on either side of the exchange:
//
//   k_ep_dest    the destination rank of every routed slot, dest = expert / (E/R); the
//                permutation kernels then order the slots by destination (stable in slot order
//                t*k + j), which gives the send counts, the send order and each slot's position
//   k_ep_gather  each slot's token row and its expert id local to the destination, in send order
//   k_rows_f32   the expert side's output rows, fp32, in arrival order (an exact copy out of the
//                permuted GEMM output)
//
// A row's GEMM output depends only on its own codes and its expert's weights, so the rows a
// rank computes for others are bit-identical to the ones a single GPU computes for itself, and the
// combine on the home rank (k_combine over the returned rows) gives the single-GPU bits.
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

__global__ void __launch_bounds__(256) k_ep_dest(EpArgs a) {
    pdl_wait_then_release();
    const int i = blockIdx.x * 256 + threadIdx.x;
    if (i >= a.A) return;
    const int e = a.idx[i];
    int d = -1;                                   // out of range: reported, and not sent
    if (e >= 0 && e < a.E) d = e / a.e_loc;
    else set_status(a.status, MOE_ERR_BOUNDS);
    a.dest[i] = d;
}

// Block (i, cb): send position i, 16-byte pieces cb*256 + thread of the token row.
__global__ void __launch_bounds__(256) k_ep_gather(EpArgs a) {
    pdl_wait_then_release();
    // every position is filled when every slot's expert id is valid (else k_ep_dest has already
    // reported MOE_ERR_BOUNDS and the positions past the valid slots are not sent)
    const int i = blockIdx.x;
    const int s = a.row_src[i];
    if (s < 0 || s >= a.A) {
        if (threadIdx.x == 0) set_status(a.status, MOE_ERR_BOUNDS);
        return;
    }
    const int t = s / a.K;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.H);
    uint4* dst = reinterpret_cast<uint4*>(a.send_x + static_cast<size_t>(i) * a.H);
    for (int c = blockIdx.y * 256 + threadIdx.x; c < a.H / 8; c += gridDim.y * 256) dst[c] = src[c];
    if (blockIdx.y == 0 && threadIdx.x == 0) a.send_expert[i] = a.idx[s] % a.e_loc;
}

// out[t, :] = o[row_of[t], :] (one slot per row), fp32, 16 bytes per thread.
__global__ void __launch_bounds__(256) k_rows_f32(const float* __restrict__ o, const int32_t* __restrict__ row_of,
                                                  float* __restrict__ out, int T, int H, int32_t* status) {
    pdl_wait_then_release();
    const int t = blockIdx.x;
    int r = row_of[t];
    if (r < 0 || r >= T) {
        if (threadIdx.x == 0 && blockIdx.y == 0) set_status(status, MOE_ERR_BOUNDS);
        r = 0;
    }
    const float4* src = reinterpret_cast<const float4*>(o + static_cast<size_t>(r) * H);
    float4* dst = reinterpret_cast<float4*>(out + static_cast<size_t>(t) * H);
    for (int c = blockIdx.y * 256 + threadIdx.x; c < H / 4; c += gridDim.y * 256) dst[c] = src[c];
}

cudaError_t launch_ep_dest(const EpArgs& a, cudaStream_t s) {
    return launch_pdl(k_ep_dest, dim3((a.A + 255) / 256), dim3(256), 0, s, a);
}

cudaError_t launch_ep_gather(const EpArgs& a, cudaStream_t s) {
    if (a.A == 0) return cudaSuccess;
    const int cb = (a.H / 8 + 255) / 256;
    return launch_pdl(k_ep_gather, dim3(a.A, cb), dim3(256), 0, s, a);
}

cudaError_t launch_rows_f32(const float* o, const int32_t* row_of, float* out, int T, int H, int32_t* status,
                            cudaStream_t s) {
    const int cb = (H / 4 + 255) / 256;
    return launch_pdl(k_rows_f32, dim3(T, cb), dim3(256), 0, s, o, row_of, out, T, H, status);
}

}  // namespace moe
