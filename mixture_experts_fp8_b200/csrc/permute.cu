// permute.cu -- stable permutation of the routed rows into expert-contiguous order.
//
// "MindIE-SD Fused MoE", execution flow: dispatch reorders tokens by expert and counts each
// expert's tokens; combine restores token order.  Routed row a = t*k + j; inside an expert,
// rows keep ascending a (hence ascending token).  Three launches, no global atomics, so the
// result is the same bits on every run:
//   1. k_hist     per-chunk expert histograms (chunk = kPermuteChunk routed rows)
//   2. k_scan     per-expert exclusive bases across chunks, counts, offsets = exclusive scan,
//                 and the first 128-row GEMM tile of every expert
//   3. k_scatter  one warp per chunk walks its rows in order; rows with the same expert inside
//                 a 32-row batch are ranked with a warp match.
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

__global__ void __launch_bounds__(256) k_hist(PermuteArgs a) {
    __shared__ int cnt[MOE_MAX_EXPERTS];
    pdl_wait_then_release();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int begin = blockIdx.x * kPermuteChunk;
    const int end = min(a.A, begin + kPermuteChunk);
    for (int r = begin + threadIdx.x; r < end; r += blockDim.x) {
        const int e = a.idx[r];
        if (e >= 0 && e < a.E) atomicAdd(&cnt[e], 1);
        else set_status(a.status, MOE_ERR_BOUNDS);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        a.hist[static_cast<size_t>(blockIdx.x) * a.E + e] = cnt[e];
}

// Exclusive scan of v over the 256 threads of the block (v of threads >= n treated as 0).
__device__ int block_exclusive_scan_256(int v, int* tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < 8 ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < 8) tmp[8 + lane] = w;               // inclusive warp totals
    }
    __syncthreads();
    const int before = warp ? tmp[8 + warp - 1] : 0;
    const int excl = before + x - v;
    __syncthreads();
    return excl;
}

__global__ void __launch_bounds__(256) k_scan(PermuteArgs a) {
    __shared__ int tmp[16];
    pdl_wait_then_release();
    const int e = threadIdx.x;
    int run = 0;
    if (e < a.E) {
        for (int c = 0; c < a.chunks; ++c) {
            int32_t* h = a.hist + static_cast<size_t>(c) * a.E + e;
            const int v = *h;
            *h = run;
            run += v;
        }
    }
    const int cnt = e < a.E ? run : 0;
    const int off = block_exclusive_scan_256(cnt, tmp);
    const int mt = (cnt + kTileM - 1) / kTileM;
    const int ts = block_exclusive_scan_256(mt, tmp);
    if (e < a.E) {
        a.counts[e] = cnt;
        a.offsets[e] = off;
        a.tile_start[e] = ts;
        if (a.expert_counts) a.expert_counts[e] = cnt;
    }
    if (e == a.E - 1) {
        a.offsets[a.E] = off + cnt;
        a.tile_start[a.E] = ts + mt;
    }
}

__global__ void __launch_bounds__(32) k_scatter(PermuteArgs a) {
    __shared__ int base[MOE_MAX_EXPERTS];
    constexpr int kBatches = kPermuteChunk / 32;
    pdl_wait_then_release();
    const int lane = threadIdx.x;
    const int begin = blockIdx.x * kPermuteChunk;
    const int end = min(a.A, begin + kPermuteChunk);
    int ids[kBatches];                                  // all of the chunk's ids, loaded at once
#pragma unroll
    for (int b = 0; b < kBatches; ++b) {
        const int r = begin + 32 * b + lane;
        ids[b] = r < end ? a.idx[r] : -1;
    }
    for (int e = lane; e < a.E; e += 32)
        base[e] = a.offsets[e] + a.hist[static_cast<size_t>(blockIdx.x) * a.E + e];
    __syncwarp();
#pragma unroll
    for (int b = 0; b < kBatches; ++b) {
        const int r = begin + 32 * b + lane;
        const bool valid = r < end;
        int e = ids[b];
        if (e >= a.E) e = -1;                           // reported by k_hist
        const uint32_t active = __ballot_sync(0xffffffffu, valid && e >= 0);
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const uint32_t mine = peers & active;
        const int rank = __popc(mine & ((1u << lane) - 1u));
        int dst = 0;
        if (valid && e >= 0) dst = base[e] + rank;
        __syncwarp();
        if (valid && e >= 0 && rank == 0) base[e] += __popc(mine);
        __syncwarp();
        if (valid && e >= 0) {
            a.row_src[dst] = r;
            a.row_of[r] = dst;
        }
    }
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
    cudaError_t e = launch_pdl(k_hist, dim3(a.chunks), dim3(256), 0, s, a);
    if (e == cudaSuccess) e = launch_pdl(k_scan, dim3(1), dim3(256), 0, s, a);
    if (e == cudaSuccess) e = launch_pdl(k_scatter, dim3(a.chunks), dim3(32), 0, s, a);
    return e;
}

}  // namespace moe
