// permute.cu -- stable permutation of the routed rows into expert-contiguous order.
//
// "MindIE-SD Fused MoE", execution flow: dispatch reorders tokens by expert and counts each
// expert's tokens; combine restores token order.  Slot row a = t*KT + j (slot j < k routed,
// slot k the shared expert when there is one); inside an expert, rows keep ascending a (hence
// ascending token).  The shared expert (index E) holds every token, so its count (T) and its
// rows (token order) are known without counting; it is appended after the routed experts.
// Three launches, no atomics at all, so the result is the same bits on every run:
//   1. k_hist     per-chunk expert histograms (a chunk is a multiple of kPermuteChunk routed
//                 rows, sized so that there are at most kMaxPermuteChunks chunks), counted per
//                 warp with a warp match and a population count
//   2. k_scan     per-expert exclusive bases across chunks, counts, offsets = exclusive scan,
//                 and the first 128-row GEMM tile of every expert
//   3. k_scatter  one warp per chunk walks its rows in order; rows with the same expert inside
//                 a 32-row batch are ranked with a warp match.
// Bounding the chunk count keeps k_scan's serial walk over the chunks short for large batches.
#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

// Count 32 ids of one warp into the warp's own histogram without atomics: lanes holding the same
// expert find each other with a warp match, and the lowest of them adds the group's size.  Ids
// outside [0, E) (the shared slot's marker included) are not counted; other ids outside [0, E)
// set MOE_ERR_BOUNDS.
__device__ __forceinline__ void warp_count(int* hist_w, int e, bool valid, const PermuteArgs& a) {
    const int lane = threadIdx.x & 31;
    if (valid && e != kSharedSlot && (e < 0 || e >= a.E)) set_status(a.status, MOE_ERR_BOUNDS);
    const int key = valid && e >= 0 && e < a.E ? e : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && lane == __ffs(peers) - 1) hist_w[key] += __popc(peers);
    __syncwarp();
}

__global__ void __launch_bounds__(256) k_hist(PermuteArgs a) {
    __shared__ int cnt[8][MOE_MAX_EXPERTS];            // one histogram per warp
    pdl_wait_then_release();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = lane; e < a.E; e += 32) cnt[warp][e] = 0;
    __syncwarp();
    const int begin = blockIdx.x * a.chunk;
    const int end = min(a.A, begin + a.chunk);
    for (int r0 = begin + 32 * warp; r0 < end; r0 += 256) {
        const int r = r0 + lane;
        warp_count(cnt[warp], r < end ? slot_expert(a, r) : -1, r < end, a);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int sum = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += cnt[w][e];
        a.hist[static_cast<size_t>(blockIdx.x) * a.E + e] = sum;
    }
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

// The shared expert (index E): every token, in token order, after the routed experts' rows.
__device__ __forceinline__ void append_shared(const PermuteArgs& a, int off, int ts) {
    a.counts[a.E] = a.T;
    a.offsets[a.E + 1] = off + a.T;
    a.tile_start[a.E + 1] = ts + (a.T + kTileM - 1) / kTileM;
    if (a.expert_counts) a.expert_counts[a.E] = a.T;
}

__global__ void __launch_bounds__(256) k_scan(PermuteArgs a) {
    __shared__ int tmp[16];
    pdl_wait_then_release();
    const int e = threadIdx.x;
    // all of this expert's chunk counts are loaded at once (at most kMaxPermuteChunks), then
    // replaced by their exclusive prefix
    int v[kMaxPermuteChunks];
#pragma unroll
    for (int c = 0; c < kMaxPermuteChunks; ++c)
        v[c] = (e < a.E && c < a.chunks) ? a.hist[static_cast<size_t>(c) * a.E + e] : 0;
    int run = 0;
#pragma unroll
    for (int c = 0; c < kMaxPermuteChunks; ++c) {
        if (e < a.E && c < a.chunks) a.hist[static_cast<size_t>(c) * a.E + e] = run;
        run += v[c];
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
        if (a.KT > a.k) append_shared(a, off + cnt, ts + mt);
    }
}

__global__ void __launch_bounds__(32) k_scatter(PermuteArgs a) {
    __shared__ int base[MOE_MAX_EXPERTS];
    constexpr int kBatches = kPermuteChunk / 32;
    pdl_wait_then_release();
    const int lane = threadIdx.x;
    const int begin = blockIdx.x * a.chunk;
    const int end = min(a.A, begin + a.chunk);
    for (int e = lane; e < a.E; e += 32)
        base[e] = a.offsets[e] + a.hist[static_cast<size_t>(blockIdx.x) * a.E + e];
    const int shared_base = a.KT > a.k ? a.offsets[a.E] : 0;
    __syncwarp();
    for (int p0 = begin; p0 < end; p0 += kPermuteChunk) {
        int ids[kBatches];                              // the next 256 ids, loaded at once
#pragma unroll
        for (int b = 0; b < kBatches; ++b) {
            const int r = p0 + 32 * b + lane;
            ids[b] = r < end ? slot_expert(a, r) : -1;
        }
#pragma unroll
        for (int b = 0; b < kBatches; ++b) {
            const int r = p0 + 32 * b + lane;
            const bool valid = r < end;
            int e = ids[b];
            if (valid && e == kSharedSlot) {            // the shared expert: token order
                const int dst = shared_base + r / a.KT;
                a.row_src[dst] = r;
                a.row_of[r] = dst;
            }
            if (e >= a.E) e = -1;                       // reported by k_hist; shared slots too
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
}

// ------------------------------------------------------------------------------------------
// Small batches (A <= kSmallRows): one block does what the three kernels above do, with the same
// result: per-warp histograms over 16 contiguous chunks of routed rows, per-expert bases across
// chunks, counts / offsets / tile starts, then each warp scatters its chunk in row order.
constexpr int kSmallWarps = 16;
constexpr size_t kSmallSmem = kSmallRows * 4 + kSmallWarps * MOE_MAX_EXPERTS * 4 + MOE_MAX_EXPERTS * 4;

__global__ void __launch_bounds__(kSmallWarps * 32) k_permute_small(PermuteArgs pa, int clear_status) {
    extern __shared__ uint8_t sm[];
    __shared__ int s_shared_base;                      // first row of the shared expert
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* ids = reinterpret_cast<int*>(sm);
    int* hist = ids + kSmallRows;                      // [warp][E]
    int* off_s = hist + kSmallWarps * MOE_MAX_EXPERTS;
    const int A = pa.A, E = pa.E;
    pdl_wait_then_release();
    if (clear_status && threadIdx.x == 0 && pa.status) *pa.status = MOE_OK;
    for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) hist[i] = 0;
    for (int r = threadIdx.x; r < A; r += blockDim.x) ids[r] = slot_expert(pa, r);
    __syncthreads();
    const int C = ((A + kSmallWarps - 1) / kSmallWarps + 31) / 32 * 32;
    const int begin = warp * C, end = min(A, begin + C);
    for (int r0 = begin; r0 < end; r0 += 32) {         // each warp counts its own chunk
        const int r = r0 + lane;
        warp_count(hist + warp * E, r < end ? ids[r] : -1, r < end, pa);
    }
    __syncthreads();
    if (threadIdx.x < E) {                             // bases across chunks, totals
        const int e = threadIdx.x;
        int run = 0;
        for (int w = 0; w < kSmallWarps; ++w) {
            const int v = hist[w * E + e];
            hist[w * E + e] = run;
            run += v;
        }
        off_s[e] = run;
    }
    __syncthreads();
    if (warp == 0) {                                   // scans over experts: lane l owns 8l .. 8l+7
        int c[8], mt[8], sc = 0, sm_ = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            c[i] = e < E ? off_s[e] : 0;
            mt[i] = (c[i] + kTileM - 1) / kTileM;
            sc += c[i];
            sm_ += mt[i];
        }
        int xc = sc, xm = sm_;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int yc = __shfl_up_sync(0xffffffffu, xc, o), ym = __shfl_up_sync(0xffffffffu, xm, o);
            if (lane >= o) {
                xc += yc;
                xm += ym;
            }
        }
        int base = xc - sc, mbase = xm - sm_;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            if (e < E) {
                pa.counts[e] = c[i];
                pa.offsets[e] = base;
                pa.tile_start[e] = mbase;
                if (pa.expert_counts) pa.expert_counts[e] = c[i];
                off_s[e] = base;
            }
            base += c[i];
            mbase += mt[i];
        }
        if (lane == 31) {
            pa.offsets[E] = base;
            pa.tile_start[E] = mbase;
            s_shared_base = base;
            if (pa.KT > pa.k) append_shared(pa, base, mbase);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) hist[i] += off_s[i % E];
    __syncthreads();
    for (int r0 = begin; r0 < end; r0 += 32) {         // stable scatter of this warp's chunk
        const int r = r0 + lane;
        const bool valid = r < end;
        int e = valid ? ids[r] : -1;
        if (valid && e == kSharedSlot) {                // the shared expert: token order
            const int dst = s_shared_base + r / pa.KT;
            pa.row_src[dst] = r;
            pa.row_of[r] = dst;
        }
        if (e >= E) e = -1;
        const uint32_t active = __ballot_sync(0xffffffffu, valid && e >= 0);
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const uint32_t mine = peers & active;
        const int rank = __popc(mine & ((1u << lane) - 1u));
        int dst = 0;
        if (valid && e >= 0) dst = hist[warp * E + e] + rank;
        __syncwarp();
        if (valid && e >= 0 && rank == 0) hist[warp * E + e] += __popc(mine);
        __syncwarp();
        if (valid && e >= 0) {
            pa.row_src[dst] = r;
            pa.row_of[r] = dst;
        }
    }
}

cudaError_t launch_permute_small(const PermuteArgs& pa, bool clear_status, cudaStream_t s) {
    static bool configured[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(k_permute_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kSmallSmem));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    return launch_pdl(k_permute_small, dim3(1), dim3(kSmallWarps * 32), kSmallSmem, s, pa, clear_status ? 1 : 0);
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
    cudaError_t e = launch_pdl(k_hist, dim3(a.chunks), dim3(256), 0, s, a);
    if (e == cudaSuccess) e = launch_pdl(k_scan, dim3(1), dim3(256), 0, s, a);
    if (e == cudaSuccess) e = launch_pdl(k_scatter, dim3(a.chunks), dim3(32), 0, s, a);
    return e;
}

}  // namespace moe
