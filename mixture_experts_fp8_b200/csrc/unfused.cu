// unfused.cu -- the gate+up step taken apart, for checking the fused epilogue: a separate SwiGLU
// + requantization kernel over fp32 gate/up projections h that a GEMM stored first.
//
// "DeepGEMM PR #371", Testing: the overlapped kernel's outputs are bitwise identical to the
// non-overlapped baseline.  Here the fused gate+up GEMM (SwiGLU and requantization in its
// epilogue) must give the same E4M3 codes and scales, bit for bit, as this composition of the
// same build: the grouped GEMM storing h (its down-projection epilogue, fp32 rows, no bias), then
// k_swiglu_requant.  Both apply the same operations to the same fp32 values: + bias, silu(g) * u,
// the group's absolute maximum, its scale, the codes.
#include "gemm_common.cuh"

namespace moe {

namespace {

struct SwigluArgs {
    const float* h;             // [A, 2I] fp32, columns in the transformed (interleaved) order
    const __nv_bfloat16* bias;  // [E', 2I] original column order, or null
    const int32_t* offsets;     // [E' + 1]
    uint8_t* act_q;             // [A, I]
    void* act_s;                // [I/128][a_pad] 4-byte words
    int A, I, E, recipe, a_pad;
};

// One warp per (row, 128 act columns); lane l owns act columns 4l .. 4l+3 of the group.
__global__ void __launch_bounds__(256) k_swiglu_requant(SwigluArgs a) {
    const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int ng = a.I >> 7;
    if (gw >= a.A * ng) return;
    const int r = gw / ng, g = gw - r * ng;
    int lo = 0, hi = a.E - 1;                    // the row's expert: the last with offsets[e] <= r
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.offsets[mid] <= r) lo = mid;
        else hi = mid - 1;
    }
    const int e = lo;
    const int blk = w13_block(a.recipe);
    const int N = 2 * a.I;
    float act[4];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int c = g * 128 + 4 * lane + i;
        float gv = a.h[static_cast<size_t>(r) * N + w13_interleaved_row(c, a.I, blk)];
        float uv = a.h[static_cast<size_t>(r) * N + w13_interleaved_row(a.I + c, a.I, blk)];
        if (a.bias) {
            gv += __bfloat162float(a.bias[static_cast<size_t>(e) * N + c]);
            uv += __bfloat162float(a.bias[static_cast<size_t>(e) * N + a.I + c]);
        }
        act[i] = silu(gv) * uv;
        amax = fmaxf(amax, fabsf(act[i]));
    }
    uint32_t q;
    if (a.recipe == 0) {
        amax = warp_max(amax);
        const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        q = e4m3x4(__fdiv_rn(act[0], sc), __fdiv_rn(act[1], sc), __fdiv_rn(act[2], sc), __fdiv_rn(act[3], sc));
        if (lane == 0) static_cast<float*>(a.act_s)[static_cast<size_t>(g) * a.a_pad + r] = sc;
    } else {                                     // UE8M0 per 32 columns: eight lanes
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const int ex = mx_exponent(amax);
        const float inv = exp2_int(-ex);
        q = e4m3x4(act[0] * inv, act[1] * inv, act[2] * inv, act[3] * inv);
        if ((lane & 7) == 0)
            static_cast<uint8_t*>(a.act_s)[(static_cast<size_t>(g) * a.a_pad + r) * 4 + (lane >> 3)] =
                static_cast<uint8_t>(ex + 127);
    }
    reinterpret_cast<uint32_t*>(a.act_q + static_cast<size_t>(r) * a.I + g * 128)[lane] = q;
}

}  // namespace

cudaError_t launch_swiglu_requant(const float* h, const __nv_bfloat16* bias, const int32_t* offsets, uint8_t* act_q,
                                  void* act_s, int A, int I, int E, int recipe, int a_pad, cudaStream_t s) {
    SwigluArgs a{h, bias, offsets, act_q, act_s, A, I, E, recipe, a_pad};
    const long long warps = static_cast<long long>(A) * (I >> 7);
    if (warps == 0) return cudaSuccess;
    k_swiglu_requant<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
