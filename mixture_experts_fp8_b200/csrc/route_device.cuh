// route_device.cuh -- per-token router top-k, one warp per token (the body of the router kernel,
// k_route, for moe_route, the forward and the gate).
//
// "MindIE-SD Fused MoE", routing selection and parameter table: softmax or sigmoid scores,
// optional expert-group pre-selection (group score = max, or sum of the two largest), top_k
// inside the kept groups, renormalize (softmax), normalized weights (sigmoid),
// routed_scaling_factor applied at selection.  "mlx_native ops/moe_gate.rs": top-K, softmax,
// per_expert_scale, ids and fp32 weights [T, k].
//
// Experts are ranked by their raw logits (softmax and sigmoid are monotone), ties to the lower
// index; group scores are fp32 scores, ties to the lower group.  Lane l holds experts
// l, l+32, ... (E <= 256 -> at most 8 per lane); each top-k round is a warp arg-max over
// (value desc, index asc) keys.
#pragma once

#include <math.h>

#include "moe_common.cuh"
#include "moe_kernels.h"

namespace moe {

// Keep the better of (v, i) and the partner lanes' keys; i < 0 marks "none".
__device__ __forceinline__ void argmax_reduce(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, v, o);
        int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (oi >= 0 && (i < 0 || ov > v || (ov == v && oi < i))) {
            v = ov;
            i = oi;
        }
    }
}

// Route token t with one warp (all 32 lanes).  Writes topk_idx/topk_weights [t, :] and, when
// ids_out is non-null, the ids to ids_out[t*K + j] as well.  Scratch: four per-warp arrays of 256.
__device__ __forceinline__ void route_token(const RouteArgs& a, int t, int lane, float* s_score, float* s_gscore,
                                            int* s_sel, unsigned char* s_elig, int* ids_out) {
    const float* l = a.logits + static_cast<size_t>(t) * a.E;
    const int E = a.E;

    float lv[8];
    uint32_t okmask = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        lv[i] = -INFINITY;
        if (e < E) {
            lv[i] = l[e];
            okmask |= 1u << i;
        }
    }
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (okmask >> i & 1) m = fmaxf(m, lv[i]);
    m = warp_max(m);
    float z = 0.0f;
    if (a.routing == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (okmask >> i & 1) z += expf(lv[i] - m);
        z = warp_sum(z);
    }

    // ---- expert-group pre-selection
    if (a.G > 1) {
        const int G = a.G, gs = E / G;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (okmask >> i & 1)
                s_score[lane + 32 * i] =
                    a.routing == 1 ? 1.0f / (1.0f + expf(-lv[i])) : expf(lv[i] - m) / z;
        __syncwarp();
        for (int g = lane; g < G; g += 32) {
            const float* s = &s_score[g * gs];
            float sc;
            if (a.mode == 0) {
                sc = s[0];
                for (int i = 1; i < gs; ++i) sc = fmaxf(sc, s[i]);
            } else {
                int i1 = 0, i2 = -1;
                for (int i = 1; i < gs; ++i)
                    if (s[i] > s[i1]) i1 = i;
                for (int i = 0; i < gs; ++i)
                    if (i != i1 && (i2 < 0 || s[i] > s[i2])) i2 = i;
                sc = s[i1] + s[i2];
            }
            s_gscore[g] = sc;
            s_sel[g] = 0;                          // group taken flags
        }
        __syncwarp();
        for (int r = 0; r < a.kg; ++r) {
            float bv = -INFINITY;
            int bi = -1;
            for (int g = lane; g < G; g += 32) {
                const float v = s_gscore[g];
                if (!s_sel[g] && (bi < 0 || v > bv)) {   // ascending g: ties keep lower
                    bv = v;
                    bi = g;
                }
            }
            argmax_reduce(bv, bi);
            if (lane == 0) s_sel[bi] = 1;
            __syncwarp();
        }
        for (int e = lane; e < E; e += 32) s_elig[e] = static_cast<unsigned char>(s_sel[e / gs]);
    } else {
        for (int e = lane; e < E; e += 32) s_elig[e] = 1;
    }
    __syncwarp();

    // ---- top-k experts by logit among the eligible ones
    uint32_t avail = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if ((okmask >> i & 1) && s_elig[lane + 32 * i]) avail |= 1u << i;
    for (int j = 0; j < a.K; ++j) {
        float bv = -INFINITY;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if ((avail >> i & 1) && (bi < 0 || lv[i] > bv)) {   // ascending index: ties keep lower
                bv = lv[i];
                bi = lane + 32 * i;
            }
        }
        argmax_reduce(bv, bi);
        if (bi >= 0 && (bi & 31) == lane) avail &= ~(1u << (bi >> 5));
        if (lane == 0) {
            s_sel[j] = bi;
            s_score[j] = bv;                       // the selected logit
        }
    }
    __syncwarp();

    // ---- weights (slot order, fp32)
    if (lane == 0) {
        const int K = a.K;
        float* wv = s_gscore;
        float sum = 0.0f;
        for (int j = 0; j < K; ++j) {
            const float lj = s_score[j];
            const float v = a.routing == 1 ? 1.0f / (1.0f + expf(-lj)) : expf(lj - m) / z;
            wv[j] = v;
            sum += v;
        }
        const bool norm = a.routing == 1 || a.renorm;
        for (int j = 0; j < K; ++j) {
            const int e = s_sel[j];
            float v = norm ? wv[j] / sum : wv[j];
            if (a.pes) v *= a.pes[e];
            v *= a.rsf;
            a.idx[static_cast<size_t>(t) * K + j] = e;
            a.w[static_cast<size_t>(t) * K + j] = v;
            if (ids_out) ids_out[static_cast<size_t>(t) * K + j] = e;
        }
    }
}

}  // namespace moe
