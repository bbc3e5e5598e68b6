// moe_kernels.h -- host-side launchers of the kernels of libmoefp8.so (internal header).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kPermuteChunk = 256;    // granularity of the histogram / scatter chunks (routed rows)
constexpr int kMaxPermuteChunks = 64; // the per-expert scan over chunks stays this short
// Rows per chunk: a multiple of kPermuteChunk, large enough that there are at most
// kMaxPermuteChunks chunks.
inline int permute_chunk_rows(long long A) {
    const long long units = (A + kPermuteChunk - 1) / kPermuteChunk;
    const long long per = (units + kMaxPermuteChunks - 1) / kMaxPermuteChunks;
    return kPermuteChunk * static_cast<int>(per > 0 ? per : 1);
}
inline int permute_chunks(long long A) {
    const int rows = permute_chunk_rows(A);
    return static_cast<int>((A + rows - 1) / rows);
}
constexpr int kSmallRows = 2048;      // batches up to this many routed rows are permuted by one block
constexpr int kTileM = 128;           // GEMM rows per tile
constexpr int kTileN = 256;           // GEMM output columns per tile
constexpr int kTileK = 128;           // K bytes (= E4M3 elements) per pipeline stage

struct RouteArgs {
    const float* logits;        // [T, E]
    const float* pes;           // [E] or null
    int32_t* idx;               // [T, K]
    float* w;                   // [T, K]
    int T, E, K, routing, renorm, G, kg, mode;
    float rsf;
    int32_t* status;            // cleared to MOE_OK by the first thread when non-null
    // Gate mode (moe_gate): when gate_x is set, logits holds the router matmul's sums
    // sum_h x[t,h] * w'[e,h]; each token's row is first scaled in place by its RMS-Norm factor
    // 1 / sqrt(mean_h x[t,h]^2 + gate_eps), then routed.
    const __nv_bfloat16* gate_x = nullptr;   // [T, gate_H]
    int gate_H = 0;
    float gate_eps = 0.0f;
};

// The gate's router matmul (k_gate_mma): logits[t, e] = sum_h x[t,h] * w'[e,h] from the tensor
// maps of x and of the three bf16 parts of w'.
struct GateArgs {
    float* logits;              // [T, E] out
    int T, H, E;
};

// Rows r = t * KT + j of the permutation: slot j < k is routed to idx[t * k + j]; slot k (when
// KT > k) is the shared expert, index E, which every token uses.
struct PermuteArgs {
    const int32_t* idx;         // [T, k] routed expert ids
    int32_t* hist;              // [chunks, E]  (per-chunk counts, then exclusive bases)
    int32_t* counts;            // [E]
    int32_t* offsets;           // [E + 1]
    int32_t* tile_start;        // [E + 1]
    int32_t* row_src;           // [A]
    int32_t* row_of;            // [A]
    int32_t* expert_counts;     // [E] or null (caller's copy)
    int32_t* status;
    int A, E, chunks, chunk;    // A = T * KT rows; E routed experts; chunk = rows per chunk
    int T, k, KT;
};

// The expert of permutation row r: a routed expert id (range-checked by the callers), or
// kSharedSlot for the shared expert's slot.
constexpr int kSharedSlot = -2;
__host__ __device__ inline int slot_expert(const PermuteArgs& a, int r) {
    const int t = r / a.KT, j = r - t * a.KT;
    return j < a.k ? a.idx[static_cast<size_t>(t) * a.k + j] : kSharedSlot;
}

struct QuantArgs {
    const __nv_bfloat16* x;     // [T, H]
    const int32_t* row_of;      // [T, K]
    uint8_t* xq;                // [A, H]
    void* xs;                   // [H/128][a_pad] 4-byte words (fp32, or 4 x UE8M0)
    int32_t* status;
    int T, H, K, recipe, a_pad;
};

struct CombineArgs {
    const float* o;             // [rows, H]
    const int32_t* row_of;      // [T, K]  (K slots per token)
    const float* w;             // [T, k]  routing weights of the k routed slots
    __nv_bfloat16* y;           // [T, H]
    int T, H, K, k;             // slots j >= k (the shared expert's) have weight 1
    int rows;                   // rows of o: a slot whose position is outside [0, rows) adds nothing
    int32_t* status;            // and is reported here as MOE_ERR_BOUNDS (when non-null)
};

// Expert parallelism (ep.cu): slot i = t * K + j of this rank's routing.
struct EpArgs {
    const int32_t* idx;           // [A] routed expert ids (global numbering)
    int32_t* dest;                // [A] out (k_ep_dest): destination rank, -1 for an invalid id
    const int32_t* row_src;       // [A] send order -> slot (from the permutation by destination)
    const __nv_bfloat16* x;       // [T, H] this rank's tokens
    __nv_bfloat16* send_x;        // [A, H] out: token rows in send order
    int32_t* send_expert;         // [A] out: expert id local to the destination rank
    int32_t* status;
    int A, K, H, E, e_loc;        // e_loc = E / ranks
};

struct TransformArgs {
    const uint8_t* w13; const void* w13s; const uint8_t* w2; const void* w2s;
    uint8_t* w13_t; void* w13s_t; uint8_t* w2_t; void* w2s_t;
    int E, H, I, recipe;
};

struct GemmArgs {
    int mode;                   // 0: gate+up, SwiGLU, requantize; 1: down projection
    int recipe;
    int N, K, E, A;
    int a_pad;                  // row stride of the stage-major activation scales
    const int32_t* offsets;     // [E + 1]
    const int32_t* tile_start;  // [E + 1]
    const void* a_scale;        // [K/128][a_pad] 4-byte words: fp32, or 4 x UE8M0 (one per 32-block)
    const void* w_scale;        // recipe 0: fp32 [E, K/128, N]; recipe 1: 512-byte atoms [E, N/128, K/128]
    const __nv_bfloat16* bias;  // [E, N] in the caller's column order, or null
    uint8_t* act_q;             // mode 0: [A, N/2]
    void* act_s;                // mode 0: [(N/2)/128][a_pad] 4-byte words
    float* out;                 // mode 1: [A, N]
    int32_t* status;
    int fault;                  // MOE_FAULT_* (acted on only in a MOE_FAULT_INJECTION build)
};

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);
cudaError_t launch_gate(const CUtensorMap& tmX, const CUtensorMap& tmW, const GateArgs& g, const RouteArgs& ra,
                        cudaStream_t s);
cudaError_t launch_gate_split(const float* norm_w, const float* router_w, void* out, int E, int H, cudaStream_t s);
// Rows of the tensor-map boxes k_gate_mma expects: tokens (x) and experts (w' parts).
uint32_t gate_token_box();
uint32_t gate_weight_box();
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s);
cudaError_t launch_permute_small(const PermuteArgs& pa, bool clear_status, cudaStream_t s);
cudaError_t launch_quant(const QuantArgs& a, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);
cudaError_t launch_transform(const TransformArgs& a, cudaStream_t s);
cudaError_t launch_ep_dest(const EpArgs& a, cudaStream_t s);
cudaError_t launch_ep_gather(const EpArgs& a, cudaStream_t s);
cudaError_t launch_rows_f32(const float* o, const int32_t* row_of, float* out, int T, int H, int32_t* status,
                            cudaStream_t s);
// Rows of the weight tensor-map box the wide kernel expects for each mode.
uint32_t gemm_weight_box(int mode);
cudaError_t launch_gemm(const GemmArgs& a, const CUtensorMap& tmA, const CUtensorMap& tmB,
                        int num_sms, cudaStream_t s);

cudaError_t launch_gemm_mx(const GemmArgs& a, const CUtensorMap& tmA, const CUtensorMap& tmB, int num_sms,
                           cudaStream_t s);
cudaError_t launch_gemm_mx_narrow(const GemmArgs& a, const CUtensorMap& tmW, const CUtensorMap& tmT, int num_sms,
                                  cudaStream_t s);
uint32_t gemm_mx_narrow_tokens();
cudaError_t launch_gemm_narrow(const GemmArgs& a, const CUtensorMap& tmW, const CUtensorMap& tmT,
                               int num_sms, cudaStream_t s);
// The narrow (swap-AB) GEMMs take problems averaging at most this many routed rows per expert.
constexpr int kNarrowRowsPerExpert = 32;
// The SwiGLU + requantization step on its own (unfused.cu): h [A, 2I] fp32 in the transformed
// column order -> act codes and scales, as the gate+up epilogue computes them.
cudaError_t launch_swiglu_requant(const float* h, const __nv_bfloat16* bias, const int32_t* offsets, uint8_t* act_q,
                                  void* act_s, int A, int I, int E, int recipe, int a_pad, cudaStream_t s);
int set_last_error(int code, const char* msg);
cudaError_t launch_selftest_wait(int32_t* status, uint32_t timeout_us, cudaStream_t s);

// Column permutation applied to w13 by the transform: the act columns are cut into blocks of
// `blk` (128 for the fp32-scale recipe, 32 for MXFP8), and block j of gate columns is followed by
// block j of up columns: transformed rows [2*blk*j, +blk) = gate j*blk .., [2*blk*j + blk, +blk) =
// up I + j*blk ..  A GEMM epilogue thread then finds the gate and up columns of one act column in
// the same place of the two halves of a 2*blk-column tile.  Returns the transformed row index of
// original column n (0 <= n < 2I); I is a multiple of blk.
__host__ __device__ inline int w13_interleaved_row(int n, int I, int blk) {
    const int is_up = n >= I;
    const int i = is_up ? n - I : n;
    return (i / blk) * 2 * blk + is_up * blk + i % blk;
}

// Its inverse: the original column of transformed row r.
__host__ __device__ inline int w13_original_col(int r, int I, int blk) {
    const int j = r / (2 * blk), is_up = (r / blk) & 1, i = r % blk;
    const int act = j * blk + i;
    return is_up ? I + act : act;
}

// The gate/up block of each recipe.
__host__ __device__ inline int w13_block(int recipe) { return recipe != 0 ? 32 : 128; }

}  // namespace moe
