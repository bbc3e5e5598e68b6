// moefp8_api.cu -- the C ABI of libmoefp8.so (declared in include/moefp8.h): argument
// validation before any launch, workspace layout, TMA descriptors, and the launch sequence of
// the layer forward on the caller's stream.
//
// "metrale_model_layers fp8_grouped_tc_w8a8.rs": the step launches nothing unless the shapes
// fit; "mlx_native ops/moe_gate.rs": every dimension > 0, top_k <= n_experts, buffer checks,
// an InvalidArgument message; "MindIE-SD Fused MoE", routing selection: the grouped-routing
// constraints; "MATE Mega MoE", Current Limits and Typical Flow.
#include <cudaTypedefs.h>

#include <array>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "moe_common.cuh"
#include "moe_kernels.h"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok() {
    g_err.clear();
    return MOE_OK;
}

#define MOE_CUDA_TRY(expr)                                                                      \
    do {                                                                                        \
        cudaError_t _e = (expr);                                                                \
        if (_e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(_e)); \
    } while (0)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int check_config(const moe_config_t* c) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "config is NULL");
    if (c->num_tokens <= 0) return fail(MOE_ERR_INVALID_ARG, "num_tokens must be > 0 (got %d)", c->num_tokens);
    if (c->hidden <= 0) return fail(MOE_ERR_INVALID_ARG, "hidden must be > 0 (got %d)", c->hidden);
    if (c->inter <= 0) return fail(MOE_ERR_INVALID_ARG, "inter must be > 0 (got %d)", c->inter);
    if (c->num_experts <= 0) return fail(MOE_ERR_INVALID_ARG, "num_experts must be > 0 (got %d)", c->num_experts);
    if (c->top_k < 1 || c->top_k > c->num_experts)
        return fail(MOE_ERR_INVALID_ARG, "top_k (%d) must be in [1, num_experts=%d]", c->top_k, c->num_experts);
    if (c->routing != 0 && c->routing != 1)
        return fail(MOE_ERR_INVALID_ARG, "routing must be 0 (softmax) or 1 (sigmoid), got %d", c->routing);
    if (c->recipe < 0 || c->recipe > 2)
        return fail(MOE_ERR_INVALID_ARG, "recipe must be 0 (fp32 per 128), 1 (MXFP8) or 2 (W4A8), got %d",
                    c->recipe);
    if (c->hidden % 128) return fail(MOE_ERR_UNSUPPORTED, "hidden (%d) must be a multiple of 128", c->hidden);
    if (c->inter % 128) return fail(MOE_ERR_UNSUPPORTED, "inter (%d) must be a multiple of 128", c->inter);
    if (c->num_experts > MOE_MAX_EXPERTS)
        return fail(MOE_ERR_UNSUPPORTED, "num_experts (%d) exceeds %d", c->num_experts, MOE_MAX_EXPERTS);
    if (c->shared_experts != 0 && c->shared_experts != 1)
        return fail(MOE_ERR_UNSUPPORTED, "shared_experts must be 0 or 1, got %d", c->shared_experts);
    if (c->group_count < 1 || c->num_experts % c->group_count)
        return fail(MOE_ERR_UNSUPPORTED, "num_experts (%d) must be divisible by group_count (%d)", c->num_experts,
                    c->group_count);
    if (c->k_group < 1 || c->k_group > c->group_count)
        return fail(MOE_ERR_UNSUPPORTED, "k_group (%d) must be in [1, group_count=%d]", c->k_group, c->group_count);
    const int per_group = c->num_experts / c->group_count;
    if (c->top_k > c->k_group * per_group)
        return fail(MOE_ERR_UNSUPPORTED, "top_k (%d) exceeds the experts in the selected groups (%d)", c->top_k,
                    c->k_group * per_group);
    if (c->group_select_mode != 0 && c->group_select_mode != 1)
        return fail(MOE_ERR_INVALID_ARG, "group_select_mode must be 0 or 1, got %d", c->group_select_mode);
    if (c->group_select_mode == 1 && per_group < 2)
        return fail(MOE_ERR_UNSUPPORTED, "group_select_mode 1 needs at least 2 experts per group");
    const long long A = 1LL * c->num_tokens * (c->top_k + c->shared_experts);
    const long long ET = c->num_experts + c->shared_experts;
    if (A > (1LL << 30) || ET * 2 * c->inter > (1LL << 30) || ET * c->hidden > (1LL << 30))
        return fail(MOE_ERR_UNSUPPORTED, "problem too large for 32-bit row indices");
    return MOE_OK;
}

// Row stride of the stage-major scale arrays: every routed row, plus room for a 128-row tile
// read starting at a 16-byte-aligned row just before the last row.
// Fault armed by moe_debug_inject_fault for the next forward on this host thread (debug
// library only; always MOE_FAULT_NONE in the release library).
thread_local int t_armed_fault = MOE_FAULT_NONE;
int take_armed_fault() {
    const int f = t_armed_fault;
    t_armed_fault = MOE_FAULT_NONE;
    return f;
}

// Rows of the stage-major activation scales: every routed row, plus the reach of the last GEMM
// tile's 16-byte-aligned scale run (132 words from its first row rounded down to 4).
size_t scale_rows_of(size_t A) { return align_up(A + moe::kTileM + 4, 4); }

void layout_of(const moe_config_t* c, moe_workspace_layout_t* L) {
    // k routed slots per token (the router's output), KT = k + shared slots, E routed experts,
    // ET = E + shared, A = T * KT permuted rows
    const size_t T = c->num_tokens, K = c->top_k, E = c->num_experts, H = c->hidden, I = c->inter;
    const size_t KT = K + c->shared_experts, ET = E + c->shared_experts;
    const size_t A = T * KT, SR = scale_rows_of(A);
    const size_t chunks = moe::permute_chunks(static_cast<long long>(A));
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 1024);
        return o;
    };
    L->status = take(16);
    L->topk_idx = take(4 * T * K);
    L->topk_weights = take(4 * T * K);
    L->counts = take(4 * ET);
    L->offsets = take(4 * (ET + 1));
    L->tile_start = take(4 * (ET + 1));
    L->row_src = take(4 * A);
    L->row_of = take(4 * A);
    L->hist = take(4 * chunks * E);
    L->xq = take(A * H);
    L->xs = take((H / 128) * SR * 4);
    L->act_q = take(A * I);
    L->act_s = take((I / 128) * SR * 4);
    L->o = take(4 * A * H);
    L->scale_rows = SR;
    L->total = off;
}

// ---- device facts, looked up once per device
struct DeviceInfo {
    int sms = 0;
    int cc_major = 0, cc_minor = 0;
};

int device_info(DeviceInfo* out) {
    static std::mutex mu;
    static std::array<DeviceInfo, 64> cache{};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev].sms == 0) {
        DeviceInfo d;
        MOE_CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        MOE_CUDA_TRY(cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev));
        MOE_CUDA_TRY(cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev));
        cache[dev] = d;
    }
    *out = cache[dev];
    if (out->cc_major != 10 || out->cc_minor != 0)
        return fail(MOE_ERR_UNSUPPORTED, "libmoefp8 is built for sm_100a (B200); device is sm_%d%d", out->cc_major,
                    out->cc_minor);
    return MOE_OK;
}

// ---- TMA descriptors (the driver entry point is fetched through the runtime; no -lcuda)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2D map over a row-major matrix [rows, cols] of 8-bit codes (cols = K, contiguous), box
// box_rows x 128, 128-byte swizzle; rows past the end read as zero.  fp4: the codes are E2M1
// packed two per byte (a row is cols / 2 bytes); each 16 codes land in a 16-byte slot of shared
// memory (8 bytes of codes, 8 bytes of gap), the layout the tensor core takes for 4-bit operands.
int make_kmajor_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                    bool fp4 = false) {
    auto fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {fp4 ? cols / 2 : cols};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                    const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return MOE_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

namespace moe {
// Record a message as the calling thread's last error (for entry points in other files).
int set_last_error(int code, const char* msg) {
    g_err = msg ? msg : "";
    return code;
}
}  // namespace moe

// ============================================================================ profiler
struct moe_profile {
    std::vector<std::array<cudaEvent_t, MOE_NUM_STAGES + 1>> sets;
    size_t used = 0;
    double totals[MOE_NUM_STAGES] = {0};
    int32_t calls = 0;
};

namespace {

int prof_next(moe_profile* p, cudaEvent_t** ev) {
    if (p->used == p->sets.size()) {
        if (p->sets.size() >= 4096) return fail(MOE_ERR_INVALID_ARG, "profiler holds 4096 unread calls; read it");
        std::array<cudaEvent_t, MOE_NUM_STAGES + 1> s{};
        for (auto& e : s) MOE_CUDA_TRY(cudaEventCreate(&e));
        p->sets.push_back(s);
    }
    *ev = p->sets[p->used++].data();
    return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_last_error(void) { return g_err.c_str(); }

int moe_check_config(const moe_config_t* cfg) {
    int rc = check_config(cfg);
    return rc ? rc : ok();
}

int moe_transformed_weights_size(const moe_config_t* cfg, size_t* w13_bytes, size_t* w13s_bytes, size_t* w2_bytes,
                                 size_t* w2s_bytes) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!w13_bytes || !w13s_bytes || !w2_bytes || !w2s_bytes) return fail(MOE_ERR_INVALID_ARG, "NULL size pointer");
    const size_t E = cfg->num_experts + cfg->shared_experts, H = cfg->hidden, I = cfg->inter;
    const size_t pk = cfg->recipe == 2 ? 2 : 1;   // W4A8: two E2M1 codes per byte
    *w13_bytes = E * 2 * I * H / pk;
    *w13s_bytes = E * (H / 128) * 2 * I * 4;
    *w2_bytes = E * H * I / pk;
    *w2s_bytes = E * (I / 128) * H * 4;
    return ok();
}

int moe_transform_weights(const moe_config_t* cfg, const void* w13, const void* w13_scale, const void* w2,
                          const void* w2_scale, void* w13_t, void* w13s_t, void* w2_t, void* w2s_t, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!w13 || !w13_scale || !w2 || !w2_scale || !w13_t || !w13s_t || !w2_t || !w2s_t)
        return fail(MOE_ERR_INVALID_ARG, "moe_transform_weights: NULL pointer");
    if (!aligned(w13_scale, 4) || !aligned(w2_scale, 4) || !aligned(w13s_t, 16) || !aligned(w2s_t, 16) ||
        !aligned(w13_t, 32) || !aligned(w2_t, 32))
        return fail(MOE_ERR_INVALID_ARG,
                    "moe_transform_weights: misaligned buffer (transformed codes need 32 bytes, scales 16)");
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    moe::TransformArgs a{static_cast<const uint8_t*>(w13), w13_scale, static_cast<const uint8_t*>(w2), w2_scale,
                         static_cast<uint8_t*>(w13_t), w13s_t, static_cast<uint8_t*>(w2_t), w2s_t,
                         cfg->num_experts + cfg->shared_experts, cfg->hidden, cfg->inter, cfg->recipe};
    MOE_CUDA_TRY(moe::launch_transform(a, static_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!bytes) return fail(MOE_ERR_INVALID_ARG, "NULL bytes pointer");
    moe_workspace_layout_t L;
    layout_of(cfg, &L);
    *bytes = L.total;
    return ok();
}

int moe_workspace_layout(const moe_config_t* cfg, moe_workspace_layout_t* layout) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!layout) return fail(MOE_ERR_INVALID_ARG, "NULL layout pointer");
    layout_of(cfg, layout);
    return ok();
}

int moe_route(const moe_config_t* cfg, const float* router_logits, const float* per_expert_scale, int32_t* topk_idx,
              float* topk_weights, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!router_logits || !topk_idx || !topk_weights) return fail(MOE_ERR_INVALID_ARG, "moe_route: NULL pointer");
    if (!aligned(router_logits, 4) || !aligned(topk_idx, 4) || !aligned(topk_weights, 4))
        return fail(MOE_ERR_INVALID_ARG, "moe_route: misaligned buffer");
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    moe::RouteArgs a{router_logits, per_expert_scale, topk_idx, topk_weights, cfg->num_tokens, cfg->num_experts,
                     cfg->top_k, cfg->routing, cfg->renormalize, cfg->group_count, cfg->k_group,
                     cfg->group_select_mode, cfg->routed_scaling_factor, nullptr};
    MOE_CUDA_TRY(moe::launch_route(a, static_cast<cudaStream_t>(stream)));
    return ok();
}

namespace {

// The forward.  Its last stage is the combine into bf16 y, or, with o_rows set (one slot per row,
// the expert side of expert parallelism), the fp32 GEMM2 rows copied out in row order.
int forward_impl(const moe_config_t* cfg, const void* hidden_states, const float* router_logits,
                 const float* per_expert_scale, const int32_t* topk_idx, const float* topk_weights,
                 const void* w13_t, const void* w13s_t, const void* w2_t, const void* w2s_t,
                 const void* w13_bias, const void* w2_bias, void* y, float* o_rows, int32_t* expert_counts,
                 void* workspace, size_t workspace_bytes, moe_profile_t* prof, void* stream_) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!hidden_states || (!y && !o_rows) || !w13_t || !w13s_t || !w2_t || !w2s_t || !workspace)
        return fail(MOE_ERR_INVALID_ARG, "moe_forward: NULL pointer");
    if ((router_logits == nullptr) == (topk_idx == nullptr))
        return fail(MOE_ERR_INVALID_ARG, "moe_forward: pass exactly one of router_logits and topk_idx");
    if (topk_idx && !topk_weights && !o_rows)
        return fail(MOE_ERR_INVALID_ARG, "moe_forward: topk_idx needs topk_weights");
    if (!aligned(hidden_states, 16) || !aligned(y ? y : static_cast<void*>(o_rows), 16) || !aligned(w13_t, 32) ||
        !aligned(w2_t, 32) ||
        !aligned(w13s_t, 16) || !aligned(w2s_t, 16) || !aligned(workspace, 256) ||
        (router_logits && !aligned(router_logits, 4)) || (topk_idx && !aligned(topk_idx, 4)) ||
        (topk_weights && !aligned(topk_weights, 4)) || (w13_bias && !aligned(w13_bias, 16)) ||
        (w2_bias && !aligned(w2_bias, 16)) || (expert_counts && !aligned(expert_counts, 4)))
        return fail(MOE_ERR_INVALID_ARG,
                    "moe_forward: misaligned buffer (hidden_states, y, biases and scales need 16 bytes, "
                    "weight codes 32, workspace 256)");
    moe_workspace_layout_t L;
    layout_of(cfg, &L);
    if (workspace_bytes < L.total)
        return fail(MOE_ERR_INVALID_ARG, "moe_forward: workspace has %zu bytes, needs %zu", workspace_bytes, L.total);
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;

    // K routed slots per token, KT with the shared expert's slot; E routed experts, ET in all
    const int T = cfg->num_tokens, K = cfg->top_k, E = cfg->num_experts, H = cfg->hidden, I = cfg->inter;
    const int KT = K + cfg->shared_experts, ET = E + cfg->shared_experts;
    const int A = T * KT;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
    int32_t* status = static_cast<int32_t*>(at(L.status));
    const int32_t* idx = topk_idx ? topk_idx : static_cast<const int32_t*>(at(L.topk_idx));
    const float* wts = topk_idx ? topk_weights : static_cast<const float*>(at(L.topk_weights));

    // Few rows per expert (decode, at most kNarrowRowsPerExpert on average) take the swap-AB
    // kernels, the weights as the M operand; else the wide kernels.  fp32 scales: both compute every
    // row with the same operations in the same order.  MXFP8 and W4A8 run the block-scaled tensor
    // core kernels, swap-AB (gemm_mx_narrow.cu) or wide (gemm_mx.cu).
    const bool mx = cfg->recipe != 0;     // MXFP8 and W4A8: the block-scaled kernels
    const bool fp4 = cfg->recipe == 2;
    const bool narrow = A <= moe::kNarrowRowsPerExpert * ET;
    CUtensorMap tm_x, tm_w13, tm_act, tm_w2;
    const uint32_t tok_box = !narrow ? moe::kTileM : mx ? moe::gemm_mx_narrow_tokens() : 16;
    const uint32_t w13_box = mx ? 128 : narrow ? moe::kTileN : moe::gemm_weight_box(0);
    const uint32_t w2_box = mx ? 128 : narrow ? moe::kTileN : moe::gemm_weight_box(1);
    if ((rc = make_kmajor_map(&tm_x, at(L.xq), A, H, tok_box))) return rc;
    if ((rc = make_kmajor_map(&tm_w13, w13_t, static_cast<uint64_t>(ET) * 2 * I, H, w13_box, fp4))) return rc;
    if ((rc = make_kmajor_map(&tm_act, at(L.act_q), A, I, tok_box))) return rc;
    if ((rc = make_kmajor_map(&tm_w2, w2_t, static_cast<uint64_t>(ET) * H, I, w2_box, fp4))) return rc;

    cudaEvent_t* ev = nullptr;
    if (prof && (rc = prof_next(prof, &ev))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream_);
    auto mark = [&](int i) -> cudaError_t { return ev ? cudaEventRecord(ev[i], s) : cudaSuccess; };

    moe::RouteArgs ra{router_logits, per_expert_scale, static_cast<int32_t*>(at(L.topk_idx)),
                      static_cast<float*>(at(L.topk_weights)), T, E, K, cfg->routing, cfg->renormalize,
                      cfg->group_count, cfg->k_group, cfg->group_select_mode, cfg->routed_scaling_factor,
                      nullptr};
    moe::PermuteArgs pa{idx, static_cast<int32_t*>(at(L.hist)), static_cast<int32_t*>(at(L.counts)),
                        static_cast<int32_t*>(at(L.offsets)), static_cast<int32_t*>(at(L.tile_start)),
                        static_cast<int32_t*>(at(L.row_src)), static_cast<int32_t*>(at(L.row_of)), expert_counts,
                        status, A, E, moe::permute_chunks(A), moe::permute_chunk_rows(A), T, K, KT};
    MOE_CUDA_TRY(mark(0));
    // The first kernel of the forward clears the status word: the router when it runs, else the
    // small-batch permutation; a memset otherwise.
    if (router_logits) {
        ra.status = status;
        MOE_CUDA_TRY(moe::launch_route(ra, s));
    } else if (A > moe::kSmallRows) {
        MOE_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
    }
    MOE_CUDA_TRY(mark(1));
    if (A <= moe::kSmallRows) MOE_CUDA_TRY(moe::launch_permute_small(pa, router_logits == nullptr, s));
    else MOE_CUDA_TRY(moe::launch_permute(pa, s));
    MOE_CUDA_TRY(mark(2));
    moe::QuantArgs qa{static_cast<const __nv_bfloat16*>(hidden_states), static_cast<const int32_t*>(at(L.row_of)),
                      static_cast<uint8_t*>(at(L.xq)), at(L.xs), status, T, H, KT, cfg->recipe,
                      static_cast<int>(L.scale_rows)};
    MOE_CUDA_TRY(moe::launch_quant(qa, s));
    MOE_CUDA_TRY(mark(3));
    moe::GemmArgs g1{};
    g1.mode = 0;
    g1.recipe = cfg->recipe;
    g1.N = 2 * I;
    g1.K = H;
    g1.E = ET;
    g1.A = A;
    g1.a_pad = static_cast<int>(L.scale_rows);
    g1.offsets = static_cast<const int32_t*>(at(L.offsets));
    g1.tile_start = static_cast<const int32_t*>(at(L.tile_start));
    g1.a_scale = at(L.xs);
    g1.w_scale = w13s_t;
    g1.bias = static_cast<const __nv_bfloat16*>(w13_bias);
    g1.act_q = static_cast<uint8_t*>(at(L.act_q));
    g1.act_s = at(L.act_s);
    g1.status = status;
    g1.fault = take_armed_fault();
    MOE_CUDA_TRY(mx ? (narrow ? moe::launch_gemm_mx_narrow(g1, tm_w13, tm_x, di.sms, s)
                              : moe::launch_gemm_mx(g1, tm_x, tm_w13, di.sms, s))
                    : (narrow ? moe::launch_gemm_narrow(g1, tm_w13, tm_x, di.sms, s)
                              : moe::launch_gemm(g1, tm_x, tm_w13, di.sms, s)));
    MOE_CUDA_TRY(mark(4));
    moe::GemmArgs g2 = g1;
    g2.mode = 1;
    g2.fault = MOE_FAULT_NONE;
    g2.N = H;
    g2.K = I;
    g2.a_scale = at(L.act_s);
    g2.w_scale = w2s_t;
    g2.bias = static_cast<const __nv_bfloat16*>(w2_bias);
    g2.act_q = nullptr;
    g2.act_s = nullptr;
    g2.out = static_cast<float*>(at(L.o));
    MOE_CUDA_TRY(mx ? (narrow ? moe::launch_gemm_mx_narrow(g2, tm_w2, tm_act, di.sms, s)
                              : moe::launch_gemm_mx(g2, tm_act, tm_w2, di.sms, s))
                    : (narrow ? moe::launch_gemm_narrow(g2, tm_w2, tm_act, di.sms, s)
                              : moe::launch_gemm(g2, tm_act, tm_w2, di.sms, s)));
    MOE_CUDA_TRY(mark(5));
    if (o_rows) {
        MOE_CUDA_TRY(moe::launch_rows_f32(static_cast<const float*>(at(L.o)),
                                          static_cast<const int32_t*>(at(L.row_of)), o_rows, T, H, status, s));
    } else {
        moe::CombineArgs ca{static_cast<const float*>(at(L.o)), static_cast<const int32_t*>(at(L.row_of)), wts,
                            static_cast<__nv_bfloat16*>(y), T, H, KT, K, A, status};
        MOE_CUDA_TRY(moe::launch_combine(ca, s));
    }
    MOE_CUDA_TRY(mark(6));
    return ok();
}

int check_ep(const moe_config_t* cfg, int ranks, const char* who) {
    if (cfg->shared_experts != 0)
        return fail(MOE_ERR_UNSUPPORTED, "%s: expert parallelism takes no shared expert", who);
    if (ranks < 1 || ranks > cfg->num_experts || cfg->num_experts % ranks != 0)
        return fail(MOE_ERR_UNSUPPORTED, "%s: ranks (%d) must divide num_experts (%d)", who, ranks,
                    cfg->num_experts);
    return MOE_OK;
}

}  // namespace

int moe_forward_profiled(const moe_config_t* cfg, const void* hidden_states, const float* router_logits,
                         const float* per_expert_scale, const int32_t* topk_idx, const float* topk_weights,
                         const void* w13_t, const void* w13s_t, const void* w2_t, const void* w2s_t,
                         const void* w13_bias, const void* w2_bias, void* y, int32_t* expert_counts, void* workspace,
                         size_t workspace_bytes, moe_profile_t* prof, void* stream_) {
    if (!y) return fail(MOE_ERR_INVALID_ARG, "moe_forward: NULL pointer");
    return forward_impl(cfg, hidden_states, router_logits, per_expert_scale, topk_idx, topk_weights, w13_t, w13s_t,
                        w2_t, w2s_t, w13_bias, w2_bias, y, nullptr, expert_counts, workspace, workspace_bytes, prof,
                        stream_);
}

int moe_forward_rows(const moe_config_t* cfg, const void* rows, const int32_t* expert_of_row, const void* w13_t,
                     const void* w13s_t, const void* w2_t, const void* w2s_t, const void* w13_bias,
                     const void* w2_bias, float* o_rows, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (cfg->top_k != 1 || cfg->shared_experts != 0)
        return fail(MOE_ERR_INVALID_ARG, "moe_forward_rows: one slot per row (top_k 1, no shared expert)");
    if (!rows || !expert_of_row || !o_rows) return fail(MOE_ERR_INVALID_ARG, "moe_forward_rows: NULL pointer");
    return forward_impl(cfg, rows, nullptr, nullptr, expert_of_row, nullptr, w13_t, w13s_t, w2_t, w2s_t, w13_bias,
                        w2_bias, nullptr, o_rows, nullptr, workspace, workspace_bytes, nullptr, stream);
}

int moe_debug_unfused_gate_up(const moe_config_t* cfg, const void* hidden_states, const int32_t* topk_idx,
                              const void* w13_t, const void* w13s_t, const void* w13_bias, float* h,
                              void* workspace, size_t workspace_bytes, void* stream_) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!hidden_states || !topk_idx || !w13_t || !w13s_t || !h || !workspace)
        return fail(MOE_ERR_INVALID_ARG, "moe_debug_unfused_gate_up: NULL pointer");
    if (!aligned(hidden_states, 16) || !aligned(topk_idx, 4) || !aligned(w13_t, 32) || !aligned(w13s_t, 16) ||
        !aligned(h, 32) || !aligned(workspace, 256) || (w13_bias && !aligned(w13_bias, 16)))
        return fail(MOE_ERR_INVALID_ARG, "moe_debug_unfused_gate_up: misaligned buffer");
    moe_workspace_layout_t L;
    layout_of(cfg, &L);
    if (workspace_bytes < L.total)
        return fail(MOE_ERR_INVALID_ARG, "moe_debug_unfused_gate_up: workspace has %zu bytes, needs %zu",
                    workspace_bytes, L.total);
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    const int T = cfg->num_tokens, K = cfg->top_k, E = cfg->num_experts, H = cfg->hidden, I = cfg->inter;
    const int KT = K + cfg->shared_experts, ET = E + cfg->shared_experts;
    const int A = T * KT;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
    int32_t* status = static_cast<int32_t*>(at(L.status));
    // the forward's choice of GEMM kernel and tensor-map boxes (see forward_impl)
    const bool mx = cfg->recipe != 0;
    const bool fp4 = cfg->recipe == 2;
    const bool narrow = A <= moe::kNarrowRowsPerExpert * ET;
    CUtensorMap tm_x, tm_w13;
    const uint32_t tok_box = !narrow ? moe::kTileM : mx ? moe::gemm_mx_narrow_tokens() : 16;
    const uint32_t w13_box = mx ? 128 : narrow ? moe::kTileN : moe::gemm_weight_box(0);
    if ((rc = make_kmajor_map(&tm_x, at(L.xq), A, H, tok_box))) return rc;
    if ((rc = make_kmajor_map(&tm_w13, w13_t, static_cast<uint64_t>(ET) * 2 * I, H, w13_box, fp4))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream_);
    MOE_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
    moe::PermuteArgs pa{topk_idx, static_cast<int32_t*>(at(L.hist)), static_cast<int32_t*>(at(L.counts)),
                        static_cast<int32_t*>(at(L.offsets)), static_cast<int32_t*>(at(L.tile_start)),
                        static_cast<int32_t*>(at(L.row_src)), static_cast<int32_t*>(at(L.row_of)), nullptr,
                        status, A, E, moe::permute_chunks(A), moe::permute_chunk_rows(A), T, K, KT};
    if (A <= moe::kSmallRows) MOE_CUDA_TRY(moe::launch_permute_small(pa, false, s));
    else MOE_CUDA_TRY(moe::launch_permute(pa, s));
    moe::QuantArgs qa{static_cast<const __nv_bfloat16*>(hidden_states), static_cast<const int32_t*>(at(L.row_of)),
                      static_cast<uint8_t*>(at(L.xq)), at(L.xs), status, T, H, KT, cfg->recipe,
                      static_cast<int>(L.scale_rows)};
    MOE_CUDA_TRY(moe::launch_quant(qa, s));
    // GEMM1 with the down projection's epilogue: h = the promoted gate/up sums, fp32, no bias
    moe::GemmArgs g{};
    g.mode = 1;
    g.recipe = cfg->recipe;
    g.N = 2 * I;
    g.K = H;
    g.E = ET;
    g.A = A;
    g.a_pad = static_cast<int>(L.scale_rows);
    g.offsets = static_cast<const int32_t*>(at(L.offsets));
    g.tile_start = static_cast<const int32_t*>(at(L.tile_start));
    g.a_scale = at(L.xs);
    g.w_scale = w13s_t;
    g.bias = nullptr;
    g.out = h;
    g.status = status;
    g.fault = MOE_FAULT_NONE;
    MOE_CUDA_TRY(mx ? (narrow ? moe::launch_gemm_mx_narrow(g, tm_w13, tm_x, di.sms, s)
                              : moe::launch_gemm_mx(g, tm_x, tm_w13, di.sms, s))
                    : (narrow ? moe::launch_gemm_narrow(g, tm_w13, tm_x, di.sms, s)
                              : moe::launch_gemm(g, tm_x, tm_w13, di.sms, s)));
    MOE_CUDA_TRY(moe::launch_swiglu_requant(h, static_cast<const __nv_bfloat16*>(w13_bias),
                                            static_cast<const int32_t*>(at(L.offsets)),
                                            static_cast<uint8_t*>(at(L.act_q)), at(L.act_s), A, I, ET, cfg->recipe,
                                            static_cast<int>(L.scale_rows), s));
    return ok();
}

int moe_ep_dispatch(const moe_config_t* cfg, int ranks, const void* hidden_states, const int32_t* topk_idx,
                    int32_t* send_counts, void* send_x, int32_t* send_expert, int32_t* slot_pos, void* workspace,
                    size_t workspace_bytes, void* stream_) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if ((rc = check_ep(cfg, ranks, "moe_ep_dispatch"))) return rc;
    if (!hidden_states || !topk_idx || !send_counts || !send_x || !send_expert || !slot_pos || !workspace)
        return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: NULL pointer");
    if (!aligned(hidden_states, 16) || !aligned(send_x, 16) || !aligned(topk_idx, 4) || !aligned(send_counts, 4) ||
        !aligned(send_expert, 4) || !aligned(slot_pos, 4) || !aligned(workspace, 256))
        return fail(MOE_ERR_INVALID_ARG,
                    "moe_ep_dispatch: misaligned buffer (rows need 16 bytes, workspace 256, ids 4)");
    moe_workspace_layout_t L;
    layout_of(cfg, &L);
    if (workspace_bytes < L.total)
        return fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch: workspace has %zu bytes, needs %zu", workspace_bytes,
                    L.total);
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    const int T = cfg->num_tokens, K = cfg->top_k, E = cfg->num_experts, A = T * K;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
    int32_t* status = static_cast<int32_t*>(at(L.status));
    int32_t* dest = static_cast<int32_t*>(at(L.topk_idx));     // [A], free while topk_idx is the caller's
    int32_t* row_src = static_cast<int32_t*>(at(L.row_src));
    cudaStream_t s = static_cast<cudaStream_t>(stream_);
    MOE_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
    // a slot that is not sent (an expert id out of range) keeps position -1
    MOE_CUDA_TRY(cudaMemsetAsync(slot_pos, 0xFF, sizeof(int32_t) * static_cast<size_t>(A), s));
    moe::EpArgs ea{topk_idx, dest, row_src, static_cast<const __nv_bfloat16*>(hidden_states),
                   static_cast<__nv_bfloat16*>(send_x), send_expert, status, A, K, cfg->hidden, E, E / ranks};
    MOE_CUDA_TRY(moe::launch_ep_dest(ea, s));
    // the permutation with the destination ranks as its "experts": counts = send counts,
    // row_src = send order, row_of = each slot's position in it
    moe::PermuteArgs pa{dest, static_cast<int32_t*>(at(L.hist)), send_counts, static_cast<int32_t*>(at(L.offsets)),
                        static_cast<int32_t*>(at(L.tile_start)), row_src, slot_pos, nullptr, status, A, ranks,
                        moe::permute_chunks(A), moe::permute_chunk_rows(A), T, K, K};
    if (A <= moe::kSmallRows) MOE_CUDA_TRY(moe::launch_permute_small(pa, false, s));
    else MOE_CUDA_TRY(moe::launch_permute(pa, s));
    MOE_CUDA_TRY(moe::launch_ep_gather(ea, s));
    return ok();
}

int moe_combine_rows(const moe_config_t* cfg, const float* o_rows, int32_t num_rows, const int32_t* slot_pos,
                     const float* topk_weights, void* y, int32_t* status, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (cfg->shared_experts != 0)
        return fail(MOE_ERR_UNSUPPORTED, "moe_combine_rows: expert parallelism takes no shared expert");
    if (num_rows < 0 || static_cast<long long>(num_rows) > static_cast<long long>(cfg->num_tokens) * cfg->top_k)
        return fail(MOE_ERR_INVALID_ARG, "moe_combine_rows: num_rows %d outside [0, T*k]", num_rows);
    if ((!o_rows && num_rows > 0) || !slot_pos || !topk_weights || !y)
        return fail(MOE_ERR_INVALID_ARG, "moe_combine_rows: NULL pointer");
    if (!aligned(o_rows, 16) || !aligned(y, 16) || !aligned(slot_pos, 4) || !aligned(topk_weights, 4) ||
        !aligned(status, 4))
        return fail(MOE_ERR_INVALID_ARG, "moe_combine_rows: misaligned buffer (rows need 16 bytes)");
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    moe::CombineArgs ca{o_rows, slot_pos, topk_weights, static_cast<__nv_bfloat16*>(y), cfg->num_tokens, cfg->hidden,
                        cfg->top_k, cfg->top_k, num_rows, status};
    MOE_CUDA_TRY(moe::launch_combine(ca, static_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_gate_weights_size(const moe_config_t* cfg, size_t* bytes) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!bytes) return fail(MOE_ERR_INVALID_ARG, "moe_gate_weights_size: NULL output");
    *bytes = static_cast<size_t>(3) * cfg->num_experts * cfg->hidden * 2;
    return ok();
}

int moe_transform_gate_weights(const moe_config_t* cfg, const float* norm_weight, const float* router_weight,
                               void* gate_weights, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!norm_weight || !router_weight || !gate_weights)
        return fail(MOE_ERR_INVALID_ARG, "moe_transform_gate_weights: NULL pointer");
    if (!aligned(norm_weight, 16) || !aligned(router_weight, 16) || !aligned(gate_weights, 16))
        return fail(MOE_ERR_INVALID_ARG, "moe_transform_gate_weights: buffers need 16-byte alignment");
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    MOE_CUDA_TRY(moe::launch_gate_split(norm_weight, router_weight, gate_weights, cfg->num_experts, cfg->hidden,
                                        static_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_gate(const moe_config_t* cfg, const void* hidden_states, const void* gate_weights, float rms_eps,
             const float* per_expert_scale, float* logits, int32_t* topk_idx, float* topk_weights, void* stream) {
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!hidden_states || !gate_weights || !logits || !topk_idx || !topk_weights)
        return fail(MOE_ERR_INVALID_ARG, "moe_gate: NULL pointer");
    if (!aligned(hidden_states, 16) || !aligned(gate_weights, 16) || !aligned(logits, 4) || !aligned(topk_idx, 4) ||
        !aligned(topk_weights, 4) || (per_expert_scale && !aligned(per_expert_scale, 4)))
        return fail(MOE_ERR_INVALID_ARG, "moe_gate: misaligned buffer (hidden_states and gate_weights need 16 bytes)");
    if (!(rms_eps >= 0.0f)) return fail(MOE_ERR_INVALID_ARG, "moe_gate: rms_eps must be >= 0");
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    const int T = cfg->num_tokens, H = cfg->hidden, E = cfg->num_experts;
    // bf16 rows viewed as bytes: 64 columns = one 128-byte box row
    CUtensorMap tm_x, tm_w;
    if ((rc = make_kmajor_map(&tm_x, hidden_states, T, 2ull * H, moe::gate_token_box()))) return rc;
    if ((rc = make_kmajor_map(&tm_w, gate_weights, 3ull * E, 2ull * H, moe::gate_weight_box()))) return rc;
    moe::GateArgs g{logits, T, H, E};
    moe::RouteArgs ra{logits, per_expert_scale, topk_idx, topk_weights, T, E, cfg->top_k, cfg->routing,
                      cfg->renormalize, cfg->group_count, cfg->k_group, cfg->group_select_mode,
                      cfg->routed_scaling_factor, nullptr};
    ra.gate_x = static_cast<const __nv_bfloat16*>(hidden_states);
    ra.gate_H = H;
    ra.gate_eps = rms_eps;
    MOE_CUDA_TRY(moe::launch_gate(tm_x, tm_w, g, ra, static_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_forward(const moe_config_t* cfg, const void* hidden_states, const float* router_logits,
                const float* per_expert_scale, const int32_t* topk_idx, const float* topk_weights, const void* w13_t,
                const void* w13s_t, const void* w2_t, const void* w2s_t, const void* w13_bias, const void* w2_bias,
                void* y, int32_t* expert_counts, void* workspace, size_t workspace_bytes, void* stream) {
    return moe_forward_profiled(cfg, hidden_states, router_logits, per_expert_scale, topk_idx, topk_weights, w13_t,
                                w13s_t, w2_t, w2s_t, w13_bias, w2_bias, y, expert_counts, workspace, workspace_bytes,
                                nullptr, stream);
}

int moe_profile_create(moe_profile_t** prof) {
    if (!prof) return fail(MOE_ERR_INVALID_ARG, "NULL profiler pointer");
    *prof = new moe_profile();
    return ok();
}

int moe_profile_destroy(moe_profile_t* prof) {
    if (!prof) return ok();
    for (auto& s : prof->sets)
        for (auto& e : s) cudaEventDestroy(e);
    delete prof;
    return ok();
}

int moe_profile_read(moe_profile_t* prof, float* stage_ms, int32_t* calls) {
    if (!prof) return fail(MOE_ERR_INVALID_ARG, "NULL profiler");
    for (size_t i = 0; i < prof->used; ++i) {
        auto& s = prof->sets[i];
        MOE_CUDA_TRY(cudaEventSynchronize(s[MOE_NUM_STAGES]));
        for (int k = 0; k < MOE_NUM_STAGES; ++k) {
            float ms = 0.f;
            MOE_CUDA_TRY(cudaEventElapsedTime(&ms, s[k], s[k + 1]));
            prof->totals[k] += ms;
        }
        prof->calls++;
    }
    prof->used = 0;
    if (stage_ms)
        for (int k = 0; k < MOE_NUM_STAGES; ++k) stage_ms[k] = static_cast<float>(prof->totals[k]);
    if (calls) *calls = prof->calls;
    return ok();
}

int moe_profile_reset(moe_profile_t* prof) {
    if (!prof) return fail(MOE_ERR_INVALID_ARG, "NULL profiler");
    prof->used = 0;
    prof->calls = 0;
    for (double& t : prof->totals) t = 0;
    return ok();
}

int moe_read_status(const void* workspace, int32_t* status, void* stream) {
    if (!workspace || !status) return fail(MOE_ERR_INVALID_ARG, "moe_read_status: NULL pointer");
    MOE_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    MOE_CUDA_TRY(cudaMemcpy(status, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost));
    return ok();
}

int moe_selftest_bounded_wait(int32_t* status, uint32_t timeout_us, void* stream) {
    if (!status) return fail(MOE_ERR_INVALID_ARG, "moe_selftest_bounded_wait: NULL status");
    if (timeout_us == 0 || timeout_us > 10000000u)
        return fail(MOE_ERR_INVALID_ARG, "timeout_us must be in [1, 10000000]");
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    MOE_CUDA_TRY(moe::launch_selftest_wait(status, timeout_us, static_cast<cudaStream_t>(stream)));
    return ok();
}

int moe_debug_inject_fault(int fault) {
    if (fault != MOE_FAULT_NONE && fault != MOE_FAULT_SKIP_STAGE)
        return fail(MOE_ERR_INVALID_ARG, "unknown fault code %d", fault);
#ifdef MOE_FAULT_INJECTION
    t_armed_fault = fault;
    return ok();
#else
    return fail(MOE_ERR_UNSUPPORTED, "fault injection needs the debug library (libmoefp8_debug.so)");
#endif
}

}  // extern "C"
