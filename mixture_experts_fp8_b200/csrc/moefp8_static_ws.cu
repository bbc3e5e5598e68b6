// moefp8_static_ws.cu -- moe_forward_static_workspace: the layer forward for callers that
// cannot allocate device memory.
//
// Who needs it: code that runs inside a host framework which owns every byte of device memory
// (a serving engine with a pre-reserved pool, or a plugin interface that hands its kernels no
// scratch buffer).  Such callers may not call cudaMalloc: it can synchronize the device and
// stall every stream in flight, and it can fail under memory pressure in the middle of serving.
// They still own and pass the inputs and outputs; only the forward's scratch moves into a
// fixed array that lives in this library's device image.
//
// The scratch is one file-scope device array of kStaticWorkspaceBytes (16 MiB).  Every GPU that
// loads the library keeps these 16 MiB until the process exits.  Host code cannot use the
// array's name as a device address, so the address is looked up with cudaGetSymbolAddress once
// per device, on the first call made with that device current; make that first call before any
// stream capture begins.  All calls on a device share the array and it keeps the last call's
// contents; the forward clears what must start at zero (its status word) itself.  Calls that
// overlap on the GPU (different streams, or different host threads, without ordering between
// them) race on the array and corrupt each other's results.  Faults the kernels find on the
// device (a bounded wait that ran out, an index out of range) land in the array's status word;
// moe_static_workspace_status reads it.
#include <cstdio>
#include <mutex>

#include "moe_common.cuh"
#include "moe_kernels.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = 16u << 20;

__device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_addr[kMaxDevices] = {nullptr};

// The device address of the array on the current device (looked up once per device).
int static_ws_addr(const char* who, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return moe::set_last_error(MOE_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) {
        char msg[160];
        snprintf(msg, sizeof(msg), "%s: device ordinal out of range", who);
        return moe::set_last_error(MOE_ERR_UNSUPPORTED, msg);
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ws_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_workspace);
        if (e != cudaSuccess || !p)
            return moe::set_last_error(MOE_ERR_CUDA, e != cudaSuccess ? cudaGetErrorString(e)
                                                                        : "cudaGetSymbolAddress returned NULL");
        g_ws_addr[dev] = p;
    }
    *out = g_ws_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" {

int moe_forward_static_workspace(const moe_config_t* cfg, const void* hidden_states,
                                 const float* router_logits, const float* per_expert_scale,
                                 const int32_t* topk_idx, const float* topk_weights,
                                 const void* w13_t, const void* w13s_t, const void* w2_t,
                                 const void* w2s_t, const void* w13_bias, const void* w2_bias,
                                 void* y, int32_t* expert_counts, void* stream) {
    size_t need = 0;
    int rc = moe_workspace_size(cfg, &need);
    if (rc != MOE_OK) return rc;
    if (need > kStaticWorkspaceBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "moe_forward_static_workspace: this problem needs %zu bytes of scratch, more than the "
                 "library's fixed %zu-byte array; use moe_forward with a caller-owned workspace",
                 need, kStaticWorkspaceBytes);
        return moe::set_last_error(MOE_ERR_UNSUPPORTED, msg);
    }
    void* ws = nullptr;
    if ((rc = static_ws_addr("moe_forward_static_workspace", &ws)) != MOE_OK) return rc;
    return moe_forward(cfg, hidden_states, router_logits, per_expert_scale, topk_idx, topk_weights, w13_t,
                       w13s_t, w2_t, w2s_t, w13_bias, w2_bias, y, expert_counts, ws, kStaticWorkspaceBytes,
                       stream);
}

// The status word of the last forward run through the array (it sits at the start of every
// workspace): after synchronizing `stream`, a blocking 4-byte copy, like moe_read_status.
int moe_static_workspace_status(int32_t* status, void* stream) {
    if (!status) return moe::set_last_error(MOE_ERR_INVALID_ARG, "moe_static_workspace_status: NULL status");
    void* ws = nullptr;
    const int rc = static_ws_addr("moe_static_workspace_status", &ws);
    if (rc != MOE_OK) return rc;
    return moe_read_status(ws, status, stream);
}

}  // extern "C"
