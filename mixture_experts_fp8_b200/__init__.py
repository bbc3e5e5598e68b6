"""mixture_experts_fp8_b200 -- a B200-native fused FP8 routed-expert MoE layer (forward).

Thin Python binding over ``libmoefp8.so`` (C ABI in ``include/moefp8.h``).  This module only
marshals arguments: every step of the layer runs in the library's sm_100a kernels.  PyTorch
supplies device memory and streams.  There is no CPU fallback: if the library is missing it is
built in-tree with nvcc, and if that is impossible, importing this package fails.

Entry points (same names as the C ABI):
    check_config, transformed_weights_size, transform_weights, workspace_size,
    workspace_layout, route, forward, forward_profiled, forward_static_workspace, read_status,
    selftest_bounded_wait,
    Profile (moe_profile_create / read / reset / destroy).
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import asdict, dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoefp8.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_TIMEOUT = -4
MOE_ERR_BOUNDS = -5
MOE_NUM_STAGES = 6
STAGE_NAMES = ("route", "permute", "quantize", "gemm1_swiglu_requant", "gemm2", "combine")

EXPORTED = (
    "moe_last_error", "moe_check_config", "moe_transformed_weights_size", "moe_transform_weights",
    "moe_workspace_size", "moe_workspace_layout", "moe_route", "moe_forward", "moe_forward_profiled",
    "moe_profile_create", "moe_profile_destroy", "moe_profile_read", "moe_profile_reset",
    "moe_read_status", "moe_selftest_bounded_wait", "moe_forward_static_workspace", "moe_static_workspace_status",
    "moe_debug_unfused_gate_up",
    "moe_debug_inject_fault", "moe_gate", "moe_gate_weights_size", "moe_transform_gate_weights",
    "moe_ep_dispatch", "moe_forward_rows", "moe_combine_rows",
)
MOE_FAULT_NONE = 0
MOE_FAULT_SKIP_STAGE = 1


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("num_tokens", "hidden", "inter", "num_experts", "top_k", "routing",
                 "renormalize", "group_count", "k_group", "group_select_mode")] + \
               [("routed_scaling_factor", ctypes.c_float), ("recipe", ctypes.c_int32),
                ("shared_experts", ctypes.c_int32)]


_LAYOUT_FIELDS = ("status", "topk_idx", "topk_weights", "counts", "offsets", "tile_start",
                  "row_src", "row_of", "hist", "xq", "xs", "act_q", "act_s", "o", "scale_rows",
                  "total")


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in _LAYOUT_FIELDS]


@dataclass
class Config:
    """One problem (moe_config_t).  routing: 0 softmax, 1 sigmoid; recipe: 0 fp32 scale per
    (row, 128), 1 MXFP8 (UE8M0 per 32); shared_experts: 1 adds an expert (index num_experts)
    that every token uses with weight 1."""
    num_tokens: int
    hidden: int
    inter: int
    num_experts: int
    top_k: int
    routing: int = 0
    renormalize: int = 0
    group_count: int = 1
    k_group: int = 1
    group_select_mode: int = 0
    routed_scaling_factor: float = 1.0
    recipe: int = 0
    shared_experts: int = 0

    def c(self) -> _Cfg:
        d = asdict(self)
        return _Cfg(*(int(d[n]) for n in ("num_tokens", "hidden", "inter", "num_experts", "top_k",
                                          "routing", "renormalize", "group_count", "k_group",
                                          "group_select_mode")),
                    float(d["routed_scaling_factor"]), int(d["recipe"]), int(d["shared_experts"]))

    @property
    def group(self) -> int:
        return 128 if self.recipe == 0 else 32


_lock = threading.Lock()
_lib = None


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            from . import build as _build
            _build.build()
        if not os.path.exists(LIB_PATH):
            raise ImportError("libmoefp8.so is missing and could not be built")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        CP = ctypes.POINTER(_Cfg)
        lib.moe_last_error.restype = ctypes.c_char_p
        lib.moe_last_error.argtypes = []
        sig = {
            "moe_check_config": [CP],
            "moe_transformed_weights_size": [CP, ctypes.POINTER(S), ctypes.POINTER(S),
                                             ctypes.POINTER(S), ctypes.POINTER(S)],
            "moe_transform_weights": [CP] + [P] * 9,
            "moe_workspace_size": [CP, ctypes.POINTER(S)],
            "moe_workspace_layout": [CP, ctypes.POINTER(_Layout)],
            "moe_route": [CP, P, P, P, P, P],
            "moe_forward": [CP] + [P] * 14 + [S, P],
            "moe_forward_profiled": [CP] + [P] * 14 + [S, P, P],
            "moe_profile_create": [ctypes.POINTER(P)],
            "moe_profile_destroy": [P],
            "moe_profile_read": [P, P, P],
            "moe_profile_reset": [P],
            "moe_read_status": [P, P, P],
            "moe_selftest_bounded_wait": [P, ctypes.c_uint32, P],
            "moe_forward_static_workspace": [CP] + [P] * 13 + [P],
            "moe_static_workspace_status": [P, P],
            "moe_debug_unfused_gate_up": [CP] + [P] * 7 + [S, P],
            "moe_debug_inject_fault": [I],
            "moe_gate": [CP, P, P, ctypes.c_float, P, P, P, P, P],
            "moe_gate_weights_size": [CP, ctypes.POINTER(S)],
            "moe_transform_gate_weights": [CP, P, P, P, P],
            "moe_ep_dispatch": [CP, I, P, P, P, P, P, P, P, S, P],
            "moe_forward_rows": [CP] + [P] * 10 + [S, P],
            "moe_combine_rows": [CP, P, ctypes.c_int32, P, P, P, P, P],
        }
        for name, args in sig.items():
            f = getattr(lib, name)
            f.restype = I
            f.argtypes = args
        _lib = lib
        return lib


def lib():
    return _load()


def _check(rc: int):
    if rc != MOE_OK:
        raise MoeError(rc, _load().moe_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# --------------------------------------------------------------------------------------------
def check_config(cfg: Config) -> None:
    c = cfg.c()
    _check(_load().moe_check_config(ctypes.byref(c)))


def transformed_weights_size(cfg: Config):
    c = cfg.c()
    out = [ctypes.c_size_t() for _ in range(4)]
    _check(_load().moe_transformed_weights_size(ctypes.byref(c), *[ctypes.byref(o) for o in out]))
    return tuple(o.value for o in out)


def transform_weights(cfg: Config, w13, w13_scale, w2, w2_scale, stream=None):
    """Device tensors in the pages' layout -> (w13_t, w13s_t, w2_t, w2s_t) uint8 device tensors."""
    import torch
    sizes = transformed_weights_size(cfg)
    outs = [torch.empty(n, dtype=torch.uint8, device=w13.device) for n in sizes]
    c = cfg.c()
    _check(_load().moe_transform_weights(ctypes.byref(c), _ptr(w13), _ptr(w13_scale), _ptr(w2),
                                         _ptr(w2_scale), *[_ptr(o) for o in outs], _stream(stream)))
    return tuple(outs)


def workspace_size(cfg: Config) -> int:
    c = cfg.c()
    n = ctypes.c_size_t()
    _check(_load().moe_workspace_size(ctypes.byref(c), ctypes.byref(n)))
    return n.value


def workspace_layout(cfg: Config) -> dict:
    c = cfg.c()
    L = _Layout()
    _check(_load().moe_workspace_layout(ctypes.byref(c), ctypes.byref(L)))
    return {n: getattr(L, n) for n in _LAYOUT_FIELDS}


def new_workspace(cfg: Config, device="cuda"):
    import torch
    return torch.empty(workspace_size(cfg), dtype=torch.uint8, device=device)


def route(cfg: Config, router_logits, per_expert_scale=None, topk_idx=None, topk_weights=None,
          stream=None):
    """-> (topk_idx int32 [T,k], topk_weights fp32 [T,k]) on the logits' device."""
    import torch
    T, k = cfg.num_tokens, cfg.top_k
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=router_logits.device)
    if topk_weights is None:
        topk_weights = torch.empty((T, k), dtype=torch.float32, device=router_logits.device)
    c = cfg.c()
    _check(_load().moe_route(ctypes.byref(c), _ptr(router_logits), _ptr(per_expert_scale),
                             _ptr(topk_idx), _ptr(topk_weights), _stream(stream)))
    return topk_idx, topk_weights


def gate_weights_size(cfg: Config) -> int:
    c = cfg.c()
    n = ctypes.c_size_t()
    _check(_load().moe_gate_weights_size(ctypes.byref(c), ctypes.byref(n)))
    return n.value


def transform_gate_weights(cfg: Config, norm_weight, router_weight, stream=None):
    """norm_weight fp32 [H] and router_weight fp32 [E, H] (device) -> the gate's weights: a uint8
    device tensor holding w' = norm_weight * router_weight as three bf16 parts [3, E, H]."""
    import torch
    out = torch.empty(gate_weights_size(cfg), dtype=torch.uint8, device=router_weight.device)
    c = cfg.c()
    _check(_load().moe_transform_gate_weights(ctypes.byref(c), _ptr(norm_weight), _ptr(router_weight), _ptr(out),
                                              _stream(stream)))
    return out


def gate(cfg: Config, hidden_states, gate_weights, rms_eps: float, per_expert_scale=None, logits=None,
         topk_idx=None, topk_weights=None, stream=None):
    """RMSNorm + router matmul + router top-k (gate_weights from transform_gate_weights).
    -> (logits fp32 [T, E], topk_idx int32 [T, k], topk_weights fp32 [T, k])."""
    import torch
    T, E, k = cfg.num_tokens, cfg.num_experts, cfg.top_k
    dev = hidden_states.device
    if logits is None:
        logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    if topk_weights is None:
        topk_weights = torch.empty((T, k), dtype=torch.float32, device=dev)
    c = cfg.c()
    _check(_load().moe_gate(ctypes.byref(c), _ptr(hidden_states), _ptr(gate_weights), ctypes.c_float(rms_eps),
                            _ptr(per_expert_scale), _ptr(logits), _ptr(topk_idx), _ptr(topk_weights),
                            _stream(stream)))
    return logits, topk_idx, topk_weights


def ep_dispatch(cfg: Config, ranks: int, hidden_states, topk_idx, workspace, stream=None):
    """Order this rank's routed slots by destination rank (rank r owns experts r*E/R ..) ->
    (send_counts int32 [R], send_x bf16 [T*k, H], send_expert int32 [T*k], slot_pos int32 [T, k])."""
    import torch
    T, H, k = cfg.num_tokens, cfg.hidden, cfg.top_k
    dev = hidden_states.device
    send_counts = torch.empty(ranks, dtype=torch.int32, device=dev)
    send_x = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    send_expert = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    c = cfg.c()
    _check(_load().moe_ep_dispatch(ctypes.byref(c), int(ranks), _ptr(hidden_states), _ptr(topk_idx),
                                   _ptr(send_counts), _ptr(send_x), _ptr(send_expert), _ptr(slot_pos),
                                   _ptr(workspace), workspace.numel(), _stream(stream)))
    return send_counts, send_x, send_expert, slot_pos


def forward_rows(cfg: Config, rows, expert_of_row, weights, w13_bias=None, w2_bias=None, o_rows=None,
                 workspace=None, stream=None):
    """Each row through one local expert with weight 1 (cfg: num_tokens = rows, top_k = 1,
    num_experts = this rank's experts) -> o_rows fp32 [N, H]."""
    import torch
    N, H = cfg.num_tokens, cfg.hidden
    if o_rows is None:
        o_rows = torch.empty((N, H), dtype=torch.float32, device=rows.device)
    if workspace is None:
        workspace = new_workspace(cfg, rows.device)
    c = cfg.c()
    w13_t, w13s_t, w2_t, w2s_t = weights
    _check(_load().moe_forward_rows(ctypes.byref(c), _ptr(rows), _ptr(expert_of_row), _ptr(w13_t), _ptr(w13s_t),
                                    _ptr(w2_t), _ptr(w2s_t), _ptr(w13_bias), _ptr(w2_bias), _ptr(o_rows),
                                    _ptr(workspace), workspace.numel(), _stream(stream)))
    return o_rows


def combine_rows(cfg: Config, o_rows, slot_pos, topk_weights, y=None, status=None, stream=None):
    """y[t] = bf16(sum_j w[t,j] * o_rows[slot_pos[t,j]]) in slot order -> y bf16 [T, H].  A slot
    whose position is outside o_rows adds nothing and sets `status` (device int32) to
    MOE_ERR_BOUNDS."""
    import torch
    T, H = cfg.num_tokens, cfg.hidden
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=slot_pos.device)
    c = cfg.c()
    n = int(o_rows.shape[0])
    _check(_load().moe_combine_rows(ctypes.byref(c), _ptr(o_rows) if n else None, n, _ptr(slot_pos),
                                    _ptr(topk_weights), _ptr(y), _ptr(status), _stream(stream)))
    return y


def forward(cfg: Config, hidden_states, weights, router_logits=None, per_expert_scale=None,
            topk_idx=None, topk_weights=None, w13_bias=None, w2_bias=None, y=None,
            expert_counts=None, workspace=None, stream=None, profile: "Profile | None" = None):
    """The fused layer forward.  `weights` = (w13_t, w13s_t, w2_t, w2s_t) from
    transform_weights.  Returns y (bf16 [T, H])."""
    import torch
    if y is None:
        y = torch.empty((cfg.num_tokens, cfg.hidden), dtype=torch.bfloat16, device=hidden_states.device)
    if workspace is None:
        workspace = new_workspace(cfg, hidden_states.device)
    c = cfg.c()
    args = [ctypes.byref(c), _ptr(hidden_states), _ptr(router_logits), _ptr(per_expert_scale),
            _ptr(topk_idx), _ptr(topk_weights), *[_ptr(w) for w in weights], _ptr(w13_bias),
            _ptr(w2_bias), _ptr(y), _ptr(expert_counts), _ptr(workspace),
            ctypes.c_size_t(workspace.numel() * workspace.element_size())]
    if profile is None:
        _check(_load().moe_forward(*args, _stream(stream)))
    else:
        _check(_load().moe_forward_profiled(*args, profile.handle, _stream(stream)))
    return y


def forward_static_workspace(cfg: Config, hidden_states, weights, router_logits=None,
                             per_expert_scale=None, topk_idx=None, topk_weights=None, w13_bias=None,
                             w2_bias=None, y=None, expert_counts=None, stream=None):
    """The layer forward with its scratch in the library's fixed device array (no workspace
    argument, nothing allocated by the library).  For callers that may not allocate device
    memory; `y` should be preallocated by such callers."""
    import torch
    if y is None:
        y = torch.empty((cfg.num_tokens, cfg.hidden), dtype=torch.bfloat16, device=hidden_states.device)
    c = cfg.c()
    _check(_load().moe_forward_static_workspace(
        ctypes.byref(c), _ptr(hidden_states), _ptr(router_logits), _ptr(per_expert_scale),
        _ptr(topk_idx), _ptr(topk_weights), *[_ptr(w) for w in weights], _ptr(w13_bias),
        _ptr(w2_bias), _ptr(y), _ptr(expert_counts), _stream(stream)))
    return y


def read_status(workspace, stream=None) -> int:
    st = ctypes.c_int32()
    _check(_load().moe_read_status(_ptr(workspace), ctypes.byref(st), _stream(stream)))
    return st.value


def debug_unfused_gate_up(cfg: Config, hidden_states, topk_idx, weights, workspace, w13_bias=None, stream=None):
    """The gate+up step taken apart (test hook): the GEMM stores the fp32 gate/up sums h, then a
    separate SwiGLU + requantization kernel writes the act codes and scales into `workspace`.
    Returns h [A, 2I] fp32 (columns in the transformed order)."""
    import torch
    A = cfg.num_tokens * (cfg.top_k + cfg.shared_experts)
    h = torch.empty((A, 2 * cfg.inter), dtype=torch.float32, device=hidden_states.device)
    c = cfg.c()
    w13_t, w13s_t = weights[0], weights[1]
    _check(_load().moe_debug_unfused_gate_up(ctypes.byref(c), _ptr(hidden_states), _ptr(topk_idx), _ptr(w13_t),
                                             _ptr(w13s_t), _ptr(w13_bias), _ptr(h), _ptr(workspace),
                                             workspace.numel(), _stream(stream)))
    return h


def static_workspace_status(stream=None) -> int:
    """The status word of the last moe_forward_static_workspace call on the current device."""
    st = ctypes.c_int32()
    _check(_load().moe_static_workspace_status(ctypes.byref(st), _stream(stream)))
    return st.value


def selftest_bounded_wait(status_tensor, timeout_us: int, stream=None) -> None:
    _check(_load().moe_selftest_bounded_wait(_ptr(status_tensor), int(timeout_us), _stream(stream)))


def debug_inject_fault(fault: int) -> None:
    """Arm a fault for the next forward on this thread (the debug library only; the release
    library raises MoeError with MOE_ERR_UNSUPPORTED)."""
    _check(_load().moe_debug_inject_fault(int(fault)))


class Profile:
    """Per-stage device time of moe_forward_profiled calls (CUDA events inside the library)."""

    def __init__(self):
        h = ctypes.c_void_p()
        _check(_load().moe_profile_create(ctypes.byref(h)))
        self.handle = h

    def read(self):
        ms = (ctypes.c_float * MOE_NUM_STAGES)()
        calls = ctypes.c_int32()
        _check(_load().moe_profile_read(self.handle, ms, ctypes.byref(calls)))
        return dict(zip(STAGE_NAMES, list(ms))), calls.value

    def reset(self):
        _check(_load().moe_profile_reset(self.handle))

    def close(self):
        if self.handle:
            _load().moe_profile_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
