"""CPU oracle for the fused FP8 routed-expert MoE forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
package.  The CUDA library (``mixture_experts_fp8_b200``) never imports it and shares no code
with it.  The arithmetic lives in ``moe_oracle.c`` (plain C, fp64 accumulation, fp32 decisions);
this module only marshals numpy arrays into it.

Every function cites the page passage it restates in ``moe_oracle.c``:
  * routing            -- "MindIE-SD Fused MoE", routing selection / parameter table;
                          "mlx_native ops/moe_gate.rs", moe_gate doc.
  * permutation        -- "MindIE-SD Fused MoE", execution flow (dispatch, combine).
  * quantization       -- "metrale_model_layers fp8_grouped_tc_w8a8.rs", module doc (E4M3 per
                          (row, 128)); "DeepGEMM PR #371", Changes (UE8M0 per 32).
  * expert MLP, combine -- "metrale ... fp8_grouped_tc_w8a8.rs", run_fp8_grouped_w8a8;
                          "MATE Mega MoE", API (swiglu) and Current Limits (bf16 output).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")
_lock = threading.Lock()
_lib = None

OK, EINVAL, EUNSUPPORTED = 0, -1, -2


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into _liboracle.so (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("num_tokens", "hidden", "inter", "num_experts", "top_k", "routing",
                 "renormalize", "group_count", "k_group", "group_select_mode")] + \
               [("routed_scaling_factor", ctypes.c_float), ("recipe", ctypes.c_int32),
                ("shared_experts", ctypes.c_int32)]


@dataclass
class Config:
    """Problem description; field meanings follow the pages' fused_moe signature."""
    num_tokens: int
    hidden: int
    inter: int
    num_experts: int
    top_k: int
    routing: int = 0             # 0 softmax, 1 sigmoid
    renormalize: int = 0
    group_count: int = 1
    k_group: int = 1
    group_select_mode: int = 0
    routed_scaling_factor: float = 1.0
    recipe: int = 0              # 0 fp32 scale per (row,128); 1 UE8M0 per 32 (MXFP8);
                                 # 2 W4A8: E2M1 weights (two per byte) + UE8M0 per 32, MXFP8 acts
    shared_experts: int = 0      # 1: one more expert (index num_experts), every token, weight 1

    @property
    def slots(self) -> int:
        """Expert slots per token: the routed top_k plus the shared expert."""
        return self.top_k + self.shared_experts

    @property
    def group(self) -> int:
        return 128 if self.recipe == 0 else 32

    @property
    def scale_dtype(self):
        return np.float32 if self.recipe == 0 else np.uint8

    def c(self) -> _Cfg:
        return _Cfg(*(int(getattr(self, n)) for n in
                      ("num_tokens", "hidden", "inter", "num_experts", "top_k", "routing",
                       "renormalize", "group_count", "k_group", "group_select_mode")),
                    float(self.routed_scaling_factor), int(self.recipe), int(self.shared_experts))


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            lib.orc_e4m3_decode.restype = ctypes.c_double
            lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e2m1_decode.restype = ctypes.c_double
            lib.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_encode.restype = ctypes.c_uint8
            lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
            lib.orc_mx_exponent.restype = ctypes.c_int
            lib.orc_mx_exponent.argtypes = [ctypes.c_float]
            lib.orc_bf16_from_double.restype = ctypes.c_uint16
            lib.orc_bf16_from_double.argtypes = [ctypes.c_double]
            lib.orc_quant_row.restype = None
            lib.orc_quant_row.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P]
            lib.orc_check_cfg.restype = ctypes.c_int
            lib.orc_check_cfg.argtypes = [ctypes.POINTER(_Cfg)]
            lib.orc_route.restype = ctypes.c_int
            lib.orc_route.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P]
            lib.orc_group_scores.restype = ctypes.c_int
            lib.orc_group_scores.argtypes = [ctypes.POINTER(_Cfg), P, P]
            lib.orc_route_weights.restype = ctypes.c_int
            lib.orc_route_weights.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P]
            lib.orc_gate_logits.restype = None
            lib.orc_gate_logits.argtypes = [ctypes.c_int] * 3 + [P] * 3 + [ctypes.c_float, P]
            lib.orc_permute.restype = None
            lib.orc_permute.argtypes = [ctypes.c_int] * 3 + [P] * 5
            lib.orc_scaled_gemv.restype = None
            lib.orc_scaled_gemv.argtypes = [ctypes.c_int] * 3 + [P] * 5
            lib.orc_forward.restype = ctypes.c_int
            lib.orc_forward.argtypes = [ctypes.POINTER(_Cfg)] + [P] * 11 + [P, ctypes.c_int, P, P, P]
            lib.orc_expert_rows.restype = ctypes.c_int
            lib.orc_expert_rows.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int] + [P] * 9
            lib.orc_combine_rows.restype = ctypes.c_int
            lib.orc_combine_rows.argtypes = [ctypes.c_int] * 3 + [P] * 4
            lib.orc_forward_permuted.restype = ctypes.c_int
            lib.orc_forward_permuted.argtypes = [ctypes.POINTER(_Cfg)] + [P] * 10
            lib.orc_quantize_tokens.restype = None
            lib.orc_quantize_tokens.argtypes = [ctypes.c_int] * 3 + [P] * 3
            lib.orc_num_threads.restype = ctypes.c_int
            lib.orc_set_num_threads.restype = None
            lib.orc_set_num_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "need C-contiguous numpy"
    return a.ctypes.data_as(ctypes.c_void_p)


def _arr(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------------------- scalar pieces
def e4m3_decode(code: int) -> float:
    return _load().orc_e4m3_decode(int(code) & 0xFF)


def e2m1_decode(code: int) -> float:
    return float(_load().orc_e2m1_decode(code))


def e4m3_encode(v: float) -> int:
    return int(_load().orc_e4m3_encode(float(v)))


def e4m3_encode_array(x: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.ascontiguousarray(x, dtype=np.float32).ravel()
    return np.array([lib.orc_e4m3_encode(float(v)) for v in flat], dtype=np.uint8).reshape(np.shape(x))


def mx_exponent(amax: float) -> int:
    return int(_load().orc_mx_exponent(float(amax)))


def bf16_from_double(v: float) -> int:
    return int(_load().orc_bf16_from_double(float(v)))


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(n: int) -> None:
    _load().orc_set_num_threads(int(n))


# ----------------------------------------------------------------------------- stages
def quant_row(x: np.ndarray, recipe: int):
    """Quantize one fp32 row; returns (codes uint8 [n], scales fp32 [n/128] | uint8 [n/32])."""
    x = _arr(x, np.float32).ravel()
    n = x.size
    g = 128 if recipe == 0 else 32
    q = np.zeros(n, np.uint8)
    s = np.zeros(n // g, np.float32 if recipe == 0 else np.uint8)
    _load().orc_quant_row(_p(x), n, recipe, _p(q), _p(s))
    return q, s


def quantize_tokens(x_bf16: np.ndarray, recipe: int):
    """x bf16 bits uint16 [T,H] -> (codes [T,H], scales [T,H/g])."""
    x = _arr(x_bf16, np.uint16)
    T, H = x.shape
    g = 128 if recipe == 0 else 32
    q = np.zeros((T, H), np.uint8)
    s = np.zeros((T, H // g), np.float32 if recipe == 0 else np.uint8)
    _load().orc_quantize_tokens(T, H, recipe, _p(x), _p(q), _p(s))
    return q, s


def check_cfg(cfg: Config) -> int:
    c = cfg.c()
    return int(_load().orc_check_cfg(ctypes.byref(c)))


def route(cfg: Config, logits: np.ndarray, per_expert_scale=None):
    """-> (topk_idx int32 [T,k], topk_weights fp32 [T,k], near_tie uint8 [T])."""
    logits = _arr(logits, np.float32)
    pes = _arr(per_expert_scale, np.float32)
    T, k = cfg.num_tokens, cfg.top_k
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    tie = np.zeros(T, np.uint8)
    c = cfg.c()
    rc = _load().orc_route(ctypes.byref(c), _p(logits), _p(pes), _p(idx), _p(w), _p(tie))
    if rc:
        raise ValueError(f"oracle route: invalid configuration ({rc})")
    return idx, w, tie


def group_scores(cfg: Config, logits: np.ndarray) -> np.ndarray:
    """-> fp32 group scores [T, group_count], the values the group choice is taken on."""
    logits = _arr(logits, np.float32)
    g = np.zeros((cfg.num_tokens, cfg.group_count), np.float32)
    c = cfg.c()
    rc = _load().orc_group_scores(ctypes.byref(c), _p(logits), _p(g))
    if rc:
        raise ValueError(f"oracle group_scores: invalid configuration ({rc})")
    return g


def route_weights(cfg: Config, logits: np.ndarray, topk_idx: np.ndarray, per_expert_scale=None) -> np.ndarray:
    """-> fp32 [T, k]: the routing weights of the given expert ids under cfg's weight rule."""
    logits = _arr(logits, np.float32)
    idx = _arr(topk_idx, np.int32)
    pes = _arr(per_expert_scale, np.float32)
    w = np.zeros((cfg.num_tokens, cfg.top_k), np.float32)
    c = cfg.c()
    rc = _load().orc_route_weights(ctypes.byref(c), _p(logits), _p(pes), _p(idx), _p(w))
    if rc:
        raise ValueError(f"oracle route_weights: invalid configuration or ids ({rc})")
    return w


def permute(topk_idx: np.ndarray, num_experts: int):
    """-> (counts [E], offsets [E+1], row_src [A], row_of [T,k]), all int32."""
    idx = _arr(topk_idx, np.int32)
    T, k = idx.shape
    E = num_experts
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    row_src = np.zeros(T * k, np.int32)
    row_of = np.zeros((T, k), np.int32)
    _load().orc_permute(T, k, E, _p(idx), _p(counts), _p(offsets), _p(row_src), _p(row_of))
    return counts, offsets, row_src, row_of


def scaled_gemv(recipe: int, aq, as_, wq, ws):
    """One block-scaled GEMM row: aq [K] E4M3 codes, as_ [K/g], wq [K,N] codes (recipe 2:
    [K,N/2] bytes of two E2M1 codes, the even column in the low nibble), ws [K/g,N]."""
    aq = _arr(aq, np.uint8).ravel()
    wq = _arr(wq, np.uint8)
    sd = np.float32 if recipe == 0 else np.uint8
    as_ = _arr(as_, sd).ravel()
    ws = _arr(ws, sd)
    K, N = wq.shape[0], wq.shape[1] * (2 if recipe == 2 else 1)
    out = np.zeros(N, np.float64)
    _load().orc_scaled_gemv(recipe, K, N, _p(aq), _p(as_), _p(wq), _p(ws), _p(out))
    return out


def gate_logits(x_bf16, norm_w, router_w, eps: float) -> np.ndarray:
    """RMSNorm + router matmul (the gate in front of the router): fp32 logits [T, E]."""
    x = _arr(x_bf16, np.uint16)
    nw = _arr(norm_w, np.float32)
    rw = _arr(router_w, np.float32)
    T, H = x.shape
    E = rw.shape[0]
    out = np.zeros((T, E), np.float32)
    _load().orc_gate_logits(T, H, E, _p(x), _p(nw), _p(rw), ctypes.c_float(eps), _p(out))
    return out


def forward(cfg: Config, x_bf16, w13, w13s, w2, w2s, logits=None, per_expert_scale=None,
            topk_idx=None, topk_weights=None, b13=None, b2=None, tokens=None,
            want_act: bool = False):
    """Full layer forward.  x_bf16 uint16 [T,H]; weights in the pages' layout:
    w13 uint8 [E,H,2I], w13s [E,H/g,2I]; w2 uint8 [E,I,H], w2s [E,I/g,H]; biases bf16 bits.
    Returns y bf16 bits uint16 [n_sel,H] (and, with want_act, the per-slot act codes/scales)."""
    x = _arr(x_bf16, np.uint16)
    sd = cfg.scale_dtype
    args = [x, _arr(logits, np.float32), _arr(per_expert_scale, np.float32),
            _arr(topk_idx, np.int32), _arr(topk_weights, np.float32),
            _arr(w13, np.uint8), _arr(w13s, sd), _arr(w2, np.uint8), _arr(w2s, sd),
            _arr(b13, np.uint16), _arr(b2, np.uint16)]
    tok = _arr(tokens, np.int32)
    n_sel = cfg.num_tokens if tok is None else int(tok.size)
    y = np.zeros((n_sel, cfg.hidden), np.uint16)
    act_q = act_s = None
    if want_act:
        act_q = np.zeros((n_sel, cfg.slots, cfg.inter), np.uint8)
        act_s = np.zeros((n_sel, cfg.slots, cfg.inter // cfg.group), sd)
    c = cfg.c()
    rc = _load().orc_forward(ctypes.byref(c), *[_p(a) for a in args], _p(tok), n_sel, _p(y),
                             _p(act_q), _p(act_s))
    if rc:
        raise ValueError(f"oracle forward: invalid configuration ({rc})")
    return (y, act_q, act_s) if want_act else y


def expert_rows(cfg: Config, x_bf16, expert_of_row, w13, w13s, w2, w2s, b13=None, b2=None) -> np.ndarray:
    """Expert parallelism, the owning rank's side: each row x_n (bf16 bits) quantized as the layer
    does, then through expert e_n's MLP (local numbering; cfg.num_experts = that rank's experts).
    Returns the fp64 outputs [N, H] (before the routing weight)."""
    x = _arr(x_bf16, np.uint16)
    e = _arr(expert_of_row, np.int32)
    N = int(e.size)
    sd = cfg.scale_dtype
    o = np.zeros((N, cfg.hidden), np.float64)
    rc = _load().orc_expert_rows(ctypes.byref(cfg.c()), N, _p(x), _p(e), _p(_arr(w13, np.uint8)), _p(_arr(w13s, sd)),
                                 _p(_arr(w2, np.uint8)), _p(_arr(w2s, sd)), _p(_arr(b13, np.uint16)),
                                 _p(_arr(b2, np.uint16)), _p(o))
    if rc:
        raise ValueError(f"oracle expert_rows: expert id out of range ({rc})")
    return o


def combine_rows(o_rows, slot_pos, topk_weights) -> np.ndarray:
    """Expert parallelism, the home rank's side: y_t = bf16(sum_j w_tj * o[pos_tj]) in slot order
    (fp64 sum).  o_rows fp64 [T*k, H], slot_pos int32 [T, k], topk_weights fp32 [T, k]."""
    o = _arr(o_rows, np.float64)
    pos = _arr(slot_pos, np.int32)
    w = _arr(topk_weights, np.float32)
    T, K = pos.shape
    H = o.shape[1]
    y = np.zeros((T, H), np.uint16)
    rc = _load().orc_combine_rows(T, K, H, _p(o), _p(pos), _p(w), _p(y))
    if rc:
        raise ValueError(f"oracle combine_rows: position out of range ({rc})")
    return y


def forward_permuted(cfg: Config, x_bf16, w13, w13s, w2, w2s, logits, per_expert_scale=None,
                     b13=None, b2=None):
    """The same forward computed expert by expert over permuted rows (route, permute, mlp,
    combine); must agree bit for bit with forward()."""
    sd = cfg.scale_dtype
    args = [_arr(x_bf16, np.uint16), _arr(logits, np.float32), _arr(per_expert_scale, np.float32),
            _arr(w13, np.uint8), _arr(w13s, sd), _arr(w2, np.uint8), _arr(w2s, sd),
            _arr(b13, np.uint16), _arr(b2, np.uint16)]
    y = np.zeros((cfg.num_tokens, cfg.hidden), np.uint16)
    c = cfg.c()
    rc = _load().orc_forward_permuted(ctypes.byref(c), *[_p(a) for a in args], _p(y))
    if rc:
        raise ValueError(f"oracle forward_permuted: invalid configuration ({rc})")
    return y
