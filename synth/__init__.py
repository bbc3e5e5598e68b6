"""Seeded synthetic inputs for the fused FP8 MoE layer forward.

This module is shared by the tests, the benchmark and the smoke check.  It holds the problem
shapes and the recipe for every input and none of the layer's own arithmetic: no routing, no
permutation, no activation quantization, no GEMM.  Weights arrive at the layer already
quantized (E4M3 codes plus block scales), so preparing them is input generation: fp32 normal
weights are divided by a per-block scale and cast with torch's own float8_e4m3fn conversion.

Every tensor is drawn from a torch.Generator seeded by (problem seed, tensor id, expert), so a
problem is reproducible for a given device type.  Inputs for the large problems can be drawn
directly on a CUDA device (``device="cuda"``); the values then differ from a CPU draw but are
the same on every run.

Shapes and distributions (one line per problem):
  tiny    16 tok, H 256,  I 256,  E 8,   k 2, softmax + renormalize, fp32 per-128 scales, seed 0
  decode  64 tok, H 2816, I 768,  E 128, k 8, softmax (renormalized over the selected
          experts), per-expert scale U(0.5,1.5), rsf 1.0, seed 1
  prefill 4096 tok, H 7168, I 2048, E 256, k 8, sigmoid, 8 groups, k_group 4, top-2-sum group
          score, rsf 2.5; logits N(0,1) + per-expert bias N(0,0.1), seed 2
  skewed  2048 tok, H 768, I 1152, E 256, k 8, softmax without renormalize; logits N(0,1) +
          ln p_e with p_e ~ rank(e)^-1.2 (Zipf, rank a seeded permutation); MXFP8, seed 3
  large   16384 tok, H 4096, I 1536, E 128, k 8, softmax + renormalize; biases bf16
          N(0,0.02), seed 4
  decode_w4a8 / prefill_w4a8: the decode and prefill shapes with W4A8 weights (E2M1 codes,
          UE8M0 per 32, nearest-even rounding) and MXFP8 activations, seeds 5 and 6
  x ~ N(0,1) rounded to bf16; logits fp32; weights N(0, 1/sqrt(K)) with K the contraction dim.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

E4M3_MAX = 448.0

# tensor ids folded into the seeds
_X, _LOGITS, _BIAS_ROUTE, _PES, _W13, _W2, _B13, _B2, _RANK, _NORM_W, _ROUTER_W = range(11)


@dataclass(frozen=True)
class Shape:
    name: str
    num_tokens: int
    hidden: int
    inter: int
    num_experts: int
    top_k: int
    routing: int = 0                 # 0 softmax, 1 sigmoid
    renormalize: int = 0
    group_count: int = 1
    k_group: int = 1
    group_select_mode: int = 0
    routed_scaling_factor: float = 1.0
    recipe: int = 0                  # 0 fp32 per (row,128); 1 MXFP8 (UE8M0 per 32);
                                     # 2 W4A8: E2M1 weights + UE8M0 per 32, MXFP8 activations
    seed: int = 0
    logit_bias_std: float = 0.0      # per-expert bias added to the logits
    zipf_s: float = 0.0              # > 0: add ln p_e, p_e ~ rank^-s
    per_expert_scale: bool = False   # draw per_expert_scale ~ U(0.5, 1.5)
    biases: bool = False             # draw w13_bias / w2_bias ~ N(0, 0.02) in bf16
    shared_experts: int = 0          # 1: weights for one more expert, which every token uses

    @property
    def group(self) -> int:
        return 128 if self.recipe == 0 else 32

    def cfg(self) -> dict:
        """The problem's configuration fields, with the names the library and oracle use."""
        return dict(num_tokens=self.num_tokens, hidden=self.hidden, inter=self.inter,
                    num_experts=self.num_experts, top_k=self.top_k, routing=self.routing,
                    renormalize=self.renormalize, group_count=self.group_count,
                    k_group=self.k_group, group_select_mode=self.group_select_mode,
                    routed_scaling_factor=self.routed_scaling_factor, recipe=self.recipe,
                    shared_experts=self.shared_experts)

    def with_tokens(self, n: int) -> "Shape":
        return replace(self, num_tokens=n)


SHAPES = {
    "tiny": Shape("tiny", 16, 256, 256, 8, 2, routing=0, renormalize=1, seed=0),
    "decode": Shape("decode", 64, 2816, 768, 128, 8, routing=0, renormalize=1, seed=1,
                    per_expert_scale=True),
    "prefill": Shape("prefill", 4096, 7168, 2048, 256, 8, routing=1, renormalize=1,
                     group_count=8, k_group=4, group_select_mode=1, routed_scaling_factor=2.5,
                     seed=2, logit_bias_std=0.1),
    "skewed": Shape("skewed", 2048, 768, 1152, 256, 8, routing=0, renormalize=0, recipe=1,
                    seed=3, zipf_s=1.2),
    "large": Shape("large", 16384, 4096, 1536, 128, 8, routing=0, renormalize=1, seed=4,
                   biases=True),
    # W4A8 (E2M1 weights, UE8M0 per 32; MXFP8 activations) on the decode and prefill shapes
    "decode_w4a8": Shape("decode_w4a8", 64, 2816, 768, 128, 8, routing=0, renormalize=1,
                         recipe=2, seed=5, per_expert_scale=True),
    "prefill_w4a8": Shape("prefill_w4a8", 4096, 7168, 2048, 256, 8, routing=1, renormalize=1,
                          group_count=8, k_group=4, group_select_mode=1,
                          routed_scaling_factor=2.5, recipe=2, seed=6, logit_bias_std=0.1),
}


def _gen(device, *key) -> torch.Generator:
    """A generator seeded from a tuple of small integers (stable across runs)."""
    s = 0x9E3779B97F4A7C15
    for k in key:
        s = (s ^ (int(k) + 0x632BE59BD9B4E019 + ((s << 6) & (2**64 - 1)) + (s >> 2))) & (2**64 - 1)
    g = torch.Generator(device=device)
    g.manual_seed(s & (2**63 - 1))
    return g


def _randn(shape, std, device, *key, dtype=torch.float32):
    return torch.randn(shape, generator=_gen(device, *key), device=device, dtype=dtype) * std


def bf16_bits(t: torch.Tensor) -> torch.Tensor:
    """torch bf16 tensor -> int16 view of its bits (same storage)."""
    return t.contiguous().view(torch.int16)


E2M1_MAX = 6.0
_E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)     # magnitudes of codes 0..7


def _e2m1_codes(v: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 code of each value (ties to the even code, saturating at 6): the input
    recipe for the FP4 weights.  Returns uint8 codes 0..15 (bit 3 = sign)."""
    grid = torch.tensor(_E2M1_GRID, dtype=torch.float32, device=v.device)
    a = v.abs().clamp(max=E2M1_MAX)
    lo = (torch.bucketize(a, grid, right=True) - 1).clamp(0, 7)
    hi = (lo + 1).clamp(max=7)
    dlo, dhi = a - grid[lo], grid[hi] - a
    up = (dhi < dlo) | ((dhi == dlo) & (lo % 2 == 1))
    code = torch.where(up, hi, lo)
    return (code | ((v < 0) & (code > 0)).to(code.dtype) * 8).to(torch.uint8)


def quantize_weight_block(w: torch.Tensor, recipe: int):
    """Prepare one expert's weight w [K, N] (fp32) as codes plus block scales [K/g, N]: E4M3
    codes [K, N] with fp32 amax/448 per 128-deep block (recipe 0) or a UE8M0 power of two per
    32-deep block (recipe 1), or E2M1 codes packed two per byte along N, [K, N/2] (the even
    column in the low nibble), with a UE8M0 power of two per 32-deep block, the smallest with
    amax <= 6 * 2^e (recipe 2, the W4A8 weights).  Input preparation only; the E4M3 cast is
    torch's."""
    K, N = w.shape
    g = 128 if recipe == 0 else 32
    blocks = w.reshape(K // g, g, N)
    amax = blocks.abs().amax(dim=1)                                   # [K/g, N]
    if recipe == 2:
        e = torch.ceil(torch.log2(torch.clamp(amax, min=1e-30) / E2M1_MAX)).clamp(-127, 127)
        codes = _e2m1_codes((blocks / torch.exp2(e)[:, None, :]).reshape(K, N))
        packed = codes[:, 0::2] | (codes[:, 1::2] << 4)
        return packed.contiguous(), (e + 127).to(torch.uint8)
    if recipe == 0:
        scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
        sc_store = scale
    else:
        e = torch.ceil(torch.log2(torch.clamp(amax, min=1e-30) / E4M3_MAX)).clamp(-127, 127)
        scale = torch.exp2(e)
        sc_store = (e + 127).to(torch.uint8)
    q = (blocks / scale[:, None, :]).clamp(-E4M3_MAX, E4M3_MAX).reshape(K, N)
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, sc_store


@dataclass
class Problem:
    shape: Shape
    x: torch.Tensor                      # bf16 [T,H]
    logits: torch.Tensor                 # fp32 [T,E]
    per_expert_scale: torch.Tensor | None
    w13: torch.Tensor                    # uint8 [E,H,2I] (W4A8: [E,H,I], two E2M1 codes a byte)
    w13_scale: torch.Tensor              # fp32 [E,H/128,2I] | uint8 [E,H/32,2I]
    w2: torch.Tensor                     # uint8 [E,I,H]  (W4A8: [E,I,H/2])
    w2_scale: torch.Tensor               # fp32 [E,I/128,H]  | uint8 [E,I/32,H]
    w13_bias: torch.Tensor | None        # bf16 [E,2I]
    w2_bias: torch.Tensor | None         # bf16 [E,H]
    extra: dict = field(default_factory=dict)

    def to(self, device) -> "Problem":
        mv = lambda t: None if t is None else t.to(device)
        return Problem(self.shape, mv(self.x), mv(self.logits), mv(self.per_expert_scale),
                       mv(self.w13), mv(self.w13_scale), mv(self.w2), mv(self.w2_scale),
                       mv(self.w13_bias), mv(self.w2_bias), dict(self.extra))

    def numpy_inputs(self) -> dict:
        """Host numpy views of every input (bf16 tensors as uint16 bits)."""
        def npy(t):
            if t is None:
                return None
            t = t.detach().cpu().contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16)
            return t.numpy()
        return dict(x=npy(self.x), logits=npy(self.logits),
                    per_expert_scale=npy(self.per_expert_scale), w13=npy(self.w13),
                    w13s=npy(self.w13_scale), w2=npy(self.w2), w2s=npy(self.w2_scale),
                    b13=npy(self.w13_bias), b2=npy(self.w2_bias))


def make_weights(shape: Shape, device="cpu"):
    """Per-expert fp32 N(0, 1/sqrt(K)) weights, prepared as codes + block scales; the shared
    expert, if any, is expert index num_experts (drawn from its own seed, so the routed
    experts' weights do not depend on it)."""
    E, H, I, r = shape.num_experts + shape.shared_experts, shape.hidden, shape.inter, shape.recipe
    g = shape.group
    sdt = torch.float32 if r == 0 else torch.uint8
    pk = 2 if r == 2 else 1                                  # E2M1 codes: two per byte
    w13 = torch.empty((E, H, 2 * I // pk), dtype=torch.uint8, device=device)
    w13s = torch.empty((E, H // g, 2 * I), dtype=sdt, device=device)
    w2 = torch.empty((E, I, H // pk), dtype=torch.uint8, device=device)
    w2s = torch.empty((E, I // g, H), dtype=sdt, device=device)
    for e in range(E):
        c, s = quantize_weight_block(_randn((H, 2 * I), 1.0 / math.sqrt(H), device, shape.seed, _W13, e), r)
        w13[e].copy_(c); w13s[e].copy_(s)
        c, s = quantize_weight_block(_randn((I, H), 1.0 / math.sqrt(I), device, shape.seed, _W2, e), r)
        w2[e].copy_(c); w2s[e].copy_(s)
    return w13, w13s, w2, w2s


def make_activations(shape: Shape, device="cpu", num_tokens: int | None = None):
    """x (bf16), logits (fp32) and the optional per-expert routing inputs."""
    T = shape.num_tokens if num_tokens is None else num_tokens
    E, H = shape.num_experts, shape.hidden
    x = _randn((T, H), 1.0, device, shape.seed, _X).to(torch.bfloat16)
    logits = _randn((T, E), 1.0, device, shape.seed, _LOGITS)
    if shape.logit_bias_std > 0:
        logits = logits + _randn((E,), shape.logit_bias_std, device, shape.seed, _BIAS_ROUTE)[None, :]
    if shape.zipf_s > 0:
        rank = torch.randperm(E, generator=_gen("cpu", shape.seed, _RANK)).to(device) + 1
        logits = logits + (-shape.zipf_s * torch.log(rank.to(torch.float32)))[None, :]
    pes = None
    if shape.per_expert_scale:
        pes = torch.rand((E,), generator=_gen(device, shape.seed, _PES), device=device) + 0.5
    return x, logits.contiguous(), pes


def make_gate(shape: Shape, device="cpu"):
    """Inputs of the gate in front of the router: the RMSNorm weight fp32 [H] ~ 1 + N(0, 0.1),
    the router weight fp32 [E, H] ~ N(0, 1/sqrt(H)) (so the logits are about N(0, 1)), and the
    norm epsilon."""
    H, E = shape.hidden, shape.num_experts
    norm_w = 1.0 + _randn((H,), 0.1, device, shape.seed, _NORM_W)
    router_w = _randn((E, H), 1.0 / math.sqrt(H), device, shape.seed, _ROUTER_W)
    return norm_w.contiguous(), router_w.contiguous(), 1e-6


def make_problem(name_or_shape, device="cpu", num_tokens: int | None = None) -> Problem:
    shape = SHAPES[name_or_shape] if isinstance(name_or_shape, str) else name_or_shape
    if num_tokens is not None:
        shape = shape.with_tokens(num_tokens)
    x, logits, pes = make_activations(shape, device)
    w13, w13s, w2, w2s = make_weights(shape, device)
    b13 = b2 = None
    if shape.biases:
        E, H, I = shape.num_experts, shape.hidden, shape.inter
        b13 = _randn((E, 2 * I), 0.02, device, shape.seed, _B13).to(torch.bfloat16)
        b2 = _randn((E, H), 0.02, device, shape.seed, _B2).to(torch.bfloat16)
        if shape.shared_experts:                     # the shared expert's rows, own seed
            b13 = torch.cat([b13, _randn((1, 2 * I), 0.02, device, shape.seed, _B13, E).to(torch.bfloat16)])
            b2 = torch.cat([b2, _randn((1, H), 0.02, device, shape.seed, _B2, E).to(torch.bfloat16)])
    return Problem(shape, x, logits, pes, w13, w13s, w2, w2s, b13, b2)


def random_shape(seed: int, **over) -> Shape:
    """A small ragged problem for parity sweeps: odd token counts, few experts."""
    rng = np.random.default_rng(1000 + seed)
    E = int(rng.choice([1, 2, 3, 6, 8, 16]))
    k = int(rng.integers(1, min(E, 4) + 1))
    s = Shape(f"rand{seed}", num_tokens=int(rng.choice([1, 3, 37, 127, 200])),
              hidden=int(rng.choice([128, 256, 384, 640])),
              inter=int(rng.choice([128, 256, 384])), num_experts=E, top_k=k,
              routing=int(rng.integers(0, 2)), renormalize=int(rng.integers(0, 2)),
              recipe=int(rng.integers(0, 2)), seed=10_000 + seed,
              routed_scaling_factor=float(rng.choice([1.0, 2.5])),
              per_expert_scale=bool(rng.integers(0, 2)), biases=bool(rng.integers(0, 2)))
    return replace(s, **over)


def random_grouped_shape(seed: int, **over) -> Shape:
    """A small ragged problem with grouped routing: the experts form group_count groups, the
    k_group best (max or top-2-sum group score) are kept, top_k is chosen inside them."""
    rng = np.random.default_rng(2000 + seed)
    E = int(rng.choice([8, 16, 32, 64]))
    G = int(rng.choice([g for g in (2, 4, 8) if E % g == 0 and E // g >= 2]))
    kg = int(rng.integers(1, G + 1))
    k = int(rng.integers(1, min(8, kg * (E // G)) + 1))
    s = Shape(f"grp{seed}", num_tokens=int(rng.choice([5, 64, 129, 300])),
              hidden=int(rng.choice([128, 256, 384])), inter=int(rng.choice([128, 256])),
              num_experts=E, top_k=k, routing=int(rng.integers(0, 2)),
              renormalize=int(rng.integers(0, 2)), group_count=G, k_group=kg,
              group_select_mode=int(rng.integers(0, 2)), recipe=int(rng.integers(0, 3)),
              seed=20_000 + seed, routed_scaling_factor=float(rng.choice([1.0, 2.5])),
              logit_bias_std=float(rng.choice([0.0, 0.1])), biases=bool(rng.integers(0, 2)))
    return replace(s, **over)
