"""The C ABI library on a machine without a GPU: it loads, exports every entry point that
include/moefp8.h declares, and validates arguments before touching the device (errors carry a
message; "mlx_native ops/moe_gate.rs" validation and "MindIE-SD Fused MoE" constraints)."""
import ctypes
import os
import re

import pytest

import mixture_experts_fp8_b200 as moe

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "moefp8.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(moe.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(moe.EXPORTED)


def test_config_struct_layout():
    # moe_config_t: twelve 4-byte fields in header order, shared_experts last
    assert ctypes.sizeof(moe._Cfg) == 52
    assert moe._Cfg.shared_experts.offset == 48
    assert moe._Cfg.recipe.offset == 44


def cfg(**kw):
    base = dict(num_tokens=16, hidden=256, inter=256, num_experts=8, top_k=2)
    base.update(kw)
    return moe.Config(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(num_tokens=0), moe.MOE_ERR_INVALID_ARG),
    (dict(hidden=-128), moe.MOE_ERR_INVALID_ARG),
    (dict(top_k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(top_k=9), moe.MOE_ERR_INVALID_ARG),
    (dict(routing=2), moe.MOE_ERR_INVALID_ARG),
    (dict(recipe=3), moe.MOE_ERR_INVALID_ARG),
    (dict(hidden=200), moe.MOE_ERR_UNSUPPORTED),
    (dict(inter=192), moe.MOE_ERR_UNSUPPORTED),
    (dict(num_experts=512, top_k=2), moe.MOE_ERR_UNSUPPORTED),
    (dict(group_count=3), moe.MOE_ERR_UNSUPPORTED),
    (dict(group_count=4, k_group=5), moe.MOE_ERR_UNSUPPORTED),
    (dict(group_count=4, k_group=1, top_k=3), moe.MOE_ERR_UNSUPPORTED),
    (dict(group_count=8, group_select_mode=1), moe.MOE_ERR_UNSUPPORTED),
    (dict(shared_experts=2), moe.MOE_ERR_UNSUPPORTED),
    (dict(shared_experts=-1), moe.MOE_ERR_UNSUPPORTED),
])
def test_validation(kw, code):
    with pytest.raises(moe.MoeError) as e:
        moe.check_config(cfg(**kw))
    assert e.value.code == code
    assert len(str(e.value)) > 10


def test_valid_configs_and_sizes():
    import synth
    for name, s in synth.SHAPES.items():
        c = moe.Config(**s.cfg())
        moe.check_config(c)
        lay = moe.workspace_layout(c)
        assert lay["total"] == moe.workspace_size(c)
        A = s.num_tokens * s.top_k
        assert lay["o"] + 4 * A * s.hidden <= lay["total"]
        assert all(v % 1024 == 0 for k, v in lay.items() if k not in ("total", "scale_rows"))
        assert lay["scale_rows"] >= A and lay["scale_rows"] % 4 == 0
        w13, w13s, w2, w2s = moe.transformed_weights_size(c)
        pk = 2 if s.recipe == 2 else 1          # W4A8: two E2M1 codes per byte
        assert w13 * pk == s.num_experts * s.hidden * 2 * s.inter and w2 * pk == s.num_experts * s.inter * s.hidden
        assert w13s == s.num_experts * (s.hidden // 128) * 2 * s.inter * 4


def test_shared_expert_sizes():
    """A shared expert adds one expert's weights and one row per token to the workspace."""
    import synth
    from dataclasses import replace
    s = replace(synth.SHAPES["decode"], shared_experts=1)
    c = moe.Config(**s.cfg())
    moe.check_config(c)
    c0 = moe.Config(**replace(s, shared_experts=0).cfg())
    w = moe.transformed_weights_size(c)
    w0 = moe.transformed_weights_size(c0)
    E = s.num_experts
    assert all(a * E == b * (E + 1) for a, b in zip(w, w0))
    lay = moe.workspace_layout(c)
    A = s.num_tokens * (s.top_k + 1)
    assert lay["o"] + 4 * A * s.hidden <= lay["total"]
    assert lay["scale_rows"] >= A
    assert lay["total"] > moe.workspace_size(c0)
    # 256 routed experts plus a shared one are accepted
    moe.check_config(moe.Config(**replace(synth.SHAPES["prefill"], shared_experts=1).cfg()))


def test_forward_rejects_bad_pointers_before_any_cuda_call():
    lib = moe.lib()
    c = cfg().c()
    rc = lib.moe_forward(ctypes.byref(c), None, None, None, None, None, None, None, None, None,
                         None, None, None, None, None, 0, None)
    assert rc == moe.MOE_ERR_INVALID_ARG
    assert b"NULL" in lib.moe_last_error()


def test_interleave_is_a_permutation():
    # mirror of the transform's gate/up column order (blocks of 128 for the fp32-scale recipe,
    # 32 for MXFP8), checked for bijectivity and for gate/up pairing at the same offset
    for blk in (128, 32):
        I = 384
        def row(n):
            up = n >= I
            i = n - I if up else n
            return (i // blk) * 2 * blk + up * blk + i % blk
        rows = [row(n) for n in range(2 * I)]
        assert sorted(rows) == list(range(2 * I))
        for i in range(I):
            assert rows[I + i] - rows[i] == blk

def test_gate_entry_points_validate_before_any_cuda_call():
    """moe_gate_weights_size reports 3 bf16 parts of [E, H]; the gate's transform and call reject
    NULL and misaligned buffers and a negative epsilon with a message, touching no device."""
    lib = moe.lib()
    c = cfg(num_experts=24, hidden=384, top_k=3)
    assert moe.gate_weights_size(c) == 3 * 24 * 384 * 2
    cc = c.c()
    rc = lib.moe_transform_gate_weights(ctypes.byref(cc), None, None, None, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"NULL" in lib.moe_last_error()
    buf = ctypes.create_string_buffer(64)
    odd = ctypes.addressof(buf) | 4                 # 4-byte aligned, not 16
    rc = lib.moe_transform_gate_weights(ctypes.byref(cc), odd, odd, odd, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"16-byte" in lib.moe_last_error()
    rc = lib.moe_gate(ctypes.byref(cc), None, None, ctypes.c_float(1e-6), None, None, None, None, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"NULL" in lib.moe_last_error()
    al = (ctypes.addressof(buf) + 15) & ~15
    rc = lib.moe_gate(ctypes.byref(cc), al, al, ctypes.c_float(-1.0), None, al, al, al, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"rms_eps" in lib.moe_last_error()
    bad = moe.Config(num_tokens=0, hidden=384, inter=128, num_experts=24, top_k=3).c()
    n = ctypes.c_size_t(0)
    assert lib.moe_gate_weights_size(ctypes.byref(bad), ctypes.byref(n)) == moe.MOE_ERR_INVALID_ARG


def test_expert_parallel_entry_points_validate_before_any_cuda_call():
    """Ranks must divide the expert count, no shared expert, one slot per row on the expert side,
    no NULL buffers: each rejected with a message and nothing launched."""
    lib = moe.lib()
    buf = ctypes.create_string_buffer(4096)
    al = (ctypes.addressof(buf) + 255) & ~255
    c = cfg(num_experts=8, top_k=2).c()
    rc = lib.moe_ep_dispatch(ctypes.byref(c), 3, al, al, al, al, al, al, al, 1 << 20, None)
    assert rc == moe.MOE_ERR_UNSUPPORTED and b"divide" in lib.moe_last_error()
    rc = lib.moe_ep_dispatch(ctypes.byref(c), 2, None, al, al, al, al, al, al, 1 << 20, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"NULL" in lib.moe_last_error()
    rc = lib.moe_ep_dispatch(ctypes.byref(c), 2, al, al, al, al, al, al, al, 16, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"workspace" in lib.moe_last_error()
    sh = cfg(num_experts=8, top_k=2, shared_experts=1).c()
    rc = lib.moe_ep_dispatch(ctypes.byref(sh), 2, al, al, al, al, al, al, al, 1 << 20, None)
    assert rc == moe.MOE_ERR_UNSUPPORTED and b"shared" in lib.moe_last_error()
    rc = lib.moe_forward_rows(ctypes.byref(c), al, al, al, al, al, al, None, None, al, al, 1 << 20, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"one slot per row" in lib.moe_last_error()
    one = cfg(num_experts=4, top_k=1).c()
    rc = lib.moe_forward_rows(ctypes.byref(one), al, None, al, al, al, al, None, None, al, al, 1 << 20, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"NULL" in lib.moe_last_error()
    rc = lib.moe_combine_rows(ctypes.byref(c), al, 4, None, al, al, None, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"NULL" in lib.moe_last_error()
    rc = lib.moe_combine_rows(ctypes.byref(c), al | 4, 4, al, al, al, None, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"misaligned" in lib.moe_last_error()
    rc = lib.moe_combine_rows(ctypes.byref(c), al, 1 << 30, al, al, al, None, None)
    assert rc == moe.MOE_ERR_INVALID_ARG and b"num_rows" in lib.moe_last_error()
