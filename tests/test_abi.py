"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function include/moe_b200.h declares,
and reject bad arguments with the documented status before touching the
device (every call below returns before any CUDA call, so it runs on a
machine without a GPU).
"""

import ctypes
import os
import re
import subprocess

import pytest

from quantized_routed_expert_bit_b200 import build as moe_build
from quantized_routed_expert_bit_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    moe_build.build()
    yield


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for required in ("moe_route_topk", "moe_expert_ffn", "moe_layer_forward", "moe_stack_forward",
                     "moe_workspace_size", "moe_get_device_status", "moe_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = moe.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", moe._LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert set(declared_functions()) <= exported


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "use.c"
    src.write_text('#include "moe_b200.h"\nint main(void){moe_config c={0};(void)c;return 0;}\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), "-c", str(src),
                    "-o", str(tmp_path / "use.o")], check=True)


def cfg35(**kw):
    c = dict(hidden=2048, num_experts=256, top_k=8, inter=512, shared_inter=512, bits=4, group=64, renorm=1)
    c.update(kw)
    return moe.Config(**c)


def test_status_strings():
    lib = moe.lib()
    assert lib.moe_status_string(0) == b"MOE_OK"
    assert lib.moe_status_string(6) == b"MOE_ERR_BOUNDS"
    assert lib.moe_status_string(99) == b"MOE_ERR_UNKNOWN"


@pytest.mark.parametrize("bad", [dict(bits=3), dict(group=128), dict(hidden=100), dict(top_k=0),
                                 dict(top_k=17), dict(num_experts=4, top_k=8), dict(num_experts=1024),
                                 dict(inter=48), dict(shared_inter=40), dict(renorm=2), dict(hidden=16384)])
def test_workspace_size_rejects_unsupported_configs(bad):
    assert moe.lib().moe_workspace_size(ctypes.byref(cfg35(**bad)), 1, 1) == 0


@pytest.mark.parametrize("shape", ["tiny", "35b", "80b", "35b8"])
def test_workspace_for_t_tokens_serves_every_smaller_call(shape):
    """A workspace sized for T tokens is large enough for every call of fewer tokens (the grouped
    GEMV's partial outputs need more planes at some small sizes than at larger ones)."""
    from quantized_routed_expert_bit_b200 import synth
    c = moe.make_config(synth.SHAPES[shape])
    sizes = [moe.lib().moe_workspace_size(ctypes.byref(c), T, 1) for T in range(1, 300)]
    assert all(b >= a for a, b in zip(sizes, sizes[1:]))


def test_workspace_size_grows_with_tokens():
    lib = moe.lib()
    a = lib.moe_workspace_size(ctypes.byref(cfg35()), 1, 40)
    b = lib.moe_workspace_size(ctypes.byref(cfg35()), 512, 40)
    assert 0 < a < b and a % 256 == 0


FAKE = 1 << 40  # 16-byte aligned, never dereferenced: every call below fails validation first


def call_route(cfg, x=FAKE, T=1, wr=FAKE, idx=FAKE, w=FAKE, ws=FAKE, nbytes=1 << 30):
    return moe.lib().moe_route_topk(ctypes.byref(cfg) if cfg is not None else None, x, T, wr, None, idx, w,
                                    ws, nbytes, None)


def test_route_validation_errors():
    assert call_route(None) == moe.MOE_ERR_INVALID_ARG
    assert call_route(cfg35(bits=2)) == moe.MOE_ERR_UNSUPPORTED
    assert call_route(cfg35(), T=-1) == moe.MOE_ERR_INVALID_ARG
    assert call_route(cfg35(), x=None) == moe.MOE_ERR_INVALID_ARG
    assert call_route(cfg35(), x=FAKE + 2) == moe.MOE_ERR_INVALID_ARG     # misaligned
    assert call_route(cfg35(), idx=None) == moe.MOE_ERR_INVALID_ARG
    assert call_route(cfg35(), ws=None) == moe.MOE_ERR_WORKSPACE
    assert call_route(cfg35(), ws=FAKE + 16) == moe.MOE_ERR_WORKSPACE     # not 256-byte aligned
    assert call_route(cfg35(), nbytes=100) == moe.MOE_ERR_WORKSPACE
    assert b"needs" in moe.lib().moe_last_error_string()
    assert call_route(cfg35(), T=0, x=None) == moe.MOE_OK                 # T = 0 is a no-op


def fake_qt(stride_q, stride_sb):
    return moe.QTensor(FAKE, FAKE, FAKE, stride_q, stride_sb)


def fake_weights(cfg, **over):
    H, I, Is, b, g = cfg.hidden, cfg.inter, cfg.shared_inter, cfg.bits, cfg.group
    w = moe.LayerWeights(FAKE, None, fake_qt(2 * I * H * b // 8, 2 * I * H // g), fake_qt(H * I * b // 8, H * I // g),
                         fake_qt(0, 0), fake_qt(0, 0), FAKE)
    for k, v in over.items():
        setattr(w, k, v)
    return w


def call_ffn(cfg, w, T=1):
    return moe.lib().moe_expert_ffn(ctypes.byref(cfg), ctypes.byref(w), FAKE, T, FAKE, FAKE, FAKE, FAKE, 1 << 34, None)


def test_expert_ffn_validation_errors():
    c = cfg35()
    assert call_ffn(c, fake_weights(c), T=0) == moe.MOE_OK
    assert call_ffn(c, fake_weights(c, gate_up=fake_qt(100, 2 * 512 * 32))) == moe.MOE_ERR_INVALID_ARG  # short stride
    assert call_ffn(c, fake_weights(c, down=fake_qt(2048 * 256 + 8, 2048 * 8))) == moe.MOE_ERR_INVALID_ARG  # %16
    assert call_ffn(c, fake_weights(c, down=fake_qt(2048 * 256, 2048 * 8 + 4))) == moe.MOE_ERR_INVALID_ARG  # %8
    bad = fake_weights(c)
    bad.gate_up.scales = FAKE + 2
    assert call_ffn(c, bad) == moe.MOE_ERR_INVALID_ARG
    bad = fake_weights(c)
    bad.shared_gate_w = None
    assert call_ffn(c, bad) == moe.MOE_ERR_INVALID_ARG
    assert b"shared_gate_w" in moe.lib().moe_last_error_string()
    # without a shared expert its pointers are not looked at
    c0 = cfg35(shared_inter=0)
    w0 = fake_weights(c0)
    w0.shared_gate_w = None
    assert call_ffn(c0, w0, T=0) == moe.MOE_OK


def test_stock_layout_validation_errors():
    """The stock gate/up layout (separate gate and up tensors) is checked before the device: the up
    tensors need the gate tensors' expert strides, and shared_up is set exactly when up is."""
    c = cfg35()
    H, I, b, g = c.hidden, c.inter, c.bits, c.group
    half_q, half_sb = I * H * b // 8, I * H // g

    def stock(**over):
        w = fake_weights(c, gate_up=fake_qt(half_q, half_sb), up=fake_qt(half_q, half_sb),
                         shared_gate_up=fake_qt(0, 0), shared_up=fake_qt(0, 0))
        for k, v in over.items():
            setattr(w, k, v)
        return w

    assert call_ffn(c, stock(), T=0) == moe.MOE_OK
    assert call_ffn(c, stock(up=fake_qt(half_q + 16, half_sb))) == moe.MOE_ERR_INVALID_ARG
    assert b"strides" in moe.lib().moe_last_error_string()
    assert call_ffn(c, stock(up=fake_qt(half_q, half_sb + 8))) == moe.MOE_ERR_INVALID_ARG
    assert call_ffn(c, stock(shared_up=moe.QTensor(None, None, None, 0, 0))) == moe.MOE_ERR_INVALID_ARG
    assert b"shared_up" in moe.lib().moe_last_error_string()
    assert call_ffn(c, stock(up=fake_qt(half_q, half_sb - 8))) == moe.MOE_ERR_INVALID_ARG  # too short for I rows
    # packed weights with a shared_up tensor: inconsistent
    assert call_ffn(c, fake_weights(c, shared_up=fake_qt(0, 0))) == moe.MOE_ERR_INVALID_ARG


def test_stack_and_sort_validation_errors():
    c = cfg35()
    lib = moe.lib()
    arr = (moe.LayerWeights * 2)(fake_weights(c), fake_weights(c, router_w=None))
    st = lib.moe_stack_forward(ctypes.byref(c), arr, 2, FAKE, 1, FAKE, None, FAKE, 1 << 34, None)
    assert st == moe.MOE_ERR_INVALID_ARG and b"layer 1" in lib.moe_last_error_string()
    assert lib.moe_stack_forward(ctypes.byref(c), arr, 0, FAKE, 1, FAKE, None, FAKE, 1 << 34, None) == moe.MOE_OK
    assert lib.moe_sort_by_expert(ctypes.byref(c), FAKE, 4, FAKE, None, FAKE, 1 << 30, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert lib.moe_get_device_status(None, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_workspace_init(None, 1024, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_check_wait_limit(None, 1024, FAKE, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_check_wait_limit(FAKE, 32, FAKE, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_check_wait_limit(FAKE, 1024, None, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_stack_path_name(None, 1, 1) is None
    assert lib.moe_stack_path_name(ctypes.byref(c), 0, 4) == b"none"
    assert lib.moe_stack_path_name(ctypes.byref(c), 1, 4) in (b"decode_split_kernel", b"decode_stack_kernel",
                                                               b"per_layer")


def test_batched_threshold_knob():
    """moe_set_batched_min_tokens returns the previous threshold; T < 1 restores the default 128."""
    lib = moe.lib()
    assert lib.moe_set_batched_min_tokens(3) == 128
    assert lib.moe_set_batched_min_tokens(100) == 3
    assert lib.moe_set_batched_min_tokens(0) == 100
    assert lib.moe_set_batched_min_tokens(-5) == 128
    assert lib.moe_set_batched_min_tokens(0) == 128


def test_decode_threshold_knob():
    """moe_set_decode_max_tokens returns the previous threshold; T < 1 restores the default 7."""
    lib = moe.lib()
    assert lib.moe_set_decode_max_tokens(3) == 7
    assert lib.moe_set_decode_max_tokens(0) == 3
    assert lib.moe_set_decode_max_tokens(-1) == 7


def test_gemv_threshold_knob():
    """moe_set_gemv_min_tokens returns the previous threshold; T < 1 restores the default 8."""
    lib = moe.lib()
    assert lib.moe_set_gemv_min_tokens(3) == 8
    assert lib.moe_set_gemv_min_tokens(100) == 3
    assert lib.moe_set_gemv_min_tokens(0) == 100
    assert lib.moe_set_gemv_min_tokens(-5) == 8
    assert lib.moe_set_gemv_min_tokens(0) == 8


def test_prepare_calls_validate_before_the_device():
    """The load-time re-layouts refuse bad arguments without touching the device."""
    c = cfg35()
    lib = moe.lib()
    qt = moe.QTensor(FAKE, FAKE, FAKE, 2048 * 256, 2048 * 8)
    assert lib.moe_down_sb_size(ctypes.byref(c), 256, 512) == 256 * 8 * 2048 * 4
    assert lib.moe_down_units_size(ctypes.byref(c), 256, 512) == 256 * 512 * 2048 // 2
    assert lib.moe_down_sb_size(ctypes.byref(c), 256, 500) == 0        # K not a multiple of the group
    assert lib.moe_down_units_size(ctypes.byref(c), 0, 512) == 0
    assert lib.moe_prepare_down_sb(ctypes.byref(c), None, 256, 512, FAKE, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_prepare_down_sb(ctypes.byref(c), ctypes.byref(qt), 256, 512, FAKE + 2, None) == \
        moe.MOE_ERR_INVALID_ARG                                        # misaligned output
    assert lib.moe_prepare_down_units(ctypes.byref(c), ctypes.byref(qt), 256, 96, FAKE, None) == \
        moe.MOE_ERR_INVALID_ARG                                        # K not a multiple of the group
    short = moe.QTensor(FAKE, FAKE, FAKE, 100, 2048 * 8)
    assert lib.moe_prepare_down_units(ctypes.byref(c), ctypes.byref(short), 256, 512, FAKE, None) == \
        moe.MOE_ERR_INVALID_ARG                                        # expert stride below one expert
