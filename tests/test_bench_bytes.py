"""The algorithmic bytes behind the bench's roofline figure, pinned two ways:
against the byte sizes of the tensors a generated layer actually holds (the
k selected experts and the shared expert, the router, the shared gate and
the router bias, each read once per token), and against the closed form for
the 35b shape (16,977,920 B per layer, 679,116,800 B per token)."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_routed_expert_bit_b200 import synth  # noqa: E402


def _nbytes(t):
    return t.numel() * t.element_size()


def _expert_bytes(qt):
    """Bytes of one expert of a QTensor: its slice of codes, scales and biases."""
    E = qt.q.shape[0]
    return (_nbytes(qt.q) + _nbytes(qt.scales) + _nbytes(qt.biases)) // E


@pytest.mark.parametrize("shape", [
    synth.SHAPES["tiny"],
    synth.MoEShape("bytes-8bit-bias", 256, 16, 2, 128, 128, 8, 32, 3, True, 1),
    synth.MoEShape("bytes-no-shared", 256, 16, 3, 128, 0, 4, 64, 2, False, 1),
], ids=lambda s: s.name)
def test_bytes_per_token_match_the_layer_tensors(shape):
    lw = synth.make_layer(shape, 0, "cpu")
    per_layer = shape.top_k * (_expert_bytes(lw.gate_up) + _expert_bytes(lw.down))
    if shape.shared_inter > 0:
        per_layer += _expert_bytes(lw.shared_gate_up) + _expert_bytes(lw.shared_down) + _nbytes(lw.shared_gate_w)
    per_layer += _nbytes(lw.router_w)
    if lw.router_bias is not None:
        per_layer += _nbytes(lw.router_bias)
    assert bench.touched_bytes_per_token(shape) == per_layer * shape.layers


def test_bytes_per_token_35b_closed_form():
    s = synth.SHAPES["35b"]
    codes = 2 * 512 * 2048 // 2 + 2048 * 512 // 2                 # packed gate/up + down, 4-bit
    scale_bias = 2 * (2 * 512 * (2048 // 64) + 2048 * (512 // 64)) * 2  # bf16 scales + biases
    expert = codes + scale_bias
    assert expert == 1_769_472
    per_layer = (8 + 1) * expert + 256 * 2048 * 2 + 2048 * 2
    assert per_layer == 16_977_920
    assert bench.touched_bytes_per_token(s) == 40 * per_layer == 679_116_800
