"""GPU parity of the stock (unpacked) gate/up layout, the A/B baseline of the packed routed
gate/up (Runnel README, "Streaming CLI", --stock-mlp): the same layers with each expert's gate
rows and up rows in separate tensors (synth.stock_layer) against the oracle (which reads the
packed matrices: the same codes, scales and biases), and against the packed layout bit for bit
on the paths whose arithmetic does not depend on arrival order."""

import dataclasses

import numpy as np
import pytest
import torch

from quantized_routed_expert_bit_b200 import moe, synth

from parity import DeviceLayer, ParityStats, bits, check_tokens
from test_gpu_stack import check_glue, run_stack

pytestmark = pytest.mark.gpu

S35 = dataclasses.replace(synth.SHAPES["35b"], layers=1)


def layer_call(shape, lw, x):
    cfg = moe.make_config(shape)
    T = x.shape[0]
    ws = moe.Workspace(cfg, T)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, shape.top_k, dtype=torch.float32, device="cuda")
    y = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(cfg, moe.make_layer_weights(lw, cfg), x, y, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    return idx.cpu().numpy(), w.cpu().numpy(), bits(y)


@pytest.fixture(scope="module")
def layer35():
    lw = synth.make_layer(S35, 0, "cuda", seed_id=40)
    return lw, synth.stock_layer(lw), DeviceLayer(S35, lw)


@pytest.mark.parametrize("T", [1, 4, 16])
def test_stock_layer_equals_packed(layer35, T):
    """Per-token kernels (T = 1, 4) and grouped GEMV (T = 16): the same bits in both layouts."""
    lw, st, host = layer35
    x = synth.make_batch(S35, T, 3, "cuda", seed_id=40)
    a, b = layer_call(S35, lw, x), layer_call(S35, st, x)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    s = check_tokens(host, bits(x), b[0], b[1], b[2], range(T), f"stock T={T}")
    print(f"stock T={T}: max-abs {s.max_abs:.2e} rel-L2 {s.max_rel_l2:.2e}")


def test_stock_layer_runs_the_gemv_where_packed_runs_tensor_cores(layer35):
    """130 tokens: the packed layout goes to the tensor cores, the stock layout (which they do not
    read) to the grouped GEMV; both agree with the oracle."""
    lw, st, host = layer35
    T = 130
    cfg = moe.make_config(S35)
    assert moe.moe_stack_path_name(cfg, T, 1) == "batched"
    x = synth.make_batch(S35, T, 4, "cuda", seed_id=40)
    a, b = layer_call(S35, lw, x), layer_call(S35, st, x)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    toks = list(range(0, T, 13))
    sa = check_tokens(host, bits(x), a[0], a[1], a[2], toks, "packed")
    sb = check_tokens(host, bits(x), b[0], b[1], b[2], toks, "stock")
    print(f"T={T}: packed rel-L2 {sa.max_rel_l2:.2e}, stock rel-L2 {sb.max_rel_l2:.2e}")


@pytest.mark.parametrize("key,L", [("35b", 4), ("80b", 3)])
def test_stock_decode_stack(key, L):
    """One token through a stack in the stock layout on the single-token decode kernel (80b: two
    units on some CTAs), every layer teacher-forced against the oracle, and the glue."""
    shape = dataclasses.replace(synth.SHAPES[key], layers=L)
    cfg = moe.make_config(shape)
    assert moe.moe_stack_path_name(cfg, 1, L) == "decode_split_kernel"
    layers = [synth.make_layer(shape, l, "cuda", seed_id=41) for l in range(L)]
    stock = [synth.stock_layer(lw) for lw in layers]
    x0 = synth.make_tokens(shape, [5], "cuda", seed_id=41)
    tx, ti, tw, ty, xo = run_stack(shape, stock, x0)
    total = ParityStats()
    for l in range(L):
        total.merge(check_tokens(DeviceLayer(shape, layers[l]), tx[l], ti[l], tw[l], ty[l], [0], f"{key} layer {l}"))
    check_glue(bits(x0), tx, ty, xo)
    assert total.checked == L
    print(f"{key} stock stack: max-abs {total.max_abs:.2e} rel-L2 {total.max_rel_l2:.2e}")
