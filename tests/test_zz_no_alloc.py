"""The allocation-free layer call (moe_layer_forward_static).

It is for callers that cannot allocate device memory or hand the library a
scratch buffer (code inside a framework that owns all device memory,
plugins given only their inputs and outputs, latency-critical paths where
an allocation is not allowed). It must give the same result as
moe_layer_forward with a workspace, call after call, since every call
reuses the same fixed scratch.
This file is collected last on purpose: a run that stops at its first
failure has run every other test before this one.
"""

import numpy as np
import pytest
import torch

from quantized_routed_expert_bit_b200 import moe, synth

from parity import Y_MAX_ABS, Y_REL_L2, W_TOL, bits, y_errors

pytestmark = pytest.mark.gpu


def _with_workspace(cfg, W, x, shape):
    ws = moe.Workspace(cfg, x.shape[0])
    idx = torch.empty(x.shape[0], shape.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(x.shape[0], shape.top_k, dtype=torch.float32, device="cuda")
    y = torch.empty(x.shape[0], shape.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(cfg, W, x, y, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    return idx.cpu().numpy(), w.cpu().numpy(), bits(y)


# The largest token count the 2 MiB static scratch admits at the 35b shape
# (H=2048, E=256, k=8, I=Is=512): the per-token regions of the workspace
# layout for 46 tokens take 2,063,360 bytes, for 47 tokens 2,103,296.
T_MAX_35B = 46


@pytest.mark.parametrize("key,T", [("tiny", 16), ("35b", 8), ("35b", T_MAX_35B)])
def test_static_scratch_call_matches_workspace_call(key, T):
    shape = synth.SHAPES[key]
    lw = synth.make_layer(shape, 0, "cuda")
    W = moe.make_layer_weights(lw)
    cfg = moe.make_config(shape)
    x = synth.make_tokens(shape, list(range(T)), "cuda")
    idx_ref, w_ref, y_ref = _with_workspace(cfg, W, x, shape)
    for call in range(2):  # two calls in a row share the one static scratch
        idx = torch.full((T, shape.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.zeros(T, shape.top_k, dtype=torch.float32, device="cuda")
        y = torch.zeros(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        moe.moe_layer_forward_static(cfg, W, x, y, idx, w, status)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.MOE_OK
        assert np.array_equal(idx.cpu().numpy(), idx_ref)
        assert np.max(np.abs(w.cpu().numpy() - w_ref)) <= W_TOL
        yb = bits(y)
        for t in range(T):
            ref = {"y16": y_ref[t:t + 1], "y32": y_ref[t:t + 1].astype(np.uint32) << 16}
            ref["y32"] = ref["y32"].view(np.float32)
            max_abs, rel, _ = y_errors(yb[t], ref)
            assert max_abs <= Y_MAX_ABS and rel <= Y_REL_L2, f"call {call} token {t}"


@pytest.mark.parametrize("key,T", [("35b", T_MAX_35B + 1), ("tiny", 4096)])
def test_static_scratch_rejects_too_many_tokens(key, T):
    """One token past the limit is refused before anything is enqueued (the
    35b case is the boundary itself; T_MAX_35B passes above)."""
    shape = synth.SHAPES[key]
    lw = synth.make_layer(shape, 0, "cuda")
    cfg = moe.make_config(shape)
    x = torch.zeros(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    y = torch.full_like(x, 7.0)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_layer_forward_static(cfg, moe.make_layer_weights(lw), x, y, None, None)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE and "static scratch" in str(ei.value)
    torch.cuda.synchronize()
    assert bool((y == 7.0).all()), "a refused call must not write its output"
