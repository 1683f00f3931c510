"""GPU parity of the router + softmax + top-k (moe_route_topk) against the oracle, on both of its
kernels: the CUDA-core one below 64 tokens and the tensor-core one from 64 (ragged token tiles
of 16 and expert tiles of 64 included: 16 experts, 77 and 130 tokens), with and without a router
bias, at E = 16, 256 and 512."""

import numpy as np
import pytest
import torch

import oracle
from quantized_routed_expert_bit_b200 import moe, synth

from parity import GAP_MIN, W_TOL, bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("key,T", [("tiny", 5), ("tiny", 64), ("tiny", 77), ("35b", 8), ("35b", 63), ("35b", 64),
                                   ("35b", 200), ("80b", 64), ("80b", 130), ("35b8", 70)])
def test_route_matches_oracle(key, T):
    shape = synth.SHAPES[key]
    cfg = moe.make_config(shape)
    lw = synth.make_layer(shape, 0, "cuda", seed_id=50)
    x = synth.make_batch(shape, T, 1, "cuda", seed_id=50)
    ws = moe.Workspace(cfg, T)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, shape.top_k, dtype=torch.float32, device="cuda")
    moe.moe_route_topk(cfg, x, lw.router_w, lw.router_bias, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    rb = None if lw.router_bias is None else lw.router_bias.cpu().numpy()
    lg = oracle.router_logits(bits(x), bits(lw.router_w), rb)
    checked = 0
    for t in range(T):
        s = np.sort(gi[t])
        assert np.all((s >= 0) & (s < shape.num_experts)) and np.all(s[1:] != s[:-1])
        assert abs(float(gw[t].sum()) - 1.0) <= 1e-5
        if oracle.topk_gap(lg[t], shape.top_k) <= GAP_MIN:
            continue
        ri, rw = oracle.softmax_topk(lg[t], shape.top_k)
        assert set(gi[t].tolist()) == set(ri.tolist()), f"token {t}"
        ref = dict(zip(ri.tolist(), rw.tolist()))
        assert max(abs(float(gw[t][j]) - ref[int(gi[t][j])]) for j in range(shape.top_k)) <= W_TOL
        checked += 1
    assert checked >= T - 2
    print(f"{key} T={T}: {checked} of {T} tokens checked (the rest within the 1e-4 gap)")
