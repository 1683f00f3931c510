"""GPU parity of the grouped GEMV path (a few tokens per expert, CUDA cores) against the
CPU oracle: each selected expert's weights read once for all of its tokens, in chunks of at
most 4 tokens and groups of four 32-column units. The path is forced with the dispatch knobs
(moe_set_gemv_min_tokens / moe_set_batched_min_tokens) and asserted by moe_stack_path_name."""

import numpy as np
import pytest
import torch

import oracle
from quantized_routed_expert_bit_b200 import moe, synth

from parity import DeviceLayer, ParityStats, bits, check_tokens, oracle_ffn_given_selection, \
    y_errors, Y_MAX_ABS, Y_REL_L2

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def gemv_path():
    """Grouped GEMV from 2 tokens up, never the tensor-core path, and stacks of a few tokens not a
    token at a time on the decode kernel; defaults restored after."""
    pg = moe.moe_set_gemv_min_tokens(2)
    pb = moe.moe_set_batched_min_tokens(1 << 30)
    pd = moe.moe_set_decode_max_tokens(1)
    yield
    moe.moe_set_gemv_min_tokens(pg)
    moe.moe_set_batched_min_tokens(pb)
    moe.moe_set_decode_max_tokens(pd)


def layer_call(shape, lw, x, prepared=True):
    T = x.shape[0]
    cfg = moe.make_config(shape)
    assert moe.moe_stack_path_name(cfg, T, 1) == "grouped_gemv"
    ws = moe.Workspace(cfg, T)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, shape.top_k, dtype=torch.float32, device="cuda")
    y = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(cfg, moe.make_layer_weights(lw, cfg if prepared else None), x, y, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    return idx.cpu().numpy(), w.cpu().numpy(), bits(y)


SHAPES = {
    "tiny": synth.SHAPES["tiny"],
    "no-shared": synth.MoEShape("gv-ns", 256, 16, 2, 128, 0, 4, 32, 1, False, 1),
    "e64-top8": synth.MoEShape("gv-e64", 1024, 64, 8, 256, 256, 4, 64, 1, False, 1),
    "35b": synth.SHAPES["35b"],
}


@pytest.mark.parametrize("name,T", [("tiny", 2), ("tiny", 5), ("tiny", 16), ("no-shared", 7), ("e64-top8", 9),
                                    ("35b", 3), ("35b", 16), ("35b", 64)])
def test_gemv_layer_parity(name, T):
    shape = SHAPES[name]
    lw = synth.make_layer(shape, 0, "cuda", seed_id=800 + list(SHAPES).index(name))
    host = DeviceLayer(shape, lw)
    x = synth.make_batch(shape, T, 7, "cuda", seed_id=800)
    idx, w, y = layer_call(shape, lw, x)
    st = check_tokens(host, bits(x), idx, w, y, range(T), f"{name} T={T}")
    assert st.checked == T
    print(f"{name} T={T}: max-abs {st.max_abs:.2e} rel-L2 {st.max_rel_l2:.2e} w-err {st.max_w_err:.2e}, "
          f"{st.excluded} gap-excluded")


def test_gemv_without_prepared_copies():
    """Without the decode-ready down copies the path reads the canonical layout: same results."""
    shape = SHAPES["e64-top8"]
    lw = synth.make_layer(shape, 1, "cuda", seed_id=810)
    x = synth.make_batch(shape, 6, 3, "cuda", seed_id=810)
    a = layer_call(shape, lw, x, prepared=True)
    b = layer_call(shape, lw, x, prepared=False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert np.array_equal(a[2], b[2])  # same arithmetic in the same order: bit-identical
    check_tokens(DeviceLayer(shape, lw), bits(x), b[0], b[1], b[2], range(6), "canonical layout")


def test_gemv_expert_with_many_tokens():
    """Expert 3 is every token's first choice: 40 tokens for one expert (ten chunks of four),
    besides the shared expert's ten chunks."""
    shape = SHAPES["35b"]
    cfg = moe.make_config(shape)
    lw = synth.make_layer(shape, 2, "cuda", seed_id=820)
    host = DeviceLayer(shape, lw)
    T, k = 40, shape.top_k
    rng = np.random.default_rng(5)
    idx_np = np.zeros((T, k), np.int32)
    for t in range(T):
        others = rng.choice([e for e in range(shape.num_experts) if e != 3], size=k - 1, replace=False)
        idx_np[t] = np.concatenate([[3], others])
    w_np = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    x = synth.make_batch(shape, T, 9, "cuda", seed_id=820)
    assert moe.moe_stack_path_name(cfg, T, 1) == "grouped_gemv"
    ws = moe.Workspace(cfg, T)
    y = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, moe.make_layer_weights(lw, cfg), x, torch.from_numpy(idx_np).cuda(),
                       torch.from_numpy(w_np).cuda(), y, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    yb, xb = bits(y), bits(x)
    for t in range(T):
        ref = oracle_ffn_given_selection(host, xb[t], idx_np[t], w_np[t])
        max_abs, rel, _ = y_errors(yb[t], ref)
        assert max_abs <= Y_MAX_ABS and rel <= Y_REL_L2, f"token {t}: {max_abs} {rel}"


def test_gemv_stack_parity():
    """16 tokens through 4 layers of the 35b shape on the grouped GEMV path, every layer of every
    token teacher-forced against the oracle, and the residual/RMSNorm glue between layers."""
    import dataclasses
    shape = dataclasses.replace(synth.SHAPES["35b"], layers=4, tokens=16)
    T, L, H, k = 16, 4, shape.hidden, shape.top_k
    cfg = moe.make_config(shape)
    assert moe.moe_stack_path_name(cfg, T, L) == "grouped_gemv"
    assert moe.moe_stack_kernel_launches(cfg, T, L) == 1 + 6 * L
    layers = [synth.make_layer(shape, l, "cuda", seed_id=830) for l in range(L)]
    ws = moe.Workspace(cfg, T, L=L)
    arr = moe.make_layer_array([moe.make_layer_weights(lw, cfg) for lw in layers])
    x0 = synth.make_batch(shape, T, 1, "cuda", seed_id=830)
    tx = torch.empty(L, T, H, dtype=torch.bfloat16, device="cuda")
    ti = torch.empty(L, T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(L, T, k, dtype=torch.float32, device="cuda")
    ty = torch.empty(L, T, H, dtype=torch.bfloat16, device="cuda")
    xo = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_stack_forward(cfg, arr, x0, xo, ws, trace=moe.Trace(tx.data_ptr(), ti.data_ptr(), tw.data_ptr(),
                                                               ty.data_ptr()))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    bx, bi, bw, by = bits(tx), ti.cpu().numpy(), tw.cpu().numpy(), bits(ty)
    total = ParityStats()
    for l in range(L):
        total.merge(check_tokens(DeviceLayer(shape, layers[l]), bx[l], bi[l], bw[l], by[l], range(T), f"layer {l}"))
    r = oracle.bf16_to_f32(bits(x0)).astype(np.float64)
    for l in range(L):
        r, x_ref = oracle.residual_rmsnorm(r, by[l])
        got = bits(xo) if l == L - 1 else bx[l + 1]
        assert int(np.abs(got.astype(np.int32) - x_ref.astype(np.int32)).max()) <= 1
    assert total.checked == T * L
    print(f"gemv stack: {total.checked} pairs, max-abs {total.max_abs:.2e}, rel-L2 {total.max_rel_l2:.2e}")
