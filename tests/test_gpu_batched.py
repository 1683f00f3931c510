"""GPU parity of the batched tensor-core path (token-by-expert grouping,
tcgen05 grouped dequant-GEMMs, combine) against the CPU oracle.

By default the library takes this path from 128 tokens up (moe_expert_ffn,
moe_layer_forward, moe_stack_forward), the grouped GEMV from 8 and the
per-token kernels below that. These tests move the tensor-core threshold
down to 8 tokens (moe_set_batched_min_tokens), so that 8 to 127 tokens are
covered on this path too.
"""

import numpy as np
import pytest
import torch

from quantized_routed_expert_bit_b200 import moe, synth

from parity import (DeviceLayer, ParityStats, Y_MAX_ABS, Y_REL_L2, bits, check_tokens,
                    oracle_ffn_given_selection, y_errors)

pytestmark = pytest.mark.gpu

S35 = synth.SHAPES["35b"]


@pytest.fixture(autouse=True)
def tensor_core_from_8_tokens():
    pb = moe.moe_set_batched_min_tokens(8)
    yield
    moe.moe_set_batched_min_tokens(pb)


def layer_call(shape, lw, x):
    cfg = moe.make_config(shape)
    T = x.shape[0]
    ws = moe.Workspace(cfg, T)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, shape.top_k, dtype=torch.float32, device="cuda")
    y = torch.empty(T, shape.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_forward(cfg, moe.make_layer_weights(lw), x, y, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    return idx.cpu().numpy(), w.cpu().numpy(), bits(y)


@pytest.fixture(scope="module")
def layer35():
    lw = synth.make_layer(S35, 0, "cuda", seed_id=2)
    return lw, DeviceLayer(S35, lw)


@pytest.mark.parametrize("key", ["35b", "35b8", "80b"])
def test_batched_path_is_taken(key):
    """With the thresholds at 8 (batched) and 2 (grouped GEMV), the workloads'
    shapes run on the tensor-core path from 8 tokens up (route, sort, gather,
    two GEMMs, combine, glue: 7 kernels a layer), on the grouped GEMV from 2
    to 7 tokens (route, sort, fixed-point x, GEMV, combine, glue: 6 a layer;
    4-bit shapes only), and on the token-at-a-time kernels (route, gate/up,
    down, glue: 4 a layer) when the GEMV is switched off."""
    cfg = moe.make_config(synth.SHAPES[key])
    # by default up to 7 tokens through a stack run one at a time on the decode kernel
    assert moe.moe_stack_path_name(cfg, 7, 3) == "decode_split_kernel"
    assert moe.moe_stack_kernel_launches(cfg, 7, 3) == 7
    pb, pg = moe.moe_set_batched_min_tokens(8), moe.moe_set_gemv_min_tokens(2)
    pd = moe.moe_set_decode_max_tokens(1)
    try:
        assert moe.moe_stack_kernel_launches(cfg, 8, 3) == 1 + 7 * 3
        assert moe.moe_stack_kernel_launches(cfg, 512, 3) == 1 + 7 * 3
        assert moe.moe_stack_path_name(cfg, 8, 3) == moe.moe_stack_path_name(cfg, 512, 3) == "batched"
        if synth.SHAPES[key].bits == 4:
            assert moe.moe_stack_kernel_launches(cfg, 7, 3) == 1 + 6 * 3
            assert moe.moe_stack_path_name(cfg, 7, 3) == moe.moe_stack_path_name(cfg, 2, 3) == "grouped_gemv"
        else:  # 8-bit: two buffers of 32 gate/up row pairs (2 x 136 KB) exceed shared memory
            assert moe.moe_stack_path_name(cfg, 7, 3) == "per_layer"
        moe.moe_set_gemv_min_tokens(1 << 30)
        assert moe.moe_stack_kernel_launches(cfg, 7, 3) == 1 + 4 * 3
        assert moe.moe_stack_path_name(cfg, 7, 3) == "per_layer"
    finally:
        moe.moe_set_batched_min_tokens(pb)
        moe.moe_set_gemv_min_tokens(pg)
        moe.moe_set_decode_max_tokens(pd)


@pytest.mark.parametrize("T", [7, 8, 16])
def test_batched_matches_single_token_and_oracle(layer35, T):
    lw, host = layer35
    x = synth.make_batch(S35, T, 1, "cuda", seed_id=2)
    idx, w, y = layer_call(S35, lw, x)
    st = check_tokens(host, bits(x), idx, w, y, range(T), f"T={T}")
    for t in range(T):
        i1, w1, y1 = layer_call(S35, lw, x[t:t + 1])
        assert np.array_equal(i1[0], idx[t]) and np.array_equal(w1[0], w[t])
        ref = {"y16": y1, "y32": (y1.astype(np.uint32) << 16).view(np.float32)}
        max_abs, rel, _ = y_errors(y[t], ref)
        assert max_abs <= Y_MAX_ABS and rel <= Y_REL_L2, f"token {t}: batched vs single {max_abs} {rel}"
    print(f"T={T}: max-abs {st.max_abs:.2e} rel-L2 {st.max_rel_l2:.2e}")


@pytest.mark.parametrize("key,T", [("35b", 512), ("35b8", 64)])
def test_batched_layer_parity(key, T):
    shape = synth.SHAPES[key]
    lw = synth.make_layer(shape, 0, "cuda")
    host = DeviceLayer(shape, lw)
    x = synth.make_batch(shape, T, 2, "cuda")
    idx, w, y = layer_call(shape, lw, x)
    st = check_tokens(host, bits(x), idx, w, y, range(T), f"{key} T={T}")
    assert st.checked == T
    print(f"{key} T={T}: {st.checked} tokens, max-abs {st.max_abs:.2e} rel-L2 {st.max_rel_l2:.2e}")


def test_large_batch_layer(layer35):
    """3,000 tokens through one layer on the default path (tensor cores, router on the tensor
    cores): the sort's selection no longer fits its shared-memory copy (27,000 pairs) and is read
    through L2, the GEMMs run ~5,000 chunks; sampled tokens against the oracle, and every token's
    selection a valid set."""
    lw, host = layer35
    T = 3000
    x = synth.make_batch(S35, T, 5, "cuda", seed_id=2)
    pb = moe.moe_set_batched_min_tokens(0)  # the library's default threshold
    try:
        assert moe.moe_stack_path_name(moe.make_config(S35), T, 1) == "batched"
        idx, w, y = layer_call(S35, lw, x)
    finally:
        moe.moe_set_batched_min_tokens(pb)
    s = np.sort(idx, axis=1)
    assert np.all((s >= 0) & (s < S35.num_experts)) and np.all(s[:, 1:] != s[:, :-1])
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-5)
    toks = [0, 1, 15, 16, 1023, 1024, 2047, 2048, 2999]
    st = check_tokens(host, bits(x), idx, w, y, toks, "T=3000")
    assert st.checked == len(toks)
    print(f"T={T}: {st.checked} sampled tokens, max-abs {st.max_abs:.2e} rel-L2 {st.max_rel_l2:.2e}")


def test_expert_with_hundreds_of_tokens(layer35):
    """Expert 3 is every token's first choice: 300 tokens for one expert (three
    GEMM chunks of <= 128), besides the shared expert's three chunks."""
    lw, host = layer35
    T, k = 300, S35.top_k
    cfg = moe.make_config(S35)
    rng = np.random.default_rng(11)
    idx_np = np.zeros((T, k), np.int32)
    for t in range(T):
        others = rng.choice([e for e in range(S35.num_experts) if e != 3], size=k - 1, replace=False)
        idx_np[t] = np.concatenate([[3], others])
    w_np = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    x = synth.make_batch(S35, T, 3, "cuda", seed_id=2)
    ws = moe.Workspace(cfg, T)
    y = torch.empty(T, S35.hidden, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn(cfg, moe.make_layer_weights(lw), x, torch.from_numpy(idx_np).cuda(),
                       torch.from_numpy(w_np).cuda(), y, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    yb, xb = bits(y), bits(x)
    for t in [0, 1, 127, 128, 129, 255, 256, 299]:
        ref = oracle_ffn_given_selection(host, xb[t], idx_np[t], w_np[t])
        max_abs, rel, _ = y_errors(yb[t], ref)
        assert max_abs <= Y_MAX_ABS and rel <= Y_REL_L2, f"token {t}: {max_abs} {rel}"


def test_batched_zeroed_experts_give_exact_zero():
    shape = S35
    lw = synth.make_layer(shape, 1, "cuda", seed_id=2)
    for qt in (lw.gate_up, lw.down, lw.shared_gate_up, lw.shared_down):
        qt.scales.zero_()
        qt.biases.zero_()
    x = synth.make_batch(shape, 32, 4, "cuda")
    _, _, y = layer_call(shape, lw, x)
    assert np.all(y == 0)
