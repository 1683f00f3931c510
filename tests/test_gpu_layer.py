"""GPU parity of one MoE layer against the CPU oracle, through the C ABI.

Covers the tiny bring-up layer (H=256, E=16, top-2, I=Is=128, 4-bit g32,
100 gap-filtered tokens), format and routing variants (8-bit, no shared
expert, top-1, top-k = E, no renormalisation, router bias), ragged and
empty batches, the largest supported shape, zeroed experts, and the
device-side bounds check on caller-supplied expert indices.
"""

import re

import numpy as np
import pytest
import torch

import oracle
from quantized_routed_expert_bit_b200 import moe, synth

from parity import DeviceLayer, bits, check_tokens, gap_filtered_tokens

pytestmark = pytest.mark.gpu

TINY = synth.SHAPES["tiny"]


def _alloc_out(shape, T, dev="cuda"):
    return (torch.empty(T, shape.top_k, dtype=torch.int32, device=dev),
            torch.empty(T, shape.top_k, dtype=torch.float32, device=dev),
            torch.empty(T, shape.hidden, dtype=torch.bfloat16, device=dev))


def _run_layer(shape, lw, x, renorm=1):
    cfg = moe.make_config(shape, renorm)
    ws = moe.Workspace(cfg, x.shape[0])
    W = moe.make_layer_weights(lw)
    idx, w, y = _alloc_out(shape, x.shape[0])
    moe.moe_layer_forward(cfg, W, x, y, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    return idx.cpu().numpy(), w.cpu().numpy(), bits(y)


@pytest.fixture(scope="module")
def tiny():
    lw_cpu = synth.make_layer(TINY, 0, "cpu")
    lw = synth.LayerWeights(lw_cpu.router_w.cuda(), None, lw_cpu.gate_up.to("cuda"), lw_cpu.down.to("cuda"),
                            lw_cpu.shared_gate_up.to("cuda"), lw_cpu.shared_down.to("cuda"),
                            lw_cpu.shared_gate_w.cuda())
    host = DeviceLayer(TINY, lw)
    ids, x = gap_filtered_tokens(TINY, host, 100, "cuda")
    return lw, host, x


def test_tiny_layer_100_tokens(tiny):
    lw, host, x = tiny
    idx, w, y = _run_layer(TINY, lw, x)
    st = check_tokens(host, bits(x), idx, w, y, range(x.shape[0]), "tiny")
    assert st.checked == 100 and st.excluded == 0
    print(f"tiny: max-abs {st.max_abs:.2e} rel-L2 {st.max_rel_l2:.2e} "
          f"(unrounded {st.max_rel_l2_unrounded:.2e}) w-err {st.max_w_err:.2e}")


def test_tiny_route_and_ffn_calls_match_layer(tiny):
    lw, host, x = tiny
    cfg = moe.make_config(TINY)
    T = x.shape[0]
    ws = moe.Workspace(cfg, T)
    idx, w, y = _alloc_out(TINY, T)
    moe.moe_route_topk(cfg, x, lw.router_w, None, idx, w, ws)
    W = moe.make_layer_weights(lw)
    moe.moe_expert_ffn(cfg, W, x, idx, w, y, ws)
    idx2, w2, y2 = _run_layer(TINY, lw, x)
    assert np.array_equal(idx.cpu().numpy(), idx2)
    assert np.array_equal(w.cpu().numpy(), w2)
    assert np.array_equal(bits(y), y2)


def test_batch_equals_single_token_calls(tiny):
    """The per-token kernels give a token the same bits alone as in a batch of 13."""
    lw, host, x = tiny
    pg = moe.moe_set_gemv_min_tokens(1 << 30)  # keep 13 tokens on the per-token kernels
    try:
        assert moe.moe_stack_path_name(moe.make_config(TINY), 13, 1) == "per_layer"
        idx, w, y = _run_layer(TINY, lw, x[:13])
        for t in range(13):
            i1, w1, y1 = _run_layer(TINY, lw, x[t:t + 1])
            assert np.array_equal(i1[0], idx[t]) and np.array_equal(w1[0], w[t]) and np.array_equal(y1[0], y[t])
    finally:
        moe.moe_set_gemv_min_tokens(pg)


def test_grouped_gemv_is_batch_invariant(tiny):
    """On the grouped GEMV a token's output depends on its own x alone (its own fixed-point scale,
    partial sums combined in a fixed order, for a given number of units per work item, which
    depends on the batch size): the same bits in a batch of 13 as in a batch of 13 copies of it."""
    lw, host, x = tiny
    pg, pb = moe.moe_set_gemv_min_tokens(2), moe.moe_set_batched_min_tokens(1 << 30)
    try:
        assert moe.moe_stack_path_name(moe.make_config(TINY), 13, 1) == "grouped_gemv"
        idx, w, y = _run_layer(TINY, lw, x[:13])
        for t in range(13):
            i2, w2, y2 = _run_layer(TINY, lw, x[t:t + 1].repeat(13, 1))
            for r in (0, 6, 12):
                assert np.array_equal(i2[r], idx[t]) and np.array_equal(w2[r], w[t]) and np.array_equal(y2[r], y[t])
    finally:
        moe.moe_set_gemv_min_tokens(pg)
        moe.moe_set_batched_min_tokens(pb)


def test_empty_batch_is_noop(tiny):
    lw, host, x = tiny
    cfg = moe.make_config(TINY)
    ws = moe.Workspace(cfg, 1)
    idx, w, y = _alloc_out(TINY, 1)
    y.fill_(1.0)
    moe.moe_layer_forward(cfg, moe.make_layer_weights(lw), x[:0], y, idx, w, ws)
    torch.cuda.synchronize()
    assert torch.all(y == 1.0)


def test_bad_expert_index_is_skipped_and_reported(tiny):
    lw, host, x = tiny
    cfg = moe.make_config(TINY)
    ws = moe.Workspace(cfg, 2)
    idx, w, y = _alloc_out(TINY, 2)
    moe.moe_route_topk(cfg, x[:2], lw.router_w, None, idx, w, ws)
    idx[1, 0] = TINY.num_experts + 5
    moe.moe_expert_ffn(cfg, moe.make_layer_weights(lw), x[:2], idx, w, y, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_BOUNDS
    assert moe.moe_get_device_status(ws) == moe.MOE_OK  # cleared by the read
    # token 0 is untouched by token 1's bad index
    st = check_tokens(host, bits(x), idx.cpu().numpy(), w.cpu().numpy(), bits(y), [0], "bounds")
    assert st.checked == 1


def test_bounded_waits_give_up_and_leave_the_context_usable(tiny):
    """A word nothing writes and an mbarrier nobody arrives at: both waits end
    by their limit, the status reads MOE_ERR_TIMEOUT, and a layer run right
    after on the same stream is still exact."""
    lw, host, x = tiny
    cfg = moe.make_config(TINY)
    ws = moe.Workspace(cfg, 4)
    gave_up = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    moe.moe_check_wait_limit(ws, gave_up)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_TIMEOUT
    assert re.search(r"detail 9[12]\b", moe.last_error())  # first to give up: 91 word poll, 92 mbarrier
    assert int(gave_up.item()) == 3
    assert 1500.0 < ms < 10000.0
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    idx, w, y = _alloc_out(TINY, 4)
    moe.moe_layer_forward(cfg, moe.make_layer_weights(lw), x[:4], y, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    st = check_tokens(host, bits(x), idx.cpu().numpy(), w.cpu().numpy(), bits(y), range(4), "after timeout")
    assert st.checked == 4


def test_zeroed_experts_give_exact_zero():
    shape = TINY
    lw = synth.make_layer(shape, 0, "cuda", seed_id=55)
    for qt in (lw.gate_up, lw.down, lw.shared_gate_up, lw.shared_down):
        qt.scales.zero_()
        qt.biases.zero_()
    x = synth.make_tokens(shape, list(range(9)), "cuda")
    _, _, y = _run_layer(shape, lw, x)
    assert np.all(y == 0)


VARIANTS = {
    "8bit_g64": synth.MoEShape("v8", 256, 16, 2, 128, 128, 8, 64, 1, False, 1),
    "no_shared": synth.MoEShape("vns", 256, 16, 2, 128, 0, 4, 32, 1, False, 1),
    "top1": synth.MoEShape("vk1", 256, 16, 1, 128, 128, 4, 32, 1, False, 1),
    "topk_all": synth.MoEShape("vkE", 256, 16, 16, 128, 64, 4, 64, 1, False, 1),
    "router_bias": synth.MoEShape("vrb", 512, 64, 6, 256, 128, 8, 32, 1, True, 1),
    "e512_k10": synth.MoEShape("v512", 256, 512, 10, 64, 64, 4, 32, 1, False, 1),
}


@pytest.mark.parametrize("name", sorted(VARIANTS))
def test_layer_variants(name):
    shape = VARIANTS[name]
    lw = synth.make_layer(shape, 0, "cuda", seed_id=200 + sorted(VARIANTS).index(name))
    host = DeviceLayer(shape, lw)
    ids, x = gap_filtered_tokens(shape, host, 21, "cuda")
    idx, w, y = _run_layer(shape, lw, x)
    st = check_tokens(host, bits(x), idx, w, y, range(x.shape[0]), name)
    if shape.top_k == 1:
        assert np.all(w == 1.0)
    print(f"{name}: max-abs {st.max_abs:.2e} rel-L2 {st.max_rel_l2:.2e} w-err {st.max_w_err:.2e}")


def test_no_renorm_returns_softmax_probabilities(tiny):
    lw, host, x = tiny
    idx, w, y = _run_layer(TINY, lw, x[:20], renorm=0)
    lg = oracle.router_logits(bits(x[:20]), host.router_w)
    for t in range(20):
        i_ref, w_ref = oracle.softmax_topk(lg[t], TINY.top_k, renorm=False)
        assert set(idx[t].tolist()) == set(i_ref.tolist())
        ref = dict(zip(i_ref.tolist(), w_ref.tolist()))
        assert max(abs(w[t][j] - ref[int(idx[t][j])]) for j in range(TINY.top_k)) <= 1e-5
    assert np.all(w.sum(axis=1) < 1.0)


def test_largest_supported_shape():
    # H=8192, I=Is=2048, k=16 are the library's upper limits
    shape = synth.MoEShape("vmax", 8192, 32, 16, 2048, 2048, 4, 64, 1, False, 1)
    lw = synth.make_layer(shape, 0, "cuda", seed_id=300)
    host = DeviceLayer(shape, lw)
    ids, x = gap_filtered_tokens(shape, host, 3, "cuda")
    idx, w, y = _run_layer(shape, lw, x)
    st = check_tokens(host, bits(x), idx, w, y, range(3), "max", threads=8)
    print(f"max shape: max-abs {st.max_abs:.2e} rel-L2 {st.max_rel_l2:.2e}")
    del lw
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T,E,k,shared", [(1, 16, 2, True), (13, 16, 2, True), (64, 256, 8, True),
                                          (512, 256, 8, True), (300, 512, 10, False), (0, 8, 2, True)])
def test_sort_by_expert_is_bit_exact(T, E, k, shared):
    rng = np.random.default_rng(T + E)
    idx_np = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32) if T else \
        np.zeros((0, k), np.int32)
    shape = synth.MoEShape("s", 256, E, k, 128, 128 if shared else 0, 4, 32, 1, False, T)
    cfg = moe.make_config(shape)
    ws = moe.Workspace(cfg, max(T, 1))
    idx = torch.from_numpy(idx_np).cuda()
    n = T * k + (T if shared else 0)
    perm = torch.full((max(n, 1),), -1, dtype=torch.int32, device="cuda")
    offs = torch.full((E + (2 if shared else 1),), -1, dtype=torch.int32, device="cuda")
    moe.moe_sort_by_expert(cfg, idx, perm, offs, ws)
    p_ref, o_ref = oracle.sort_by_expert(idx_np.reshape(T, k), E, shared)
    assert np.array_equal(offs.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy()[:n], p_ref)
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
