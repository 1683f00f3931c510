"""GPU parity of full-size stacked layers against the CPU oracle.

Decode stacks (T=1, the launch configuration the benchmark times):
  35b   40 layers, H=2048, E=256, top-8, I=Is=512, 4-bit g64
  80b   48 layers, H=2048, E=512, top-10, I=Is=512, 4-bit g64
  35b8  40 layers, the 35b shape in 8-bit g64 with a per-expert router bias
Batched stacks: the 35b shape with T=64 and T=512 tokens.

Every layer is checked teacher-forced: the oracle gets the GPU's own bf16
input of that layer (recorded by the stack's trace), so one-ulp
differences do not compound through later routing. The residual/RMSNorm
glue between layers is checked separately (within one bf16 ulp).
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from quantized_routed_expert_bit_b200 import moe, synth

from parity import DeviceLayer, ParityStats, bits, check_tokens

pytestmark = pytest.mark.gpu


def run_stack(shape, layers, x0, prepared=True):
    """One stack call with a trace. prepared: hand the library the group-major down
    scale/bias copies (moe_prepare_down_sb); without them the single-token decode reads
    the canonical layout (same results, slower)."""
    T, L, H, k = x0.shape[0], len(layers), shape.hidden, shape.top_k
    cfg = moe.make_config(shape)
    ws = moe.Workspace(cfg, T, L=L)
    arr = moe.make_layer_array([moe.make_layer_weights(lw, cfg if prepared else None) for lw in layers])
    tx = torch.empty(L, T, H, dtype=torch.bfloat16, device="cuda")
    ti = torch.empty(L, T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(L, T, k, dtype=torch.float32, device="cuda")
    ty = torch.empty(L, T, H, dtype=torch.bfloat16, device="cuda")
    xo = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    tr = moe.Trace(tx.data_ptr(), ti.data_ptr(), tw.data_ptr(), ty.data_ptr())
    moe.moe_stack_forward(cfg, arr, x0, xo, ws, trace=tr)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    return bits(tx), ti.cpu().numpy(), tw.cpu().numpy(), bits(ty), bits(xo)


def check_glue(x0_bits, tx, ty, xo):
    """x_{l+1} = bf16(rmsnorm(x_0 + sum_{m<=l} y_m)) within one bf16 ulp."""
    L = ty.shape[0]
    r = oracle.bf16_to_f32(x0_bits).astype(np.float64)
    worst, flips = 0, 0
    for l in range(L):
        r, x_ref = oracle.residual_rmsnorm(r, ty[l])
        got = xo if l == L - 1 else tx[l + 1]
        d = np.abs(got.astype(np.int32) - x_ref.astype(np.int32))
        worst = max(worst, int(d.max()))
        flips += int((d > 0).sum())
    assert worst <= 1, f"glue differs by {worst} bf16 ulps"
    return flips


@pytest.mark.parametrize("key", ["35b", "80b", "35b8"])
def test_decode_stack_parity(key):
    shape = synth.SHAPES[key]
    # which persistent kernel runs each stack on a 148-SM B200 (a silent fallback would fail here)
    want = "decode_split_kernel"
    assert moe.moe_stack_path_name(moe.make_config(shape), 1, shape.layers) == want
    layers = [synth.make_layer(shape, l, "cuda") for l in range(shape.layers)]
    total = ParityStats()
    for tok in (0, 1):
        x0 = synth.make_tokens(shape, [tok], "cuda")
        tx, ti, tw, ty, xo = run_stack(shape, layers, x0)
        for l in range(shape.layers):
            host = DeviceLayer(shape, layers[l])
            total.merge(check_tokens(host, tx[l], ti[l], tw[l], ty[l], [0], f"{key} tok {tok} layer {l}"))
        flips = check_glue(bits(x0), tx, ty, xo)
    print(f"{key}: {total.checked} (token, layer) pairs, {total.excluded} gap-excluded, "
          f"max-abs {total.max_abs:.2e}, rel-L2 {total.max_rel_l2:.2e} "
          f"(unrounded {total.max_rel_l2_unrounded:.2e}), w-err {total.max_w_err:.2e}, glue flips {flips}")
    assert total.excluded <= max(2, total.checked // 20)
    del layers
    torch.cuda.empty_cache()


@pytest.mark.parametrize("key,path", [("35b_t64", "grouped_gemv"), ("35b_t64", "batched"), ("35b_t512", "batched")])
def test_batched_stack_parity(key, path):
    """The batched stacks on the path the library picks for them by default (grouped GEMV at 64
    tokens, tensor cores at 512) and, at 64 tokens, on the tensor-core path as well."""
    shape = synth.SHAPES[key]
    T = shape.tokens
    cfg = moe.make_config(shape)
    layers = [synth.make_layer(shape, l, "cuda") for l in range(shape.layers)]
    x0 = synth.make_batch(shape, T, 0, "cuda")
    forced = path != moe.moe_stack_path_name(cfg, T, shape.layers)
    pb = moe.moe_set_batched_min_tokens(1 if forced else 0)  # 0: the default threshold
    try:
        assert moe.moe_stack_path_name(cfg, T, shape.layers) == path
        tx, ti, tw, ty, xo = run_stack(shape, layers, x0)
    finally:
        moe.moe_set_batched_min_tokens(pb)
    total = ParityStats()
    rng = np.random.default_rng(T)
    # every token of every layer at T=64; at T=512 every token of the first two, a middle and the
    # last layer (2,048 pairs) and 8 sampled tokens of the others
    full = set(range(shape.layers)) if T <= 64 else {0, 1, shape.layers // 2, shape.layers - 1}
    for l in range(shape.layers):
        host = DeviceLayer(shape, layers[l])
        toks = range(T) if l in full else sorted(rng.choice(T, size=8, replace=False).tolist())
        total.merge(check_tokens(host, tx[l], ti[l], tw[l], ty[l], toks, f"{key} layer {l}"))
        del host
    flips = check_glue(bits(x0), tx, ty, xo)
    want = len(full) * T + (shape.layers - len(full)) * 8
    assert total.checked == want
    print(f"{key} on {path}: {total.checked} (token, layer) pairs checked (every token on {len(full)} of {shape.layers} "
          f"layers), {total.excluded} gap-excluded, max-abs {total.max_abs:.2e}, rel-L2 {total.max_rel_l2:.2e}, "
          f"glue flips {flips}")
    assert total.excluded <= max(2, total.checked // 50)
    # every token's selection is a valid set of k distinct experts
    assert np.all((ti >= 0) & (ti < shape.num_experts))
    s = np.sort(ti, axis=-1)
    assert np.all(s[..., 1:] != s[..., :-1])
    assert np.allclose(tw.sum(axis=-1), 1.0, atol=1e-5)
    del layers
    torch.cuda.empty_cache()


def test_decode_stack_longer_than_one_launch():
    """100 layers: the persistent path splits the stack over three launches of
    at most 48 layers and carries the residual stream between them."""
    shape = synth.MoEShape("chunk-h256-e16", 256, 16, 2, 128, 128, 4, 32, 100, False, 1)
    cfg = moe.make_config(shape)
    assert moe.moe_stack_kernel_launches(cfg, 1, shape.layers) == 3
    layers = [synth.make_layer(shape, l, "cuda", seed_id=400) for l in range(shape.layers)]
    x0 = synth.make_tokens(shape, [3], "cuda", seed_id=400)
    tx, ti, tw, ty, xo = run_stack(shape, layers, x0)
    total = ParityStats()
    for l in (0, 1, 46, 47, 48, 49, 95, 96, 99):
        total.merge(check_tokens(DeviceLayer(shape, layers[l]), tx[l], ti[l], tw[l], ty[l], [0], f"layer {l}"))
    check_glue(bits(x0), tx, ty, xo)
    assert total.checked == 9


SMALL_STACKS = {
    # name: (H, E, k, I, Is, bits, group, layers, router bias)
    "8bit": (256, 16, 2, 128, 128, 8, 32, 6, True),
    # 1536-wide 8-bit rows: 96 code segments, three per lane
    "8bit-h1536": (1536, 16, 2, 128, 128, 8, 32, 3, False),
    "no-shared": (256, 16, 2, 128, 0, 4, 32, 6, False),
    "top1-g64": (512, 32, 1, 256, 256, 4, 64, 6, False),
    "top8-e64": (1024, 64, 8, 128, 128, 4, 32, 6, False),
    # (5 * 1024 + 1024) / 32 = 192 units: more than one per SM, some CTAs take two
    "two-units": (256, 16, 5, 1024, 1024, 4, 32, 4, False),
    # (7 * 1024 + 1024) / 32 = 256 units: 108 CTAs take a second unit
    "two-units-k7": (256, 16, 7, 1024, 1024, 4, 32, 3, False),
}


@pytest.mark.parametrize("prepared", [True, False])
@pytest.mark.parametrize("name", sorted(SMALL_STACKS))
def test_small_decode_stacks(name, prepared):
    """Format and routing variants of the persistent decode path, every layer
    teacher-forced against the oracle, with and without the group-major down
    scale/bias copies."""
    H, E, k, I, Is, b, g, L, rb = SMALL_STACKS[name]
    shape = synth.MoEShape("stack-" + name, H, E, k, I, Is, b, g, L, rb, 1)
    assert moe.moe_stack_kernel_launches(moe.make_config(shape), 1, L) == 1
    layers = [synth.make_layer(shape, l, "cuda", seed_id=500) for l in range(L)]
    total = ParityStats()
    for tok in (0, 1, 2):
        x0 = synth.make_tokens(shape, [tok], "cuda", seed_id=500)
        tx, ti, tw, ty, xo = run_stack(shape, layers, x0, prepared=prepared)
        for l in range(L):
            total.merge(check_tokens(DeviceLayer(shape, layers[l]), tx[l], ti[l], tw[l], ty[l], [0], f"{name} {l}"))
        check_glue(bits(x0), tx, ty, xo)
    assert total.excluded <= 2


def test_exchange_kernel_stack():
    """A shape the split kernel's plan does not take (8-bit, 1536 wide, top-9 of 256: 160 units
    need a second unit on some CTAs, and two units' 8-bit rows do not fit in its shared memory)
    runs on decode_stack_kernel; two tokens, every layer teacher-forced against the oracle, and
    the glue."""
    shape = synth.MoEShape("stack-8bit-h1536-top9", 1536, 256, 9, 512, 512, 8, 64, 2, False, 1)
    cfg = moe.make_config(shape)
    assert moe.moe_stack_path_name(cfg, 1, shape.layers) == "decode_stack_kernel"
    layers = [synth.make_layer(shape, l, "cuda", seed_id=70) for l in range(shape.layers)]
    total = ParityStats()
    for tok in (0, 1):
        x0 = synth.make_tokens(shape, [tok], "cuda", seed_id=70)
        tx, ti, tw, ty, xo = run_stack(shape, layers, x0)
        for l in range(shape.layers):
            total.merge(check_tokens(DeviceLayer(shape, layers[l]), tx[l], ti[l], tw[l], ty[l], [0], f"layer {l}"))
        check_glue(bits(x0), tx, ty, xo)
    assert total.checked == 2 * shape.layers
    print(f"exchange kernel: max-abs {total.max_abs:.2e} rel-L2 {total.max_rel_l2:.2e}")
    del layers
    torch.cuda.empty_cache()


@pytest.mark.parametrize("key,T,L", [("35b", 3, 4), ("80b", 2, 3)])
def test_small_batch_runs_a_token_at_a_time(key, T, L):
    """Up to 7 tokens through a stack run one after another on the persistent decode kernel (T
    launches), each token's trace in its row of every layer: every (token, layer) teacher-forced
    against the oracle, and the glue."""
    shape = dataclasses.replace(synth.SHAPES[key], layers=L)
    cfg = moe.make_config(shape)
    assert moe.moe_stack_path_name(cfg, T, L) == "decode_split_kernel"
    assert moe.moe_stack_kernel_launches(cfg, T, L) == T
    layers = [synth.make_layer(shape, l, "cuda", seed_id=60) for l in range(L)]
    x0 = synth.make_batch(shape, T, 2, "cuda", seed_id=60)
    tx, ti, tw, ty, xo = run_stack(shape, layers, x0)
    total = ParityStats()
    for l in range(L):
        total.merge(check_tokens(DeviceLayer(shape, layers[l]), tx[l], ti[l], tw[l], ty[l], range(T), f"{key} {l}"))
    check_glue(bits(x0), tx, ty, xo)
    assert total.checked == T * L
    print(f"{key} T={T}: {total.checked} pairs, max-abs {total.max_abs:.2e} rel-L2 {total.max_rel_l2:.2e}")


def test_single_token_path_matches_multi_kernel_path():
    """One token through the persistent kernel against the same token run
    twice in a batch of two through the multi-kernel path, layer by layer on
    the persistent kernel's own input of that layer (teacher-forced): same
    experts, routing weights within 1e-5, and outputs within twice the
    oracle tolerance of each other (each path's bf16 output is within
    max-abs 2e-2 and rel-L2 1e-3 of the oracle's rounded output, so the two
    are within twice that of each other)."""
    shape = synth.SHAPES["35b"]
    import dataclasses
    shape = dataclasses.replace(shape, layers=4)
    layers = [synth.make_layer(shape, l, "cuda", seed_id=2) for l in range(shape.layers)]
    cfg = moe.make_config(shape)
    assert moe.moe_stack_kernel_launches(cfg, 1, 4) == 1
    x1 = synth.make_tokens(shape, [7], "cuda", seed_id=2)
    tx, ti, tw, ty, _ = run_stack(shape, layers, x1)
    ws = moe.Workspace(cfg, 2)
    pg = moe.moe_set_gemv_min_tokens(1 << 30)  # the four-kernel per-token path for T=2
    pd = moe.moe_set_decode_max_tokens(1)
    try:
        assert moe.moe_stack_kernel_launches(cfg, 2, 4) == 17
        _compare_with_per_layer(shape, cfg, layers, tx, ti, tw, ty, ws)
    finally:
        moe.moe_set_gemv_min_tokens(pg)
        moe.moe_set_decode_max_tokens(pd)


def _compare_with_per_layer(shape, cfg, layers, tx, ti, tw, ty, ws):
    for l in range(shape.layers):
        xl = torch.from_numpy(tx[l].astype(np.int16)).view(torch.bfloat16).cuda().repeat(2, 1)
        y = torch.empty(2, shape.hidden, dtype=torch.bfloat16, device="cuda")
        idx = torch.empty(2, shape.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(2, shape.top_k, dtype=torch.float32, device="cuda")
        moe.moe_layer_forward(cfg, moe.make_layer_weights(layers[l]), xl, y, idx, w, ws)
        torch.cuda.synchronize()
        bi, bw, by = idx.cpu().numpy(), w.cpu().numpy(), bits(y)
        assert set(ti[l][0].tolist()) == set(bi[0].tolist()) == set(bi[1].tolist())
        ref = dict(zip(bi[0].tolist(), bw[0].tolist()))
        assert max(abs(float(tw[l][0][j]) - ref[int(ti[l][0][j])]) for j in range(shape.top_k)) <= 1e-5
        ya = oracle.bf16_to_f32(ty[l][0]).astype(np.float64)
        for t in range(2):
            yb = oracle.bf16_to_f32(by[t]).astype(np.float64)
            assert np.max(np.abs(ya - yb)) <= 2 * 2e-2, f"layer {l}"
            assert np.linalg.norm(ya - yb) <= 2 * 1e-3 * np.linalg.norm(yb), f"layer {l}"
