"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test checks one step of the oracle against something independent of its
code: a hand-worked fixture of the packing reading, a closed form, a library
routine (torch / scipy in float64) or brute force on tiny inputs. The checks
are chosen so that a plausible slip (wrong nibble order, swapped gate/up,
transposed matrix, dropped bias or scale term, sign error in the softmax or
sigmoid, wrong top-k tie rule) fails at least one of them.
"""

import itertools
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from quantized_routed_expert_bit_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BF16_ONE = 0x3F80


def _bits(t):
    return synth.bf16_bits(t)


# ---------------------------------------------------------------- formats


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        (rng.standard_normal(1000) * 1e-30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.0039062, 1.01171875, -3.5, 65504.0, 1e38], np.float32),
    ])
    # exact halfway cases between two bf16 values: tie goes to even
    halves = (np.arange(1, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    vals = np.concatenate([vals, halves, -halves])
    ours = oracle.f32_to_bf16(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = oracle.bf16_to_f32(ref)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def _read_packing_fixture():
    rows = []
    with open(os.path.join(GOLDEN, "packing_4bit_8bit.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, packed, codes = [p.strip() for p in line.split("|")]
            rows.append((int(bits), bytes.fromhex(packed.replace(" ", "")),
                         [int(c) for c in codes.split()]))
    return rows


@pytest.mark.parametrize("case", range(len(_read_packing_fixture())))
def test_dequant_unpacks_golden_packing(case):
    bits, packed, codes = _read_packing_fixture()[case]
    K = len(codes)
    q = np.frombuffer(packed, dtype=np.uint8)[None, :]
    # unit scale and zero bias: the dequantised row is the code row itself
    m = oracle.QMatrix(q, np.full((1, 1), BF16_ONE, np.uint16), np.zeros((1, 1), np.uint16), 1, K)
    out = oracle.dequant(m, bits, K)
    np.testing.assert_array_equal(out[0], np.array(codes, np.float32))


@pytest.mark.parametrize("bits", [4, 8])
def test_dequant_single_code_unit_positions(bits):
    K, group = 64, 32
    for p in range(K):
        codes = np.zeros(K, np.uint8)
        codes[p] = 1
        packed = synth.pack_codes(torch.from_numpy(codes[None, :]), bits).numpy()
        m = oracle.QMatrix(packed, np.full((1, K // group), BF16_ONE, np.uint16),
                           np.zeros((1, K // group), np.uint16), 1, K)
        out = oracle.dequant(m, bits, group)[0]
        expect = np.zeros(K, np.float32)
        expect[p] = 1.0
        np.testing.assert_array_equal(out, expect)


@pytest.mark.parametrize("bits,group", [(4, 32), (4, 64), (8, 32), (8, 64)])
def test_quantize_dequant_roundtrip_is_exact(bits, group):
    """Groups built as s*q + b with bf16 s, b and every code present round-trip exactly.

    The quantiser (input generator, torch) and the oracle's dequantiser (C)
    are separate code; agreement pins the affine form, the per-group scale
    and bias indexing, the packing and the row layout together.
    """
    rng = np.random.default_rng(bits * 100 + group)
    rows, K = 6, 4 * group
    levels = (1 << bits) - 1
    s_exp = rng.integers(-9, -4, size=(rows, K // group))
    s = np.ldexp(1.0, s_exp).astype(np.float32)                     # powers of two
    b = (rng.integers(-64, 64, size=(rows, K // group)) / 256.0).astype(np.float32)  # bf16-exact
    q = rng.integers(0, levels + 1, size=(rows, K)).astype(np.int64)
    q[:, ::group] = 0          # make min and max of every group hit the ends
    q[:, 1::group] = levels
    w = (np.repeat(s, group, axis=1) * q + np.repeat(b, group, axis=1)).astype(np.float32)
    packed, sc, bi = synth.quantize_groups(torch.from_numpy(w), bits, group)
    np.testing.assert_array_equal(sc.float().numpy(), s)
    np.testing.assert_array_equal(bi.float().numpy(), b)
    m = oracle.QMatrix(packed.numpy(), _bits(sc), _bits(bi), rows, K)
    np.testing.assert_array_equal(oracle.dequant(m, bits, group), w)


def test_dequant_constant_group_and_zero_rows():
    K, group = 64, 32
    q = np.full((2, K // 2), 0xFF, np.uint8)
    sc = np.zeros((2, 2), np.uint16)
    bi = np.array([[0x4040, 0], [0, 0]], np.uint16)  # 3.0 in group 0 of row 0, else 0
    out = oracle.dequant(oracle.QMatrix(q, sc, bi, 2, K), 4, group)
    expect = np.zeros((2, K), np.float32)
    expect[0, :32] = 3.0
    np.testing.assert_array_equal(out, expect)


# ---------------------------------------------------------------- router


def test_router_logits_exact_on_integer_inputs():
    """Integer-valued bf16 x and power-of-two weights make every logit exact."""
    rng = np.random.default_rng(1)
    T, E, H = 3, 7, 40          # E != H catches a transposed router
    x = rng.integers(-8, 9, size=(T, H)).astype(np.float32)
    pw = rng.integers(-6, 0, size=(E, H))
    sign = rng.choice([-1.0, 0.0, 1.0], size=(E, H))
    wr = (sign * np.ldexp(1.0, pw)).astype(np.float32)
    rbias = rng.integers(-4, 5, size=E).astype(np.float32) / 4
    xb = _bits(torch.from_numpy(x).to(torch.bfloat16))
    wb = _bits(torch.from_numpy(wr).to(torch.bfloat16))
    lg = oracle.router_logits(xb, wb, rbias)
    # exact integer arithmetic: scale weights by 2^6 into integers
    expect = (x.astype(np.int64) @ (wr * 64).astype(np.int64).T) / 64.0 + rbias
    np.testing.assert_array_equal(lg, expect)
    np.testing.assert_array_equal(oracle.router_logits(xb, wb, None), expect - rbias)


# ---------------------------------------------------------------- softmax / top-k


def test_two_expert_softmax_closed_form():
    for d in [0.0, 0.3, -1.7, 5.0]:
        idx, w = oracle.softmax_topk(np.array([0.25 + d, 0.25]), 2)
        hi = 1.0 / (1.0 + np.exp(-abs(d)))
        assert abs(w[0] - hi) < 1e-15 and abs(w[1] - (1 - hi)) < 1e-15
        if d != 0:
            assert idx[0] == (0 if d > 0 else 1)
        else:
            assert list(idx) == [0, 1]  # tie: lower index first


def test_topk_equal_to_all_is_full_softmax():
    rng = np.random.default_rng(2)
    lg = rng.standard_normal(16) * 3
    idx, w = oracle.softmax_topk(lg, 16)
    p = scipy.special.softmax(lg)
    np.testing.assert_allclose(w, p[idx], rtol=1e-13, atol=0)
    assert sorted(idx.tolist()) == list(range(16))
    assert np.all(np.diff(w) <= 0)


def test_top1_weight_is_exactly_one():
    rng = np.random.default_rng(3)
    for _ in range(20):
        lg = rng.standard_normal(32)
        idx, w = oracle.softmax_topk(lg, 1)
        assert idx[0] == int(np.argmax(lg)) and w[0] == 1.0


@pytest.mark.parametrize("E,k", [(8, 2), (8, 3), (10, 4), (6, 5)])
def test_topk_brute_force_over_subsets(E, k):
    """The selected set maximises the summed logit over every k-subset."""
    rng = np.random.default_rng(E * 10 + k)
    for _ in range(25):
        lg = rng.standard_normal(E)
        idx, w = oracle.softmax_topk(lg, k)
        best = max(itertools.combinations(range(E), k), key=lambda s: sum(lg[list(s)]))
        assert set(idx.tolist()) == set(best)
        ref = scipy.special.softmax(lg[list(idx)])
        np.testing.assert_allclose(w, ref, rtol=1e-13, atol=0)
        assert abs(w.sum() - 1.0) < 1e-12


def test_topk_without_renorm_returns_softmax_probabilities():
    rng = np.random.default_rng(4)
    lg = rng.standard_normal(12)
    idx, w = oracle.softmax_topk(lg, 3, renorm=False)
    np.testing.assert_allclose(w, scipy.special.softmax(lg)[idx], rtol=1e-13)


def test_topk_ties_prefer_lower_index():
    lg = np.array([1.0, 2.0, 2.0, 0.5, 2.0])
    idx, _ = oracle.softmax_topk(lg, 2)
    assert idx.tolist() == [1, 2]


# ---------------------------------------------------------------- shared gate, expert


def test_shared_gate_is_sigmoid_of_dot():
    rng = np.random.default_rng(5)
    H = 24
    x = rng.integers(-4, 5, size=H).astype(np.float32)
    w = (rng.integers(-8, 9, size=H) / 8.0).astype(np.float32)
    g = oracle.shared_gate(_bits(torch.from_numpy(x).to(torch.bfloat16)),
                           _bits(torch.from_numpy(w).to(torch.bfloat16)))
    assert abs(g - scipy.special.expit(float(x @ w))) < 1e-15


def test_expert_ffn_matches_torch_float64():
    """Gate rows first, SwiGLU on the gate, down on h; H != I catches transposes."""
    rng = np.random.default_rng(6)
    H, I = 48, 20
    wgu = (rng.standard_normal((2 * I, H)) * 0.2).astype(np.float32)
    wd = (rng.standard_normal((H, I)) * 0.2).astype(np.float32)
    x = rng.standard_normal(H)
    o, h = oracle.expert_ffn(wgu, wd, x)
    tw = torch.from_numpy(wgu).double()
    g, u = tw[:I] @ torch.from_numpy(x), tw[I:] @ torch.from_numpy(x)
    h_ref = (F.silu(g) * u).float()
    o_ref = torch.from_numpy(wd).double() @ h_ref.double()
    np.testing.assert_array_equal(h, h_ref.numpy())
    np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-12, atol=1e-15)
    # the test is sensitive to a gate/up swap
    swapped = np.concatenate([wgu[I:], wgu[:I]])
    o_sw, _ = oracle.expert_ffn(swapped, wd, x)
    assert np.max(np.abs(o_sw - o)) > 1e-3


# ---------------------------------------------------------------- whole layer


def _tiny_shape(bits=4, group=32, H=64, E=8, k=3, I=32, Is=32, rbias=False):
    return synth.MoEShape("pin", H, E, k, I, Is, bits, group, 1, rbias, 1)


def _host_layer(shape, lw):
    def trip(qt):
        return (qt.q.numpy(), _bits(qt.scales), _bits(qt.biases))
    return oracle.HostLayer(
        shape.hidden, shape.num_experts, shape.top_k, shape.inter, shape.shared_inter, shape.bits,
        shape.group, _bits(lw.router_w), None if lw.router_bias is None else lw.router_bias.numpy(),
        trip(lw.gate_up), trip(lw.down),
        trip(lw.shared_gate_up) if lw.shared_gate_up is not None else None,
        trip(lw.shared_down) if lw.shared_down is not None else None,
        None if lw.shared_gate_w is None else _bits(lw.shared_gate_w))


def _dense_unpack(qt, bits):
    """Independent numpy unpack of a QTensor to float64 [E][rows][K]."""
    q = qt.q.numpy()
    if bits == 4:
        codes = np.stack([q & 0x0F, q >> 4], axis=-1).reshape(q.shape[0], q.shape[1], -1)
    else:
        codes = q
    s = qt.scales.float().numpy().astype(np.float64)
    b = qt.biases.float().numpy().astype(np.float64)
    g = codes.shape[2] // s.shape[2]
    return codes * np.repeat(s, g, axis=2) + np.repeat(b, g, axis=2)


@pytest.mark.parametrize("bits,rbias", [(4, False), (8, True)])
def test_layer_matches_dense_brute_force(bits, rbias):
    """Evaluate every expert densely, pick the top-k subset by brute force, combine."""
    shape = _tiny_shape(bits=bits, rbias=rbias)
    lw = synth.make_layer(shape, 0, "cpu", seed_id=90 + bits)
    x = synth.make_tokens(shape, list(range(6)), "cpu", seed_id=90 + bits)
    out = oracle.layer_forward(_host_layer(shape, lw), _bits(x))
    H, I, E, k = shape.hidden, shape.inter, shape.num_experts, shape.top_k
    xd = torch.from_numpy(x.float().numpy()).double()
    WGU = torch.from_numpy(_dense_unpack(lw.gate_up, bits))
    WD = torch.from_numpy(_dense_unpack(lw.down, bits))
    SGU = torch.from_numpy(_dense_unpack(lw.shared_gate_up, bits))[0]
    SD = torch.from_numpy(_dense_unpack(lw.shared_down, bits))[0]
    wr = lw.router_w.double()
    for t in range(x.shape[0]):
        lg = (wr @ xd[t]).numpy()
        if rbias:
            lg = lg + lw.router_bias.double().numpy()
        best = max(itertools.combinations(range(E), k), key=lambda s: sum(lg[list(s)]))
        assert set(out["idx"][t].tolist()) == set(best)
        wsel = scipy.special.softmax(lg[list(best)])
        dense = []
        for e in range(E):
            gu = WGU[e] @ xd[t]
            h = F.silu(gu[:I]) * gu[I:]
            dense.append(WD[e] @ h)
        y = sum(wsel[j] * dense[e] for j, e in enumerate(best))
        gate = scipy.special.expit(float(lw.shared_gate_w.double() @ xd[t]))
        gu = SGU @ xd[t]
        y = y + gate * (SD @ (F.silu(gu[:I]) * gu[I:]))
        # the oracle rounds dequantised weights to fp32 and h to fp32: 1e-6 covers both
        np.testing.assert_allclose(out["y64"][t], y.numpy(), rtol=1e-6, atol=1e-7)


def test_zeroed_experts_give_exact_zero():
    shape = _tiny_shape()
    lw = synth.make_layer(shape, 0, "cpu", seed_id=77)
    for qt in (lw.gate_up, lw.down, lw.shared_gate_up, lw.shared_down):
        qt.scales.zero_()
        qt.biases.zero_()
    x = synth.make_tokens(shape, [0, 1, 2], "cpu", seed_id=77)
    out = oracle.layer_forward(_host_layer(shape, lw), _bits(x))
    assert np.all(out["y64"] == 0.0) and np.all(out["y16"] == 0)


def test_only_shared_expert_gives_gated_shared_output():
    shape = _tiny_shape()
    lw = synth.make_layer(shape, 0, "cpu", seed_id=78)
    lw.down.scales.zero_()
    lw.down.biases.zero_()
    x = synth.make_tokens(shape, [0, 1], "cpu", seed_id=78)
    host = _host_layer(shape, lw)
    out = oracle.layer_forward(host, _bits(x))
    sgu, sdn = host.shared()
    for t in range(2):
        xd = oracle.bf16_to_f32(_bits(x)[t]).astype(np.float64)
        o, _ = oracle.expert_ffn(oracle.dequant(sgu, 4, 32), oracle.dequant(sdn, 4, 32), xd)
        gate = scipy.special.expit(float(lw.shared_gate_w.double() @ torch.from_numpy(xd)))
        np.testing.assert_allclose(out["y64"][t], gate * o, rtol=1e-13, atol=1e-16)


def test_expert_permutation_equivariance():
    """Relabelling experts (router rows and expert weights together) relabels the selection only."""
    shape = _tiny_shape()
    lw = synth.make_layer(shape, 0, "cpu", seed_id=79)
    x = synth.make_tokens(shape, list(range(4)), "cpu", seed_id=79)
    perm = np.random.default_rng(7).permutation(shape.num_experts)
    inv = np.argsort(perm)
    base = oracle.layer_forward(_host_layer(shape, lw), _bits(x))
    P = torch.from_numpy(perm)
    lw2 = synth.LayerWeights(lw.router_w[P], None, synth.QTensor(lw.gate_up.q[P], lw.gate_up.scales[P],
                             lw.gate_up.biases[P], lw.gate_up.rows, lw.gate_up.K),
                             synth.QTensor(lw.down.q[P], lw.down.scales[P], lw.down.biases[P],
                                           lw.down.rows, lw.down.K),
                             lw.shared_gate_up, lw.shared_down, lw.shared_gate_w)
    out = oracle.layer_forward(_host_layer(shape, lw2), _bits(x))
    np.testing.assert_array_equal(perm[out["idx"]], base["idx"])
    np.testing.assert_array_equal(inv[base["idx"]], out["idx"])
    # the softmax denominator sums the experts in a different order: ulps only
    np.testing.assert_allclose(out["y64"], base["y64"], rtol=1e-13, atol=1e-18)


def test_force_idx_reproduces_own_selection():
    shape = _tiny_shape()
    lw = synth.make_layer(shape, 0, "cpu", seed_id=80)
    x = synth.make_tokens(shape, list(range(3)), "cpu", seed_id=80)
    host = _host_layer(shape, lw)
    a = oracle.layer_forward(host, _bits(x))
    b = oracle.layer_forward(host, _bits(x), force_idx=a["idx"])
    np.testing.assert_allclose(b["w"], a["w"], rtol=1e-14)
    np.testing.assert_allclose(b["y64"], a["y64"], rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- sort / permute


@pytest.mark.parametrize("T,k,E,shared", [(1, 2, 16, True), (37, 8, 256, True), (64, 3, 5, False),
                                          (0, 4, 8, True)])
def test_sort_by_expert_groups_pairs_stably(T, k, E, shared):
    rng = np.random.default_rng(T * 1000 + E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]) if T else np.zeros((0, k), np.int32)
    perm, off = oracle.sort_by_expert(idx.reshape(T, k), E, shared)
    buckets = {e: [] for e in range(E + (1 if shared else 0))}
    for t in range(T):
        for j in range(k):
            buckets[int(idx[t, j])].append(t * k + j)
    if shared:
        buckets[E] = [T * k + t for t in range(T)]
    pos = 0
    for e in range(len(buckets)):
        assert off[e] == pos
        assert perm[pos:pos + len(buckets[e])].tolist() == buckets[e]
        pos += len(buckets[e])
    assert off[-1] == pos == perm.shape[0]


# ---------------------------------------------------------------- stacking glue


def test_residual_rmsnorm_matches_torch():
    rng = np.random.default_rng(8)
    T, H = 3, 96
    r = rng.standard_normal((T, H)) * 2
    y = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16)
    r_out, x_out = oracle.residual_rmsnorm(r, _bits(y), 1e-6)
    rr = torch.from_numpy(r) + y.double()
    np.testing.assert_array_equal(r_out, rr.numpy())
    ref = F.rms_norm(rr, (H,), eps=1e-6).float().to(torch.bfloat16)
    np.testing.assert_array_equal(x_out, _bits(ref))


def test_rmsnorm_of_constant_vector():
    H = 64
    r_out, x_out = oracle.residual_rmsnorm(np.full((1, H), -3.0), np.zeros((1, H), np.uint16), 0.0)
    np.testing.assert_array_equal(oracle.bf16_to_f32(x_out), np.full((1, H), -1.0, np.float32))
