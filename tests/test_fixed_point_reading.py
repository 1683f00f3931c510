"""The fixed-point readings of the integer dot products, checked on the CPU.

The grouped GEMV holds each token's x as X = rint(x * 2^S) in two byte planes
(S from the token's largest |x|: 2^S * max|x| < 2^15) and each unit's h in three
(2^S * max|h| < 2^22), so its outputs differ from the exact layer by that
rounding alone (up to fp32 summation order). Emulating that rounding in
float64 around the oracle's dequantised weights, 400 seeded tokens of the
256-wide top-2 layer must keep their bf16 outputs within the parity bound
(rel-L2 1e-3 against the oracle's bf16 output); rounding h to 16 bits as well
must not (which is why h keeps three planes). The split decode kernel holds x
and h in three planes (2^S * max < 2^22): the same emulation must keep the
same bound. The routing is the oracle's.
"""

import numpy as np

import oracle
from parity import DeviceLayer, bits
from quantized_routed_expert_bit_b200 import synth

TINY = synth.SHAPES["tiny"]
REL_L2 = 1e-3


def _fixed(v: np.ndarray, top: int) -> np.ndarray:
    """v rounded to the fixed point 2^-S with S = top - floor(log2 max|v|)."""
    m = float(np.max(np.abs(v)))
    if m == 0.0:
        return v
    s = top - int(np.floor(np.log2(m)))
    return np.rint(v * 2.0 ** s) * 2.0 ** -s


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _rel_l2_per_token(x_top: int, h_top: int, n: int = 400) -> np.ndarray:
    lw = synth.make_layer(TINY, 0, "cpu", seed_id=synth.SHAPE_SEED_ID["tiny"])
    layer = DeviceLayer(TINY, lw)
    xb = bits(synth.make_tokens(TINY, list(range(n)), "cpu", seed_id=synth.SHAPE_SEED_ID["tiny"]))
    deq = {}

    def mats(e):
        if e not in deq:
            g, d = layer.expert(e) if e >= 0 else layer.shared()
            deq[e] = (oracle.dequant(g, TINY.bits, TINY.group).astype(np.float64),
                      oracle.dequant(d, TINY.bits, TINY.group).astype(np.float64))
        return deq[e]

    out = np.empty(n)
    for t in range(n):
        ref = oracle.layer_forward(layer, xb[t:t + 1])
        idx, w = ref["idx"][0], ref["w"][0]
        sg = oracle.shared_gate(xb[t], layer.shared_gate_w)
        x = _fixed(oracle.bf16_to_f32(xb[t]).astype(np.float64), x_top)
        y = np.zeros(TINY.hidden)
        for e, wj in list(zip(idx.tolist(), w.tolist())) + [(-1, sg)]:
            gu, dn = mats(int(e))
            i = gu.shape[0] // 2
            h = _silu(gu[:i] @ x) * (gu[i:] @ x)
            h = np.concatenate([_fixed(h[c:c + 32], h_top) for c in range(0, i, 32)])  # per 32-column unit
            y += wj * (dn @ h)
        yg = oracle.bf16_to_f32(oracle.f32_to_bf16(y.astype(np.float32))).astype(np.float64)
        yr = oracle.bf16_to_f32(ref["y16"][0]).astype(np.float64)
        out[t] = np.linalg.norm(yg - yr) / np.linalg.norm(yr)
    return out


def test_sixteen_bit_x_keeps_the_bound():
    rel = _rel_l2_per_token(x_top=14, h_top=21)
    assert rel.max() < REL_L2, f"worst rel-L2 {rel.max():.3e}"


def test_sixteen_bit_h_would_not():
    rel = _rel_l2_per_token(x_top=14, h_top=13)
    assert (rel > REL_L2).sum() > 0, f"worst rel-L2 {rel.max():.3e}"


def test_decode_fixed_point_keeps_the_bound():
    rel = _rel_l2_per_token(x_top=21, h_top=21)
    assert rel.max() < REL_L2, f"worst rel-L2 {rel.max():.3e}"
