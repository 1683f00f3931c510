"""Shared helpers of the GPU parity tests: host views of device weights for
the oracle, and the three agreement checks.

  (1) the selected expert sets are identical where the oracle's gap between
      the k-th and (k+1)-th logit exceeds 1e-4;
  (2) the routing weights agree within 1e-5 absolute;
  (3) the layer outputs agree within max-abs 2e-2 and relative L2 1e-3,
      the GPU's bf16 output against the oracle's fp32 output rounded once to
      bf16 (bf16 output rounding alone differs from the unrounded fp32 by a
      relative L2 of about 1.7e-3, so the unrounded comparison is reported,
      not asserted).
A (token, layer) pair whose gap is at most 1e-4 is excluded from (1) and
(2) and checked in (3) against the oracle run with the GPU's selection.
"""

from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
from quantized_routed_expert_bit_b200 import synth

GAP_MIN = 1e-4
W_TOL = 1e-5
Y_MAX_ABS = 2e-2
Y_REL_L2 = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    return synth.bf16_bits(t)


class DeviceLayer(oracle.HostLayer):
    """oracle.HostLayer over a synth.LayerWeights; experts are copied to the
    host when the oracle first asks for them."""

    def __init__(self, shape: synth.MoEShape, lw: synth.LayerWeights):
        def trip(qt):
            return (qt.q.cpu().numpy(), bits(qt.scales), bits(qt.biases)) if qt is not None else None
        super().__init__(shape.hidden, shape.num_experts, shape.top_k, shape.inter, shape.shared_inter,
                         shape.bits, shape.group, bits(lw.router_w),
                         None if lw.router_bias is None else lw.router_bias.cpu().numpy(), None, None,
                         trip(lw.shared_gate_up), trip(lw.shared_down),
                         None if lw.shared_gate_w is None else bits(lw.shared_gate_w))
        self.lw = lw
        self._cache = {}

    def expert(self, e: int):
        if e not in self._cache:
            g, d = self.lw.gate_up, self.lw.down
            self._cache[e] = (
                oracle.QMatrix(g.q[e].cpu().numpy(), bits(g.scales[e]), bits(g.biases[e]), 2 * self.I, self.H),
                oracle.QMatrix(d.q[e].cpu().numpy(), bits(d.scales[e]), bits(d.biases[e]), self.H, self.I))
        return self._cache[e]


@dataclasses.dataclass
class ParityStats:
    checked: int = 0
    excluded: int = 0
    max_abs: float = 0.0
    max_rel_l2: float = 0.0
    max_rel_l2_unrounded: float = 0.0
    max_w_err: float = 0.0

    def merge(self, o: "ParityStats"):
        self.checked += o.checked
        self.excluded += o.excluded
        self.max_abs = max(self.max_abs, o.max_abs)
        self.max_rel_l2 = max(self.max_rel_l2, o.max_rel_l2)
        self.max_rel_l2_unrounded = max(self.max_rel_l2_unrounded, o.max_rel_l2_unrounded)
        self.max_w_err = max(self.max_w_err, o.max_w_err)


def y_errors(y_gpu_bits: np.ndarray, ref: dict, row: int = 0):
    yg = oracle.bf16_to_f32(y_gpu_bits).astype(np.float64)
    yr = oracle.bf16_to_f32(ref["y16"][row]).astype(np.float64)
    y32 = ref["y32"][row].astype(np.float64)
    max_abs = float(np.max(np.abs(yg - yr))) if yg.size else 0.0
    nr = float(np.linalg.norm(yr))
    rel = float(np.linalg.norm(yg - yr) / nr) if nr > 0 else float(np.linalg.norm(yg))
    n32 = float(np.linalg.norm(y32))
    rel32 = float(np.linalg.norm(yg - y32) / n32) if n32 > 0 else float(np.linalg.norm(yg))
    return max_abs, rel, rel32


def _check_one(layer: oracle.HostLayer, x_bits: np.ndarray, gpu_idx: np.ndarray, gpu_w: np.ndarray,
               gpu_y_bits: np.ndarray, t: int, where: str, threads: int) -> ParityStats:
    st = ParityStats()
    ref = oracle.layer_forward(layer, x_bits[t:t + 1], threads=threads)
    gi = gpu_idx[t].astype(np.int64)
    if ref["gap"][0] > GAP_MIN:
        assert set(gi.tolist()) == set(ref["idx"][0].tolist()), \
            f"{where} token {t}: experts {sorted(gi.tolist())} != {sorted(ref['idx'][0].tolist())}"
        rw = dict(zip(ref["idx"][0].tolist(), ref["w"][0].tolist()))
        werr = max(abs(float(gpu_w[t][j]) - rw[int(gi[j])]) for j in range(len(gi)))
        assert werr <= W_TOL, f"{where} token {t}: weight error {werr}"
        st.max_w_err = werr
    else:
        st.excluded = 1
        ref = oracle.layer_forward(layer, x_bits[t:t + 1], force_idx=gpu_idx[t:t + 1], threads=threads)
    max_abs, rel, rel32 = y_errors(gpu_y_bits[t], ref)
    assert max_abs <= Y_MAX_ABS and rel <= Y_REL_L2, \
        f"{where} token {t}: max-abs {max_abs:.3e}, rel-L2 {rel:.3e}"
    st.checked = 1
    st.max_abs, st.max_rel_l2, st.max_rel_l2_unrounded = max_abs, rel, rel32
    return st


def check_tokens(layer: oracle.HostLayer, x_bits: np.ndarray, gpu_idx: np.ndarray, gpu_w: np.ndarray,
                 gpu_y_bits: np.ndarray, tokens, where: str = "", threads: int = 4) -> ParityStats:
    """Checks (1)-(3) for the given token rows; raises AssertionError on a violation.

    Several tokens are checked concurrently, one oracle call per host core
    (the oracle's C calls run without the interpreter lock)."""
    tokens = list(tokens)
    st = ParityStats()
    if len(tokens) <= 1:
        for t in tokens:
            st.merge(_check_one(layer, x_bits, gpu_idx, gpu_w, gpu_y_bits, t, where, threads))
        return st
    for e in np.unique(gpu_idx[tokens]).tolist():  # host copies of the experts, before the workers start
        if 0 <= e < layer.E:
            layer.expert(int(e))
    workers = max(1, min(len(tokens), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        for r in ex.map(lambda t: _check_one(layer, x_bits, gpu_idx, gpu_w, gpu_y_bits, t, where, 1), tokens):
            st.merge(r)
    return st


def gap_filtered_tokens(shape: synth.MoEShape, layer: oracle.HostLayer, n: int, device="cpu"):
    """The first n token seeds whose own k-th/(k+1)-th logit gap exceeds 1e-4
    (a token at or under the limit is replaced by the next seed)."""
    ids, i = [], 0
    while len(ids) < n:
        x = synth.make_tokens(shape, [i], "cpu")
        lg = oracle.router_logits(bits(x), layer.router_w, layer.router_bias)
        if oracle.topk_gap(lg[0], shape.top_k) > GAP_MIN:
            ids.append(i)
        i += 1
    return ids, synth.make_tokens(shape, ids, device)


def oracle_ffn_given_selection(layer: oracle.HostLayer, x_bits_row, idx_row, w_row, threads: int = 4):
    """Oracle expert part for one token under a given selection and weights
    (as moe_expert_ffn receives them): returns the oracle dict for y."""
    mats = [layer.expert(int(e)) for e in idx_row]
    sgu, sdn = layer.shared()
    gate = oracle.shared_gate(x_bits_row, layer.shared_gate_w) if sgu is not None else 0.0
    y64, y32, y16 = oracle.moe_token(layer.H, layer.I, layer.Is, layer.bits, layer.group, x_bits_row,
                                     [m[0] for m in mats], [m[1] for m in mats],
                                     np.asarray(w_row, dtype=np.float64), sgu, sdn, gate, threads)
    return dict(y64=y64[None], y32=y32[None], y16=y16[None])
