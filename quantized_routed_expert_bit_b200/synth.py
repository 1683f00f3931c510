"""Seeded synthetic inputs for the routed-MoE layer.

This module only *produces* inputs: random hidden states, router weights and
expert weights quantised into the packed low-bit format the layer consumes.
It computes nothing the layer computes (no routing, no expert arithmetic,
no dequantisation) and it is the one module that both the CUDA path's tests
and the CPU oracle draw their inputs from.

The packed format (the reading of "MLX-style int4/int8 group quantization",
Swiftlet article on xix.ai, paragraph 8):
  * every matrix is [rows][K], quantised in groups of `group` consecutive
    elements along K (the input dimension);
  * per group a bf16 scale and a bf16 bias with w ~= scale * q + bias, where
    scale = (max - min) / (2^bits - 1) and bias = min, both rounded to bf16
    first, and q = clamp(round_half_even((w - bias) / scale), 0, 2^bits - 1)
    (q = 0 for a constant group, scale = 0);
  * 8-bit codes are one byte per element; 4-bit codes are two per byte along
    K with the even element in the low nibble;
  * the routed experts' gate and up projections are one packed [2I][H]
    matrix per expert (Runnel README, introduction): gate rows first.
The value distributions follow the workloads the layer is measured on:
weights N(0, 0.02), router N(0, 0.02) in bf16, hidden states N(0, 1) in
bf16, and an optional per-expert router bias N(0, 1) that skews routing
toward a hot subset of experts (the Swiftlet article, paragraph 4, reports
43-70% expert-cache hit rates, i.e. strongly skewed expert popularity).
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

# Tensor ids inside one layer's seed space.
T_ROUTER, T_GATE_UP, T_DOWN, T_SH_GATE_UP, T_SH_DOWN, T_WSG, T_RBIAS = range(7)


@dataclasses.dataclass(frozen=True)
class MoEShape:
    """Shape of one routed-MoE workload."""

    name: str
    hidden: int          # H
    num_experts: int     # E
    top_k: int           # k
    inter: int           # I, routed expert intermediate size
    shared_inter: int    # Is, shared expert intermediate size (0 = none)
    bits: int            # 4 or 8
    group: int           # quantisation group along K
    layers: int          # L, stacked layers
    router_bias: bool    # per-expert logit bias N(0, 1)
    tokens: int          # tokens per batch (T)

    @property
    def row_bytes_gate_up(self) -> int:
        return self.hidden * self.bits // 8

    def expert_bytes(self, inter: Optional[int] = None) -> int:
        """Packed bytes + bf16 scales and biases of one expert (gate/up and down)."""
        i = self.inter if inter is None else inter
        gu = 2 * i * (self.hidden * self.bits // 8 + (self.hidden // self.group) * 4)
        dn = self.hidden * (i * self.bits // 8 + (i // self.group) * 4)
        return gu + dn


# The workloads, by id. 1 is the tiny bring-up layer; 2-4 are batch-1 decode
# stacks shaped like Qwen3.6-35B-A3B (256 experts, top-8) and
# Qwen3-Next-80B-A3B (512 experts, top-10) -- the routing fan-outs the
# Swiftlet article gives in paragraph 4 and Runnel's "Target" section; 5 is
# the batched (chunked-prefill / multi-sequence) form of the 35B shape.
SHAPES: Dict[str, MoEShape] = {
    "tiny": MoEShape("tiny-h256-e16-top2", 256, 16, 2, 128, 128, 4, 32, 1, False, 1),
    "35b": MoEShape("qwen35b-a3b-4bit-l40", 2048, 256, 8, 512, 512, 4, 64, 40, False, 1),
    "80b": MoEShape("qwen-next-80b-a3b-4bit-l48", 2048, 512, 10, 512, 512, 4, 64, 48, False, 1),
    "35b8": MoEShape("qwen35b-a3b-8bit-skewed-l40", 2048, 256, 8, 512, 512, 8, 64, 40, True, 1),
    "35b_t64": MoEShape("qwen35b-a3b-4bit-l40-t64", 2048, 256, 8, 512, 512, 4, 64, 40, False, 64),
    "35b_t512": MoEShape("qwen35b-a3b-4bit-l40-t512", 2048, 256, 8, 512, 512, 4, 64, 40, False, 512),
}

# Seed-space id of each workload.
SHAPE_SEED_ID = {"tiny": 1, "35b": 2, "80b": 3, "35b8": 4, "35b_t64": 5, "35b_t512": 5}


def layer_seed(cfg_id: int, layer: int, tensor: int) -> int:
    return cfg_id * 1_000_003 + layer * 1_009 + tensor


def token_seed(cfg_id: int, i: int) -> int:
    return cfg_id * 1_000_003 + 999_983 + i


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def quantize_groups(w: torch.Tensor, bits: int, group: int):
    """Quantise fp32 [rows][K] into (codes uint8 [rows][K*bits/8], scales bf16, biases bf16).

    Input preparation only (the offline repack step); the layer itself never
    quantises.
    """
    rows, K = w.shape
    assert K % group == 0 and bits in (4, 8)
    levels = (1 << bits) - 1
    wg = w.float().reshape(rows, K // group, group)
    mn = wg.amin(dim=2)
    mx = wg.amax(dim=2)
    scale = ((mx - mn) / levels).to(torch.bfloat16)
    bias = mn.to(torch.bfloat16)
    sf = scale.float().unsqueeze(2)
    bf = bias.float().unsqueeze(2)
    safe = torch.where(sf == 0, torch.ones_like(sf), sf)
    q = torch.round((wg - bf) / safe).clamp_(0, levels)
    q = torch.where(sf == 0, torch.zeros_like(q), q)
    q = q.to(torch.uint8).reshape(rows, K)
    return pack_codes(q, bits), scale.contiguous(), bias.contiguous()


def pack_codes(q: torch.Tensor, bits: int) -> torch.Tensor:
    """Pack integer codes [rows][K] (uint8) into the byte layout."""
    if bits == 8:
        return q.contiguous()
    lo = q[:, 0::2]
    hi = q[:, 1::2]
    return (lo | (hi << 4)).contiguous()


@dataclasses.dataclass
class QTensor:
    """Packed codes, scales and biases of E matrices [E][rows][K]."""

    q: torch.Tensor       # uint8 [E][rows][K*bits/8]
    scales: torch.Tensor  # bf16  [E][rows][K/group]
    biases: torch.Tensor  # bf16  [E][rows][K/group]
    rows: int
    K: int

    def to(self, device) -> "QTensor":
        return QTensor(self.q.to(device), self.scales.to(device), self.biases.to(device),
                       self.rows, self.K)

    def expert(self, e: int) -> "QTensor":
        return QTensor(self.q[e:e + 1], self.scales[e:e + 1], self.biases[e:e + 1], self.rows, self.K)

    def select(self, experts) -> "QTensor":
        ix = torch.as_tensor(experts, dtype=torch.long, device=self.q.device)
        return QTensor(self.q.index_select(0, ix), self.scales.index_select(0, ix),
                       self.biases.index_select(0, ix), self.rows, self.K)


@dataclasses.dataclass
class LayerWeights:
    router_w: torch.Tensor             # bf16 [E][H]
    router_bias: Optional[torch.Tensor]  # fp32 [E] or None
    gate_up: QTensor                   # [E][2I][H]
    down: QTensor                      # [E][H][I]
    shared_gate_up: Optional[QTensor]  # [1][2Is][H]
    shared_down: Optional[QTensor]     # [1][H][Is]
    shared_gate_w: Optional[torch.Tensor]  # bf16 [H]
    # The stock (unpacked) gate/up layout: when set, gate_up holds only the gate rows [E][I][H]
    # and up the up rows [E][I][H] (stock_layer); None in the packed layout.
    up: Optional[QTensor] = None
    shared_up: Optional[QTensor] = None


def _quantized_stack(n: int, rows: int, K: int, bits: int, group: int, seed: int, device,
                     chunk: int = 16, std: float = 0.02) -> QTensor:
    g = _gen(seed, device)
    q = torch.empty((n, rows, K * bits // 8), dtype=torch.uint8, device=device)
    s = torch.empty((n, rows, K // group), dtype=torch.bfloat16, device=device)
    b = torch.empty((n, rows, K // group), dtype=torch.bfloat16, device=device)
    for e0 in range(0, n, chunk):
        e1 = min(n, e0 + chunk)
        w = torch.randn((e1 - e0) * rows, K, generator=g, device=device) * std
        qq, ss, bb = quantize_groups(w, bits, group)
        q[e0:e1] = qq.reshape(e1 - e0, rows, -1)
        s[e0:e1] = ss.reshape(e1 - e0, rows, -1)
        b[e0:e1] = bb.reshape(e1 - e0, rows, -1)
        del w, qq, ss, bb
    return QTensor(q, s, b, rows, K)


def _split_rows(qt: QTensor, half: int) -> QTensor:
    """Rows [half*R/2, (half+1)*R/2) of every matrix of qt, as contiguous tensors of their own."""
    r = qt.rows // 2
    sl = slice(half * r, (half + 1) * r)
    return QTensor(qt.q[:, sl].contiguous(), qt.scales[:, sl].contiguous(), qt.biases[:, sl].contiguous(), r, qt.K)


def stock_layer(lw: LayerWeights) -> LayerWeights:
    """The same layer in the stock gate/up layout: the packed [2I][H] matrices split into
    separate gate [I][H] and up [I][H] tensors (new allocations; same codes, scales, biases)."""
    sg = lw.shared_gate_up
    return dataclasses.replace(lw, gate_up=_split_rows(lw.gate_up, 0), up=_split_rows(lw.gate_up, 1),
                               shared_gate_up=None if sg is None else _split_rows(sg, 0),
                               shared_up=None if sg is None else _split_rows(sg, 1))


def make_layer(shape: MoEShape, layer: int, device="cpu", seed_id: Optional[int] = None) -> LayerWeights:
    """Deterministic weights of one layer of `shape`, generated on `device`."""
    cid = SHAPE_SEED_ID.get(_key_of(shape), 0) if seed_id is None else seed_id
    H, E, I, Is = shape.hidden, shape.num_experts, shape.inter, shape.shared_inter
    gr = _gen(layer_seed(cid, layer, T_ROUTER), device)
    router = (torch.randn(E, H, generator=gr, device=device) * 0.02).to(torch.bfloat16)
    rbias = None
    if shape.router_bias:
        gb = _gen(layer_seed(cid, layer, T_RBIAS), device)
        rbias = torch.randn(E, generator=gb, device=device).float()
    gate_up = _quantized_stack(E, 2 * I, H, shape.bits, shape.group,
                               layer_seed(cid, layer, T_GATE_UP), device)
    down = _quantized_stack(E, H, I, shape.bits, shape.group,
                            layer_seed(cid, layer, T_DOWN), device)
    sh_gu = sh_dn = wsg = None
    if Is > 0:
        sh_gu = _quantized_stack(1, 2 * Is, H, shape.bits, shape.group,
                                 layer_seed(cid, layer, T_SH_GATE_UP), device)
        sh_dn = _quantized_stack(1, H, Is, shape.bits, shape.group,
                                 layer_seed(cid, layer, T_SH_DOWN), device)
        gw = _gen(layer_seed(cid, layer, T_WSG), device)
        wsg = (torch.randn(H, generator=gw, device=device) * 0.02).to(torch.bfloat16)
    return LayerWeights(router, rbias, gate_up, down, sh_gu, sh_dn, wsg)


def make_tokens(shape: MoEShape, ids: List[int], device="cpu", seed_id: Optional[int] = None) -> torch.Tensor:
    """Hidden states bf16 [len(ids)][H], token i drawn from its own seed."""
    cid = SHAPE_SEED_ID.get(_key_of(shape), 0) if seed_id is None else seed_id
    out = torch.empty(len(ids), shape.hidden, dtype=torch.bfloat16, device=device)
    for n, i in enumerate(ids):
        g = _gen(token_seed(cid, i), device)
        out[n] = torch.randn(shape.hidden, generator=g, device=device).to(torch.bfloat16)
    return out


def make_batch(shape: MoEShape, T: int, trial: int, device="cpu", seed_id: Optional[int] = None) -> torch.Tensor:
    """A batch of T hidden states for one trial (one seed per batch)."""
    cid = SHAPE_SEED_ID.get(_key_of(shape), 0) if seed_id is None else seed_id
    g = _gen(token_seed(cid, 1_000_000 + trial), device)
    return torch.randn(T, shape.hidden, generator=g, device=device).to(torch.bfloat16)


def _key_of(shape: MoEShape) -> str:
    for k, v in SHAPES.items():
        if v == shape:
            return k
    return ""


def bf16_bits(t: torch.Tensor):
    """The raw uint16 bit patterns of a bf16 tensor as a numpy array (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
