"""Python binding of libmoe_b200.so (include/moe_b200.h): argument
marshalling only. Every step of the layer runs in the library's CUDA
kernels; torch tensors are used for device memory and streams.

The functions keep the C names (moe_route_topk, moe_expert_ffn,
moe_layer_forward, moe_stack_forward, moe_sort_by_expert, ...), take torch
CUDA tensors in place of pointers, run on the current torch stream unless
one is given, and raise MoEError on a non-OK status.
"""

from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
_lib = None

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, \
    MOE_ERR_BOUNDS = range(7)

P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{status_string(status)}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("hidden", I32), ("num_experts", I32), ("top_k", I32), ("inter", I32),
                ("shared_inter", I32), ("bits", I32), ("group", I32), ("renorm", I32)]


class QTensor(ctypes.Structure):
    _fields_ = [("q", P), ("scales", P), ("biases", P), ("q_expert_stride", I64), ("sb_expert_stride", I64)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("router_w", P), ("router_bias", P), ("gate_up", QTensor), ("down", QTensor),
                ("shared_gate_up", QTensor), ("shared_down", QTensor), ("shared_gate_w", P),
                ("down_sb", P), ("shared_down_sb", P), ("down_units", P), ("shared_down_units", P),
                ("up", QTensor), ("shared_up", QTensor)]


class Trace(ctypes.Structure):
    _fields_ = [("x", P), ("idx", P), ("w", P), ("y", P), ("t", P)]


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m quantized_routed_expert_bit_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        CP, LP = ctypes.POINTER(Config), ctypes.POINTER(LayerWeights)
        L.moe_workspace_size.argtypes = [CP, I32, I32]
        L.moe_workspace_size.restype = ctypes.c_size_t
        L.moe_workspace_init.argtypes = [P, ctypes.c_size_t, P]
        L.moe_route_topk.argtypes = [CP, P, I32, P, P, P, P, P, ctypes.c_size_t, P]
        L.moe_expert_ffn.argtypes = [CP, LP, P, I32, P, P, P, P, ctypes.c_size_t, P]
        L.moe_layer_forward.argtypes = [CP, LP, P, I32, P, P, P, P, ctypes.c_size_t, P]
        L.moe_stack_forward.argtypes = [CP, LP, I32, P, I32, P, ctypes.POINTER(Trace), P, ctypes.c_size_t, P]
        L.moe_sort_by_expert.argtypes = [CP, P, I32, P, P, P, ctypes.c_size_t, P]
        L.moe_layer_forward_static.argtypes = [CP, LP, P, I32, P, P, P, P, P]
        L.moe_down_sb_size.argtypes = [CP, I32, I32]
        L.moe_down_sb_size.restype = ctypes.c_size_t
        L.moe_prepare_down_sb.argtypes = [CP, ctypes.POINTER(QTensor), I32, I32, P, P]
        L.moe_down_units_size.argtypes = [CP, I32, I32]
        L.moe_down_units_size.restype = ctypes.c_size_t
        L.moe_prepare_down_units.argtypes = [CP, ctypes.POINTER(QTensor), I32, I32, P, P]
        L.moe_set_batched_min_tokens.argtypes = [I32]
        L.moe_set_batched_min_tokens.restype = I32
        L.moe_set_gemv_min_tokens.argtypes = [I32]
        L.moe_set_gemv_min_tokens.restype = I32
        L.moe_set_decode_max_tokens.argtypes = [I32]
        L.moe_set_decode_max_tokens.restype = I32
        L.moe_stack_kernel_launches.argtypes = [CP, I32, I32]
        L.moe_stack_kernel_launches.restype = I32
        L.moe_stack_path_name.argtypes = [CP, I32, I32]
        L.moe_stack_path_name.restype = ctypes.c_char_p
        L.moe_get_device_status.argtypes = [P, P]
        L.moe_check_wait_limit.argtypes = [P, ctypes.c_size_t, P, P]
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_last_error_string.argtypes = []
        L.moe_last_error_string.restype = ctypes.c_char_p
        for f in ("moe_workspace_init", "moe_route_topk", "moe_expert_ffn", "moe_layer_forward",
                  "moe_stack_forward", "moe_sort_by_expert", "moe_get_device_status",
                  "moe_layer_forward_static", "moe_check_wait_limit"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().moe_status_string(int(s)).decode()


def last_error() -> str:
    return lib().moe_last_error_string().decode()


def _check(s: int):
    if s != MOE_OK:
        raise MoEError(s, last_error())


def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


# ---------------------------------------------------------------- structs from tensors


def make_config(shape, renorm: int = 1) -> Config:
    return Config(shape.hidden, shape.num_experts, shape.top_k, shape.inter, shape.shared_inter,
                  shape.bits, shape.group, renorm)


def _qtensor(qt) -> QTensor:
    if qt is None:
        return QTensor(None, None, None, 0, 0)
    return QTensor(qt.q.data_ptr(), qt.scales.data_ptr(), qt.biases.data_ptr(),
                   qt.q.stride(0) * qt.q.element_size(), qt.scales.stride(0))


def moe_down_sb_size(cfg: Config, n_experts: int, K: int) -> int:
    return int(lib().moe_down_sb_size(ctypes.byref(cfg), int(n_experts), int(K)))


def moe_prepare_down_sb(cfg: Config, qt, out: torch.Tensor, stream=None):
    """Group-major (scale, bias) copy of a down tensor (synth.QTensor [n][H][K]) into out
    (uint8 device tensor of moe_down_sb_size bytes)."""
    n, K = qt.q.shape[0], qt.K
    if out.numel() * out.element_size() < moe_down_sb_size(cfg, n, K):
        raise MoEError(MOE_ERR_INVALID_ARG, "out is smaller than moe_down_sb_size")
    q = _qtensor(qt)
    _check(lib().moe_prepare_down_sb(ctypes.byref(cfg), ctypes.byref(q), n, K, out.data_ptr(), _stream(stream)))


def moe_down_units_size(cfg: Config, n_experts: int, K: int) -> int:
    return int(lib().moe_down_units_size(ctypes.byref(cfg), int(n_experts), int(K)))


def moe_prepare_down_units(cfg: Config, qt, out: torch.Tensor, stream=None):
    """Unit-major copy of a down tensor's codes (synth.QTensor [n][H][K]) into out
    (uint8 device tensor of moe_down_units_size bytes)."""
    n, K = qt.q.shape[0], qt.K
    if out.numel() * out.element_size() < moe_down_units_size(cfg, n, K):
        raise MoEError(MOE_ERR_INVALID_ARG, "out is smaller than moe_down_units_size")
    q = _qtensor(qt)
    _check(lib().moe_prepare_down_units(ctypes.byref(cfg), ctypes.byref(q), n, K, out.data_ptr(), _stream(stream)))


def prepare_layer(cfg: Config, lw):
    """The decode-ready down copies of a layer on the GPU (made once, kept on lw):
    (down_sb, shared_down_sb, down_units, shared_down_units) as uint8 device tensors
    (the shared ones None without a shared expert)."""
    got = lw.__dict__.get("_decode_copies")
    if got is None:
        dev = lw.down.q.device
        n, K = lw.down.q.shape[0], lw.down.K
        dsb = torch.empty(moe_down_sb_size(cfg, n, K), dtype=torch.uint8, device=dev)
        moe_prepare_down_sb(cfg, lw.down, dsb)
        dcu = torch.empty(moe_down_units_size(cfg, n, K), dtype=torch.uint8, device=dev)
        moe_prepare_down_units(cfg, lw.down, dcu)
        sdsb = sdcu = None
        if lw.shared_down is not None and cfg.shared_inter > 0:
            sdsb = torch.empty(moe_down_sb_size(cfg, 1, lw.shared_down.K), dtype=torch.uint8, device=dev)
            moe_prepare_down_sb(cfg, lw.shared_down, sdsb)
            sdcu = torch.empty(moe_down_units_size(cfg, 1, lw.shared_down.K), dtype=torch.uint8, device=dev)
            moe_prepare_down_units(cfg, lw.shared_down, sdcu)
        got = (dsb, sdsb, dcu, sdcu)
        lw.__dict__["_decode_copies"] = got
    return got


def make_layer_weights(lw, cfg: Optional[Config] = None) -> LayerWeights:
    """LayerWeights struct over a synth.LayerWeights (the caller keeps lw alive). With cfg
    given, the weights on the GPU and a shape that decode_split_kernel runs, the decode-ready
    down copies that kernel reads (unit-major codes, group-major scales and biases) are made
    once (prepare_layer) and referenced too."""
    dsb = sdsb = dcu = sdcu = None
    if cfg is not None and lw.down.q.is_cuda and split_decode(cfg):
        dsb, sdsb, dcu, sdcu = prepare_layer(cfg, lw)
    up = getattr(lw, "up", None)  # the stock gate/up layout (synth.stock_layer)
    shared_up = getattr(lw, "shared_up", None)
    return LayerWeights(lw.router_w.data_ptr(), _p(lw.router_bias), _qtensor(lw.gate_up), _qtensor(lw.down),
                        _qtensor(lw.shared_gate_up), _qtensor(lw.shared_down), _p(lw.shared_gate_w),
                        _p(dsb), _p(sdsb), _p(dcu), _p(sdcu), _qtensor(up), _qtensor(shared_up))


def split_decode(cfg: Config) -> bool:
    """Whether one token through a stack of this shape runs decode_split_kernel on the current
    device: the only reader of the decode-ready copies, made only then."""
    return moe_stack_path_name(cfg, 1, 1) == "decode_split_kernel"


class Workspace:
    """Caller-owned scratch for the library: a torch byte tensor, initialised once."""

    def __init__(self, cfg: Config, T: int, device="cuda", L: int = 1, stream=None):
        n = lib().moe_workspace_size(ctypes.byref(cfg), int(max(T, 1)), int(L))
        if n == 0:
            raise MoEError(MOE_ERR_UNSUPPORTED, last_error())
        self.buf = torch.empty(n + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.tensor = self.buf[off:off + n]
        self.nbytes = n
        _check(lib().moe_workspace_init(self.ptr, n, _stream(stream)))

    @property
    def ptr(self) -> int:
        return self.tensor.data_ptr()


# ---------------------------------------------------------------- entry points


def moe_workspace_size(cfg: Config, T: int, L: int = 1) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(cfg), int(T), int(L)))


def moe_route_topk(cfg: Config, x: torch.Tensor, router_w: torch.Tensor, router_bias: Optional[torch.Tensor],
                   topk_idx: torch.Tensor, topk_w: torch.Tensor, ws: Workspace, stream=None):
    _check(lib().moe_route_topk(ctypes.byref(cfg), x.data_ptr(), x.shape[0], router_w.data_ptr(),
                                _p(router_bias), topk_idx.data_ptr(), topk_w.data_ptr(), ws.ptr, ws.nbytes,
                                _stream(stream)))


def moe_expert_ffn(cfg: Config, w: LayerWeights, x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor,
                   y: torch.Tensor, ws: Workspace, stream=None):
    _check(lib().moe_expert_ffn(ctypes.byref(cfg), ctypes.byref(w), x.data_ptr(), x.shape[0],
                                topk_idx.data_ptr(), topk_w.data_ptr(), y.data_ptr(), ws.ptr, ws.nbytes,
                                _stream(stream)))


def moe_layer_forward(cfg: Config, w: LayerWeights, x: torch.Tensor, y: torch.Tensor,
                      topk_idx: Optional[torch.Tensor], topk_w: Optional[torch.Tensor], ws: Workspace,
                      stream=None):
    _check(lib().moe_layer_forward(ctypes.byref(cfg), ctypes.byref(w), x.data_ptr(), x.shape[0], y.data_ptr(),
                                   _p(topk_idx), _p(topk_w), ws.ptr, ws.nbytes, _stream(stream)))


def moe_layer_forward_static(cfg: Config, w: LayerWeights, x: torch.Tensor, y: torch.Tensor,
                             topk_idx: Optional[torch.Tensor], topk_w: Optional[torch.Tensor],
                             device_status: Optional[torch.Tensor] = None, stream=None):
    """moe_layer_forward with the library's fixed scratch instead of a workspace."""
    _check(lib().moe_layer_forward_static(ctypes.byref(cfg), ctypes.byref(w), x.data_ptr(), x.shape[0],
                                          y.data_ptr(), _p(topk_idx), _p(topk_w), _p(device_status),
                                          _stream(stream)))


def make_layer_array(layers: Sequence[LayerWeights]):
    arr = (LayerWeights * len(layers))(*layers)
    return arr


def moe_stack_forward(cfg: Config, layers, x0: torch.Tensor, x_out: torch.Tensor, ws: Workspace,
                      trace: Optional[Trace] = None, stream=None):
    """layers: a ctypes array from make_layer_array (host array of LayerWeights)."""
    _check(lib().moe_stack_forward(ctypes.byref(cfg), layers, len(layers), x0.data_ptr(), x0.shape[0],
                                   x_out.data_ptr(), ctypes.byref(trace) if trace is not None else None,
                                   ws.ptr, ws.nbytes, _stream(stream)))


def moe_sort_by_expert(cfg: Config, topk_idx: torch.Tensor, perm: torch.Tensor, offsets: torch.Tensor,
                       ws: Workspace, stream=None):
    _check(lib().moe_sort_by_expert(ctypes.byref(cfg), topk_idx.data_ptr(), topk_idx.shape[0], perm.data_ptr(),
                                    offsets.data_ptr(), ws.ptr, ws.nbytes, _stream(stream)))


def moe_get_device_status(ws: Workspace, stream=None) -> int:
    return int(lib().moe_get_device_status(ws.ptr, _stream(stream)))


def moe_check_wait_limit(ws: Workspace, gave_up: torch.Tensor, stream=None):
    """Runs the bounded-wait self-check (about 2 s on the GPU); gave_up is a device int32 [1]."""
    _check(lib().moe_check_wait_limit(ws.ptr, ws.nbytes, gave_up.data_ptr(), _stream(stream)))


# ---------------------------------------------------------------- launch plan (for reporting)


def moe_stack_kernel_launches(cfg: Config, T: int, L: int) -> int:
    """Kernels one moe_stack_forward call launches on the current device."""
    return int(lib().moe_stack_kernel_launches(ctypes.byref(cfg), int(T), int(L)))


def moe_set_batched_min_tokens(T: int) -> int:
    """Token count from which the batched tensor-core path runs (process-wide); T < 1 restores
    the default. Returns the previous value."""
    return int(lib().moe_set_batched_min_tokens(int(T)))


def moe_set_gemv_min_tokens(T: int) -> int:
    """Token count from which the grouped GEMV path runs (process-wide); T < 1 restores the
    default. Returns the previous value."""
    return int(lib().moe_set_gemv_min_tokens(int(T)))


def moe_set_decode_max_tokens(T: int) -> int:
    """Token count up to which moe_stack_forward runs its tokens one at a time through the
    single-token persistent kernel (process-wide); T < 1 restores the default. Returns the
    previous value."""
    return int(lib().moe_set_decode_max_tokens(int(T)))


def moe_stack_path_name(cfg: Config, T: int, L: int) -> Optional[str]:
    """The path one moe_stack_forward call takes on the current device (None on a bad configuration)."""
    name = lib().moe_stack_path_name(ctypes.byref(cfg), int(T), int(L))
    return None if name is None else name.decode()
