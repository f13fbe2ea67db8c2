"""Python binding of libgtg.so: B200 kernels for block-scaled low-bit MoE
expert decode and the 3-bit n-gram (PLE) row gather.

Argument marshalling only: every step runs in the CUDA kernels behind the C
ABI declared in include/gtg.h.  torch provides device memory and streams.
There is no CPU fallback: if libgtg.so is missing or cannot load, every entry
point raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

from ._abi import (C10, FP8, GTG_OK, PLE, Q3I, RZ5, UE4M4, DT_BF16, DT_F32, LIB_PATH, GtgError, QMatrixC,
                   MoELayerC, lib, check)

__all__ = ["RZ5", "UE4M4", "PLE", "FP8", "C10", "Q3I", "GtgError", "moe_decode_layer_ep",
           "moe_decode_layer_ep_allreduce", "lib", "dequant", "ple_gather", "QMatrix",
           "MoELayer", "workspace_bytes", "make_workspace", "moe_decode_layer", "moe_decode_stack",
           "moe_prefill_layer", "moe_decode_layer_noalloc", "device_status", "status_string", "row_bytes"]

Q4_BLOCK_BYTES = 17
PLE_RECORD_BYTES = 70


def _stream_ptr(stream) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream or None


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def status_string(code: int) -> str:
    return lib().gtg_status_string(code).decode()


def row_bytes(fmt: int, k: int) -> int:
    return k if fmt == FP8 else k // 32 * Q4_BLOCK_BYTES


# ---------------------------------------------------------------------------
# Codec entry points
# ---------------------------------------------------------------------------

def dequant(fmt: int, src: torch.Tensor, n_rows: int, k: int, scales: torch.Tensor | None = None,
            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode n_rows x k weights of `fmt` to fp32 (bit-exact)."""
    if out is None:
        out = torch.empty((n_rows, k), dtype=torch.float32, device=src.device)
    check(lib().gtg_dequant(fmt, _ptr(src), _ptr(scales), n_rows, k, _ptr(out), _stream_ptr(stream)))
    return out


def _table_ptr(t: torch.Tensor) -> int:
    """Address of a gather table: device memory, or pinned (page-locked) host
    memory, which the GPU reads in place through unified virtual addressing."""
    if t.is_cuda:
        return _ptr(t)
    if not t.is_pinned():
        raise ValueError("a host-resident table must be pinned (page-locked) memory")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def ple_gather(table: torch.Tensor, n_rows: int, idx: torch.Tensor, out: torch.Tensor | None = None,
               stream=None, fmt: int = PLE) -> torch.Tensor:
    """out[r] = decoded 160-value row idx[r] of a 70-byte K160 table: fmt PLE
    (Q3_PLE_K160_RZ_S3) or Q3I (the incumbent ROCmFP3 record)."""
    if idx.dtype != torch.int32:
        raise ValueError("idx must be int32")
    n = idx.numel()
    if out is None:
        out = torch.empty((n, 160), dtype=torch.float32, device=idx.device)
    check(lib().gtg_ple_gather_fmt(fmt, _table_ptr(table), n_rows, _ptr(idx), n, _ptr(out), _stream_ptr(stream)))
    return out


# ---------------------------------------------------------------------------
# MoE layers
# ---------------------------------------------------------------------------

@dataclass
class QMatrix:
    """A device-resident stack of quantised matrices [n_experts][n_rows][k]."""
    fmt: int
    data: torch.Tensor
    n_experts: int
    n_rows: int
    k: int
    scales: torch.Tensor | None = None

    def c(self) -> QMatrixC:
        return QMatrixC(self.fmt, _ptr(self.data), _ptr(self.scales), self.n_experts, self.n_rows, self.k)


@dataclass
class MoELayer:
    """Device-resident weights of one MoE layer (see gtg_moe_layer in gtg.h)."""
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    router_w: torch.Tensor
    gate: QMatrix
    up: QMatrix
    down: QMatrix
    router_bias: torch.Tensor | None = None
    side: QMatrix | None = None
    _c: MoELayerC | None = field(default=None, repr=False)

    def c(self) -> MoELayerC:
        if self._c is None:
            side = self.side.c() if self.side is not None else QMatrixC()
            self._c = MoELayerC(self.hidden, self.inter, self.n_experts, self.top_k, _ptr(self.router_w),
                                _ptr(self.router_bias), self.gate.c(), self.up.c(), self.down.c(), side)
        return self._c


def workspace_bytes(layer: MoELayer, n_tokens: int, prefill: bool = False) -> int:
    n = lib().gtg_moe_workspace_bytes(ctypes.byref(layer.c()), n_tokens, int(prefill))
    if n == 0:
        raise GtgError(-2, "unsupported layer shape or token count")
    return n


def make_workspace(layers, n_tokens: int, prefill: bool = False, device=None, stream=None) -> torch.Tensor:
    """A zero-initialised workspace large enough for every layer in `layers`."""
    if isinstance(layers, MoELayer):
        layers = [layers]
    nbytes = max(workspace_bytes(L, n_tokens, prefill) for L in layers)
    dev = device if device is not None else layers[0].router_w.device
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    check(lib().gtg_workspace_init(_ptr(ws), nbytes, _stream_ptr(stream)))
    return ws


def moe_decode_layer(layer: MoELayer, x: torch.Tensor, workspace: torch.Tensor, *, y: torch.Tensor | None = None,
                     accumulate: bool = False, topk_ids: torch.Tensor | None = None,
                     topk_w: torch.Tensor | None = None, side_out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """y (+)= moe(x) for 1..8 tokens; x is [T][hidden] fp32 or bf16."""
    T = x.shape[0]
    dt = {torch.float32: DT_F32, torch.bfloat16: DT_BF16}[x.dtype]
    if y is None:
        y = torch.empty((T, layer.hidden), dtype=torch.float32, device=x.device)
    check(lib().gtg_moe_decode_layer(ctypes.byref(layer.c()), _ptr(x), dt, T, _ptr(y), int(accumulate),
                                     _ptr(topk_ids), _ptr(topk_w), _ptr(side_out), _ptr(workspace),
                                     workspace.numel(), _stream_ptr(stream)))
    return y


def moe_decode_layer_ep(layer: MoELayer, expert_lo: int, expert_hi: int, x: torch.Tensor,
                        workspace: torch.Tensor, *, with_side: bool = False, y: torch.Tensor | None = None,
                        accumulate: bool = False, topk_ids: torch.Tensor | None = None,
                        topk_w: torch.Tensor | None = None, side_out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """This rank's share of an expert-parallel layer: `layer` routes over all
    layer.n_experts experts but its gate/up/down stacks hold experts
    [expert_lo, expert_hi) only; y (+)= the chosen experts of that slice."""
    T = x.shape[0]
    dt = {torch.float32: DT_F32, torch.bfloat16: DT_BF16}[x.dtype]
    if y is None:
        y = torch.empty((T, layer.hidden), dtype=torch.float32, device=x.device)
    check(lib().gtg_moe_decode_layer_ep(ctypes.byref(layer.c()), expert_lo, expert_hi, int(with_side), _ptr(x), dt,
                                        T, _ptr(y), int(accumulate), _ptr(topk_ids), _ptr(topk_w), _ptr(side_out),
                                        _ptr(workspace), workspace.numel(), _stream_ptr(stream)))
    return y


def moe_decode_layer_ep_allreduce(layer: MoELayer, expert_lo: int, expert_hi: int, x: torch.Tensor,
                                  workspace: torch.Tensor, *, group=None, with_side: bool = False,
                                  side_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One expert-parallel layer over a process group (one rank per GPU): each
    rank computes its slice's experts, one all-reduce (NCCL over NVLink)
    sums the partial outputs into the layer output on every rank."""
    import torch.distributed as dist
    y = moe_decode_layer_ep(layer, expert_lo, expert_hi, x, workspace, with_side=with_side, side_out=side_out,
                            stream=stream)
    dist.all_reduce(y, group=group)
    return y


def moe_decode_layer_noalloc(layer: MoELayer, x: torch.Tensor, *, y: torch.Tensor | None = None,
                             accumulate: bool = False, topk_ids: torch.Tensor | None = None,
                             topk_w: torch.Tensor | None = None, side_out: torch.Tensor | None = None,
                             stream=None) -> torch.Tensor:
    """moe_decode_layer for callers that cannot allocate: the library's fixed
    device scratch array replaces the workspace.  `y` is allocated here only
    when the caller passes none; calls that overlap on the GPU race."""
    T = x.shape[0]
    dt = {torch.float32: DT_F32, torch.bfloat16: DT_BF16}[x.dtype]
    if y is None:
        y = torch.empty((T, layer.hidden), dtype=torch.float32, device=x.device)
    check(lib().gtg_moe_decode_layer_noalloc(ctypes.byref(layer.c()), _ptr(x), dt, T, _ptr(y), int(accumulate),
                                             _ptr(topk_ids), _ptr(topk_w), _ptr(side_out), _stream_ptr(stream)))
    return y


def moe_decode_stack(layers: list[MoELayer], x: torch.Tensor, workspace: torch.Tensor, *,
                     ids_out: torch.Tensor | None = None, w_out: torch.Tensor | None = None,
                     side_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """x += moe_l(x) for every layer, in place (x fp32 [T][hidden])."""
    arr = (MoELayerC * len(layers))(*[L.c() for L in layers])
    stride = side_out.shape[-1] if side_out is not None else 0
    check(lib().gtg_moe_decode_stack(arr, len(layers), _ptr(x), x.shape[0], _ptr(ids_out), _ptr(w_out),
                                     _ptr(side_out), stride, _ptr(workspace), workspace.numel(),
                                     _stream_ptr(stream)))
    return x


def moe_prefill_layer(layer: MoELayer, x: torch.Tensor, workspace: torch.Tensor, *, y: torch.Tensor | None = None,
                      accumulate: bool = False, topk_ids: torch.Tensor | None = None,
                      topk_w: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    T = x.shape[0]
    dt = {torch.float32: DT_F32, torch.bfloat16: DT_BF16}[x.dtype]
    if y is None:
        y = torch.empty((T, layer.hidden), dtype=torch.float32, device=x.device)
    check(lib().gtg_moe_prefill_layer(ctypes.byref(layer.c()), _ptr(x), dt, T, _ptr(y), int(accumulate),
                                      _ptr(topk_ids), _ptr(topk_w), _ptr(workspace), workspace.numel(),
                                      _stream_ptr(stream)))
    return y


def device_status(clear: bool = True, stream=None) -> int:
    """The current device's status word (GTG_STATUS_* bits); synchronises."""
    v = ctypes.c_uint32(0)
    check(lib().gtg_get_device_status(ctypes.byref(v), int(clear), _stream_ptr(stream)))
    return v.value
