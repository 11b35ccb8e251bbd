"""Route-layer / sliding-window attention through librdl, with torch-owned buffers.

This layer only allocates buffers (torch) and sequences the C-ABI calls; every step of the
computation runs in the CUDA library:

    summary_pool   -> s [B,Hq,C,d] f32, H [B,Hq,C] f32 (+ mask-slot rows of o)
    score_topk     -> idx [B,Hkv,Lq,K] i32, z_sel [B,Hq,Lq,K] f32
    route_attn     -> o [B,Lq,Hq,d], lse [B,Hq,Lq]
    swa_attn       -> o, lse of a sliding-window layer
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

from . import rdl
from .workloads import Workload

CHUNK = rdl.CHUNK


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def from_numpy(a: np.ndarray, dtype: str, device) -> torch.Tensor:
    """A workload array (uint16 bf16 bits or float32) as a torch tensor on `device`."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.int16).view(torch.bfloat16)
    elif a.dtype == np.float32 and dtype == "bf16":
        raise ValueError("float32 array for a bf16 workload")
    return t.to(device)


@dataclass
class DeviceInputs:
    dims: rdl.Dims
    dtype: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    x: torch.Tensor
    w_down: torch.Tensor
    w_up: torch.Tensor
    q_pos: Optional[torch.Tensor]
    q_mask: Optional[torch.Tensor]      # separate mask-slot queries (decode); None: rows of q

    @property
    def prefill(self) -> bool:
        return self.q_pos is None


def to_device(wl: Workload, device="cuda") -> DeviceInputs:
    dm = wl.dims
    f = lambda a: from_numpy(a, dm.dtype, device)  # noqa: E731
    q_pos = None if wl.q_pos is None else torch.from_numpy(wl.q_pos.astype(np.int32)).to(device)
    q_mask = None if wl.q_pos is None else f(wl.q_mask)
    return DeviceInputs(rdl.Dims.of(dm), dm.dtype, f(wl.q), f(wl.k), f(wl.v), f(wl.x),
                        f(wl.w_down), f(wl.w_up), q_pos, q_mask)


def mask_query_view(inp: DeviceInputs):
    """(pointer, chunk stride, batch stride) of the mask-slot query rows, in elements."""
    dm = inp.dims
    row = dm.Hq * dm.d
    if inp.q_mask is None:
        es = inp.q.element_size()
        return inp.q.data_ptr() + (CHUNK - 1) * row * es, CHUNK * row, dm.L * row
    C = dm.L // CHUNK
    return inp.q_mask.data_ptr(), row, C * row


@dataclass
class Outputs:
    s: torch.Tensor
    H: torch.Tensor
    idx: torch.Tensor
    z_sel: torch.Tensor
    o: torch.Tensor
    lse: torch.Tensor
    ws_score: torch.Tensor
    ws_attn: torch.Tensor
    ws_swa: torch.Tensor
    extra: dict = field(default_factory=dict)


def alloc_outputs(dims: rdl.Dims, dtype: str, device="cuda") -> Outputs:
    C = dims.L // CHUNK
    dev = torch.device(device)
    ws_s = rdl.workspace_bytes(rdl.WS_SCORE, dims, dtype)
    ws_a = rdl.workspace_bytes(rdl.WS_ATTN, dims, dtype)
    ws_w = rdl.workspace_bytes(rdl.WS_SWA, dims, dtype)
    return Outputs(
        s=torch.empty(dims.B, dims.Hq, C, dims.d, dtype=torch.float32, device=dev),
        H=torch.empty(dims.B, dims.Hq, C, dtype=torch.float32, device=dev),
        idx=torch.empty(dims.B, dims.Hkv, dims.Lq, dims.K, dtype=torch.int32, device=dev),
        z_sel=torch.empty(dims.B, dims.Hq, dims.Lq, dims.K, dtype=torch.float32, device=dev),
        o=torch.zeros(dims.B, dims.Lq, dims.Hq, dims.d, dtype=torch_dtype(dtype), device=dev),
        lse=torch.full((dims.B, dims.Hq, dims.Lq), float("nan"), dtype=torch.float32, device=dev),
        ws_score=torch.empty(max(ws_s, 256), dtype=torch.uint8, device=dev),
        ws_attn=torch.empty(max(ws_a, 256), dtype=torch.uint8, device=dev),
        ws_swa=torch.empty(max(ws_w, 256), dtype=torch.uint8, device=dev),
    )


def summary_pool(inp: DeviceInputs, out: Outputs, *, write_mask_rows=True, stream=None):
    ptr, cs, bs = mask_query_view(inp)
    o_mask = None
    if write_mask_rows and inp.prefill:
        o_mask = out.o.data_ptr() + (CHUNK - 1) * inp.dims.Hq * inp.dims.d * out.o.element_size()
    rdl.rdl_summary_pool(ptr, cs, bs, inp.k, inp.v if o_mask else None, inp.dims, inp.dtype,
                         out.s, out.H, o_mask, stream=stream)


def score_topk(inp: DeviceInputs, out: Outputs, stream=None):
    rdl.rdl_route_score_topk(inp.q, inp.q_pos, inp.x, inp.w_down, inp.w_up, out.s, out.H,
                             inp.dims, inp.dtype, out.idx, out.z_sel, out.ws_score, stream=stream)


def route_attn(inp: DeviceInputs, out: Outputs, stream=None):
    rdl.rdl_route_attn(inp.q, inp.q_pos, inp.k, inp.v, out.idx, out.z_sel, inp.dims, inp.dtype,
                       out.o, out.lse, out.ws_attn, stream=stream)


def swa_attn(inp: DeviceInputs, out: Outputs, stream=None):
    rdl.rdl_swa_attn(inp.q, inp.q_pos, inp.k, inp.v, inp.dims, inp.dtype, out.o, out.lse,
                     out.ws_swa, stream=stream)


def route_layer(inp: DeviceInputs, out: Outputs, *, with_summary=True, stream=None):
    """One route layer: summaries (prefill), scores + top-K, two-level attention."""
    if with_summary:
        summary_pool(inp, out, stream=stream)
    score_topk(inp, out, stream=stream)
    route_attn(inp, out, stream=stream)
    return out
