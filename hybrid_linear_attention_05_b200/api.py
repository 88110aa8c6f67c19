"""Tensor-level convenience calls over the C ABI.

``prefill`` and ``decode`` take torch CUDA tensors, allocate the outputs and
the workspace with torch, and call ``gdn_prefill`` / ``gdn_decode`` on the
current stream.  ``to_device`` moves a seeded workload (numpy arrays from
``workloads``) onto the GPU in the workload's dtype.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import gdn
from .workloads import DecodeInputs, PrefillInputs


def _torch_dtype(name: str):
    return torch.bfloat16 if name == "bf16" else torch.float32


@dataclass
class DevicePrefill:
    Hk: int
    Hv: int
    d: int
    chunk: int
    scale: float
    N: int
    T: int
    cu_seqlens: torch.Tensor
    mixed_qkv: torch.Tensor
    conv_w: torch.Tensor
    a: torch.Tensor
    b: torch.Tensor
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    z: torch.Tensor
    norm_w: torch.Tensor
    initial_state: Optional[torch.Tensor]
    conv_state_in: Optional[torch.Tensor]

    @property
    def dtype(self):
        return self.mixed_qkv.dtype

    @property
    def Cc(self):
        return 2 * self.Hk * self.d + self.Hv * self.d


def to_device(inp: PrefillInputs, device="cuda", chunk: Optional[int] = None) -> DevicePrefill:
    w = inp.w
    dt = _torch_dtype(w.dtype)

    def t(x, dtype=dt):
        return None if x is None else torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)

    return DevicePrefill(
        Hk=w.Hk, Hv=w.Hv, d=w.d, chunk=chunk or w.chunk, scale=w.scale, N=inp.N, T=inp.T,
        cu_seqlens=t(inp.cu_seqlens, torch.int32), mixed_qkv=t(inp.mixed_qkv), conv_w=t(inp.conv_w),
        a=t(inp.a), b=t(inp.b), A_log=t(inp.A_log, torch.float32),
        dt_bias=t(inp.dt_bias, torch.float32), z=t(inp.z), norm_w=t(inp.norm_w),
        initial_state=t(inp.initial_state, torch.float32), conv_state_in=t(inp.conv_state_in))


@dataclass
class PrefillOut:
    out: torch.Tensor            # [T, Hv, d]
    final_state: torch.Tensor    # [N, Hv, d, d] fp32
    conv_state_out: torch.Tensor  # [N, Cc, 3]


class PrefillBuffers:
    """Outputs and workspace for repeated prefill calls on one shape."""

    def __init__(self, dp: DevicePrefill):
        dev = dp.mixed_qkv.device
        self.dims = gdn.make_dims(dp.Hk, dp.Hv, dp.d, scale=dp.scale)
        self.dtype_code = gdn.dtype_code(dp.mixed_qkv)
        self.out = torch.empty((dp.T, dp.Hv, dp.d), dtype=dp.dtype, device=dev)
        self.final_state = torch.empty((dp.N, dp.Hv, dp.d, dp.d), dtype=torch.float32, device=dev)
        self.conv_state_out = torch.empty((dp.N, dp.Cc, 3), dtype=dp.dtype, device=dev)
        # room for every path, including the two-kernel tensor-core one
        self.ws_bytes = gdn.gdn_prefill_workspace_size_n(self.dims, dp.N, dp.T, self.dtype_code)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)


def prefill(dp: DevicePrefill, impl: int = gdn.GDN_IMPL_AUTO, bufs: Optional[PrefillBuffers] = None,
            core_events=None, segments: int = 0, reuse_workspace: bool = False) -> PrefillOut:
    """reuse_workspace: bufs.workspace holds a ``state_map`` of the same inputs
    (the conv and key-side kernels are skipped, conv_state_out is not written)."""
    bufs = bufs or PrefillBuffers(dp)
    ev0, ev1 = (None, None) if core_events is None else (core_events[0].cuda_event,
                                                         core_events[1].cuda_event)
    gdn.gdn_prefill(
        bufs.dims, mixed_qkv=dp.mixed_qkv, conv_w=dp.conv_w, a=dp.a, b=dp.b, A_log=dp.A_log,
        dt_bias=dp.dt_bias, z=dp.z, norm_w=dp.norm_w, cu_seqlens=dp.cu_seqlens, N=dp.N,
        T_tot=dp.T, chunk=dp.chunk, dtype=bufs.dtype_code, out=bufs.out,
        workspace=bufs.workspace, workspace_bytes=bufs.ws_bytes,
        initial_state=dp.initial_state, final_state=bufs.final_state,
        conv_state_in=dp.conv_state_in, conv_state_out=None if reuse_workspace else bufs.conv_state_out,
        impl=gdn.GDN_IMPL_TC_SPLIT if reuse_workspace else impl, core_event_begin=ev0, core_event_end=ev1,
        segments=segments, reuse_workspace=int(reuse_workspace))
    return PrefillOut(bufs.out, bufs.final_state, bufs.conv_state_out)


def state_map(dp: DevicePrefill, bufs: Optional[PrefillBuffers] = None, segments: int = 0,
              conv_state_out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """(M, R) of every sequence of dp as [N, Hv, 2, d, d] fp32: a start state S
    gives the final state S @ M + R (the initial state of dp is not used).
    bufs.workspace is left ready for ``prefill(dp, bufs=bufs, reuse_workspace=True)``."""
    bufs = bufs or PrefillBuffers(dp)
    maps = torch.empty((dp.N, dp.Hv, 2, dp.d, dp.d), dtype=torch.float32, device=dp.mixed_qkv.device)
    gdn.gdn_prefill_state_map(
        bufs.dims, mixed_qkv=dp.mixed_qkv, conv_w=dp.conv_w, a=dp.a, b=dp.b, A_log=dp.A_log,
        dt_bias=dp.dt_bias, cu_seqlens=dp.cu_seqlens, N=dp.N, T_tot=dp.T, chunk=dp.chunk,
        dtype=bufs.dtype_code, map_out=maps, workspace=bufs.workspace, workspace_bytes=bufs.ws_bytes,
        conv_state_in=dp.conv_state_in, conv_state_out=conv_state_out, z=dp.z, norm_w=dp.norm_w,
        segments=segments)
    return maps


def state_fold(maps: torch.Tensor, S_first: Optional[torch.Tensor], Hk: int, Hv: int, d: int,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Fold of maps [count, N, Hv, 2, d, d] from S_first [N, Hv, d, d] (None: zeros)."""
    count, N = int(maps.shape[0]), int(maps.shape[1])
    if out is None:
        out = torch.empty((N, Hv, d, d), dtype=torch.float32, device=maps.device)
    gdn.gdn_state_fold(gdn.make_dims(Hk, Hv, d), N=N, count=count, maps=maps.contiguous(),
                       S_out=out, S_first=S_first)
    return out


@dataclass
class DeviceDecode:
    Hk: int
    Hv: int
    d: int
    scale: float
    B: int
    mixed_qkv: torch.Tensor
    conv_w: torch.Tensor
    a: torch.Tensor
    b: torch.Tensor
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    z: torch.Tensor
    norm_w: torch.Tensor
    state: torch.Tensor
    conv_state: torch.Tensor


def decode_to_device(inp: DecodeInputs, device="cuda", state_dtype=torch.float32) -> DeviceDecode:
    """The decode inputs on the device; the state in `state_dtype` (fp32, or
    bf16 for the bf16-state step -- the caller rounds the state beforehand if
    it wants the device to hold exactly the values it has)."""
    w = inp.w
    dt = _torch_dtype(w.dtype)

    def t(x, dtype=dt):
        return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)

    return DeviceDecode(
        Hk=w.Hk, Hv=w.Hv, d=w.d, scale=w.scale, B=inp.mixed_qkv.shape[0],
        mixed_qkv=t(inp.mixed_qkv), conv_w=t(inp.conv_w), a=t(inp.a), b=t(inp.b),
        A_log=t(inp.A_log, torch.float32), dt_bias=t(inp.dt_bias, torch.float32), z=t(inp.z),
        norm_w=t(inp.norm_w), state=t(inp.state, state_dtype), conv_state=t(inp.conv_state))


def decode(dd: DeviceDecode, out: Optional[torch.Tensor] = None, T: int = 1) -> torch.Tensor:
    """One step of T tokens per sequence (token inputs [B, T, ...] when T > 1);
    dd.state and dd.conv_state are updated in place."""
    if out is None:
        shape = (dd.B, dd.Hv, dd.d) if T == 1 else (dd.B, T, dd.Hv, dd.d)
        out = torch.empty(shape, dtype=dd.mixed_qkv.dtype, device=dd.mixed_qkv.device)
    dims = gdn.make_dims(dd.Hk, dd.Hv, dd.d, scale=dd.scale)
    gdn.gdn_decode(dims, mixed_qkv=dd.mixed_qkv, conv_w=dd.conv_w, a=dd.a, b=dd.b,
                   A_log=dd.A_log, dt_bias=dd.dt_bias, z=dd.z, norm_w=dd.norm_w, state=dd.state,
                   conv_state=dd.conv_state, out=out, B=dd.B,
                   dtype=gdn.dtype_code(dd.mixed_qkv), state_dtype=gdn.dtype_code(dd.state), T=T)
    return out


def linear(x: torch.Tensor, w: torch.Tensor, splits=None):
    """y = x w^T on the tensor cores (bf16); with `splits` (column counts) the
    columns of y come back as separate tensors."""
    M, K = x.shape
    N = w.shape[0]
    splits = list(splits or [N])
    outs = [torch.empty((M, c), dtype=torch.bfloat16, device=x.device) for c in splits]
    gdn.gdn_linear(x=x, w=w, M=M, N=N, K=K, outs=[(o, c, c) for o, c in zip(outs, splits)])
    return outs if len(outs) > 1 else outs[0]


@dataclass
class DeviceLayer:
    mixer: DevicePrefill
    d_model: int
    hidden: torch.Tensor
    w_in: torch.Tensor
    w_out: torch.Tensor


def layer_to_device(li, device="cuda") -> DeviceLayer:
    dp = to_device(li.mixer, device=device)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=torch.bfloat16)  # noqa: E731
    return DeviceLayer(dp, li.d_model, t(li.hidden), t(li.w_in), t(li.w_out))


class LayerBuffers:
    def __init__(self, dl: DeviceLayer, records: bool = True):
        dp = dl.mixer
        dev = dl.hidden.device
        self.dims = gdn.make_dims(dp.Hk, dp.Hv, dp.d, scale=dp.scale)
        self.y = torch.empty((dp.T, dl.d_model), dtype=torch.bfloat16, device=dev)
        self.final_state = torch.empty((dp.N, dp.Hv, dp.d, dp.d), dtype=torch.float32, device=dev)
        self.conv_state_out = torch.empty((dp.N, dp.Cc, 3), dtype=torch.bfloat16, device=dev)
        if records:
            self.ws_bytes = gdn.gdn_layer_workspace_size(self.dims, dl.d_model, dp.N, dp.T)
        else:
            self.ws_bytes = (gdn.gdn_layer_activation_bytes(self.dims, dl.d_model, dp.T)
                             + gdn.gdn_prefill_workspace_size(self.dims, dp.T, gdn.GDN_BF16))
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)


def layer_prefill(dl: DeviceLayer, bufs: Optional[LayerBuffers] = None, impl: int = gdn.GDN_IMPL_AUTO):
    """The whole layer: in_proj, the mixer, out_proj (gdn_layer_prefill)."""
    dp = dl.mixer
    bufs = bufs or LayerBuffers(dl)
    gdn.gdn_layer_prefill(bufs.dims, hidden=dl.hidden, w_in=dl.w_in, w_out=dl.w_out, y=bufs.y,
                          d_model=dl.d_model, conv_w=dp.conv_w, A_log=dp.A_log, dt_bias=dp.dt_bias,
                          norm_w=dp.norm_w, cu_seqlens=dp.cu_seqlens, N=dp.N, T_tot=dp.T, chunk=dp.chunk,
                          workspace=bufs.workspace, workspace_bytes=bufs.ws_bytes,
                          initial_state=dp.initial_state, final_state=bufs.final_state,
                          conv_state_in=dp.conv_state_in, conv_state_out=bufs.conv_state_out, impl=impl)
    return bufs
