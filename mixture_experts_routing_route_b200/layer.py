"""MoeLayer: a user-facing handle around the C ABI's whole-layer forward.

Holds the layer's device weights and a workspace (device memory allocated by
torch: plumbing only), fills the C layer struct, and calls moe_forward /
moe_forward_host. Intermediates of the last forward can be read as torch views
of the workspace.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _abi as abi


class MoeLayer:
    def __init__(self, w_router: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor,
                 w3: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None,
                 k: int = 2, act: str = "swiglu", capacity_factor: float = 0.0,
                 gather_in_gemm: bool = False, binned: bool = False, z_loss: bool = False,
                 combine_in_gemm: bool = False, router_temperature: float = 1.0):
        if not w1.is_cuda:
            raise ValueError("weights must be CUDA tensors")
        self.E, self.d, self.F = w1.shape
        self.k = k
        self.dtype = w1.dtype
        self.act = abi.MOE_ACT_SWIGLU if act == "swiglu" else abi.MOE_ACT_GELU
        self.cf = float(capacity_factor)
        self.w_router = w_router.contiguous()
        self.w1 = w1.contiguous()
        self.w3 = None if w3 is None else w3.contiguous()
        self.w2 = w2.contiguous()
        self.bias = None if bias is None else bias.to(device=w1.device, dtype=torch.float32).contiguous()
        # gather_in_gemm: the up projection gathers x rows itself (bf16; see
        # MOE_LAYER_GATHER_IN_GEMM in include/moe_b200.h)
        # binned: the [E, C, hs] bucket layout (MOE_LAYER_BINNED); with
        # capacity_factor <= 0 the bin size is the call's largest expert count
        # combine_in_gemm: k = 1, bf16: the down projection scales its rows by
        # the top-k weight and writes out (MOE_LAYER_COMBINE_IN_GEMM)
        flags = (abi.MOE_LAYER_GATHER_IN_GEMM if gather_in_gemm else 0) | \
            (abi.MOE_LAYER_BINNED if binned else 0) | (abi.MOE_LAYER_Z_LOSS if z_loss else 0) | \
            (abi.MOE_LAYER_COMBINE_IN_GEMM if combine_in_gemm else 0)
        # router_temperature: the router softmax sees logits / tau (training
        # variant; moe_route_train in include/moe_b200.h)
        self.c = abi.layer_struct(self.d, self.E, k, self.F, abi.dtype_code(self.dtype), self.act,
                                  self.cf, self.w_router, self.bias, self.w1, self.w3, self.w2,
                                  flags, router_temperature)
        self._ws = {}

    def workspace(self, T: int, host_io: bool = False, stream=None, slot: int = 0) -> torch.Tensor:
        """The device workspace for T tokens; `slot` keeps separate ones for
        calls that may run at the same time on different streams."""
        key = (T, host_io, slot)
        if key not in self._ws:
            n = (abi.moe_forward_host_workspace_size(self.c, T) if host_io
                 else abi.moe_forward_workspace_size(self.c, T))
            ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.w1.device)
            abi.moe_workspace_init(ws, stream)
            self._ws[key] = ws
        return self._ws[key]

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                aux: Optional[torch.Tensor] = None, stream=None, events=None,
                x_router: Optional[torch.Tensor] = None,
                logit_noise: Optional[torch.Tensor] = None):
        """x_router: the router's own input (e.g. moe_router_jitter of x);
        logit_noise: [T, E] fp32 added to the gate logits (training variants)."""
        T = x.shape[0]
        self.c.x_router = None if x_router is None else x_router.data_ptr()
        self.c.logit_noise = None if logit_noise is None else logit_noise.data_ptr()
        if out is None:
            out = torch.empty(T, self.d, dtype=self.dtype, device=x.device)
        if aux is None:
            aux = torch.empty(1, dtype=torch.float32, device=x.device)
        ws = self.workspace(T, stream=stream)
        abi.moe_forward(self.c, x, T, out, aux, ws, stream, events)
        return out, aux

    __call__ = forward

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor, aux_host: torch.Tensor,
                     stream=None, slot: int = 0):
        """Pinned host x in, pinned host out and aux back, all asynchronous on
        `stream`. Calls that overlap (double-buffered serving on two streams)
        pass different `slot`s so they use different workspaces."""
        T = x_host.shape[0]
        self.c.x_router = None
        self.c.logit_noise = None
        ws = self.workspace(T, host_io=True, stream=stream, slot=slot)
        abi.moe_forward_host(self.c, x_host, T, out_host, aux_host, ws, stream)

    def device_error(self, T: int, stream=None) -> int:
        return abi.moe_get_device_error(self.workspace(T, stream=stream), stream)

    def views(self, T: int) -> dict:
        """Torch views of the intermediates moe_forward left in the workspace."""
        ws = self.workspace(T)
        v = abi.moe_forward_views(self.c, T, ws)
        base = ws.data_ptr()
        R = v.rows_max
        S = T * self.k

        def view(ptr, n, dt, shape):
            es = torch.empty(0, dtype=dt).element_size()
            off = ptr - base
            return ws[off:off + n * es].view(dt).view(*shape)

        return {
            "topk_idx": view(v.topk_idx, S, torch.int32, (T, self.k)),
            "topk_w": view(v.topk_w, S, torch.float32, (T, self.k)),
            "aux": view(v.aux_loss, 1, torch.float32, (1,)),
            "z_loss": view(v.z_loss, 1, torch.float32, (1,)),
            "counts": view(v.counts, self.E, torch.int32, (self.E,)),
            "bins": view(v.bins, self.E, torch.int32, (self.E,)),
            "kept_counts": view(v.kept_counts, self.E, torch.int32, (self.E,)),
            "seg_offsets": view(v.seg_offsets, self.E + 1, torch.int32, (self.E + 1,)),
            "sorted_slot": view(v.sorted_slot, S, torch.int32, (S,)),
            "slot_to_row": view(v.slot_to_row, S, torch.int32, (S,)),
            "row_slot": view(v.row_slot, R, torch.int32, (R,)),
            "drop": view(v.drop_mask, S, torch.uint8, (S,)),
            # no x_perm when the up projection gathers x rows itself
            "x_perm": view(v.x_perm, R * self.d, self.dtype, (R, self.d)) if v.x_perm else None,
            "h": view(v.h, R * self.F, self.dtype, (R, self.F)),
            # no y_perm when the down projection writes the output itself
            "y_perm": view(v.y_perm, R * self.d, self.dtype, (R, self.d)) if v.y_perm else None,
            "rows_max": R,
            "capacity": v.capacity,
        }
