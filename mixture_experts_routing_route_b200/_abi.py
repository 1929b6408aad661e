"""ctypes binding of libmoe_b200.so: the C entry points under the same names.

Argument marshalling only. Tensors are passed as their device addresses,
shapes as ints, the stream as torch's current CUDA stream unless given. Every
step of the layer runs in the library's CUDA kernels; there is no fallback:
if the library is missing or cannot load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG), "include", "moe_b200.h")

MOE_OK = 0
STATUS = {0: "MOE_OK", 1: "MOE_ERR_NULL", 2: "MOE_ERR_INVALID", 3: "MOE_ERR_UNSUPPORTED",
          4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_ALIGN", 6: "MOE_ERR_CUDA", 7: "MOE_ERR_DEVICE"}
MOE_F32, MOE_BF16 = 0, 1
MOE_ACT_GELU, MOE_ACT_SWIGLU = 0, 1
MOE_LAYER_GATHER_IN_GEMM, MOE_LAYER_BINNED, MOE_LAYER_Z_LOSS, MOE_LAYER_COMBINE_IN_GEMM = 1, 2, 4, 8
DEVERR_EXPERT_RANGE, DEVERR_ROW_RANGE, DEVERR_TIMEOUT = 1, 2, 4


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str = ""):
        super().__init__(f"{fn} -> {STATUS.get(status, status)} {msg}".strip())
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"libmoe_b200.so is not built ({path}); run "
                          "`python mixture_experts_routing_route_b200/build.py`")
    return ctypes.CDLL(path)


_lib = load_library()

c_void_p, c_int, c_int64, c_size_t = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
c_double, c_uint32 = ctypes.c_double, ctypes.c_uint32


class MoeLayerC(ctypes.Structure):
    _fields_ = [("d", c_int), ("E", c_int), ("k", c_int), ("F", c_int), ("dtype", c_int),
                ("act", c_int), ("capacity_factor", c_double), ("w_router", c_void_p),
                ("router_bias", c_void_p), ("w1", c_void_p), ("w3", c_void_p), ("w2", c_void_p),
                ("flags", c_int), ("x_router", c_void_p), ("logit_noise", c_void_p),
                ("router_temperature", ctypes.c_float)]


class MoeViewsC(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("topk_idx", "topk_w", "aux_loss", "z_loss", "counts", "bins",
                                        "kept_counts", "seg_offsets", "sorted_slot",
                                        "slot_to_row", "row_slot", "drop_mask", "x_perm", "h",
                                        "y_perm")] + [("rows_max", c_int64), ("capacity", c_int64)]


_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [c_int]),
    "moe_workspace_init": (c_int, [c_void_p, c_size_t, c_void_p]),
    "moe_workspace_set_wait_limit": (c_int, [c_void_p, c_size_t, c_uint32, c_void_p]),
    "moe_kernel_launches": (ctypes.c_uint64, []),
    "moe_get_device_error": (c_int, [c_void_p, c_void_p, ctypes.POINTER(c_uint32), c_int]),
    "moe_capacity": (c_int64, [c_double, c_int, c_int, c_int]),
    "moe_rows_max": (c_int64, [c_int, c_int, c_int, c_int64]),
    "moe_route_workspace_size": (c_size_t, [c_int, c_int, c_int]),
    "moe_route": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                          c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                          c_void_p]),
    "moe_permute_workspace_size": (c_size_t, [c_int, c_int, c_int]),
    "moe_permute": (c_int, [c_void_p, c_int, c_int, c_int, c_int64] + [c_void_p] * 8
                    + [c_void_p, c_size_t, c_void_p]),
    "moe_permute_noalloc": (c_int, [c_void_p, c_int, c_int, c_int, c_int64] + [c_void_p] * 9
                            + [c_void_p]),
    "moe_route_train": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, ctypes.c_float, c_int, c_int,
                                c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_route_backward_workspace_size": (c_size_t, [c_int, c_int, c_int]),
    "moe_route_backward": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int] + [c_void_p] * 5
                           + [ctypes.c_float] * 3 + [c_void_p] * 4 + [c_size_t, c_void_p]),
    "moe_router_jitter": (c_int, [c_void_p, c_int, c_int, c_int, ctypes.c_float, ctypes.c_uint64,
                                  c_void_p, c_void_p]),
    "moe_router_noise": (c_int, [c_int, c_int, ctypes.c_float, ctypes.c_uint64, c_void_p, c_void_p]),
    "moe_permute_binned": (c_int, [c_void_p, c_int, c_int, c_int, c_int64] + [c_void_p] * 8
                           + [c_void_p, c_size_t, c_void_p]),
    "moe_rows_max_binned": (c_int64, [c_int, c_int, c_int, c_int64]),
    "moe_gather": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_int,
                           c_int64, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_expert_ffn": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int64,
                               c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_size_t, c_void_p]),
    "moe_combine": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int64,
                            c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_ep_send_plan": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                 c_size_t, c_void_p]),
    "moe_ep_recv_plan": (c_int, [c_void_p, c_int, c_int, c_int64, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "moe_forward_workspace_size": (c_size_t, [ctypes.POINTER(MoeLayerC), c_int]),
    "moe_forward_host_workspace_size": (c_size_t, [ctypes.POINTER(MoeLayerC), c_int]),
    "moe_forward": (c_int, [ctypes.POINTER(MoeLayerC), c_void_p, c_int, c_void_p, c_void_p,
                            c_void_p, c_size_t, c_void_p, c_void_p]),
    "moe_forward_views": (c_int, [ctypes.POINTER(MoeLayerC), c_int, c_void_p, c_size_t,
                                  ctypes.POINTER(MoeViewsC)]),
    "moe_forward_host": (c_int, [ctypes.POINTER(MoeLayerC), c_void_p, c_int, c_void_p, c_void_p,
                                 c_void_p, c_size_t, c_void_p]),
}

for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def header_functions(path: str = HEADER_PATH):
    """Names of the functions include/moe_b200.h declares."""
    with open(path) as f:
        text = f.read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M)))


# ---------------------------------------------------------------- marshalling
def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, st: int):
    if st != MOE_OK:
        raise MoeError(fn, st, _lib.moe_status_string(st).decode())


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return MOE_BF16
    if t == torch.float32:
        return MOE_F32
    raise ValueError(f"unsupported dtype {t}")


def status_string(st: int) -> str:
    return _lib.moe_status_string(st).decode()


def moe_kernel_launches() -> int:
    """Kernels the library has launched so far in this process."""
    return int(_lib.moe_kernel_launches())


def moe_capacity(cf: float, T: int, k: int, E: int) -> int:
    return _lib.moe_capacity(float(cf), T, k, E)


def moe_rows_max(T: int, k: int, E: int, capacity: int) -> int:
    return _lib.moe_rows_max(T, k, E, capacity)


def moe_rows_max_binned(T: int, k: int, E: int, capacity: int) -> int:
    return _lib.moe_rows_max_binned(T, k, E, capacity)


def moe_route_workspace_size(T, d, E) -> int:
    return _lib.moe_route_workspace_size(T, d, E)


def moe_permute_workspace_size(T, k, E) -> int:
    return _lib.moe_permute_workspace_size(T, k, E)


def moe_workspace_init(ws: torch.Tensor, stream=None):
    _check("moe_workspace_init", _lib.moe_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))


def moe_workspace_set_wait_limit(ws: torch.Tensor, limit_us: int, stream=None):
    _check("moe_workspace_set_wait_limit",
           _lib.moe_workspace_set_wait_limit(_ptr(ws), ws.numel(), int(limit_us), _stream(stream)))


def moe_get_device_error(ws: torch.Tensor, stream=None, clear: bool = True) -> int:
    bits = c_uint32(0)
    st = _lib.moe_get_device_error(_ptr(ws), _stream(stream), ctypes.byref(bits), int(clear))
    if st not in (MOE_OK, 7):
        _check("moe_get_device_error", st)
    return bits.value


def moe_route(x, w_router, bias, T, d, E, k, topk_idx, topk_w, aux_loss, logits, probs, ws,
              stream=None):
    _check("moe_route", _lib.moe_route(
        _ptr(x), _ptr(w_router), _ptr(bias), dtype_code(x.dtype), T, d, E, k, _ptr(topk_idx),
        _ptr(topk_w), _ptr(aux_loss), _ptr(logits), _ptr(probs), _ptr(ws), ws.numel(),
        _stream(stream)))


def moe_route_train(x, w_router, bias, logit_noise, T, d, E, k, topk_idx, topk_w, aux_loss, z_loss,
                    logits, probs, ws, stream=None, temperature=1.0):
    _check("moe_route_train", _lib.moe_route_train(
        _ptr(x), _ptr(w_router), _ptr(bias), _ptr(logit_noise), float(temperature),
        dtype_code(x.dtype), T, d, E, k,
        _ptr(topk_idx), _ptr(topk_w), _ptr(aux_loss), _ptr(z_loss), _ptr(logits), _ptr(probs),
        _ptr(ws), ws.numel(), _stream(stream)))


def moe_route_backward_workspace_size(T, d, E) -> int:
    return _lib.moe_route_backward_workspace_size(T, d, E)


def moe_route_backward(x, w_router, T, d, E, k, probs, logits, topk_idx, topk_w, d_topk_w, d_aux, d_z,
                       temperature, d_logits, dx, d_wg, ws, stream=None, dtype=None):
    dt = dtype_code(x.dtype) if x is not None else dtype
    _check("moe_route_backward", _lib.moe_route_backward(
        _ptr(x), _ptr(w_router), dt, T, d, E, k, _ptr(probs), _ptr(logits), _ptr(topk_idx),
        _ptr(topk_w), _ptr(d_topk_w), float(d_aux), float(d_z), float(temperature), _ptr(d_logits),
        _ptr(dx), _ptr(d_wg), _ptr(ws), ws.numel(), _stream(stream)))


def moe_router_jitter(x, T, d, eps, seed, x_out, stream=None):
    _check("moe_router_jitter", _lib.moe_router_jitter(
        _ptr(x), dtype_code(x.dtype), T, d, float(eps), int(seed), _ptr(x_out), _stream(stream)))


def moe_router_noise(T, E, std, seed, noise_out, stream=None):
    _check("moe_router_noise", _lib.moe_router_noise(T, E, float(std), int(seed), _ptr(noise_out),
                                                     _stream(stream)))


def moe_permute(topk_idx, T, k, E, capacity, counts, bins, sorted_slot, slot_to_row, row_slot,
                drop_mask, kept_counts, seg_offsets, ws, stream=None):
    _check("moe_permute", _lib.moe_permute(
        _ptr(topk_idx), T, k, E, int(capacity), _ptr(counts), _ptr(bins), _ptr(sorted_slot),
        _ptr(slot_to_row), _ptr(row_slot), _ptr(drop_mask), _ptr(kept_counts), _ptr(seg_offsets),
        _ptr(ws), ws.numel(), _stream(stream)))


def moe_permute_binned(topk_idx, T, k, E, capacity, counts, bins, sorted_slot, slot_to_row,
                       row_slot, drop_mask, kept_counts, seg_offsets, ws, stream=None):
    _check("moe_permute_binned", _lib.moe_permute_binned(
        _ptr(topk_idx), T, k, E, int(capacity), _ptr(counts), _ptr(bins), _ptr(sorted_slot),
        _ptr(slot_to_row), _ptr(row_slot), _ptr(drop_mask), _ptr(kept_counts), _ptr(seg_offsets),
        _ptr(ws), ws.numel(), _stream(stream)))


def moe_permute_noalloc(topk_idx, T, k, E, capacity, counts, bins, sorted_slot, slot_to_row,
                        row_slot, drop_mask, kept_counts, seg_offsets, device_error=None,
                        stream=None):
    _check("moe_permute_noalloc", _lib.moe_permute_noalloc(
        _ptr(topk_idx), T, k, E, int(capacity), _ptr(counts), _ptr(bins), _ptr(sorted_slot),
        _ptr(slot_to_row), _ptr(row_slot), _ptr(drop_mask), _ptr(kept_counts), _ptr(seg_offsets),
        _ptr(device_error), _stream(stream)))


def moe_gather(x, T, d, k, row_slot, seg_offsets, E, rows_max, x_perm, ws, stream=None):
    _check("moe_gather", _lib.moe_gather(
        _ptr(x), dtype_code(x.dtype), T, d, k, _ptr(row_slot), _ptr(seg_offsets), E,
        int(rows_max), _ptr(x_perm), _ptr(ws), ws.numel(), _stream(stream)))


def moe_expert_ffn(x_perm, w1, w3, w2, act, rows_max, d, F, E, seg_offsets, h, y_perm, ws,
                   stream=None):
    _check("moe_expert_ffn", _lib.moe_expert_ffn(
        _ptr(x_perm), _ptr(w1), _ptr(w3), _ptr(w2), dtype_code(w1.dtype), act, int(rows_max), d,
        F, E, _ptr(seg_offsets), _ptr(h), _ptr(y_perm), _ptr(ws), ws.numel(), _stream(stream)))


def moe_combine(y_perm, topk_w, slot_to_row, T, d, k, rows_max, out, ws, stream=None):
    _check("moe_combine", _lib.moe_combine(
        _ptr(y_perm), _ptr(topk_w), _ptr(slot_to_row), dtype_code(out.dtype), T, d, k,
        int(rows_max), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))


def moe_ep_send_plan(kept_counts, seg_offsets, E, world, send_rows, send_offsets, ws, stream=None):
    _check("moe_ep_send_plan", _lib.moe_ep_send_plan(
        _ptr(kept_counts), _ptr(seg_offsets), E, world, _ptr(send_rows), _ptr(send_offsets), _ptr(ws),
        ws.numel(), _stream(stream)))


def moe_ep_recv_plan(recv_counts, world, experts_per_rank, rows_cap, recv_rows, recv_offsets, local_seg,
                     local_to_recv, recv_to_local, ws, stream=None):
    _check("moe_ep_recv_plan", _lib.moe_ep_recv_plan(
        _ptr(recv_counts), world, experts_per_rank, int(rows_cap), _ptr(recv_rows), _ptr(recv_offsets),
        _ptr(local_seg), _ptr(local_to_recv), _ptr(recv_to_local), _ptr(ws), ws.numel(), _stream(stream)))


def layer_struct(d, E, k, F, dtype, act, cf, w_router, bias, w1, w3, w2, flags=0,
                 router_temperature=1.0) -> MoeLayerC:
    return MoeLayerC(d, E, k, F, dtype, act, float(cf), _ptr(w_router), _ptr(bias), _ptr(w1),
                     _ptr(w3), _ptr(w2), int(flags), None, None, float(router_temperature))


def moe_forward_workspace_size(layer: MoeLayerC, T: int) -> int:
    return _lib.moe_forward_workspace_size(ctypes.byref(layer), T)


def moe_forward_host_workspace_size(layer: MoeLayerC, T: int) -> int:
    return _lib.moe_forward_host_workspace_size(ctypes.byref(layer), T)


def moe_forward(layer: MoeLayerC, x, T, out, aux_loss, ws, stream=None, events=None):
    ev = None
    if events is not None:
        # torch creates a CUDA event lazily, on its first record(): record once
        # so that the handle exists (the library then re-records it in place).
        for e in events:
            if e is not None and e.cuda_event == 0:
                e.record(torch.cuda.current_stream() if stream is None else stream)
        arr = (c_void_p * 7)(*[e.cuda_event if e is not None else None for e in events])
        ev = ctypes.cast(arr, c_void_p)
    _check("moe_forward", _lib.moe_forward(
        ctypes.byref(layer), _ptr(x), T, _ptr(out), _ptr(aux_loss), _ptr(ws), ws.numel(),
        _stream(stream), ev))


def moe_forward_views(layer: MoeLayerC, T: int, ws) -> MoeViewsC:
    v = MoeViewsC()
    _check("moe_forward_views", _lib.moe_forward_views(ctypes.byref(layer), T, _ptr(ws),
                                                       ws.numel(), ctypes.byref(v)))
    return v


def moe_forward_host(layer: MoeLayerC, x_host, T, out_host, aux_host, ws, stream=None):
    _check("moe_forward_host", _lib.moe_forward_host(
        ctypes.byref(layer), _ptr(x_host), T, _ptr(out_host), _ptr(aux_host), _ptr(ws),
        ws.numel(), _stream(stream)))
