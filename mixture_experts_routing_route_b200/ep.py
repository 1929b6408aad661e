"""Expert-parallel forward of the MoE layer: the experts live on several
ranks, each token's rows travel to the ranks that hold their experts and
their outputs travel back.

"MoE Router: who decides which expert a token goes to": the router's output
is a per-device dispatch plan (device = expert / experts_per_device); an
all-to-all-v with per-pair counts and displacements moves the rows.
"ops-transformer MoE operators", 坑2: tokens are computed on the cards that
hold their experts and sent back. "Integrating MoE into your model with
Colossal-AI", step 2: all-to-all to the expert's GPU, expert MLP, all-to-all
back.

Every arithmetic step runs in the library's kernels (route, permute, gather,
the two dispatch plans, the grouped GEMM on this rank's experts, the
combine); the exchanges are all-to-all-v collectives (NCCL through
torch.distributed by default). Experts are owned in contiguous blocks of
E / world per rank, each rank applies the capacity to its own tokens, so a
rank's output equals moe_forward on its own tokens.

The steps are passed in as an object (`LibraryOps` here) and the exchanges
as another (`DistExchange` here), so the same driver runs on any transport.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _abi as abi


def _ws(nbytes: int, dev) -> torch.Tensor:
    w = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
    abi.moe_workspace_init(w)
    return w


class LibraryOps:
    """The steps of the expert-parallel forward on this library's kernels
    (device tensors on the current stream). Control workspaces are kept so
    that check() can read every step's device error word."""

    def __init__(self):
        self._ctl = []

    def _new_ws(self, nbytes, dev):
        w = _ws(nbytes, dev)
        self._ctl.append(w)
        return w

    def dispatch(self, x, w_router, bias, k, E, cf):
        """Route, permute (this rank's capacity) and gather this rank's tokens."""
        T, d = x.shape
        dev = x.device
        i32 = dict(dtype=torch.int32, device=dev)
        idx = torch.empty(T, k, **i32)
        w = torch.empty(T, k, dtype=torch.float32, device=dev)
        aux = torch.empty(1, dtype=torch.float32, device=dev)
        rws = self._new_ws(abi.moe_route_workspace_size(T, d, E), dev)
        abi.moe_route(x, w_router, bias, T, d, E, k, idx, w, aux, None, None, rws)
        cap = abi.moe_capacity(cf, T, k, E)
        R = abi.moe_rows_max(T, k, E, cap)
        S = T * k
        st = {"T": T, "d": d, "k": k, "E": E, "rows_max": R, "idx": idx, "w": w, "aux": aux}
        for name, n in (("counts", E), ("bins", E), ("kept", E), ("seg", E + 1), ("sorted_slot", S),
                        ("slot_to_row", S), ("row_slot", R)):
            st[name] = torch.empty(max(n, 1), **i32)
        st["drop"] = torch.empty(max(S, 1), dtype=torch.uint8, device=dev)
        pws = self._new_ws(abi.moe_permute_workspace_size(T, k, E), dev)
        abi.moe_permute(idx, T, k, E, cap, st["counts"], st["bins"], st["sorted_slot"], st["slot_to_row"],
                        st["row_slot"], st["drop"], st["kept"], st["seg"], pws)
        st["x_perm"] = torch.empty(max(R, 1), d, dtype=x.dtype, device=dev)
        abi.moe_gather(x, T, d, k, st["row_slot"], st["seg"], E, R, st["x_perm"], self._new_ws(256, dev))
        return st

    def send_plan(self, st, world):
        """Rows of x_perm for each rank and where they start (device)."""
        dev = st["idx"].device
        send_rows = torch.empty(world, dtype=torch.int32, device=dev)
        send_offsets = torch.empty(world + 1, dtype=torch.int32, device=dev)
        abi.moe_ep_send_plan(st["kept"], st["seg"], st["E"], world, send_rows, send_offsets,
                             self._new_ws(256, dev))
        return send_rows, send_offsets

    def expert_counts(self, st):
        """Per-expert kept counts; rank g's slice goes to rank g."""
        return st["kept"][:st["E"]]

    def recv_plan(self, recv_counts, world, e_loc, rows):
        dev = recv_counts.device
        i32 = dict(dtype=torch.int32, device=dev)
        rp = {"recv_rows": torch.empty(world, **i32), "recv_offsets": torch.empty(world + 1, **i32),
              "local_seg": torch.empty(e_loc + 1, **i32), "local_to_recv": torch.empty(max(rows, 1), **i32),
              "recv_to_local": torch.empty(max(rows, 1), **i32)}
        abi.moe_ep_recv_plan(recv_counts, world, e_loc, rows, rp["recv_rows"], rp["recv_offsets"],
                             rp["local_seg"], rp["local_to_recv"], rp["recv_to_local"], self._new_ws(256, dev))
        return rp

    def gather_rows(self, src, rows_map, seg, nseg, rows):
        """dst[r] = src[rows_map[r]] for r < seg[nseg] (the gather kernel, k = 1)."""
        d = src.shape[1]
        dst = torch.empty(max(rows, 1), d, dtype=src.dtype, device=src.device)
        if rows > 0:
            abi.moe_gather(src, rows, d, 1, rows_map, seg, nseg, rows, dst, self._new_ws(256, src.device))
        return dst

    def expert_ffn(self, x_loc, local_seg, e_loc, w1, w3, w2, act, rows):
        d, F = w1.shape[1], w1.shape[2]
        dev = x_loc.device
        h = torch.empty(max(rows, 1), F, dtype=x_loc.dtype, device=dev)
        y = torch.empty(max(rows, 1), d, dtype=x_loc.dtype, device=dev)
        code = abi.MOE_ACT_SWIGLU if act == "swiglu" else abi.MOE_ACT_GELU
        abi.moe_expert_ffn(x_loc, w1, w3, w2, code, rows, d, F, e_loc, local_seg, h, y, self._new_ws(256, dev))
        return y

    def combine(self, st, y_perm):
        T, d, k = st["T"], st["d"], st["k"]
        out = torch.empty(T, d, dtype=y_perm.dtype, device=y_perm.device)
        abi.moe_combine(y_perm, st["w"], st["slot_to_row"], T, d, k, st["rows_max"], out,
                        self._new_ws(256, y_perm.device))
        return out

    def check(self):
        """Raise if any step set its device error word (synchronises)."""
        for w in self._ctl:
            bits = abi.moe_get_device_error(w)
            if bits:
                raise abi.MoeError("expert-parallel step", 7, f"device error bits {bits}")
        self._ctl.clear()


class DistExchange:
    """All-to-all-v over a torch.distributed process group (NCCL for CUDA
    tensors, gloo for CPU tensors)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def equal(self, out, inp):
        self.dist.all_to_all_single(out, inp, group=self.group)

    def rows(self, out, inp, out_splits, in_splits):
        self.dist.all_to_all_single(out, inp, output_split_sizes=out_splits, input_split_sizes=in_splits,
                                    group=self.group)


def ep_forward(x: torch.Tensor, w_router: torch.Tensor, bias: Optional[torch.Tensor], w1_local: torch.Tensor,
               w3_local: Optional[torch.Tensor], w2_local: torch.Tensor, k: int, act: str, E: int,
               capacity_factor: float = 0.0, ops=None, exchange=None):
    """This rank's layer output and its router's aux loss (over its own
    tokens). w1_local / w3_local / w2_local hold this rank's E / world
    experts, [E/world, d, F] / [E/world, F, d]; w_router [d, E] and bias are
    the whole router's."""
    ops = LibraryOps() if ops is None else ops
    ex = DistExchange() if exchange is None else exchange
    world = ex.world
    if E % world != 0:
        raise ValueError("the experts must split evenly over the ranks")
    e_loc = E // world
    st = ops.dispatch(x, w_router, bias, k, E, capacity_factor)
    send_rows, _ = ops.send_plan(st, world)
    # per-expert counts: rank g receives this rank's counts of g's experts
    counts = ops.expert_counts(st).contiguous()
    recv_counts = torch.empty_like(counts)
    ex.equal(recv_counts, counts)
    # all-to-all-v takes its split sizes on the host
    send_h = [int(v) for v in send_rows.cpu().tolist()]
    recv_h = [int(v) for v in recv_counts.view(world, e_loc).sum(dim=1).cpu().tolist()]
    n_send, n_recv = sum(send_h), sum(recv_h)
    d = st["d"]
    x_recv = torch.empty(max(n_recv, 1), d, dtype=x.dtype, device=x.device)
    ex.rows(x_recv[:n_recv], st["x_perm"][:n_send], recv_h, send_h)
    rp = ops.recv_plan(recv_counts, world, e_loc, n_recv)
    x_loc = ops.gather_rows(x_recv, rp["local_to_recv"], rp["local_seg"], e_loc, n_recv)
    y_loc = ops.expert_ffn(x_loc, rp["local_seg"], e_loc, w1_local, w3_local, w2_local, act, n_recv)
    y_recv = ops.gather_rows(y_loc, rp["recv_to_local"], rp["recv_offsets"], world, n_recv)
    y_back = torch.empty(max(st["rows_max"], 1), d, dtype=x.dtype, device=x.device)
    ex.rows(y_back[:n_send], y_recv[:n_recv], send_h, recv_h)
    out = ops.combine(st, y_back)
    if hasattr(ops, "check"):
        ops.check()
    return out, st["aux"]
