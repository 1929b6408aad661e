"""The expert-parallel driver (mixture_experts_routing_route_b200.ep.ep_forward)
over a real torch.distributed group: world size 2 with gloo on CPU tensors,
the oracle's steps plugged in where the library's kernels run on a GPU (the
kernels themselves are checked on one GPU by tests/test_gpu_ep.py). Each
rank's output must be the oracle's single-GPU forward of its own tokens: the
dispatch plans, both all-to-all-v exchanges (uneven splits) and the regroup
in between only move rows. The exchange itself is unmeasured on hardware:
every run available here has one GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """ep_forward's steps computed by the CPU oracle on float64 tensors."""

    def __init__(self):
        from oracle import moe_oracle as O
        self.O = O

    def dispatch(self, x, w_router, bias, k, E, cf):
        O = self.O
        xn = x.numpy()
        T, d = xn.shape
        r = O.route(xn, w_router.numpy(), None if bias is None else bias.numpy(), k)
        pm = O.permute(r["topk_idx"], E, O.capacity(cf, k, T, E))
        xp = O.gather(xn, pm["row_slot"], k)
        plan = O.ep_send_plan(r["topk_idx"], pm["drop"], E, dist.get_world_size())
        return {"T": T, "d": d, "k": k, "E": E, "rows_max": pm["rows"], "route": r, "permute": pm,
                "plan": plan, "x_perm": torch.from_numpy(np.ascontiguousarray(xp, dtype=np.float64)),
                "aux": torch.tensor([r["aux"]])}

    def send_plan(self, st, world):
        return torch.from_numpy(st["plan"]["send_rows"]), torch.from_numpy(st["plan"]["send_offsets"])

    def expert_counts(self, st):
        return torch.from_numpy(st["plan"]["expert_counts"].astype(np.int64))

    def recv_plan(self, recv_counts, world, e_loc, rows):
        rp = self.O.ep_recv_plan(recv_counts.view(world, e_loc).numpy())
        return {n: torch.from_numpy(v) for n, v in rp.items()}

    def gather_rows(self, src, rows_map, seg, nseg, rows):
        return src[rows_map[:rows].long()]

    def expert_ffn(self, x_loc, local_seg, e_loc, w1, w3, w2, act, rows):
        W = lambda t: None if t is None else [t[e].numpy() for e in range(t.shape[0])]  # noqa: E731
        y = self.O.expert_ffn(x_loc[:rows].numpy(), local_seg.numpy(), W(w1), W(w3), W(w2), act)
        return torch.from_numpy(y)

    def combine(self, st, y_perm):
        R = st["rows_max"]
        out = self.O.combine(y_perm[:R].numpy(), st["route"]["topk_w64"], st["permute"]["slot_to_row"],
                             st["T"], st["k"])
        return torch.from_numpy(out)


CASES = [
    # T0, T1, d, E, k, F, act, cf
    (37, 50, 16, 4, 2, 24, "swiglu", 0.0),
    (64, 20, 8, 8, 3, 12, "gelu", 1.0),    # capacity drops on each rank, uneven token counts
    (5, 0, 8, 2, 1, 8, "swiglu", 0.0),     # a rank with no tokens
]


def _worker(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mixture_experts_routing_route_b200.ep import ep_forward
        from oracle import moe_oracle as O
        T0, T1, d, E, k, F, act, cf = case
        g = torch.Generator().manual_seed(1234)  # the same weights on every rank
        wg = torch.randn(d, E, generator=g, dtype=torch.float64)
        w1 = torch.randn(E, d, F, generator=g, dtype=torch.float64) * 0.3
        w3 = torch.randn(E, d, F, generator=g, dtype=torch.float64) * 0.3
        w2 = torch.randn(E, F, d, generator=g, dtype=torch.float64) * 0.3
        T = (T0, T1)[rank]
        x = torch.randn(T, d, generator=torch.Generator().manual_seed(77 + rank), dtype=torch.float64)
        e_loc = E // world
        sl = slice(rank * e_loc, (rank + 1) * e_loc)
        got, aux = ep_forward(x, wg, None, w1[sl].contiguous(), w3[sl].contiguous() if act == "swiglu" else None,
                              w2[sl].contiguous(), k, act, E, cf, ops=OracleOps())
        W = lambda t: [t[e].numpy() for e in range(E)]  # noqa: E731
        ref = O.forward(x.numpy(), wg.numpy(), None, W(w1), W(w3) if act == "swiglu" else None, W(w2), k, act, cf)
        err = float(np.max(np.abs(got.numpy() - ref["out"]))) if T else 0.0
        out[rank] = (err, float(np.max(np.abs(ref["out"]))) if T else 0.0, tuple(got.shape))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_ep_forward_two_ranks_gloo(case):
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, case, out), nprocs=world, join=True)
    for rank in range(world):
        err, scale, shape = out[rank]
        assert shape == ((case[0], case[1])[rank], case[2])
        assert err <= 1e-10 * max(scale, 1.0), (rank, err, scale)
