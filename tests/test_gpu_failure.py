"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The permute's multi-CTA kernel has one barrier between its CTAs (every CTA
publishes its per-expert counts, then waits for all the others). Its wait is
bounded by the workspace's wait limit. Here the barrier's arrival counter is
pre-loaded from the host so that the barrier can never complete (the flag
that releases it is never set); with a 1 ms limit every CTA gives up, sets
MOE_DEVERR_TIMEOUT and returns, and the context stays usable. After
moe_workspace_init the same workspace gives the oracle's result bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from tests.gpu_helpers import npi

pytestmark = pytest.mark.gpu
DEV = "cuda"
BAR_COUNT_OFFSET = 8  # byte offset of the barrier's arrival counter in the control block


def _permute(abi, idx, T, k, E, cap, ws):
    S = T * k
    R = abi.moe_rows_max(T, k, E, cap)
    o = {n: torch.full((max(m, 1),), -3, dtype=torch.int32, device=DEV)
         for n, m in (("counts", E), ("bins", E), ("sorted_slot", S), ("slot_to_row", S),
                      ("row_slot", R), ("kept_counts", E), ("seg_offsets", E + 1))}
    o["drop"] = torch.full((max(S, 1),), 9, dtype=torch.uint8, device=DEV)
    abi.moe_permute(idx, T, k, E, cap, o["counts"], o["bins"], o["sorted_slot"], o["slot_to_row"],
                    o["row_slot"], o["drop"], o["kept_counts"], o["seg_offsets"], ws)
    return o


def _check_against_oracle(o, idx_np, T, k, E, cap):
    ref = O.permute(idx_np, E, None if cap < 0 else cap)
    S = T * k
    for key, n in (("counts", E), ("bins", E), ("kept_counts", E), ("seg_offsets", E + 1),
                   ("sorted_slot", S), ("slot_to_row", S)):
        assert np.array_equal(npi(o[key])[:n], ref[key]), key
    assert np.array_equal(npi(o["drop"])[:S], ref["drop"])
    assert np.array_equal(npi(o["row_slot"])[:ref["rows"]], ref["row_slot"])


@pytest.mark.parametrize("cap", [-1, 900])
def test_grid_barrier_wait_runs_out_then_workspace_init_recovers(cap):
    from mixture_experts_routing_route_b200 import _abi as abi
    T, k, E = 4096, 2, 8  # 8192 slots: the multi-CTA permute with a grid barrier
    rng = np.random.default_rng(77)
    idx_np = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    idx = torch.from_numpy(idx_np).to(DEV)
    ws = torch.empty(abi.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
    abi.moe_workspace_init(ws)

    # a 1 ms limit alone changes nothing: the barrier completes in microseconds
    abi.moe_workspace_set_wait_limit(ws, 1000)
    o = _permute(abi, idx, T, k, E, cap, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    _check_against_oracle(o, idx_np, T, k, E, cap)

    # no arrival count can reach the release value: every CTA's wait runs out
    ws[BAR_COUNT_OFFSET:BAR_COUNT_OFFSET + 4].view(torch.int32).fill_(0x40000000)
    _permute(abi, idx, T, k, E, cap, ws)
    torch.cuda.synchronize()
    bits = abi.moe_get_device_error(ws)
    assert bits & abi.DEVERR_TIMEOUT, bits

    # the context is usable and the re-initialised workspace is exact again
    abi.moe_workspace_init(ws)
    o = _permute(abi, idx, T, k, E, cap, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    _check_against_oracle(o, idx_np, T, k, E, cap)
