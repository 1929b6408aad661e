"""moe_permute_noalloc: the permute for callers that cannot allocate device
memory (its scratch is a static device array inside the library, so such a
caller passes only its inputs and outputs). Checked against the workspace
entry point moe_permute and against the CPU oracle on the same inputs,
bit-exact as every integer stage is, over two calls in a row so that the
second call runs on the scratch the first one left behind. An out-of-range
expert id must reach the caller's device_error word, and the next valid call
must start from a cleared one.

Collected last (file name) so that a run stopping at its first failure has
already run every other test; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _outputs(T, k, E, cap):
    from mixture_experts_routing_route_b200 import _abi
    S = T * k
    R = _abi.moe_rows_max(T, k, E, cap)
    t = lambda n: torch.full((max(n, 1),), -3, dtype=torch.int32, device=DEV)  # noqa: E731
    return {"counts": t(E), "bins": t(E), "sorted_slot": t(S), "slot_to_row": t(S),
            "row_slot": t(R), "drop": torch.full((max(S, 1),), 9, dtype=torch.uint8, device=DEV),
            "kept_counts": t(E), "seg_offsets": t(E + 1)}, R


def _with_workspace(idx, T, k, E, cap):
    from mixture_experts_routing_route_b200 import _abi
    o, R = _outputs(T, k, E, cap)
    ws = torch.empty(_abi.moe_permute_workspace_size(T, k, E), dtype=torch.uint8, device=DEV)
    _abi.moe_workspace_init(ws)
    _abi.moe_permute(idx, T, k, E, cap, o["counts"], o["bins"], o["sorted_slot"], o["slot_to_row"],
                     o["row_slot"], o["drop"], o["kept_counts"], o["seg_offsets"], ws)
    torch.cuda.synchronize()
    assert _abi.moe_get_device_error(ws) == 0
    return o, R


def _no_alloc(idx, T, k, E, cap, want_err=0):
    from mixture_experts_routing_route_b200 import _abi
    o, R = _outputs(T, k, E, cap)
    err = torch.full((1,), 0x55, dtype=torch.int32, device=DEV)
    _abi.moe_permute_noalloc(idx, T, k, E, cap, o["counts"], o["bins"], o["sorted_slot"],
                             o["slot_to_row"], o["row_slot"], o["drop"], o["kept_counts"],
                             o["seg_offsets"], err)
    torch.cuda.synchronize()
    assert int(err.item()) == want_err
    return o, R


def _same_as_oracle(o, idx_np, T, k, E, cap):
    ref = O.permute(idx_np, E, None if cap < 0 else cap)
    S = T * k
    for key, n in (("counts", E), ("bins", E), ("kept_counts", E), ("seg_offsets", E + 1),
                   ("sorted_slot", S), ("slot_to_row", S)):
        assert np.array_equal(o[key][:n].cpu().numpy(), ref[key]), key
    assert np.array_equal(o["drop"][:S].cpu().numpy(), ref["drop"])
    assert np.array_equal(o["row_slot"][:ref["rows"]].cpu().numpy(), ref["row_slot"])


def _same(a, b, T, k, E, R):
    S = T * k
    for key, n in (("counts", E), ("bins", E), ("kept_counts", E), ("seg_offsets", E + 1),
                   ("sorted_slot", S), ("slot_to_row", S), ("drop", S)):
        assert torch.equal(a[key][:n], b[key][:n]), key
    rows = int(a["seg_offsets"][E].item())
    assert rows <= R
    assert torch.equal(a["row_slot"][:rows], b["row_slot"][:rows])


def test_no_alloc_matches_workspace_entry_point_twice():
    rng = np.random.default_rng(123)
    cases = [(4096, 2, 8, -1), (3000, 3, 64, 100)]  # two calls in a row, different shapes
    for T, k, E, cap in cases:
        idx_np = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        idx = torch.from_numpy(idx_np).to(DEV)
        ref, R = _with_workspace(idx, T, k, E, cap)
        got, _ = _no_alloc(idx, T, k, E, cap)
        _same(got, ref, T, k, E, R)
        _same_as_oracle(got, idx_np, T, k, E, cap)


def test_no_alloc_reports_a_bad_expert_id_then_clears_it():
    """The kernel guards every expert id it reads: an id outside [0, E) is
    skipped (its slot marked dropped) and recorded in the error word, which
    reaches the caller's device_error. The next call clears the shared
    control block first, so a valid call after it reports 0."""
    from mixture_experts_routing_route_b200 import _abi
    rng = np.random.default_rng(9)
    T, k, E = 1000, 2, 16
    idx_np = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    bad = idx_np.copy()
    bad[123, 1] = E + 5
    _no_alloc(torch.from_numpy(bad).to(DEV), T, k, E, -1, want_err=_abi.DEVERR_EXPERT_RANGE)
    got, _ = _no_alloc(torch.from_numpy(idx_np).to(DEV), T, k, E, -1, want_err=0)
    _same_as_oracle(got, idx_np, T, k, E, -1)


def test_no_alloc_rejects_sizes_beyond_its_static_scratch():
    from mixture_experts_routing_route_b200 import _abi
    T, k = 32769, 2  # 65538 slots > MOE_PERMUTE_NOALLOC_MAX_SLOTS (65536)
    with pytest.raises(_abi.MoeError) as ex:
        _abi.moe_permute_noalloc(torch.empty(1, dtype=torch.int32, device=DEV), T, k, 8, -1,
                                 *[torch.empty(1, dtype=torch.int32, device=DEV)] * 8)
    assert ex.value.status == 4  # MOE_ERR_WORKSPACE: nothing was launched
