"""The C-ABI library without a GPU: it builds, loads, exports every function
include/moe_b200.h declares, and its host-only logic (capacity, row bounds,
workspace sizes, argument checks that return before any launch) is right."""
import ctypes

import pytest

import __graft_entry__


@pytest.fixture(scope="module")
def abi():
    __graft_entry__.build()
    from mixture_experts_routing_route_b200 import _abi
    return _abi


def test_exports_every_declared_function(abi):
    declared = abi.header_functions()
    assert len(declared) >= 15
    lib = ctypes.CDLL(abi.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def test_capacity_matches_oracle_formula(abi):
    from oracle import moe_oracle as O
    for cf, k, T, E in [(1.25, 1, 256, 4), (1.0, 2, 16384, 64), (1.25, 2, 32768, 8), (1.1, 3, 10, 4),
                        (0.05, 1, 64, 4), (0.0, 2, 100, 8), (-1.0, 2, 5, 2), (2.5, 8, 4096, 256)]:
        ref = O.capacity(cf, k, T, E)
        assert abi.moe_capacity(cf, T, k, E) == (-1 if ref is None else ref)


def test_rows_max_binned(abi):
    assert abi.moe_rows_max_binned(100, 2, 8, 10) == 80
    assert abi.moe_rows_max_binned(100, 2, 8, -1) == 8 * 200   # dynamic: worst case C = T*k
    assert abi.moe_rows_max_binned(100, 2, 8, 0) == 0
    L = abi.MoeLayerC(4096, 8, 2, 14336, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16,
                      abi.MOE_LAYER_BINNED)
    Ld = abi.MoeLayerC(4096, 8, 2, 14336, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16)
    assert abi.moe_forward_workspace_size(L, 4096) > abi.moe_forward_workspace_size(Ld, 4096)


def test_rows_max(abi):
    assert abi.moe_rows_max(100, 2, 8, -1) == 200
    assert abi.moe_rows_max(100, 2, 8, 10) == 80
    assert abi.moe_rows_max(100, 2, 8, 1000) == 200
    assert abi.moe_rows_max(0, 2, 8, -1) == 0


def test_workspace_sizes_grow(abi):
    a = abi.moe_route_workspace_size(4096, 4096, 8)
    b = abi.moe_route_workspace_size(32768, 4096, 8)
    assert 256 < a < b
    assert abi.moe_permute_workspace_size(4096, 2, 8) >= 256 + 4096 * 2 * 4
    L = abi.MoeLayerC(4096, 8, 2, 14336, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16)
    n = abi.moe_forward_workspace_size(L, 4096)
    # x_perm + h + y_perm alone: 8192 rows of (4096 + 14336 + 4096) bf16
    assert n >= 8192 * (4096 + 14336 + 4096) * 2
    # gathering inside the up projection drops x_perm
    Lg = abi.MoeLayerC(4096, 8, 2, 14336, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16,
                       abi.MOE_LAYER_GATHER_IN_GEMM)
    assert abi.moe_forward_workspace_size(Lg, 4096) == n - 8192 * 4096 * 2
    # the combine inside the down projection (k = 1) drops y_perm
    L1 = abi.MoeLayerC(4096, 8, 1, 14336, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16)
    Lc = abi.MoeLayerC(4096, 8, 1, 14336, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16,
                       abi.MOE_LAYER_COMBINE_IN_GEMM)
    assert abi.moe_forward_workspace_size(Lc, 4096) == abi.moe_forward_workspace_size(L1, 4096) - 4096 * 4096 * 2
    assert abi.moe_forward_host_workspace_size(L, 4096) >= n + 2 * 4096 * 4096 * 2


def _call_route(abi, **over):
    a = dict(x=16, wg=16, bias=None, dt=abi.MOE_BF16, T=8, d=128, E=8, k=2, idx=16, w=16, aux=16,
             logits=None, probs=None, ws=16, ws_bytes=1 << 30)
    a.update(over)
    return abi._lib.moe_route(a["x"], a["wg"], a["bias"], a["dt"], a["T"], a["d"], a["E"], a["k"],
                              a["idx"], a["w"], a["aux"], a["logits"], a["probs"], a["ws"],
                              a["ws_bytes"], None)


def test_argument_checks_return_before_launch(abi):
    # every case here fails a host check, so nothing is launched
    n0 = abi.moe_kernel_launches()
    assert _call_route(abi, x=None) == 1                      # MOE_ERR_NULL
    assert _call_route(abi, k=9) == 2                         # k > 8
    assert _call_route(abi, E=4, k=5) == 2                    # k > E
    assert _call_route(abi, E=257) == 2                       # E > 256
    assert _call_route(abi, d=96) == 3                        # bf16 needs d % 128 == 0
    assert _call_route(abi, x=24) == 5                        # misaligned pointer
    assert _call_route(abi, ws_bytes=100) == 4                # workspace too small
    assert _call_route(abi, T=-1) == 2
    assert abi._lib.moe_workspace_init(None, 256, None) == 1
    L = abi.MoeLayerC(4096, 8, 2, 100, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16)
    assert abi._lib.moe_forward(ctypes.byref(L), 16, 4, 16, None, 16, 1 << 40, None, None) == 3
    L2 = abi.MoeLayerC(4096, 8, 2, 128, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, None, 16)
    assert abi._lib.moe_forward(ctypes.byref(L2), 16, 4, 16, None, 16, 1 << 40, None, None) == 1
    assert abi._lib.moe_permute(16, 4, 2, 0, -1, *([16] * 8), 16, 1 << 20, None) == 2
    L3 = abi.MoeLayerC(4096, 8, 2, 128, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16, 16)
    assert abi._lib.moe_forward(ctypes.byref(L3), 16, 4, 16, None, 16, 1 << 40, None, None) == 2
    # the combine in the down projection: bf16 and k = 1 only
    L5 = abi.MoeLayerC(4096, 8, 2, 128, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16,
                       abi.MOE_LAYER_COMBINE_IN_GEMM)
    assert abi._lib.moe_forward(ctypes.byref(L5), 16, 4, 16, None, 16, 1 << 40, None, None) == 3
    L6 = abi.MoeLayerC(4096, 8, 1, 128, abi.MOE_F32, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16,
                       abi.MOE_LAYER_COMBINE_IN_GEMM)
    assert abi._lib.moe_forward(ctypes.byref(L6), 16, 4, 16, None, 16, 1 << 40, None, None) == 3
    L4 = abi.MoeLayerC(4096, 8, 2, 128, abi.MOE_F32, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16,
                       abi.MOE_LAYER_GATHER_IN_GEMM)
    assert abi._lib.moe_forward(ctypes.byref(L4), 16, 4, 16, None, 16, 1 << 40, None, None) == 3
    # the router temperature must be > 0 (moe_route_train) or >= 0 (layer, 0 = 1)
    assert abi._lib.moe_route_train(16, 16, None, None, 0.0, abi.MOE_BF16, 8, 128, 8, 2, 16, 16, 16,
                                    None, None, None, 16, 1 << 30, None) == 2
    L7 = abi.MoeLayerC(4096, 8, 2, 128, abi.MOE_BF16, abi.MOE_ACT_SWIGLU, 0.0, 16, None, 16, 16, 16,
                       0, None, None, -1.0)
    assert abi._lib.moe_forward(ctypes.byref(L7), 16, 4, 16, None, 16, 1 << 40, None, None) == 2
    # router backward: tau > 0, a workspace, probs when T > 0
    assert abi._lib.moe_route_backward(16, 16, abi.MOE_BF16, 8, 128, 8, 2, 16, None, 16, 16, None, 0.0,
                                       0.0, 0.0, None, None, None, 16, 1 << 30, None) == 2
    assert abi._lib.moe_route_backward(16, 16, abi.MOE_BF16, 8, 128, 8, 2, None, None, 16, 16, None,
                                       0.0, 0.0, 1.0, None, None, None, 16, 1 << 30, None) == 1
    assert abi._lib.moe_route_backward(16, 16, abi.MOE_BF16, 8, 128, 8, 2, 16, None, 16, 16, None, 0.0,
                                       1.0, 1.0, None, None, None, 16, 1 << 30, None) == 1  # d_z needs logits
    assert abi._lib.moe_route_backward(16, 16, abi.MOE_BF16, 8, 128, 8, 2, 16, None, 16, 16, None, 0.0,
                                       0.0, 1.0, None, None, None, 16, 16, None) == 4
    # router backward: d limits as everywhere (bf16 d % 128, fp32 d % 4)
    assert abi._lib.moe_route_backward(16, 16, abi.MOE_BF16, 8, 96, 8, 2, 16, None, 16, 16, None, 0.0,
                                       0.0, 1.0, None, None, None, 16, 1 << 30, None) == 3
    assert abi._lib.moe_route_backward(16, 16, abi.MOE_F32, 8, 66, 8, 2, 16, None, 16, 16, None, 0.0,
                                       0.0, 1.0, None, None, None, 16, 1 << 30, None) == 3
    assert abi.moe_route_backward_workspace_size(4096, 4096, 8) >= 4096 * 8 * 4
    assert abi.moe_kernel_launches() == n0


def test_status_strings(abi):
    for st in range(8):
        assert abi.status_string(st)
