"""GPU parity of each C-ABI stage entry point on its own (moe_route,
moe_permute, moe_gather, moe_expert_ffn, moe_combine), stage-chained against
the CPU oracle, plus the permute's edge cases and its device error word."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_route_b200 import _abi as abi
from workloads import small_case
from oracle import moe_oracle as O
from tests.gpu_helpers import (check_topk_end_to_end, TOL_AUX_REL, TOL_BF16_OUT, TOL_PROB_REL, ExpertWeights,
                               max_err_ratio, new_ws, np32, npi, rel_err)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def route_on_gpu(x, wg, bias, T, d, E, k):
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    aux = torch.empty(1, dtype=torch.float32, device=DEV)
    logits = torch.empty(T, E, dtype=torch.float32, device=DEV)
    probs = torch.empty(T, E, dtype=torch.float32, device=DEV)
    ws = new_ws(abi.moe_route_workspace_size(T, d, E))
    abi.moe_route(x, wg, bias, T, d, E, k, idx, w, aux, logits, probs, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    return idx, w, aux, logits, probs


@pytest.mark.parametrize("T,d,E,k,dt,bias", [
    (1000, 512, 8, 2, "bf16", "none"),     # fused E <= 8 path
    (77, 4096, 8, 2, "bf16", "expert0"),   # fused, d = 4096, ragged quad
    (300, 256, 5, 3, "bf16", "none"),      # fused with E < 8 (padded experts)
    (513, 256, 64, 2, "bf16", "zipf"),     # tensor cores, TMA Wg + router_select, 2 experts per lane
    (700, 256, 64, 8, "bf16", "none"),     # E = 64, k = 8: eight warp arg-max rounds
    (300, 4096, 64, 2, "bf16", "zipf"),    # E = 64, d = 4096 split over KS CTAs (partials added in ks order)
    (20000, 512, 64, 2, "bf16", "expert0"),  # E = 64, more token tiles than SMs
    (129, 256, 256, 8, "bf16", "none"),    # tensor cores, TMA Wg, 8 experts per lane, k = 8
    (300, 512, 16, 2, "bf16", "zipf"),     # tensor cores, staged Wg^T (E <= 32)
    (1000, 1024, 32, 4, "bf16", "none"),   # tensor cores, staged Wg^T, split over d
    (2000, 1024, 64, 2, "bf16", "zipf"),   # tensor cores, TMA Wg, one tile per CTA
    (97, 128, 128, 3, "bf16", "none"),     # tensor cores, 4 experts per lane
    (10000, 4096, 8, 2, "bf16", "expert0"),  # tensor cores, no d split: 64 k-blocks in 32 slots
    (20000, 1024, 8, 2, "bf16", "zipf"),   # more tiles than SMs: the persistent kernel
    (24000, 512, 24, 3, "bf16", "none"),   # persistent, E = 24 (Epad 32: padding rows from the next k-block)
    (19000, 256, 16, 2, "bf16", "expert0"),  # persistent, E = 16, 149 tiles (one SM takes two)
    (1000, 1024, 24, 2, "bf16", "expert0"),  # E = 24, split over d in a cluster
    (200, 64, 4, 1, "f32", "none"),        # fp32 fused
    (90, 64, 40, 4, "f32", "none"),        # fp32 general
])
def test_route(T, d, E, k, dt, bias):
    inp = small_case("r", T=T, d=d, E=E, k=k, F=128, act="gelu", dtype=dt, bias=bias, seed=T + E)
    x, wg = inp.x.to(DEV), inp.wg.to(DEV)
    b = None if inp.bias is None else inp.bias.to(DEV)
    idx, w, aux, logits, probs = route_on_gpu(x, wg, b, T, d, E, k)
    r = O.route(np32(inp.x), np32(inp.wg), None if inp.bias is None else inp.bias.numpy(), k)
    g_logits = np32(logits)
    # fp32 accumulation of the gate GEMM: close to the exact logits
    assert np.max(np.abs(g_logits - r["logits"])) <= 1e-5 * max(1.0, np.max(np.abs(r["logits"])))
    # top-k decided on the GPU's own fp32 logits: bit-exact with the oracle's selection of them
    assert np.array_equal(npi(idx), O.topk_select(g_logits, k))
    check_topk_end_to_end(npi(idx), r)
    assert rel_err(np32(probs), r["probs64"]) <= TOL_PROB_REL
    g_idx = npi(idx).astype(np.int64)
    assert rel_err(np32(w), O.renormalise(r["probs64"], g_idx)) <= TOL_PROB_REL
    aux_ref = O.aux_loss(r["probs64"], g_idx, E)
    assert abs(float(aux.item()) - aux_ref) <= TOL_AUX_REL * aux_ref


def test_route_exact_ties_lower_index():
    """Hand-placed exact ties (integer-valued logits) go to the lower expert."""
    T, d, E, k = 64, 128, 8, 3
    rng = np.random.default_rng(5)
    x = np.zeros((T, d), np.float32)
    x[:, :E] = rng.integers(-2, 3, size=(T, E))
    wg = np.zeros((d, E), np.float32)
    wg[:E, :E] = np.eye(E)
    for dt in (torch.bfloat16, torch.float32):
        xt = torch.from_numpy(x).to(dt).to(DEV)
        wt = torch.from_numpy(wg).to(dt).to(DEV)
        idx, *_ = route_on_gpu(xt, wt, None, T, d, E, k)
        assert np.array_equal(npi(idx), O.topk_select(x[:, :E], k))
    # E = 16, 32 (tensor cores, staged Wg^T), 40 (CUDA cores), 64 (tensor cores, TMA Wg)
    for E2 in (16, 32, 40, 64):
        wg2 = np.zeros((d, E2), np.float32)
        wg2[:E2, :E2] = np.eye(E2)
        x2 = np.zeros((T, d), np.float32)
        x2[:, :E2] = rng.integers(-1, 2, size=(T, E2))
        for dt in (torch.bfloat16, torch.float32):
            idx, *_ = route_on_gpu(torch.from_numpy(x2).to(dt).to(DEV),
                                   torch.from_numpy(wg2).to(dt).to(DEV), None, T, d, E2, 5)
            assert np.array_equal(npi(idx), O.topk_select(x2[:, :E2], 5)), (E2, dt)


def permute_on_gpu(idx_np, E, cap):
    T, k = idx_np.shape
    S = T * k
    R = abi.moe_rows_max(T, k, E, cap)
    t = lambda n: torch.full((max(n, 1),), -7, dtype=torch.int32, device=DEV)
    out = {"counts": t(E), "bins": t(E), "sorted_slot": t(S), "slot_to_row": t(S),
           "row_slot": t(R), "kept_counts": t(E), "seg_offsets": t(E + 1)}
    drop = torch.full((max(S, 1),), 7, dtype=torch.uint8, device=DEV)
    ws = new_ws(abi.moe_permute_workspace_size(T, k, E))
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).to(DEV)
    abi.moe_permute(idx, T, k, E, cap, out["counts"], out["bins"], out["sorted_slot"],
                    out["slot_to_row"], out["row_slot"], drop, out["kept_counts"],
                    out["seg_offsets"], ws)
    torch.cuda.synchronize()
    res = {kk: npi(vv) for kk, vv in out.items()}
    res["drop"] = npi(drop)
    res["err"] = abi.moe_get_device_error(ws)
    return res


def assert_permute_equal(g, ref, S, E):
    assert g["err"] == 0
    for key in ("counts", "bins", "kept_counts"):
        assert np.array_equal(g[key][:E], ref[key]), key
    assert np.array_equal(g["seg_offsets"][:E + 1], ref["seg_offsets"])
    for key in ("sorted_slot", "slot_to_row"):
        assert np.array_equal(g[key][:S], ref[key]), key
    assert np.array_equal(g["drop"][:S], ref["drop"])
    assert np.array_equal(g["row_slot"][:ref["rows"]], ref["row_slot"])


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (5, 2, 3), (512, 2, 8), (1025, 1, 7), (3000, 8, 256),
                                   (4096, 2, 64), (20000, 3, 17)])
def test_permute_random(T, k, E):
    rng = np.random.default_rng(T * 31 + E)
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)])
    S = T * k
    for cap in (-1, 0, 1, max(1, S // E), S):
        g = permute_on_gpu(idx, E, cap)
        ref = O.permute(idx, E, None if cap < 0 else cap)
        assert_permute_equal(g, ref, S, E)


def test_permute_skewed_and_forced():
    """Skew (most slots on one expert) and the forced uniform assignment
    (slot s -> expert s mod E, MegaBlocks section 5)."""
    T, k, E = 3333, 2, 8
    rng = np.random.default_rng(1)
    idx = np.where(rng.random((T, k)) < 0.8, 0, rng.integers(1, E, size=(T, k)))
    idx[:, 1] = np.where(idx[:, 1] == idx[:, 0], (idx[:, 0] + 1) % E, idx[:, 1])
    for cap in (-1, 512, 2000):
        assert_permute_equal(permute_on_gpu(idx, E, cap), O.permute(idx, E, None if cap < 0 else cap),
                             T * k, E)
    forced = (np.arange(T * k) % E).reshape(T, k)
    assert_permute_equal(permute_on_gpu(forced, E, -1), O.permute(forced, E, None), T * k, E)


def test_permute_bad_expert_id_sets_error_bit():
    """An id outside [0, E) is reported in the device error word; the slot is
    marked dropped and nothing is written out of bounds."""
    idx = np.array([[0, 1], [2, 9], [3, 1]])
    g = permute_on_gpu(idx, 4, -1)
    assert g["err"] & abi.DEVERR_EXPERT_RANGE
    assert g["slot_to_row"][3] == -1 and g["drop"][3] == 1


def test_gather_ffn_combine_entry_points():
    T, d, E, k, F = 400, 256, 8, 2, 256
    inp = small_case("s", T=T, d=d, E=E, k=k, F=F, act="swiglu", seed=21)
    x = inp.x.to(DEV)
    idx, w, aux, logits, probs = route_on_gpu(x, inp.wg.to(DEV), None, T, d, E, k)
    pm_ref = O.permute(npi(idx).astype(np.int64), E, None)
    R = pm_ref["rows"]
    row_slot = torch.from_numpy(pm_ref["row_slot"]).to(DEV)
    seg = torch.from_numpy(pm_ref["seg_offsets"]).to(DEV)
    s2r = torch.from_numpy(pm_ref["slot_to_row"]).to(DEV)
    ws = new_ws(256)
    x_perm = torch.empty(R, d, dtype=torch.bfloat16, device=DEV)
    abi.moe_gather(x, T, d, k, row_slot, seg, E, R, x_perm, ws)
    h = torch.empty(R, F, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(R, d, dtype=torch.bfloat16, device=DEV)
    abi.moe_expert_ffn(x_perm, inp.w1.to(DEV), inp.w3.to(DEV), inp.w2.to(DEV), abi.MOE_ACT_SWIGLU,
                       R, d, F, E, seg, h, y, ws)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    abi.moe_combine(y, w, s2r, T, d, k, R, out, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    xp_ref = O.gather(np32(inp.x), pm_ref["row_slot"], k)
    assert np.array_equal(np32(x_perm), xp_ref)
    w1, w3, w2 = ExpertWeights(inp.w1), ExpertWeights(inp.w3), ExpertWeights(inp.w2)
    # h: activation output before the down projection
    h_ref = np.zeros((R, F))
    for e in range(E):
        a, b = pm_ref["seg_offsets"][e], pm_ref["seg_offsets"][e + 1]
        if b > a:
            h_ref[a:b] = O.activation(xp_ref[a:b] @ w1[e].astype(np.float64), "swiglu",
                                      xp_ref[a:b] @ w3[e].astype(np.float64))
    assert max_err_ratio(np32(h), h_ref) <= 1e-2
    y_ref = O.expert_ffn(xp_ref, pm_ref["seg_offsets"], w1, w3, w2, "swiglu")
    assert max_err_ratio(np32(y), y_ref) <= TOL_BF16_OUT
    out_ref = O.combine(np32(y), np32(w), pm_ref["slot_to_row"], T, k)
    assert max_err_ratio(np32(out), out_ref) <= 1e-2


@pytest.mark.parametrize("act,d,F", [("swiglu", 256, 256), ("gelu", 256, 512), ("gelu", 384, 384),
                                     ("swiglu", 512, 128)])
def test_expert_ffn_segment_boundaries(act, d, F):
    """Segment sizes on both sides of the 64-row (M = 64 MMA) and 128-row
    tiles, empty experts, and slack rows past the last segment; the rows
    outside every segment are never written."""
    m = [0, 1, 63, 64, 65, 127, 128, 129, 192, 193, 255, 256, 257, 300, 0, 513]
    E = len(m)
    seg = np.concatenate([[0], np.cumsum(m)]).astype(np.int32)
    R = int(seg[-1]) + 77
    g = torch.Generator().manual_seed(d + F)
    x = torch.randn(R, d, generator=g).to(torch.bfloat16)
    w1 = (torch.randn(E, d, F, generator=g) * 0.05).to(torch.bfloat16)
    w3 = (torch.randn(E, d, F, generator=g) * 0.05).to(torch.bfloat16) if act == "swiglu" else None
    w2 = (torch.randn(E, F, d, generator=g) * 0.05).to(torch.bfloat16)
    sentinel = -3.0
    h = torch.full((R, F), sentinel, dtype=torch.bfloat16, device=DEV)
    y = torch.full((R, d), sentinel, dtype=torch.bfloat16, device=DEV)
    ws = new_ws(256)
    code = abi.MOE_ACT_SWIGLU if act == "swiglu" else abi.MOE_ACT_GELU
    abi.moe_expert_ffn(x.to(DEV), w1.to(DEV), None if w3 is None else w3.to(DEV), w2.to(DEV), code,
                       R, d, F, E, torch.from_numpy(seg).to(DEV), h, y, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    xs = np32(x)
    W1, W2 = ExpertWeights(w1), ExpertWeights(w2)
    W3 = ExpertWeights(w3) if w3 is not None else None
    y_ref = O.expert_ffn(xs[:seg[-1]], seg, W1, W3, W2, act)
    assert max_err_ratio(np32(y)[:seg[-1]], y_ref) <= TOL_BF16_OUT
    assert np.all(np32(y)[seg[-1]:] == sentinel) and np.all(np32(h)[seg[-1]:] == sentinel)


@pytest.mark.parametrize("act,d,F,m", [
    ("swiglu", 256, 256, [0, 1, 127, 128, 129, 255, 256, 257, 383, 384, 385, 600, 1000]),
    ("gelu", 512, 256, [0, 1, 127, 128, 129, 255, 256, 257, 383, 384, 385, 600, 1000]),
    ("swiglu", 256, 256, [1, 200, 256, 300, 700]),   # few tiles: half-width gate/up units
    ("gelu", 256, 512, [513, 0, 64, 1024]),
])
def test_expert_ffn_pair_tiles(act, d, F, m):
    """Row counts that select the CTA-pair kernel (256-row tiles, each CTA
    128 rows): segments on both sides of 128 (the second CTA has no valid
    rows) and 256, empty experts, a last wave split into half-width units,
    and slack rows past the last segment that are never written."""
    E = len(m)
    seg = np.concatenate([[0], np.cumsum(m)]).astype(np.int32)
    R = max(int(seg[-1]) + 77, 768 * E + 1)  # enough rows for the pair kernel
    g = torch.Generator().manual_seed(d + F + E)
    x = torch.randn(R, d, generator=g).to(torch.bfloat16)
    w1 = (torch.randn(E, d, F, generator=g) * 0.05).to(torch.bfloat16)
    w3 = (torch.randn(E, d, F, generator=g) * 0.05).to(torch.bfloat16) if act == "swiglu" else None
    w2 = (torch.randn(E, F, d, generator=g) * 0.05).to(torch.bfloat16)
    sentinel = -3.0
    h = torch.full((R, F), sentinel, dtype=torch.bfloat16, device=DEV)
    y = torch.full((R, d), sentinel, dtype=torch.bfloat16, device=DEV)
    ws = new_ws(256)
    code = abi.MOE_ACT_SWIGLU if act == "swiglu" else abi.MOE_ACT_GELU
    abi.moe_expert_ffn(x.to(DEV), w1.to(DEV), None if w3 is None else w3.to(DEV), w2.to(DEV), code,
                       R, d, F, E, torch.from_numpy(seg).to(DEV), h, y, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    xs = np32(x)
    W1, W2 = ExpertWeights(w1), ExpertWeights(w2)
    W3 = ExpertWeights(w3) if w3 is not None else None
    n = int(seg[-1])
    h_ref = O.expert_hidden(xs[:n], seg, W1, W3, act)
    assert max_err_ratio(np32(h)[:n], h_ref) <= TOL_BF16_OUT
    y_ref = O.expert_ffn(xs[:n], seg, W1, W3, W2, act)
    assert max_err_ratio(np32(y)[:n], y_ref) <= TOL_BF16_OUT
    # every expert's rows, not only the largest values
    for e in range(E):
        a, b = int(seg[e]), int(seg[e + 1])
        if b > a:
            assert max_err_ratio(np32(y)[a:b], y_ref[a:b]) <= TOL_BF16_OUT, e
    assert np.all(np32(y)[n:] == sentinel) and np.all(np32(h)[n:] == sentinel)


@pytest.mark.parametrize("act,T,d,E,k,F,cf", [("swiglu", 700, 256, 8, 2, 512, 0.0),
                                             ("gelu", 555, 384, 16, 2, 384, 1.0),
                                             ("swiglu", 300, 256, 64, 8, 256, 0.0)])
def test_fused_gather_equals_gather_then_ffn(act, T, d, E, k, F, cf):
    """With MOE_LAYER_GATHER_IN_GEMM, moe_forward's up projection gathers x
    rows itself (tile::gather4). Its h and y must equal, bit for bit,
    moe_gather followed by moe_expert_ffn on the same permutation: the same
    products in the same order, only the A rows' source differs."""
    from mixture_experts_routing_route_b200 import MoeLayer
    inp = small_case("fused", T=T, d=d, E=E, k=k, F=F, act=act, cf=cf, seed=T + d)
    dv = {n: (None if t is None else t.to(DEV)) for n, t in
          (("x", inp.x), ("wg", inp.wg), ("w1", inp.w1), ("w3", inp.w3), ("w2", inp.w2), ("bias", inp.bias))}
    layer = MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], bias=dv["bias"], k=k, act=act,
                     capacity_factor=cf, gather_in_gemm=True)
    out, _ = layer.forward(dv["x"])
    plain = MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], bias=dv["bias"], k=k, act=act,
                     capacity_factor=cf)
    out_plain, _ = plain.forward(dv["x"])
    torch.cuda.synchronize()
    assert layer.device_error(T) == 0
    v = layer.views(T)
    assert v["x_perm"] is None
    R = int(v["seg_offsets"][-1].item())
    Rm = v["rows_max"]
    ws = new_ws(256)
    x_perm = torch.empty(Rm, d, dtype=torch.bfloat16, device=DEV)
    abi.moe_gather(dv["x"], T, d, k, v["row_slot"], v["seg_offsets"], E, Rm, x_perm, ws)
    h = torch.empty(Rm, F, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(Rm, d, dtype=torch.bfloat16, device=DEV)
    code = abi.MOE_ACT_SWIGLU if act == "swiglu" else abi.MOE_ACT_GELU
    abi.moe_expert_ffn(x_perm, dv["w1"], dv["w3"], dv["w2"], code, Rm, d, F, E, v["seg_offsets"], h, y, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    assert torch.equal(h[:R], v["h"][:R])
    assert torch.equal(y[:R], v["y_perm"][:R])
    assert torch.equal(out, out_plain)


def permute_binned_on_gpu(idx_np, E, cap):
    T, k = idx_np.shape
    S = T * k
    R = abi.moe_rows_max_binned(T, k, E, cap)
    t = lambda n: torch.full((max(n, 1),), -7, dtype=torch.int32, device=DEV)
    out = {"counts": t(E), "bins": t(E), "sorted_slot": t(S), "slot_to_row": t(S),
           "row_slot": t(R), "kept_counts": t(E), "seg_offsets": t(E + 1)}
    drop = torch.full((max(S, 1),), 7, dtype=torch.uint8, device=DEV)
    ws = new_ws(abi.moe_permute_workspace_size(T, k, E))
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).to(DEV)
    abi.moe_permute_binned(idx, T, k, E, cap, out["counts"], out["bins"], out["sorted_slot"],
                           out["slot_to_row"], out["row_slot"], drop, out["kept_counts"],
                           out["seg_offsets"], ws)
    torch.cuda.synchronize()
    res = {kk: npi(vv) for kk, vv in out.items()}
    res["drop"] = npi(drop)
    res["err"] = abi.moe_get_device_error(ws)
    return res


@pytest.mark.parametrize("T,k,E", [(5, 2, 3), (512, 2, 8), (1025, 1, 7), (3000, 8, 256), (20000, 3, 17)])
def test_permute_binned(T, k, E):
    """[E, C] bucket layout (MegaBlocks page, sections 4.3-4.6): bit-exact with
    the oracle for fixed capacities and for dynamic capacity (C = the largest
    count), single- and multi-CTA permute."""
    rng = np.random.default_rng(T * 7 + E)
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)])
    S = T * k
    for cap in (-1, 0, 1, max(1, S // E), S):
        g = permute_binned_on_gpu(idx, E, cap)
        ref = O.permute_binned(idx, E, None if cap < 0 else cap)
        assert g["err"] == 0
        for key in ("counts", "bins", "kept_counts"):
            assert np.array_equal(g[key][:E], ref[key]), (cap, key)
        assert np.array_equal(g["seg_offsets"][:E + 1], ref["seg_offsets"]), cap
        for key in ("sorted_slot", "slot_to_row"):
            assert np.array_equal(g[key][:S], ref[key]), (cap, key)
        assert np.array_equal(g["drop"][:S], ref["drop"]), cap
        assert np.array_equal(g["row_slot"][:ref["rows"]], ref["row_slot"]), cap


def test_permute_binned_skewed_dynamic():
    """80% of the slots on expert 0: the dynamic bin is expert 0's count and
    the other bins are mostly padding."""
    T, k, E = 3333, 2, 8
    rng = np.random.default_rng(1)
    idx = np.where(rng.random((T, k)) < 0.8, 0, rng.integers(1, E, size=(T, k)))
    idx[:, 1] = np.where(idx[:, 1] == idx[:, 0], (idx[:, 0] + 1) % E, idx[:, 1])
    g = permute_binned_on_gpu(idx, E, -1)
    ref = O.permute_binned(idx, E, None)
    assert g["err"] == 0 and g["seg_offsets"][1] == ref["bin"] == ref["counts"].max()
    assert np.array_equal(g["row_slot"][:ref["rows"]], ref["row_slot"])
    assert np.array_equal(g["slot_to_row"][:T * k], ref["slot_to_row"])


@pytest.mark.parametrize("T,d,dt", [(37, 128, "bf16"), (1000, 512, "f32"), (4096, 4096, "bf16")])
def test_router_jitter_matches_oracle(T, d, dt):
    """Philox4x32-10 multipliers and x * m (MegaBlocks page, section 5), bit
    for bit: the same generator and the same fp32 operations on both sides."""
    g = torch.Generator().manual_seed(T)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    x = torch.randn(T, d, generator=g).to(tdt)
    out = torch.empty(T, d, dtype=tdt, device=DEV)
    seed = 0x1234_5678_9ABC + T
    abi.moe_router_jitter(x.to(DEV), T, d, 0.01, seed, out)
    torch.cuda.synchronize()
    m = O.jitter_multipliers(T, d, 0.01, seed)
    ref = O.apply_jitter(np32(x), m, dt == "bf16")
    assert np.array_equal(np32(out), ref)


@pytest.mark.parametrize("T,E", [(33, 8), (4096, 64), (999, 7)])
def test_router_noise_matches_oracle(T, E):
    """Box-Muller normals from the same Philox words: fp32 on the GPU, float64
    in the oracle."""
    out = torch.empty(T, E, dtype=torch.float32, device=DEV)
    abi.moe_router_noise(T, E, 1.0 / E, 99 + T, out)
    torch.cuda.synchronize()
    ref = O.logit_noise(T, E, 1.0 / E, 99 + T)
    g = np32(out).astype(np.float64)
    assert np.all(np.abs(g - ref) <= 2e-6 * (1.0 + np.abs(ref) * E))


@pytest.mark.parametrize("T,d,E,k,dt,tau", [
    (1000, 1024, 8, 2, "bf16", 1.0),    # fused tensor-core router, KS split in a cluster
    (1000, 1024, 8, 2, "bf16", 0.6),    # ... at a temperature
    (19500, 512, 8, 2, "bf16", 2.0),    # persistent fused router (more tiles than SMs)
    (300, 512, 32, 4, "bf16", 1.0),     # fused, E = 32
    (300, 512, 32, 4, "bf16", 3.0),
    (513, 256, 64, 2, "bf16", 1.0),     # tensor cores (TMA Wg) + router_select + aux_reduce
    (513, 256, 64, 2, "bf16", 0.5),
    (300, 256, 128, 2, "bf16", 0.8),    # the same at E = 128 (4 experts per lane)
    (90, 64, 40, 4, "f32", 1.5),        # CUDA-core gate + router_select
    (200, 64, 4, 1, "f32", 1.0),        # fp32 E <= 8: the general path when noise / z-loss are asked
    (200, 64, 4, 1, "f32", 2.5),
])
def test_route_train(T, d, E, k, dt, tau):
    """moe_route_train: logits = x Wg + b + noise, softmax of logits / tau;
    top-k, weights, aux loss and the z-loss, against the oracle."""
    inp = small_case("rt", T=T, d=d, E=E, k=k, F=128, act="gelu", dtype=dt, bias="zipf", seed=T + E)
    noise = torch.empty(T, E, dtype=torch.float32, device=DEV)
    abi.moe_router_noise(T, E, 1.0 / E, 7, noise)
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    aux = torch.empty(1, dtype=torch.float32, device=DEV)
    z = torch.empty(1, dtype=torch.float32, device=DEV)
    logits = torch.empty(T, E, dtype=torch.float32, device=DEV)
    probs = torch.empty(T, E, dtype=torch.float32, device=DEV)
    ws = new_ws(abi.moe_route_workspace_size(T, d, E))
    abi.moe_route_train(inp.x.to(DEV), inp.wg.to(DEV), inp.bias.to(DEV), noise, T, d, E, k, idx, w,
                        aux, z, logits, probs, ws, temperature=tau)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    n64 = np32(noise).astype(np.float64)
    r = O.route(np32(inp.x), np32(inp.wg), inp.bias.numpy(), k, noise=n64, temperature=tau)
    g_logits = np32(logits)
    assert np.max(np.abs(g_logits - r["logits"])) <= 1e-5 * max(1.0, np.max(np.abs(r["logits"])))
    assert np.array_equal(npi(idx), O.topk_select(g_logits, k))
    assert rel_err(np32(probs), r["probs64"]) <= TOL_PROB_REL
    g_idx = npi(idx).astype(np.int64)
    assert rel_err(np32(w), O.renormalise(r["probs64"], g_idx)) <= TOL_PROB_REL
    aux_ref = O.aux_loss(r["probs64"], g_idx, E)
    assert abs(float(aux.item()) - aux_ref) <= TOL_AUX_REL * aux_ref
    assert abs(float(z.item()) - r["z"]) <= TOL_AUX_REL * r["z"]


@pytest.mark.parametrize("T,d,E,k,dt", [(1000, 1024, 8, 2, "bf16"), (513, 256, 64, 2, "bf16"),
                                        (200, 64, 4, 1, "f32")])
def test_route_train_at_unit_temperature_is_route(T, d, E, k, dt):
    """moe_route_train with no noise, no z-loss and tau = 1 gives moe_route's
    outputs bit for bit (the temperature multiplies by exactly 1)."""
    inp = small_case("rt1", T=T, d=d, E=E, k=k, F=128, act="gelu", dtype=dt, bias="zipf", seed=T + 3)
    x, wg, b = inp.x.to(DEV), inp.wg.to(DEV), inp.bias.to(DEV)
    ref = route_on_gpu(x, wg, b, T, d, E, k)
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    aux = torch.empty(1, dtype=torch.float32, device=DEV)
    logits = torch.empty(T, E, dtype=torch.float32, device=DEV)
    probs = torch.empty(T, E, dtype=torch.float32, device=DEV)
    ws = new_ws(abi.moe_route_workspace_size(T, d, E))
    abi.moe_route_train(x, wg, b, None, T, d, E, k, idx, w, aux, None, logits, probs, ws, temperature=1.0)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(ws) == 0
    for g, r in zip((idx, w, aux, logits, probs), ref):
        assert torch.equal(g, r)


@pytest.mark.parametrize("T,d,E,k,dt,tau,d_aux,d_z", [
    (1000, 1024, 8, 2, "bf16", 1.0, 0.01, 0.001),   # Mixtral's router shape at a reduced T
    (777, 512, 8, 2, "bf16", 0.7, 0.5, 0.0),        # temperature, no z-loss term
    (513, 256, 64, 2, "bf16", 1.3, 0.1, 0.02),      # E = 64: K = 128, two swizzle atoms
    (129, 256, 256, 8, "bf16", 1.0, 0.05, 0.01),    # E = 256, k = 8
    (300, 512, 24, 3, "bf16", 2.0, 0.0, 0.1),       # E not a multiple of 32, no aux term
    (200, 64, 40, 4, "f32", 1.0, 0.3, 0.05),        # fp32 (dx in fp32)
    (64, 384, 16, 4, "bf16", 1.0, 0.1, 0.01),       # tensor-core passes, E = 16, a half-width dx column tile
    (5, 256, 12, 2, "bf16", 1.0, 0.2, 0.0),         # five tokens, E = 12 (zero expert columns)
    (2500, 2048, 8, 2, "bf16", 1.3, 0.01, 0.001),   # dWg tiles shared by several blocks, a ragged last unit
    (333, 128, 5, 2, "bf16", 1.0, 0.1, 0.01),       # one column tile, E = 5, a ragged last unit
    (4100, 256, 16, 3, "bf16", 0.8, 0.05, 0.0),     # 2 column tiles x 65 units: 22 blocks per tile
    (5462, 256, 8, 3, "bf16", 1.0, 0.2, 0.0),       # 16386 picks: thread per token, counts over a grid barrier
    (9000, 128, 16, 2, "bf16", 1.0, 0.0, 0.01),     # thread per token without the aux term (no barrier)
    (2000, 1024, 32, 2, "bf16", 1.0, 0.05, 0.01),   # EC = 32: K = 64, one swizzle atom of [hi | lo]
    (1, 128, 8, 2, "bf16", 1.0, 0.1, 0.01),         # one token: one dx tile, one dWg unit, mostly padding
    (64, 256, 16, 1, "bf16", 1.0, 0.1, 0.0),        # exactly one 64-token dWg unit per column tile, k = 1
    (700, 384, 48, 4, "bf16", 0.9, 0.1, 0.0),       # EC = 64 with 16 zero columns; 128-column dx tiles
    (300, 64, 8, 2, "f32", 1.0, 0.1, 0.01),         # fp32, E = 8: CUDA-core passes
    (270000, 128, 8, 2, "bf16", 1.0, 0.01, 0.001),  # > 1024 x 256 tokens: grid-stride d_logits, 147 blocks on one tile
    (7001, 128, 24, 2, "bf16", 1.0, 0.2, 0.0),      # 14002 picks, E = 24: one counting block, warp-per-token d_logits
    (8192, 128, 20, 2, "bf16", 1.0, 0.1, 0.01),     # 16384 picks: the largest count taken by one block
])
def test_route_backward(T, d, E, k, dt, tau, d_aux, d_z):
    """moe_route_backward from the GPU's own forward (moe_route_train at tau)
    against the oracle's chain rule of that forward: d_logits, dx and d_wg;
    two runs give the same bits."""
    inp = small_case("rb", T=T, d=d, E=E, k=k, F=128, act="gelu", dtype=dt, bias="zipf", seed=T + E)
    x, wg, b = inp.x.to(DEV), inp.wg.to(DEV), inp.bias.to(DEV)
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    aux = torch.empty(1, dtype=torch.float32, device=DEV)
    logits = torch.empty(T, E, dtype=torch.float32, device=DEV)
    probs = torch.empty(T, E, dtype=torch.float32, device=DEV)
    ws = new_ws(abi.moe_route_workspace_size(T, d, E))
    abi.moe_route_train(x, wg, b, None, T, d, E, k, idx, w, aux, None, logits, probs, ws, temperature=tau)
    g = torch.from_numpy(np.random.default_rng(T).standard_normal((T, k)).astype(np.float32)).to(DEV)
    bws = new_ws(abi.moe_route_backward_workspace_size(T, d, E))
    outs = []
    for _ in range(2):
        d_logits = torch.empty(T, E, dtype=torch.float32, device=DEV)
        dx = torch.empty(T, d, dtype=x.dtype, device=DEV)
        d_wg = torch.empty(d, E, dtype=torch.float32, device=DEV)
        abi.moe_route_backward(x, wg, T, d, E, k, probs, logits if d_z else None, idx, w, g, d_aux, d_z,
                               tau, d_logits, dx, d_wg, bws)
        torch.cuda.synchronize()
        assert abi.moe_get_device_error(bws) == 0
        outs.append((d_logits, dx, d_wg))
    for a, c in zip(*outs):
        assert torch.equal(a, c)
    d_logits, dx, d_wg = outs[0]
    ref = O.route_backward_from(np32(probs).astype(np.float64), npi(idx), np32(w).astype(np.float64),
                                np32(logits).astype(np.float64), np32(inp.x), np32(inp.wg),
                                d_w=np32(g).astype(np.float64), d_aux=d_aux, d_z=d_z, temperature=tau)
    assert max_err_ratio(np32(d_logits), ref["d_logits"]) <= 1e-5
    assert max_err_ratio(np32(d_wg), ref["dwg"]) <= 1e-4
    assert max_err_ratio(np32(dx), ref["dx"]) <= (TOL_BF16_OUT if dt == "bf16" else 1e-5)


@pytest.mark.parametrize("T,d,E", [(3000, 1024, 8), (777, 512, 16), (700, 384, 48), (900, 256, 32)])
def test_route_backward_one_output(T, d, E):
    """With both dx and d_wg requested (bf16, E <= 16) the two tensor-core
    passes run in one launch; asked for one of them, each runs alone. Same
    arithmetic and the same dWg split, so the results are bit-identical."""
    k = 2
    inp = small_case("rb1", T=T, d=d, E=E, k=k, F=128, act="gelu", dtype="bf16", bias="zipf", seed=T + E)
    x, wg, b = inp.x.to(DEV), inp.wg.to(DEV), inp.bias.to(DEV)
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    aux = torch.empty(1, dtype=torch.float32, device=DEV)
    logits = torch.empty(T, E, dtype=torch.float32, device=DEV)
    probs = torch.empty(T, E, dtype=torch.float32, device=DEV)
    ws = new_ws(abi.moe_route_workspace_size(T, d, E))
    abi.moe_route_train(x, wg, b, None, T, d, E, k, idx, w, aux, None, logits, probs, ws)
    g = torch.from_numpy(np.random.default_rng(T).standard_normal((T, k)).astype(np.float32)).to(DEV)
    bws = new_ws(abi.moe_route_backward_workspace_size(T, d, E))
    res = {}
    for name, want_dx, want_wg in (("both", True, True), ("dx", True, False), ("wg", False, True)):
        dl = torch.empty(T, E, dtype=torch.float32, device=DEV)
        dx = torch.full((T, d), 7.0, dtype=x.dtype, device=DEV) if want_dx else None
        d_wg = torch.full((d, E), 7.0, dtype=torch.float32, device=DEV) if want_wg else None
        abi.moe_route_backward(x, wg, T, d, E, k, probs, logits, idx, w, g, 0.05, 0.01, 1.0, dl, dx, d_wg, bws)
        torch.cuda.synchronize()
        assert abi.moe_get_device_error(bws) == 0
        res[name] = (dl, dx, d_wg)
    assert torch.equal(res["both"][0], res["dx"][0]) and torch.equal(res["both"][0], res["wg"][0])
    assert torch.equal(res["both"][1], res["dx"][1])
    assert torch.equal(res["both"][2], res["wg"][2])
    ref = O.route_backward_from(np32(probs).astype(np.float64), npi(idx), np32(w).astype(np.float64),
                                np32(logits).astype(np.float64), np32(inp.x), np32(inp.wg),
                                d_w=np32(g).astype(np.float64), d_aux=0.05, d_z=0.01)
    assert max_err_ratio(np32(res["both"][2]), ref["dwg"]) <= 1e-4
    assert max_err_ratio(np32(res["both"][1]), ref["dx"]) <= TOL_BF16_OUT


def test_pair_gemm_repeats_on_one_workspace():
    """The CTA-pair GEMM hands out its tiles from a counter in the
    workspace's control block, reset by the last pair of each launch: three
    forwards on one workspace (six pair launches) give the same output bit
    for bit, and both counter words are zero afterwards."""
    from mixture_experts_routing_route_b200 import MoeLayer
    inp = small_case("rep", T=1600, d=256, E=4, k=2, F=256, act="swiglu", seed=44)
    layer = MoeLayer(inp.wg.to(DEV), inp.w1.to(DEV), inp.w2.to(DEV), w3=inp.w3.to(DEV), k=2, act="swiglu")
    x = inp.x.to(DEV)
    outs = []
    for _ in range(3):
        out, _ = layer.forward(x)
        outs.append(out.clone())
    torch.cuda.synchronize()
    assert layer.device_error(1600) == 0
    assert all(torch.equal(o, outs[0]) for o in outs[1:])
    ctl = layer.workspace(1600)[:256].view(torch.int32).cpu()
    assert int(ctl[5]) == 0 and int(ctl[6]) == 0  # next unit, pairs done
