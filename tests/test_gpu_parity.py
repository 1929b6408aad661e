"""GPU parity: the whole-layer forward (the path bench.py times) against the
CPU oracle, stage by stage, on reduced sizes that span several tiles and a
ragged tail.

Checks are stage-chained: each oracle stage is fed the GPU's own input to that
stage, so integer stages are compared bit-exactly and float stages with the
stated tolerances. End-to-end top-k agreement is checked on tokens the oracle
does not flag as near-ties.
"""
import numpy as np
import pytest
import torch

from workloads import small_case, worked_example_a, make_inputs, CONFIGS
from oracle import moe_oracle as O
from tests.gpu_helpers import (check_topk_end_to_end, TOL_AUX_REL, TOL_BF16_OUT, TOL_F32_OUT, TOL_PROB_REL, ExpertWeights,
                               device_inputs, max_err_ratio, np32, npi, rel_err)

pytestmark = pytest.mark.gpu

CASES = {
    # name: (T, d, E, k, F, act, dtype, cf, bias)
    "swiglu_e8_ragged": (300, 256, 8, 2, 384, "swiglu", "bf16", 0.0, "none"),
    "swiglu_multi_mtile": (1000, 512, 4, 2, 512, "swiglu", "bf16", 0.0, "none"),
    "gelu_capacity_zipf": (1000, 256, 16, 2, 512, "gelu", "bf16", 1.0, "zipf"),
    "gelu_n128_paths": (333, 384, 8, 2, 384, "gelu", "bf16", 0.0, "none"),
    "router_e256_k8": (200, 256, 256, 8, 256, "swiglu", "bf16", 0.0, "none"),
    "router_e64_capacity": (700, 128, 64, 2, 256, "gelu", "bf16", 1.25, "zipf"),
    "single_expert": (130, 128, 1, 1, 128, "swiglu", "bf16", 0.0, "none"),
    "k_equals_e": (150, 128, 4, 4, 256, "swiglu", "bf16", 0.0, "none"),
    "expert0_skew_cf": (900, 256, 8, 2, 256, "swiglu", "bf16", 1.25, "expert0"),
    "f32_swiglu": (200, 64, 6, 2, 96, "swiglu", "f32", 0.0, "none"),
    "f32_gelu_capacity": (256, 64, 4, 1, 128, "gelu", "f32", 1.25, "none"),
    # >= 768 slots per expert: the CTA-pair grouped GEMM (256-row tiles)
    "pair_gelu_capacity_zipf": (3200, 256, 8, 2, 512, "gelu", "bf16", 1.25, "zipf"),
    "pair_swiglu_skew_cf": (1600, 256, 4, 2, 256, "swiglu", "bf16", 1.0, "expert0"),
    "pair_swiglu_dropless": (1600, 512, 4, 2, 768, "swiglu", "bf16", 0.0, "none"),
}


def run_layer(inp):
    from mixture_experts_routing_route_b200 import MoeLayer
    sh = inp.shape
    dv = device_inputs(inp)
    layer = MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], bias=dv["bias"], k=sh.k,
                     act=sh.act, capacity_factor=sh.cf)
    out, aux = layer.forward(dv["x"])
    torch.cuda.synchronize()
    err = layer.device_error(sh.T)
    v = layer.views(sh.T)
    return layer, out, aux, v, err


def check_layer(inp, n_sample=None):
    sh = inp.shape
    T, k, E = sh.T, sh.k, sh.E
    layer, out, aux, v, err = run_layer(inp)
    assert err == 0, f"device error bits {err}"
    x = np32(inp.x)
    wg = np32(inp.wg)
    bias = None if inp.bias is None else inp.bias.numpy()
    r = O.route(x, wg, bias, k)

    # ---- route: top-k on the GPU's own fp32 logits is the oracle's top-k of them
    g_idx = npi(v["topk_idx"]).astype(np.int64)
    g_w = np32(v["topk_w"])
    # logits are not dumped by moe_forward; re-derive the decision check end to end
    check_topk_end_to_end(g_idx, r)
    w_ref = O.renormalise(r["probs64"], g_idx)
    assert rel_err(g_w, w_ref) <= TOL_PROB_REL, rel_err(g_w, w_ref)
    aux_ref = O.aux_loss(r["probs64"], g_idx, E)
    assert abs(float(aux.item()) - aux_ref) <= TOL_AUX_REL * abs(aux_ref), (float(aux.item()), aux_ref)
    assert abs(float(v["aux"].item()) - aux_ref) <= TOL_AUX_REL * abs(aux_ref)

    # ---- permute on the GPU's routing: bit-exact
    cap = O.capacity(sh.cf, k, T, E)
    assert v["capacity"] == (-1 if cap is None else cap)
    pm = O.permute(g_idx, E, cap)
    for key in ("counts", "bins", "kept_counts", "seg_offsets", "sorted_slot", "slot_to_row"):
        assert np.array_equal(npi(v[key]), pm[key]), key
    assert np.array_equal(npi(v["drop"]), pm["drop"])
    R = pm["rows"]
    assert np.array_equal(npi(v["row_slot"])[:R], pm["row_slot"])

    # ---- gather: bit-exact copy of rows (fp32 writes x_perm; bf16 gathers
    # inside the up projection, checked through y below)
    xp = O.gather(x, pm["row_slot"], k)
    if v["x_perm"] is not None:
        assert np.array_equal(np32(v["x_perm"])[:R], xp)

    # ---- expert FFN on the GPU's gathered rows
    w1, w2 = ExpertWeights(inp.w1), ExpertWeights(inp.w2)
    w3 = None if inp.w3 is None else ExpertWeights(inp.w3)
    y_ref = O.expert_ffn(xp, pm["seg_offsets"], w1, w3, w2, sh.act)
    y_gpu = np32(v["y_perm"])[:R]
    tol = TOL_BF16_OUT if sh.dtype == "bf16" else TOL_F32_OUT
    assert max_err_ratio(y_gpu, y_ref) <= tol, max_err_ratio(y_gpu, y_ref)

    # ---- combine on the GPU's y and weights
    out_ref_chain = O.combine(y_gpu, g_w, npi(v["slot_to_row"]), T, k)
    assert max_err_ratio(np32(out), out_ref_chain) <= tol
    # ---- whole layer from the oracle's own FFN of the GPU's routing
    out_ref = O.combine(y_ref, w_ref, pm["slot_to_row"], T, k)
    e2e = max_err_ratio(np32(out), out_ref)
    assert e2e <= tol, e2e
    # dropped-everywhere tokens are exactly zero
    all_dropped = pm["drop"].reshape(T, k).all(axis=1)
    assert np.all(np32(out)[all_dropped] == 0.0)
    return {"e2e_err": e2e, "rows": R}


@pytest.mark.parametrize("name", sorted(CASES))
def test_layer_small(name):
    T, d, E, k, F, act, dt, cf, bias = CASES[name]
    inp = small_case(name, T=T, d=d, E=E, k=k, F=F, act=act, dtype=dt, cf=cf, bias=bias,
                     seed=11 + len(name))
    check_layer(inp)


def test_tiny_fp32_config():
    check_layer(make_inputs(CONFIGS["tiny_fp32"]))


def test_worked_example_a_counts():
    """MegaBlocks page section 2: 8 tokens, 4 experts, top-1 -> counts 3/0/4/1."""
    inp = worked_example_a()
    layer, out, aux, v, err = run_layer(inp)
    assert err == 0
    assert npi(v["topk_idx"])[:, 0].tolist() == inp.extra["ids"]
    assert npi(v["counts"]).tolist() == [3, 0, 4, 1]
    assert npi(v["bins"]).tolist() == [3, 3, 7, 8]
    assert np.all(np32(v["topk_w"]) == 1.0)
    check_layer(inp)


def test_all_slots_dropped():
    """cf small enough that C = int(cf*k*T/E) = 0: every output row is zero."""
    inp = small_case("drop_all", T=64, d=128, E=4, k=1, F=128, act="gelu", cf=0.05)
    assert O.capacity(0.05, 1, 64, 4) == 0
    layer, out, aux, v, err = run_layer(inp)
    assert err == 0
    assert int(v["seg_offsets"][-1].item()) == 0
    assert torch.count_nonzero(out).item() == 0
    assert np.all(npi(v["drop"]) == 1)


def test_empty_batch():
    inp = small_case("empty", T=0, d=128, E=4, k=2, F=128, act="swiglu")
    layer, out, aux, v, err = run_layer(inp)
    assert err == 0 and out.shape == (0, 128)
    assert float(aux.item()) == 0.0


def test_repeat_is_deterministic():
    inp = small_case("det", T=513, d=256, E=8, k=2, F=256, act="swiglu", seed=3)
    _, out1, aux1, _, _ = run_layer(inp)
    _, out2, aux2, _, _ = run_layer(inp)
    assert torch.equal(out1, out2) and torch.equal(aux1, aux2)


@pytest.mark.parametrize("T,d,E,k,F,act,dt,cf,bias", [
    (700, 256, 8, 2, 512, "swiglu", "bf16", 0.0, "none"),      # dynamic capacity (no drop)
    (900, 256, 8, 2, 256, "swiglu", "bf16", 0.0, "expert0"),   # dynamic, skewed: big padding
    (1000, 256, 16, 2, 512, "gelu", "bf16", 1.0, "zipf"),      # fixed capacity with drops
    (256, 64, 4, 1, 128, "gelu", "f32", 1.25, "none"),         # fp32, fixed capacity
    (200, 64, 6, 2, 96, "swiglu", "f32", 0.0, "none"),         # fp32, dynamic
])
def test_layer_binned(T, d, E, k, F, act, dt, cf, bias):
    """The [E, C, hs] bucket layout (MOE_LAYER_BINNED): the same output as the
    default layout, bit for bit; the bucket's rows (zero padding included) and
    the expert outputs of the kept rows match the oracle's binned stages."""
    from mixture_experts_routing_route_b200 import MoeLayer
    inp = small_case("binned", T=T, d=d, E=E, k=k, F=F, act=act, dtype=dt, cf=cf, bias=bias,
                     seed=T + E)
    dv = device_inputs(inp)
    mk = lambda b: MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], bias=dv["bias"], k=k,
                            act=act, capacity_factor=cf, binned=b)
    lb, ld = mk(True), mk(False)
    out_b, aux_b = lb.forward(dv["x"])
    out_d, aux_d = ld.forward(dv["x"])
    torch.cuda.synchronize()
    assert lb.device_error(T) == 0 and ld.device_error(T) == 0
    assert torch.equal(out_b, out_d) and torch.equal(aux_b, aux_d)
    v = lb.views(T)
    g_idx = npi(v["topk_idx"]).astype(np.int64)
    cap = O.capacity(cf, k, T, E)
    bn = O.permute_binned(g_idx, E, cap)
    assert int(v["seg_offsets"][1].item()) == bn["bin"]
    assert np.array_equal(npi(v["row_slot"])[:bn["rows"]], bn["row_slot"])
    assert np.array_equal(npi(v["slot_to_row"]), bn["slot_to_row"])
    xb = O.gather_binned(np32(inp.x), bn["row_slot"], k)
    assert np.array_equal(np32(v["x_perm"])[:bn["rows"]], xb)
    w1, w2 = ExpertWeights(inp.w1), ExpertWeights(inp.w2)
    w3 = None if inp.w3 is None else ExpertWeights(inp.w3)
    y_ref = O.expert_ffn_binned(xb, bn["kept_counts"], bn["bin"], w1, w3, w2, act)
    live = bn["row_slot"] >= 0
    tol = TOL_BF16_OUT if dt == "bf16" else TOL_F32_OUT
    assert max_err_ratio(np32(v["y_perm"])[:bn["rows"]][live], y_ref[live]) <= tol


@pytest.mark.parametrize("T,d,E,F,act,cf,bias,binned,gig", [
    (700, 256, 8, 512, "swiglu", 0.0, "none", False, False),      # dropless
    (1000, 256, 16, 512, "gelu", 1.0, "zipf", False, False),      # capacity drops: zeroed rows
    (900, 256, 8, 256, "swiglu", 1.25, "expert0", True, False),   # bucket layout
    (1000, 256, 16, 512, "gelu", 1.0, "zipf", False, True),       # gather in the up projection too
    (333, 384, 8, 384, "gelu", 0.0, "none", False, False),        # d % 256 != 0: 128-column tiles
    (300, 256, 8, 256, "swiglu", 0.02, "none", False, False),     # C = 0: every token dropped
    (3200, 256, 4, 256, "swiglu", 0.0, "none", False, False),     # CTA-pair GEMMs, dropless
    (3200, 256, 4, 512, "gelu", 1.0, "expert0", True, False),     # CTA pairs, bucket layout, drops
])
def test_layer_combine_in_gemm(T, d, E, F, act, cf, bias, binned, gig):
    """k = 1: the combine in the down projection's epilogue
    (MOE_LAYER_COMBINE_IN_GEMM) writes every output row, the default path's
    output bit for bit, zero for dropped tokens, within the bf16 tolerance
    of the oracle."""
    from mixture_experts_routing_route_b200 import MoeLayer
    inp = small_case("comb", T=T, d=d, E=E, k=1, F=F, act=act, dtype="bf16", cf=cf, bias=bias,
                     seed=T + E)
    dv = device_inputs(inp)
    mk = lambda c: MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], bias=dv["bias"], k=1, act=act,
                            capacity_factor=cf, binned=binned and c, gather_in_gemm=gig and c,
                            combine_in_gemm=c)
    lc, ld = mk(True), mk(False)
    out_c = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")  # rows left unwritten stay NaN
    lc.forward(dv["x"], out_c)
    out_d, aux_d = ld.forward(dv["x"])
    torch.cuda.synchronize()
    assert lc.device_error(T) == 0 and ld.device_error(T) == 0
    assert torch.equal(out_c, out_d)
    v = lc.views(T)
    assert v["y_perm"] is None
    # against the oracle, from the GPU's routing
    g_idx = npi(v["topk_idx"]).astype(np.int64)
    r = O.route(np32(inp.x), np32(inp.wg), None if inp.bias is None else inp.bias.numpy(), 1)
    w_ref = O.renormalise(r["probs64"], g_idx)
    pm = O.permute(g_idx, E, O.capacity(cf, 1, T, E))
    xp = O.gather(np32(inp.x), pm["row_slot"], 1)
    w1, w2 = ExpertWeights(inp.w1), ExpertWeights(inp.w2)
    w3 = None if inp.w3 is None else ExpertWeights(inp.w3)
    y_ref = O.expert_ffn(xp, pm["seg_offsets"], w1, w3, w2, act)
    out_ref = O.combine(y_ref, w_ref, pm["slot_to_row"], T, 1)
    assert max_err_ratio(np32(out_c), out_ref) <= TOL_BF16_OUT
    dropped = pm["drop"].reshape(T, 1).all(axis=1)
    assert np.all(np32(out_c)[dropped] == 0.0)


@pytest.mark.parametrize("tau", [1.0, 1.7])
def test_layer_training_router_inputs(tau):
    """The router reads jittered x and adds logit noise (and, tau != 1, runs
    its softmax at that temperature) while the experts read x; the z-loss
    comes back through the views."""
    from mixture_experts_routing_route_b200 import MoeLayer, _abi as abi
    T, d, E, k, F = 700, 256, 8, 2, 256
    inp = small_case("train", T=T, d=d, E=E, k=k, F=F, act="swiglu", seed=77)
    dv = device_inputs(inp)
    xj = torch.empty_like(dv["x"])
    abi.moe_router_jitter(dv["x"], T, d, 0.01, 5, xj)
    noise = torch.empty(T, E, dtype=torch.float32, device="cuda")
    abi.moe_router_noise(T, E, 1.0 / E, 6, noise)
    layer = MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], k=k, act="swiglu", z_loss=True,
                     router_temperature=tau)
    out, aux = layer.forward(dv["x"], x_router=xj, logit_noise=noise)
    torch.cuda.synchronize()
    assert layer.device_error(T) == 0
    v = layer.views(T)
    xj_ref = O.apply_jitter(np32(inp.x), O.jitter_multipliers(T, d, 0.01, 5), True)
    assert np.array_equal(np32(xj), xj_ref)
    r = O.route(xj_ref, np32(inp.wg), None, k, noise=np32(noise).astype(np.float64), temperature=tau)
    g_idx = npi(v["topk_idx"]).astype(np.int64)
    check_topk_end_to_end(g_idx, r)
    w_ref = O.renormalise(r["probs64"], g_idx)
    assert rel_err(np32(v["topk_w"]), w_ref) <= TOL_PROB_REL
    assert abs(float(v["z_loss"].item()) - r["z"]) <= TOL_AUX_REL * r["z"]
    pm = O.permute(g_idx, E, None)
    xp = O.gather(np32(inp.x), pm["row_slot"], k)      # the experts see x, not the jittered x
    y_ref = O.expert_ffn(xp, pm["seg_offsets"], ExpertWeights(inp.w1), ExpertWeights(inp.w3),
                         ExpertWeights(inp.w2), "swiglu")
    out_ref = O.combine(y_ref, w_ref, pm["slot_to_row"], T, k)
    assert max_err_ratio(np32(out), out_ref) <= TOL_BF16_OUT
