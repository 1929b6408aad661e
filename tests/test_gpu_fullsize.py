"""GPU parity at the workloads' full sizes, in the launch configuration
bench.py times (MoeLayer.forward -> moe_forward). Route and permute are
checked on every token / slot; the layer output on a seeded sample of tokens
that the oracle evaluates one by one (each sampled token's kept slots through
its experts' MLPs), plus every token whose slots were all dropped."""
import numpy as np
import pytest
import torch

from workloads import CONFIGS, make_inputs
from oracle import moe_oracle as O
from tests.gpu_helpers import (check_topk_end_to_end, TOL_AUX_REL, TOL_BF16_OUT, TOL_PROB_REL, ExpertWeights,
                               device_inputs, max_err_ratio, np32, npi, rel_err)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

N_SAMPLE = 48


@pytest.mark.parametrize("name", ["mixtral", "fine_grained", "capacity_skew", "long_skewed",
                                  "long_skewed_cf"])
def test_full_size(name):
    from mixture_experts_routing_route_b200 import MoeLayer
    sh = CONFIGS[name]
    inp = make_inputs(sh)
    dv = device_inputs(inp)
    layer = MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], bias=dv["bias"], k=sh.k,
                     act=sh.act, capacity_factor=sh.cf)
    out, aux = layer.forward(dv["x"])
    torch.cuda.synchronize()
    assert layer.device_error(sh.T) == 0
    v = layer.views(sh.T)
    T, k, E = sh.T, sh.k, sh.E

    x = np32(inp.x)
    r = O.route(x, np32(inp.wg), None if inp.bias is None else inp.bias.numpy(), k)
    g_idx = npi(v["topk_idx"]).astype(np.int64)
    check_topk_end_to_end(g_idx, r)
    w_ref = O.renormalise(r["probs64"], g_idx)
    assert rel_err(np32(v["topk_w"]), w_ref) <= TOL_PROB_REL
    aux_ref = O.aux_loss(r["probs64"], g_idx, E)
    assert abs(float(aux.item()) - aux_ref) <= TOL_AUX_REL * aux_ref

    cap = O.capacity(sh.cf, k, T, E)
    pm = O.permute(g_idx, E, cap)
    for key in ("counts", "bins", "kept_counts", "seg_offsets", "sorted_slot", "slot_to_row"):
        assert np.array_equal(npi(v[key]), pm[key]), key
    assert np.array_equal(npi(v["drop"]), pm["drop"])
    assert np.array_equal(npi(v["row_slot"])[:pm["rows"]], pm["row_slot"])

    rng = np.random.default_rng(sh.seed)
    sample = np.sort(rng.choice(T, size=min(N_SAMPLE, T), replace=False))
    all_dropped = np.nonzero(pm["drop"].reshape(T, k).all(axis=1))[0]
    got = np32(out)
    if len(all_dropped):
        assert np.all(got[all_dropped] == 0.0)
    # gathered rows of the sampled tokens are exact copies (where a forward
    # keeps x_perm; the bf16 forward gathers inside the up projection)
    if v["x_perm"] is not None:
        rows = pm["slot_to_row"].reshape(T, k)[sample]
        xp = np32(v["x_perm"])
        for i, t in enumerate(sample):
            for rr in rows[i]:
                if rr >= 0:
                    assert np.array_equal(xp[rr], x[t])
    ref = O.forward_tokens(x, sample, g_idx, w_ref, pm["slot_to_row"], ExpertWeights(inp.w1),
                           None if inp.w3 is None else ExpertWeights(inp.w3),
                           ExpertWeights(inp.w2), sh.act)
    err = max_err_ratio(got[sample], ref)
    assert err <= TOL_BF16_OUT, err


@pytest.mark.parametrize("name", ["mixtral", "long_skewed_cf"])
def test_full_size_layout_variants_equal(name):
    """The padded-binned layout (dynamic or fixed capacity) and the gather
    inside the up projection change where rows live or where they are read
    from, not what is computed: at full size the layer output and aux loss
    are bit-identical to the default layout's."""
    from mixture_experts_routing_route_b200 import MoeLayer
    sh = CONFIGS[name]
    inp = make_inputs(sh)
    dv = device_inputs(inp)

    def run(**kw):
        layer = MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], bias=dv["bias"], k=sh.k,
                         act=sh.act, capacity_factor=sh.cf, **kw)
        out, aux = layer.forward(dv["x"])
        torch.cuda.synchronize()
        assert layer.device_error(sh.T) == 0
        res = (out.clone(), aux.clone())
        del layer
        torch.cuda.empty_cache()
        return res

    out0, aux0 = run()
    for kw in ({"binned": True}, {"gather_in_gemm": True}):
        out1, aux1 = run(**kw)
        assert torch.equal(out1, out0), kw
        assert torch.equal(aux1, aux0), kw


def test_full_size_combine_in_gemm_k1():
    """The Mixtral-shaped layer at top-1 (dropless, and with capacity 1.25):
    the combine in the down projection's epilogue gives the default path's
    output bit for bit at full size."""
    from mixture_experts_routing_route_b200 import MoeLayer
    sh = CONFIGS["mixtral"].with_(k=1)
    inp = make_inputs(sh)
    dv = device_inputs(inp)
    for cf in (0.0, 1.25):
        outs = []
        for comb in (False, True):
            layer = MoeLayer(dv["wg"], dv["w1"], dv["w2"], w3=dv["w3"], bias=dv["bias"], k=1,
                             act=sh.act, capacity_factor=cf, combine_in_gemm=comb)
            out = torch.full((sh.T, sh.d), float("nan"), dtype=dv["x"].dtype, device="cuda")
            layer.forward(dv["x"], out)
            torch.cuda.synchronize()
            assert layer.device_error(sh.T) == 0
            outs.append(out)
            del layer
        assert torch.equal(outs[0], outs[1]), cf
        torch.cuda.empty_cache()


def test_full_size_router_backward():
    """The router backward on the Mixtral router at full size (T = 4096,
    d = 4096, E = 8, k = 2) from the GPU's own forward, against the oracle's
    chain rule: d_logits, dx and dWg."""
    from mixture_experts_routing_route_b200 import _abi as abi
    sh = CONFIGS["mixtral"]
    inp = make_inputs(sh)
    T, d, E, k = sh.T, sh.d, sh.E, sh.k
    x, wg = inp.x.to("cuda"), inp.wg.to("cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    aux = torch.empty(1, dtype=torch.float32, device="cuda")
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    probs = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ws = torch.empty(abi.moe_route_workspace_size(T, d, E), dtype=torch.uint8, device="cuda")
    abi.moe_workspace_init(ws)
    abi.moe_route_train(x, wg, None, None, T, d, E, k, idx, w, aux, None, logits, probs, ws)
    g = torch.from_numpy(np.random.default_rng(5).standard_normal((T, k)).astype(np.float32)).to("cuda")
    d_logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    dx = torch.empty(T, d, dtype=x.dtype, device="cuda")
    d_wg = torch.empty(d, E, dtype=torch.float32, device="cuda")
    bws = torch.empty(abi.moe_route_backward_workspace_size(T, d, E), dtype=torch.uint8, device="cuda")
    abi.moe_workspace_init(bws)
    abi.moe_route_backward(x, wg, T, d, E, k, probs, logits, idx, w, g, 0.01, 0.001, 1.0, d_logits, dx,
                           d_wg, bws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_error(bws) == 0
    ref = O.route_backward_from(np32(probs).astype(np.float64), npi(idx), np32(w).astype(np.float64),
                                np32(logits).astype(np.float64), np32(inp.x), np32(inp.wg),
                                d_w=np32(g).astype(np.float64), d_aux=0.01, d_z=0.001)
    assert max_err_ratio(np32(d_logits), ref["d_logits"]) <= 1e-5
    assert max_err_ratio(np32(d_wg), ref["dwg"]) <= 1e-4
    assert max_err_ratio(np32(dx), ref["dx"]) <= TOL_BF16_OUT
