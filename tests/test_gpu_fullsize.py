"""GPU parity at the workloads' full sizes, in the launch configuration
bench.py times (MoeLayer.forward -> moe_forward). Route and permute are
checked on every token / slot; the layer output on a seeded sample of tokens
that the oracle evaluates one by one (each sampled token's kept slots through
its experts' MLPs), plus every token whose slots were all dropped."""
import numpy as np
import pytest
import torch

from mixture_experts_routing_route_b200.inputs import CONFIGS, make_inputs
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
