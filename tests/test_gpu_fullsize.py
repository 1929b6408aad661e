"""GPU parity at the workloads' full sizes, in the launch configuration
bench.py times (MoeLayer.forward -> moe_forward).

* Route and permute on every token and slot.
* The gathered rows x_perm: every row an exact copy of its token.
* The layer output: every token for the T = 4096 and T = 16384 workloads; for
  the T = 32768 workloads, 4096 seeded tokens that the oracle evaluates one by
  one (each sampled token's kept slots through its experts' MLPs), plus every
  token whose slots were all dropped (exact zeros).
* The hidden rows h and the expert outputs y_perm stage-chained: for the
  largest and the smallest non-empty expert, every row of h against the
  oracle's hidden rows of the GPU's x_perm, and every row of y_perm against
  the oracle's MLP of those rows.

The float stages run on the GPU's routing (verified first): in a capacity
workload one flipped near tie would shift later arrival ranks."""
import numpy as np
import pytest
import torch

from workloads import CONFIGS, make_inputs
from oracle import moe_oracle as O
from tests.gpu_helpers import (check_topk_end_to_end, TOL_AUX_REL, TOL_BF16_OUT, TOL_PROB_REL, ExpertWeights,
                               device_inputs, max_err_ratio, np32, npi, rel_err)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ALL_TOKENS = ("mixtral", "fine_grained", "capacity_skew")
N_SAMPLE = 4096  # tokens of the T = 32768 workloads the oracle evaluates


def _check_expert_rows(v, pm, inp, sh):
    """h and y_perm of the largest and the smallest non-empty expert, every
    row, from the GPU's own x_perm (stage-chained)."""
    seg = pm["seg_offsets"].astype(np.int64)
    sizes = np.diff(seg)
    live = np.nonzero(sizes > 0)[0]
    experts = sorted({int(live[np.argmax(sizes[live])]), int(live[np.argmin(sizes[live])])})
    w1 = ExpertWeights(inp.w1)
    w3 = None if inp.w3 is None else ExpertWeights(inp.w3)
    w2 = ExpertWeights(inp.w2)
    for e in experts:
        a, b = int(seg[e]), int(seg[e + 1])
        xe = np32(v["x_perm"][a:b])
        one = [0, b - a]
        pick = lambda w: None if w is None else _One(w, e)  # noqa: E731
        h_ref = O.expert_hidden(xe, one, pick(w1), pick(w3), sh.act)
        h_got = np32(v["h"][a:b])
        assert max_err_ratio(h_got, h_ref) <= TOL_BF16_OUT, ("h", e)
        y_ref = O.expert_ffn(xe, one, pick(w1), pick(w3), pick(w2), sh.act)
        assert max_err_ratio(np32(v["y_perm"][a:b]), y_ref) <= TOL_BF16_OUT, ("y_perm", e)
    return experts


class _One:
    """Expert e of an [E, r, c] weight seen as a one-expert list."""

    def __init__(self, w, e):
        self.w, self.e = w, e

    def __getitem__(self, i):
        assert i == 0
        return self.w[self.e]


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
    bias = None if inp.bias is None else inp.bias.numpy()
    r = O.route(x, np32(inp.wg), bias, k)
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

    # every gathered row is an exact copy of its token's row
    R = pm["rows"]
    xp = np32(v["x_perm"][:R])
    assert np.array_equal(xp, x[pm["row_slot"].astype(np.int64) // k])
    del xp

    got = np32(out)
    all_dropped = np.nonzero(pm["drop"].reshape(T, k).all(axis=1))[0]
    if len(all_dropped):
        assert np.all(got[all_dropped] == 0.0)

    W = lambda w: None if w is None else ExpertWeights(w)  # noqa: E731
    if name in ALL_TOKENS:
        ref = O.forward(x, np32(inp.wg), bias, W(inp.w1), W(inp.w3), W(inp.w2), k, sh.act, sh.cf,
                        topk_idx=g_idx, topk_w=w_ref)["out"]
        err = max_err_ratio(got, ref)
    else:
        rng = np.random.default_rng(sh.seed)
        sample = np.sort(rng.choice(T, size=min(N_SAMPLE, T), replace=False))
        ref = O.forward_tokens(x, sample, g_idx, w_ref, pm["slot_to_row"], W(inp.w1), W(inp.w3),
                               W(inp.w2), sh.act)
        err = max_err_ratio(got[sample], ref)
    assert err <= TOL_BF16_OUT, err

    _check_expert_rows(v, pm, inp, sh)


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


@pytest.mark.parametrize("name", ["mixtral", "capacity_skew"])
def test_full_size_router_backward(name):
    """The router backward at full size from the GPU's own forward, against
    the oracle's chain rule (d_logits, dx and dWg): the Mixtral router (T =
    4096, d = 4096, E = 8, k = 2) and the capacity workload's (T = 16384,
    d = 1024, E = 64, k = 2: the tensor-core passes with K = 128)."""
    from mixture_experts_routing_route_b200 import _abi as abi
    sh = CONFIGS[name]
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
