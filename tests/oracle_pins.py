"""Pins for the CPU oracle: checks against facts the pages and mathematics
fix, not against the oracle's own formulas.

Each ``pin_*`` takes the oracle namespace ``o`` and raises AssertionError when
the oracle is wrong. tests/test_oracle_pins.py runs every pin on the real
oracle; tests/test_oracle_mutations.py plants mistakes in a copy of the oracle
and checks that some pin fails for each of them.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as Fn

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------
# brute-force helpers (pure Python loops on tiny inputs)
# ----------------------------------------------------------------------------

def _bf_topk(row, k):
    """k largest, largest first, ties to the lower index, by explicit selection."""
    taken = []
    for _ in range(k):
        best = None
        for e, v in enumerate(row):
            if e in taken:
                continue
            if best is None or v > row[best]:
                best = e
        taken.append(best)
    return taken


def _bf_permute(flat, E, cap):
    """Counting, ranks, drops and rows by walking the slots in arrival order."""
    seen = [0] * E
    rank = []
    for e in flat:
        rank.append(seen[e])
        seen[e] += 1
    counts = seen
    bins = list(itertools.accumulate(counts))
    buckets = [[] for _ in range(E)]
    for s, e in enumerate(flat):
        buckets[e].append(s)
    sorted_slot = [s for b in buckets for s in b]
    drop = [cap is not None and r >= cap for r in rank]
    kept = [min(c, cap) if cap is not None else c for c in counts]
    seg = [0]
    for c in kept:
        seg.append(seg[-1] + c)
    slot_to_row = [-1 if drop[s] else seg[e] + rank[s] for s, e in enumerate(flat)]
    return counts, bins, sorted_slot, rank, drop, kept, seg, slot_to_row


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------

def pin_example_a(o):
    """MegaBlocks page section 2: counts 3/0/4/1 from the forced routing."""
    g = _golden("worked_example_a.json")
    ids = [2, 0, 2, 3, 0, 2, 0, 2]
    x = np.zeros((8, 4))
    for t, e in enumerate(ids):
        x[t, e] = 5.0
    r = o.route(x, np.eye(4), None, 1)
    assert r["topk_idx"][:, 0].tolist() == ids
    assert np.all(r["topk_w"] == 1.0)
    pm = o.permute(r["topk_idx"], 4, o.capacity(0.0, 1, 8, 4))
    assert pm["counts"].tolist() == g["counts"]
    assert pm["bins"].tolist() == list(itertools.accumulate(g["counts"]))
    assert np.diff(pm["seg_offsets"]).tolist() == g["gemm_rows"]


def pin_example_b(o):
    """ops-transformer blog 原理: picks experts 0 and 6, weights softmax([0.9, 0.7])."""
    g = _golden("worked_example_b.json")
    a = 1.0 / (1.0 + math.exp(-(0.9 - 0.7)))    # closed form of softmax([0.9,0.7])[0]
    for seed in range(20):
        rng = _rng(seed)
        s = rng.uniform(-3.0, g["filler_upper_bound"] - 1e-3, size=g["E"])
        for e, v in g["known_scores"].items():
            s[int(e)] = v
        r = o.route(s[None, :], np.eye(g["E"]), None, g["k"])
        assert r["topk_idx"][0].tolist() == g["selected"]
        w = r["topk_w64"][0]
        assert abs(w[0] - a) < 1e-12 and abs(w[1] - (1 - a)) < 1e-12
    assert abs(a - 0.549834) < 5e-7


def pin_topk_vs_torch(o):
    """Top-k on tie-free inputs equals torch.topk (largest first)."""
    rng = _rng(1)
    for E, k in [(4, 1), (8, 2), (64, 2), (256, 8), (5, 5)]:
        l = rng.standard_normal((50, E)).astype(np.float32)
        ref = torch.topk(torch.from_numpy(l), k, dim=1).indices.numpy()
        assert np.array_equal(o.topk_select(l, k), ref)


def pin_topk_ties(o):
    """Exact ties go to the lower expert index (brute-force selection)."""
    rng = _rng(2)
    for _ in range(200):
        E = int(rng.integers(2, 9))
        k = int(rng.integers(1, E + 1))
        row = rng.integers(-2, 3, size=E).astype(np.float32)  # many exact ties
        assert o.topk_select(row[None, :], k)[0].tolist() == _bf_topk(row.tolist(), k)
    z = np.array([[0.0, -0.0, 0.0, -0.0]], dtype=np.float32)  # +0 and -0 compare equal
    assert o.topk_select(z, 2)[0].tolist() == [0, 1]


def pin_softmax_vs_torch(o):
    rng = _rng(3)
    l = rng.standard_normal((40, 16)) * 4
    ref = torch.softmax(torch.from_numpy(l), dim=1).numpy()
    assert np.allclose(o.softmax_rows(l), ref, rtol=1e-13, atol=0)
    assert np.allclose(o.softmax_rows(l + 123.0), ref, rtol=1e-12, atol=0)


def pin_renormalise(o):
    rng = _rng(4)
    x = rng.standard_normal((30, 16))
    wg = rng.standard_normal((16, 8))
    for k in (1, 2, 3, 8):
        r = o.route(x, wg, None, k)
        assert np.allclose(r["topk_w64"].sum(1), 1.0, rtol=0, atol=1e-14)
        if k == 1:
            assert np.all(r["topk_w"] == 1.0)
        # weights are the selected probabilities scaled by one factor per token
        sel = np.take_along_axis(torch.softmax(torch.from_numpy(x @ wg), 1).numpy(),
                                 r["topk_idx"].astype(np.int64), 1)
        assert np.allclose(r["topk_w64"], sel / sel.sum(1, keepdims=True), rtol=1e-12)
    # changing an unselected logit changes nothing after renormalisation
    l = np.array([[3.0, 1.0, 2.5, -1.0]])
    l2 = l.copy()
    l2[0, 3] = 0.9
    w1 = o.renormalise(o.softmax_rows(l), [[0, 2]])
    w2 = o.renormalise(o.softmax_rows(l2), [[0, 2]])
    assert np.allclose(w1, w2, rtol=1e-14)


def pin_aux(o):
    """Balanced routing with uniform probabilities gives 1; collapse gives E;
    small cases match a double loop."""
    E, T, k = 4, 8, 2
    probs = np.full((T, E), 1.0 / E)
    idx = np.array([[t % E, (t + 1) % E] for t in range(T)])
    assert abs(o.aux_loss(probs, idx, E) - 1.0) < 1e-15
    onehot = np.zeros((T, E))
    onehot[:, 2] = 1.0
    assert abs(o.aux_loss(onehot, np.full((T, 1), 2), E) - E) < 1e-15
    rng = _rng(5)
    for _ in range(20):
        E = int(rng.integers(2, 7))
        T = int(rng.integers(1, 9))
        k = int(rng.integers(1, E + 1))
        p = rng.random((T, E))
        p /= p.sum(1, keepdims=True)
        idx = np.array([rng.permutation(E)[:k] for _ in range(T)])
        tot = 0.0
        for i in range(E):
            f = sum(1 for t in range(T) for j in range(k) if idx[t][j] == i) / (T * k)
            P = sum(p[t][i] for t in range(T)) / T
            tot += f * P
        assert abs(o.aux_loss(p, idx, E) - E * tot) < 1e-12


def pin_capacity(o):
    for c in _golden("capacity_values.json")["cases"]:
        assert o.capacity(c["cf"], c["k"], c["T"], c["E"]) == c["C"], c
    assert o.capacity(0.0, 2, 100, 4) is None
    assert o.sort_end_bit(1) == 1 and o.sort_end_bit(2) == 1
    assert o.sort_end_bit(8) == 3 and o.sort_end_bit(64) == 6
    assert o.sort_end_bit(65) == 7 and o.sort_end_bit(256) == 8


def pin_permute_bruteforce(o):
    """Every capacity on tiny inputs matches the arrival-order walk."""
    rng = _rng(6)
    for _ in range(60):
        T = int(rng.integers(1, 17))
        E = int(rng.integers(1, 6))
        k = int(rng.integers(1, min(3, E) + 1))
        idx = np.array([rng.permutation(E)[:k] for _ in range(T)])
        flat = idx.reshape(-1).tolist()
        for cap in [None] + list(range(0, T * k + 1)):
            pm = o.permute(idx, E, cap)
            counts, bins, ss, rank, drop, kept, seg, s2r = _bf_permute(flat, E, cap)
            assert pm["counts"].tolist() == counts
            assert pm["bins"].tolist() == bins
            assert pm["sorted_slot"].tolist() == ss
            assert pm["rank"].tolist() == rank
            assert pm["drop"].astype(bool).tolist() == drop
            assert pm["kept_counts"].tolist() == kept
            assert pm["seg_offsets"].tolist() == seg
            assert pm["slot_to_row"].tolist() == s2r
            for r, s in enumerate(pm["row_slot"].tolist()):
                assert s2r[s] == r


def pin_permute_vs_torch_sort(o):
    """Stable sort order equals torch.sort(stable=True); a bijection; forced
    uniform assignment (slot s -> expert s mod E) gives equal counts."""
    rng = _rng(7)
    for E in (3, 8, 64, 256):
        idx = rng.integers(0, E, size=(500, 2))
        pm = o.permute(idx, E, None)
        ref = torch.sort(torch.from_numpy(idx.reshape(-1)), stable=True).indices.numpy()
        assert np.array_equal(pm["sorted_slot"], ref)
        assert np.array_equal(np.sort(pm["sorted_slot"]), np.arange(idx.size))
    T, k, E = 64, 2, 8
    forced = (np.arange(T * k) % E).reshape(T, k)   # MegaBlocks section 5 uniform assignment
    pm = o.permute(forced, E, None)
    assert pm["counts"].tolist() == [T * k // E] * E
    assert pm["sorted_slot"][:T * k // E].tolist() == list(range(0, T * k, E))


def pin_activations(o):
    """Known values: GELU(z) = z * Phi(z); silu(z) = z * sigmoid(z)."""
    z = np.array([-3.0, -1.0, 0.0, 0.5, 1.0, 2.0])
    phi = np.array([0.0013498980316300946, 0.15865525393145707, 0.5,
                    0.6914624612740131, 0.8413447460685429, 0.9772498680518208])
    assert np.allclose(o.activation(z, "gelu"), z * phi, rtol=1e-14, atol=1e-16)
    sig = np.array([0.04742587317756678, 0.2689414213699951, 0.5,
                    0.6224593312018546, 0.7310585786300049, 0.8807970779778823])
    up = np.array([2.0, -1.0, 3.0, 1.0, 1.0, 0.5])
    assert np.allclose(o.activation(z, "swiglu", up), z * sig * up, rtol=1e-14, atol=1e-16)


def pin_dense_mlp(o):
    """One expert, top-1: the layer is a dense MLP (torch F.linear/F.gelu/F.silu, fp64)."""
    rng = _rng(8)
    T, d, F = 7, 12, 20
    x = rng.standard_normal((T, d))
    w1 = rng.standard_normal((1, d, F)) * 0.3
    w3 = rng.standard_normal((1, d, F)) * 0.3
    w2 = rng.standard_normal((1, F, d)) * 0.3
    tx = torch.from_numpy(x)
    t1, t3, t2 = (torch.from_numpy(w[0].T.copy()) for w in (w1, w3, w2))
    ref_g = Fn.linear(Fn.gelu(Fn.linear(tx, t1), approximate="none"), t2).numpy()
    ref_s = Fn.linear(Fn.silu(Fn.linear(tx, t1)) * Fn.linear(tx, t3), t2).numpy()
    wg = rng.standard_normal((d, 1))
    og = o.forward(x, wg, None, w1, None, w2, 1, "gelu")["out"]
    os_ = o.forward(x, wg, None, w1, w3, w2, 1, "swiglu")["out"]
    assert np.allclose(og, ref_g, rtol=1e-12, atol=1e-12)
    assert np.allclose(os_, ref_s, rtol=1e-12, atol=1e-12)


def pin_expert_hidden_segments(o):
    """The hidden rows of each expert's segment are that expert's first
    projection and activation (torch F.linear/F.gelu/F.silu, fp64); an
    expert with an empty segment contributes no rows, and the rows of
    expert_ffn are the hidden rows times that expert's W2."""
    rng = _rng(42)
    d, F, E = 10, 14, 3
    seg = [0, 3, 3, 7]
    x = rng.standard_normal((7, d))
    w1 = rng.standard_normal((E, d, F)) * 0.4
    w3 = rng.standard_normal((E, d, F)) * 0.4
    w2 = rng.standard_normal((E, F, d)) * 0.4
    lin = lambda a, w: Fn.linear(torch.from_numpy(a), torch.from_numpy(w.T.copy()))  # noqa: E731
    for act in ("gelu", "swiglu"):
        h = o.expert_hidden(x, seg, w1, w3 if act == "swiglu" else None, act)
        assert h.shape == (7, F)
        for e, (a, b) in enumerate(zip(seg[:-1], seg[1:])):
            if b == a:
                continue
            z = lin(x[a:b], w1[e])
            ref = Fn.gelu(z, approximate="none") if act == "gelu" else Fn.silu(z) * lin(x[a:b], w3[e])
            assert np.allclose(h[a:b], ref.numpy(), rtol=1e-12, atol=1e-12), (act, e)
            y = o.expert_ffn(x, seg, w1, w3 if act == "swiglu" else None, w2, act)
            assert np.allclose(y[a:b], lin(np.ascontiguousarray(h[a:b]), w2[e]).numpy(),
                               rtol=1e-12, atol=1e-12)


def _dense_dispatch_reference(x, idx, w, kept_mask, w1, w3, w2, act):
    """The dispatch-mask / combine-weight formulation: every expert runs on
    every token (torch fp64), and a dense [T, E] combine weight picks and
    scales the outputs. No sort, no gather."""
    T, k = idx.shape
    E = w1.shape[0]
    cw = torch.zeros(T, E, dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            if kept_mask[t, j]:
                cw[t, idx[t, j]] += w[t, j]
    tx = torch.from_numpy(np.asarray(x, dtype=np.float64))
    out = torch.zeros(T, w2.shape[2], dtype=torch.float64)
    for e in range(E):
        z = tx @ torch.from_numpy(w1[e])
        if act == "gelu":
            h = Fn.gelu(z, approximate="none")
        else:
            h = Fn.silu(z) * (tx @ torch.from_numpy(w3[e]))
        out += cw[:, e:e + 1] * (h @ torch.from_numpy(w2[e]))
    return out.numpy()


def pin_forward_dense_formulation(o):
    """Sorted/gathered/combined output equals the dense dispatch-mask form,
    with and without capacity drops."""
    rng = _rng(9)
    for act, cf, k, E in [("gelu", 0.0, 1, 4), ("swiglu", 0.0, 2, 5),
                          ("swiglu", 0.75, 2, 4), ("gelu", 1.0, 3, 6)]:
        T, d, F = 23, 8, 12
        x = rng.standard_normal((T, d))
        wg = rng.standard_normal((d, E))
        w1 = rng.standard_normal((E, d, F)) * 0.4
        w3 = rng.standard_normal((E, d, F)) * 0.4
        w2 = rng.standard_normal((E, F, d)) * 0.4
        res = o.forward(x, wg, None, w1, w3 if act == "swiglu" else None, w2, k, act, cf)
        idx = res["route"]["topk_idx"]
        # arrival-order capacity by brute force
        cap = None if cf <= 0 else int(cf * (k * T / E))
        seen = [0] * E
        kept_mask = np.zeros((T, k), dtype=bool)
        for t in range(T):
            for j in range(k):
                e = idx[t, j]
                kept_mask[t, j] = cap is None or seen[e] < cap
                seen[e] += 1
        ref = _dense_dispatch_reference(x, idx, res["route"]["topk_w64"], kept_mask,
                                        w1, w3, w2, act)
        assert np.allclose(res["out"], ref, rtol=1e-11, atol=1e-11), (act, cf)
        sub = [0, 5, 22]
        ft = o.forward_tokens(x, sub, idx, res["route"]["topk_w64"],
                              res["permute"]["slot_to_row"], w1,
                              w3 if act == "swiglu" else None, w2, act)
        assert np.allclose(ft, ref[sub], rtol=1e-11, atol=1e-11)


def pin_all_dropped_token_is_zero(o):
    """Capacity 0 drops every slot, so the output is all zeros."""
    rng = _rng(10)
    T, d, F, E = 6, 4, 8, 2
    x = rng.standard_normal((T, d))
    w1 = rng.standard_normal((E, d, F))
    w2 = rng.standard_normal((E, F, d))
    res = o.forward(x, rng.standard_normal((d, E)), None, w1, None, w2, 1, "gelu", cf=0.1)
    assert res["permute"]["rows"] == 0 and np.all(res["out"] == 0.0)


ALL_PINS = [
    pin_example_a, pin_example_b, pin_topk_vs_torch, pin_topk_ties,
    pin_softmax_vs_torch, pin_renormalise, pin_aux, pin_capacity,
    pin_permute_bruteforce, pin_permute_vs_torch_sort, pin_activations,
    pin_dense_mlp, pin_forward_dense_formulation, pin_all_dropped_token_is_zero,
]


def pin_bias(o):
    """With a zero gate weight, every token's probabilities are softmax(b)
    and its top-k is b's order (closed form)."""
    b = np.array([0.3, -1.0, 2.0, 0.3, 1.5])
    x = np.ones((3, 4))
    r = o.route(x, np.zeros((4, 5)), b, 3)
    e = np.exp(b - b.max())
    assert np.allclose(r["probs64"], np.tile(e / e.sum(), (3, 1)), rtol=1e-14)
    assert r["topk_idx"].tolist() == [[2, 4, 0]] * 3


ALL_PINS.append(pin_bias)


def pin_binned_example_a(o):
    """The worked example in the [E, C, hs] bucket layout (MegaBlocks page,
    sections 2 and 4.3-4.6), dynamic capacity and C = 2; padding rows of the
    gathered bucket are zero."""
    g = _golden("worked_example_a_binned.json")
    ids = np.array(g["ids"]).reshape(-1, 1)
    for c in g["cases"]:
        b = o.permute_binned(ids, g["E"], c["capacity"])
        assert b["bin"] == c["bin"]
        for key in ("seg_offsets", "kept_counts", "slot_to_row", "row_slot", "drop"):
            assert np.array_equal(np.asarray(b[key]), np.asarray(c[key])), (c["capacity"], key)
        x = np.arange(1, 9, dtype=np.float64)[:, None] * np.ones((1, 3))
        xb = o.gather_binned(x, b["row_slot"], 1)
        assert np.array_equal(xb[:, 0], [0.0 if r < 0 else float(r + 1) for r in c["row_slot"]])


def pin_binned_bruteforce(o):
    """Tiny random routings: walking each expert's slots in ascending order,
    the i-th lands in row e*C + i when i < C; C defaults to the largest count
    (no drops)."""
    rng = _rng(21)
    for trial in range(60):
        E = int(rng.integers(1, 6))
        k = int(rng.integers(1, min(E, 3) + 1))
        T = int(rng.integers(1, 9))
        idx = np.array([rng.permutation(E)[:k] for _ in range(T)])
        flat = idx.reshape(-1)
        counts = [int(np.sum(flat == e)) for e in range(E)]
        for cap in (None, 0, 1, 2, 5):
            C = max(counts) if cap is None else cap
            rows = [-1] * len(flat)
            row_slot = [-1] * (E * C)
            for e in range(E):
                i = 0
                for s in range(len(flat)):
                    if flat[s] == e:
                        if i < C:
                            rows[s] = e * C + i
                            row_slot[e * C + i] = s
                        i += 1
            b = o.permute_binned(idx, E, cap)
            assert b["bin"] == C and b["rows"] == E * C
            assert list(b["slot_to_row"]) == rows, (trial, cap)
            assert list(b["row_slot"]) == row_slot, (trial, cap)
            assert list(b["drop"]) == [1 if r < 0 else 0 for r in rows]
            assert list(b["kept_counts"]) == [min(c, C) for c in counts]
            assert list(b["seg_offsets"]) == [e * C for e in range(E + 1)]


def pin_binned_forward_equals_dense(o):
    """The bucket layout changes where rows live, not the layer: gathered,
    expert MLP and combined output are the same as the dense layout's, for a
    fixed capacity (same drops) and for capacity 0 (dynamic, nothing dropped,
    equal to dropless)."""
    rng = _rng(22)
    T, d, E, k, F = 20, 6, 4, 2, 5
    x = rng.standard_normal((T, d))
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)])
    w = rng.random((T, k))
    w1 = [rng.standard_normal((d, F)) for _ in range(E)]
    w3 = [rng.standard_normal((d, F)) for _ in range(E)]
    w2 = [rng.standard_normal((F, d)) for _ in range(E)]
    for cap in (None, 3, 7):
        dn = o.permute(idx, E, cap)
        bn = o.permute_binned(idx, E, cap)
        y_d = o.expert_ffn(o.gather(x, dn["row_slot"], k), dn["seg_offsets"], w1, w3, w2, "swiglu")
        xb = o.gather_binned(x, bn["row_slot"], k)
        y_b = o.expert_ffn_binned(xb, bn["kept_counts"], bn["bin"], w1, w3, w2, "swiglu")
        keep = dn["slot_to_row"] >= 0
        assert np.array_equal(y_d[dn["slot_to_row"][keep]], y_b[bn["slot_to_row"][keep]])
        assert np.all(xb[bn["row_slot"] < 0] == 0) and np.all(y_b[bn["row_slot"] < 0] == 0)
        out_d = o.combine(y_d, w, dn["slot_to_row"], T, k)
        out_b = o.combine(y_b, w, bn["slot_to_row"], T, k)
        assert np.array_equal(out_d, out_b), cap


ALL_PINS.extend([pin_binned_example_a, pin_binned_bruteforce, pin_binned_forward_equals_dense])


def pin_philox_kat(o):
    """Philox4x32-10 reproduces the generator's published known-answer vectors."""
    for c in _golden("philox_kat.json")["cases"]:
        got = o.philox4x32_10([int(v, 16) for v in c["ctr"]], tuple(int(v, 16) for v in c["key"]))
        assert [int(v) for v in got] == [int(v, 16) for v in c["out"]], c


def pin_jitter(o):
    """Multipliers lie in [1 - eps, 1 + eps) with the uniform's mean and
    variance (eps^2 / 3); eps = 0 gives exactly 1; seeds give different
    streams; bf16 rounding of x * m is round-to-nearest-even."""
    m = o.jitter_multipliers(256, 256, 0.01, 7).astype(np.float64)
    assert m.min() >= 1 - 0.01 - 1e-7 and m.max() < 1 + 0.01 + 1e-7
    assert abs(m.mean() - 1.0) < 2e-4
    assert abs(m.var() - 0.01 ** 2 / 3) < 0.05 * 0.01 ** 2 / 3
    assert np.all(o.jitter_multipliers(4, 8, 0.0, 7) == 1.0)
    assert not np.array_equal(o.jitter_multipliers(4, 8, 0.1, 7), o.jitter_multipliers(4, 8, 0.1, 8))
    # bf16 spacing at 1 is 2^-7: 1 + 2^-8 is a tie (to even: 1); 1 + 3*2^-8 is a
    # tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even); 1 + 2^-7 + 2^-9 is below
    # the tie and rounds down to 1 + 2^-7
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -7 + 2.0 ** -9], dtype=np.float32)
    assert list(o.bf16_round(x)) == [1.0, 1.0 + 2.0 ** -6, 1.0 + 2.0 ** -7]


def pin_logit_noise(o):
    """Box-Muller normals: mean 0, standard deviation std, 68.3% within one
    std; std = 0 gives zeros."""
    z = o.logit_noise(512, 256, 0.5, 11)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 0.5) < 0.01
    assert abs(np.mean(np.abs(z) < 0.5) - 0.6827) < 0.01
    assert np.all(o.logit_noise(3, 4, 0.0, 11) == 0.0)


def pin_z_loss(o):
    """Equal logits c: (c + ln E)^2; a dominant logit L: close to L^2; small
    random cases: a direct double loop."""
    E = 8
    assert abs(o.z_loss(np.full((5, E), 2.0)) - (2.0 + math.log(E)) ** 2) < 1e-12
    l = np.zeros((3, E))
    l[:, 3] = 40.0
    assert abs(o.z_loss(l) - 40.0 ** 2) < 1e-6
    rng = _rng(30)
    l = rng.standard_normal((6, 5)) * 3
    ref = sum(math.log(sum(math.exp(v) for v in row)) ** 2 for row in l) / 6
    assert abs(o.z_loss(l) - ref) < 1e-12


def pin_route_noise(o):
    """Noise enters as a per-token additive logit term: routing with noise n
    equals routing the gate logits plus n (closed form with a zero gate)."""
    rng = _rng(31)
    T, d, E, k = 12, 4, 6, 2
    n = rng.standard_normal((T, E))
    r = o.route(np.zeros((T, d)), np.zeros((d, E)), None, k, noise=n)
    assert np.array_equal(r["topk_idx"], o.topk_select(n.astype(np.float32), k))
    p = np.exp(n - n.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    assert np.allclose(r["probs64"], p, rtol=0, atol=1e-15)
    assert abs(r["z"] - o.z_loss(n)) < 1e-12


def pin_temperature(o):
    """Router temperature: two experts give the logistic closed form
    1 / (1 + exp((b - a) / tau)); the pick does not move; tau = 1 is the
    plain router; a huge tau gives uniform probabilities, hence aux = 1 for
    any routing; the z-loss of equal logits c is (c / tau + ln E)^2."""
    T, d, k = 7, 3, 1
    x, wg = np.zeros((T, d)), np.zeros((d, 2))
    a, b = 0.9, 0.2
    for tau in (0.25, 0.5, 2.0, 10.0):
        r = o.route(x, wg, np.array([a, b]), k, temperature=tau)
        assert np.allclose(r["probs64"][:, 0], 1.0 / (1.0 + math.exp((b - a) / tau)), rtol=0, atol=1e-15)
        assert np.all(r["topk_idx"][:, 0] == 0)
    rng = _rng(32)
    T, d, E, k = 40, 16, 8, 2
    x, wg = rng.standard_normal((T, d)), rng.standard_normal((d, E))
    base = o.route(x, wg, None, k)
    same = o.route(x, wg, None, k, temperature=1.0)
    for key in ("probs64", "topk_w64", "topk_idx"):
        assert np.array_equal(base[key], same[key])
    assert base["aux"] == same["aux"] and base["z"] == same["z"]
    for tau in (0.3, 3.0):
        assert np.array_equal(o.route(x, wg, None, k, temperature=tau)["topk_idx"], base["topk_idx"])
    flat = o.route(x, wg, None, k, temperature=1e9)
    assert np.allclose(flat["probs64"], 1.0 / E, rtol=0, atol=1e-8)
    assert abs(flat["aux"] - 1.0) < 1e-7
    c, tau = 2.0, 4.0
    assert abs(o.z_loss(o.tempered_logits(np.full((3, E), c), tau)) - (c / tau + math.log(E)) ** 2) < 1e-12


def _router_loss(o, x, wg, bias, k, g, d_aux, d_z, noise, tau):
    r = o.route(x, wg, bias, k, noise=noise, temperature=tau)
    return float((g * r["topk_w64"]).sum() + d_aux * r["aux"] + d_z * r["z"])


def pin_route_backward_finite_differences(o):
    """The router backward against central differences of the forward's own
    loss sum(d_w * w) + d_aux * aux + d_z * z (float64, step 1e-6; inputs
    drawn without near-ties, so the pick does not move): d_logits through the
    additive noise input, dx and dWg through x and Wg, at tau = 1 and 0.7,
    with a bias and noise."""
    rng = _rng(33)
    T, d, E, k = 6, 5, 6, 2
    h = 1e-6
    for tau in (1.0, 0.7):
        x, wg = rng.standard_normal((T, d)), rng.standard_normal((d, E))
        bias, noise = rng.standard_normal(E), 0.3 * rng.standard_normal((T, E))
        g = rng.standard_normal((T, k))
        d_aux, d_z = 0.8, 0.35
        b = o.route_backward(x, wg, bias, k, d_w=g, d_aux=d_aux, d_z=d_z, noise=noise, temperature=tau)
        loss = lambda x_, wg_, n_: _router_loss(o, x_, wg_, bias, k, g, d_aux, d_z, n_, tau)
        fd = np.zeros((T, E))
        for t in range(T):
            for e in range(E):
                up, dn = noise.copy(), noise.copy()
                up[t, e] += h
                dn[t, e] -= h
                fd[t, e] = (loss(x, wg, up) - loss(x, wg, dn)) / (2 * h)
        assert np.max(np.abs(fd - b["d_logits"])) < 1e-7
        for (t, i) in ((0, 0), (2, 3), (5, 4)):
            up, dn = x.copy(), x.copy()
            up[t, i] += h
            dn[t, i] -= h
            assert abs((loss(up, wg, noise) - loss(dn, wg, noise)) / (2 * h) - b["dx"][t, i]) < 1e-7
        for (i, e) in ((0, 0), (1, 5), (4, 2)):
            up, dn = wg.copy(), wg.copy()
            up[i, e] += h
            dn[i, e] -= h
            assert abs((loss(x, up, noise) - loss(x, dn, noise)) / (2 * h) - b["dwg"][i, e]) < 1e-7


def pin_route_backward_identities(o):
    """Renormalised weights sum to 1, so a constant d_w passes no gradient;
    without the z-loss every row of d_logits sums to 0 (softmax); with k = 1
    the single weight is 1 whatever the logits."""
    rng = _rng(34)
    T, d, E = 9, 4, 5
    x, wg = rng.standard_normal((T, d)), rng.standard_normal((d, E))
    b = o.route_backward(x, wg, None, 2, d_w=np.full((T, 2), 1.7))
    assert np.max(np.abs(b["d_logits"])) < 1e-13
    b = o.route_backward(x, wg, None, 2, d_w=rng.standard_normal((T, 2)), d_aux=0.5, temperature=1.9)
    assert np.max(np.abs(b["d_logits"].sum(axis=1))) < 1e-13
    b = o.route_backward(x, wg, None, 1, d_w=rng.standard_normal((T, 1)))
    assert np.max(np.abs(b["d_logits"])) < 1e-13


def _bf_near_tie(row, k, eps):
    """Gap between the k-th and (k+1)-th largest values of one row, by an
    explicit descending walk; no (k+1)-th value (k = E) means no near tie."""
    s = sorted((float(v) for v in row), reverse=True)
    if k >= len(s):
        return False
    return s[k - 1] - s[k] < eps


def pin_near_tie(o):
    """Which tokens the end-to-end top-k checks leave out: those whose k-th
    and (k+1)-th largest logits are less than 1e-3 apart (the acceptance
    rule's "within 1e-3", read as strictly less; an exact gap of eps is not a
    near tie). Hand-built rows put gaps of 0.999e-3 and 1.001e-3 at the k /
    k+1 boundary, a small gap one position earlier, unsorted rows, exact ties
    and k = E; a gap that is exactly eps pins the strict comparison; random
    rows on a 2^-10 grid (gaps of 0, ~0.98e-3 and ~1.95e-3) are checked
    against the explicit walk for every k."""
    eps = 1e-3
    rows = np.array([
        [3.0, 2.0, 2.0 - 0.999e-3, -1.0],      # k = 2 boundary gap just below eps
        [3.0, 2.0, 2.0 - 1.001e-3, -1.0],      # just above eps
        [2.0, 2.0 - 0.5e-3, 0.5, 0.0],         # small gap between 1st and 2nd only
        [-1.0, 2.0 - 0.999e-3, 3.0, 2.0],      # first row, unsorted
        [1.0, 1.0, 1.0, 0.0],                  # exact tie across the boundary
        [0.0, 1.0, 1.0 + 1.001e-3, 5.0],       # 2nd/3rd gap above eps, unsorted
    ], dtype=np.float32)
    assert o.near_tie_tokens(rows, 2, eps).tolist() == [True, False, False, True, True, False]
    assert o.near_tie_tokens(rows, 1, eps).tolist() == [False, False, True, False, True, False]
    assert o.near_tie_tokens(rows, 4, eps).tolist() == [False] * len(rows)  # k = E
    exact = np.array([[1.0, 0.5, 0.25, 0.0]], dtype=np.float32)  # gaps are exact in binary
    assert o.near_tie_tokens(exact, 1, 0.5).tolist() == [False]
    assert o.near_tie_tokens(exact, 1, 0.5 + 2.0 ** -20).tolist() == [True]
    assert o.near_tie_tokens(exact, 2, 0.25).tolist() == [False]
    rng = _rng(41)
    grid = (rng.integers(0, 40, size=(300, 8)) * 2.0 ** -10).astype(np.float32)
    for k in range(1, 9):
        want = [_bf_near_tie(r, k, eps) for r in grid.tolist()]
        assert o.near_tie_tokens(grid, k, eps).tolist() == want, k
    # the flags route() reports are these, on its own fp32 logits
    x, wg = rng.standard_normal((64, 6)), rng.standard_normal((6, 8))
    r = o.route(x, wg, None, 3)
    want = [_bf_near_tie(row, 3, eps) for row in r["logits"].tolist()]
    assert r["near_tie"].tolist() == want


def pin_ep_forward_equals_each_rank_alone(o):
    """Expert parallelism moves rows, not arithmetic: on every rank the
    layer's output is the single-GPU forward of that rank's own tokens
    (world 1, 2 and 4; SwiGLU and GELU; with and without capacity drops;
    ranks with different token counts). A wrong destination, a wrong
    regroup order or rows returned to the wrong place change some rank's
    output."""
    rng = _rng(51)
    d, F = 8, 12
    for world, E, k, act, cf in [(1, 4, 2, "swiglu", 0.0), (2, 8, 2, "swiglu", 1.0),
                                 (4, 8, 3, "gelu", 0.0), (2, 4, 1, "gelu", 1.25), (4, 16, 2, "swiglu", 0.5)]:
        xs = [rng.standard_normal((int(rng.integers(5, 40)), d)) for _ in range(world)]
        wg = rng.standard_normal((d, E))
        w1 = rng.standard_normal((E, d, F)) * 0.3
        w3 = rng.standard_normal((E, d, F)) * 0.3 if act == "swiglu" else None
        w2 = rng.standard_normal((E, F, d)) * 0.3
        r = o.ep_forward(xs, wg, None, w1, w3, w2, k, act, cf)
        for i, x in enumerate(xs):
            ref = o.forward(x, wg, None, w1, w3, w2, k, act, cf)["out"]
            assert np.allclose(r["out"][i], ref, rtol=1e-12, atol=1e-12), (world, E, k, act, cf, i)


def pin_ep_plans_bruteforce(o):
    """Send plan: rows per destination = kept slots whose expert lies in that
    rank's block, counted by a mask over the slots; they start where the
    permute's segment of the rank's first expert starts. Receive plan: the
    maps are inverse permutations and expert-major row r holds, for its
    expert, source 0's rows before source 1's, each in arrival order."""
    rng = _rng(52)
    for _ in range(30):
        world = int(rng.choice([1, 2, 4]))
        E = world * int(rng.integers(1, 4))
        k = int(rng.integers(1, min(E, 3) + 1))
        T = int(rng.integers(0, 30))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).reshape(T, k) if T else np.zeros((0, k), int)
        cap = int(rng.integers(0, 6)) if rng.random() < 0.5 else None
        pm = o.permute(idx, E, cap)
        plan = o.ep_send_plan(idx, pm["drop"], E, world)
        e_loc = E // world
        flat = idx.reshape(-1)
        keep = pm["drop"].astype(bool) == False  # noqa: E712
        for g in range(world):
            mask = keep & (flat >= g * e_loc) & (flat < (g + 1) * e_loc)
            assert plan["send_rows"][g] == int(mask.sum())
            assert plan["send_offsets"][g] == pm["seg_offsets"][g * e_loc]
        assert plan["send_offsets"][world] == pm["seg_offsets"][E]
        assert np.array_equal(plan["expert_counts"], pm["kept_counts"])
        c = rng.integers(0, 5, size=(world, e_loc))
        rp = o.ep_recv_plan(c)
        n = int(c.sum())
        assert sorted(rp["local_to_recv"].tolist()) == list(range(n))
        assert np.array_equal(rp["recv_to_local"][rp["local_to_recv"]], np.arange(n))
        tags = []  # (src, e, i) of each received row, source-major
        for src in range(world):
            for e in range(e_loc):
                tags += [(src, e, i) for i in range(c[src, e])]
        got = [tags[q] for q in rp["local_to_recv"]]
        want = [(src, e, i) for e in range(e_loc) for src in range(world) for i in range(c[src, e])]
        assert got == want
        assert rp["local_seg"].tolist() == [0] + np.cumsum(c.sum(axis=0)).tolist()
        assert rp["recv_offsets"].tolist() == [0] + np.cumsum(c.sum(axis=1)).tolist()


ALL_PINS.extend([pin_philox_kat, pin_jitter, pin_logit_noise, pin_z_loss, pin_route_noise,
                 pin_temperature, pin_route_backward_finite_differences,
                 pin_route_backward_identities, pin_near_tie, pin_expert_hidden_segments,
                 pin_ep_forward_equals_each_rank_alone, pin_ep_plans_bruteforce])

