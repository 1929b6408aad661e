"""CPU oracle for the single-GPU MoE-layer forward (route, permute, gather,
expert FFN, combine).

TEST INFRASTRUCTURE. This module is the plain, slow, obviously correct
reference that the CUDA path is checked against. Only the tests, the package's
smoke check and the benchmark's CPU-baseline / reference arm may import it. The
product path never calls it, and it shares no code with the CUDA kernels: it
imports numpy and scipy only.

Everything is float64 unless stated. Inputs are numpy arrays; bf16 inputs are
passed already widened to float32 (the widening is exact).

Sources (page title, then section):

* "ops-transformer MoE operators" blog (aicoding.csdn.net), 原理 Steps 1-4 and
  实现 (MoEGatingForward: softmax, top-k by selection, renormalise the K
  weights to sum 1).
* "MoE Router: who decides which expert a token goes to" (lpnh.cn): gate is
  Linear(hidden, E, bias=False), softmax, top-k, renormalise; capacity
  limit with dropped tokens taking the residual path.
* "MegaBlocks 01 - why MoE is hard" (ai-reference-codex), section 1 (router
  = bias-free linear + softmax + top-k), section 3 (capacity
  C = cf * tokens * top_k / E, overflow dropped, dropped output zero), section
  4.1 (sort by expert id, histogram, inclusive cumsum = bins; sort only the
  low ceil(log2 E) key bits), section 4.2 (capacity formula with int()),
  section 4.3 (gather into expert-contiguous rows, bmm -> activation -> bmm,
  weights [E, hs, ffn], scatter multiplied by the router weight and summed
  over top-k), section 4.5 (which rows get dropped), section 5 (top-k sum).
* "Integrating MoE into your model with Colossal-AI" (blog.gitcode.com), step
  2: gate logits cast to fp32 before routing; gated MLP option.

Readings where the pages are silent or disagree (the same list is kept with
the design notes):

* No learned router bias. An optional fixed fp32 logit bias b[E] is added
  before the softmax (it is how the skewed workloads are made).
* Top-k selects on the fp32 logits (the precision the kernel routes in);
  softmax is monotone, so this is the order the pages' top-k on softmax
  scores gives, with exact ties broken toward the lower expert index.
* Capacity C = int(cf * (k * T / E)) truncated toward zero; cf <= 0 means
  dropless. Drop order is arrival order: flat slot s = t * k + j ascending.
  A dropped slot contributes zero; the surviving weights are not
  renormalised again.
* Auxiliary loss aux = E * sum_i f_i * P_i, f_i = (slots routed to i before
  any drop) / (T * k), P_i = mean over tokens of the full softmax p[t, i].
* GELU is the exact erf form; SwiGLU is silu(x W_gate) * (x W_up), then
  W_down; silu(z) = z / (1 + exp(-z)).
* The router weight multiplies the expert output in the combine, in the
  combine's own precision, summed over j = 0..k-1 in ascending order.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "gate_logits", "softmax_rows", "topk_select", "renormalise", "aux_loss",
    "near_tie_tokens", "route", "capacity", "sort_end_bit", "permute", "gather",
    "activation", "expert_hidden", "expert_ffn", "combine", "forward", "forward_tokens",
    "permute_binned", "gather_binned", "expert_ffn_binned",
    "philox4x32_10", "jitter_multipliers", "apply_jitter", "bf16_round", "logit_noise", "z_loss",
    "ep_send_plan", "ep_recv_plan", "ep_forward",
]


# --------------------------------------------------------------------------
# route
# --------------------------------------------------------------------------

def gate_logits(x, wg, bias=None):
    """Router gate: logits[t, e] = sum_i x[t, i] * Wg[i, e] (+ b[e]).

    "MoE Router" page: the gate is Linear(hidden, E) without bias; Colossal-AI
    step 2: logits are taken to fp32 before routing. Returns float64 [T, E]
    (exact dot products up to float64 rounding); callers round to float32.
    """
    l = np.asarray(x, dtype=np.float64) @ np.asarray(wg, dtype=np.float64)
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def softmax_rows(logits):
    """p[t, :] = softmax(logits[t, :]) over the E experts, float64.

    ops-transformer blog, 实现 step 1 (softmax over num_experts).
    """
    l = np.asarray(logits, dtype=np.float64)
    m = l.max(axis=1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=1, keepdims=True)


def topk_select(logits32, k):
    """Indices of the k largest logits per token, largest first.

    ops-transformer blog, 实现 step 2 (top-K over the E scores). Equal values
    are ordered by the lower expert index (a stable ordering of -logit). The
    comparison is made on the float32 values given.
    """
    l = np.asarray(logits32, dtype=np.float32).astype(np.float64)
    order = np.argsort(-l, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def renormalise(probs, idx):
    """w[t, j] = p[t, idx[t, j]] / sum_j' p[t, idx[t, j']].

    ops-transformer blog, 实现 step 3; "MoE Router" page (the K chosen
    weights are made to sum to 1). float64.
    """
    p = np.asarray(probs, dtype=np.float64)
    sel = np.take_along_axis(p, np.asarray(idx, dtype=np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def aux_loss(probs, idx, E):
    """Load-balance loss E * sum_i f_i * P_i.

    The pages name the loss (ops-transformer blog 坑1; CANN page 2.2; "MoE
    Router": every expert should get about 1/E of the tokens) but print no
    formula; the Switch/GShard form is used. f_i counts slots routed to expert
    i before any capacity drop, over all T * k slots; P_i is the mean routing
    probability of expert i over the T tokens.
    """
    p = np.asarray(probs, dtype=np.float64)
    idx = np.asarray(idx)
    T, k = idx.shape
    f = np.bincount(idx.reshape(-1), minlength=E).astype(np.float64) / (T * k)
    P = p.mean(axis=0)
    return float(E * np.sum(f * P))


def near_tie_tokens(logits32, k, eps=1e-3):
    """Tokens whose k-th and (k+1)-th largest logits are closer than eps.

    Their top-k set can flip under a different (equally valid) float
    summation order, so end-to-end index checks leave them out. "Within eps"
    is read as a strict gap < eps (a gap of exactly eps is not a near tie);
    with k = E there is no (k+1)-th logit and no token is flagged.
    """
    l = np.sort(np.asarray(logits32, dtype=np.float64), axis=1)[:, ::-1]
    if k >= l.shape[1]:
        return np.zeros(l.shape[0], dtype=bool)
    return (l[:, k - 1] - l[:, k]) < eps


def tempered_logits(logits, temperature):
    """What the router's softmax sees under a temperature tau > 0: l / tau.

    ops-transformer blog, 坑3 (numerical stability): instead of a hard top-K
    the router takes a softmax with a temperature, so experts that are not
    picked keep a little probability. The page gives no formula; the plain
    reading is softmax(l / tau): tau > 1 flattens the probabilities, tau < 1
    sharpens them, tau = 1 is the plain router. The top-k pick is unchanged
    (l / tau is increasing in l); the renormalised weights, the aux loss's
    P_i and the z-loss see l / tau.
    """
    if not temperature > 0:
        raise ValueError("temperature must be > 0")
    return np.asarray(logits, dtype=np.float64) / float(temperature)


def route(x, wg, bias, k, noise=None, temperature=1.0):
    """Router stage: logits, softmax, top-k, renormalised weights, aux loss,
    z-loss. noise: optional [T, E] values added to the logits (the training
    variant's Gaussian noise); temperature: the softmax's tau (see
    tempered_logits)."""
    l64 = gate_logits(x, wg, bias)
    if noise is not None:
        l64 = l64 + np.asarray(noise, dtype=np.float64)
    logits32 = l64.astype(np.float32)
    lt = tempered_logits(l64, temperature)
    p64 = softmax_rows(lt)
    idx = topk_select(logits32, k)
    w64 = renormalise(p64, idx)
    E = l64.shape[1]
    return {
        "logits": logits32,
        "probs64": p64,
        "probs": p64.astype(np.float32),
        "topk_idx": idx,
        "topk_w64": w64,
        "topk_w": w64.astype(np.float32),
        "aux": aux_loss(p64, idx, E),
        "z": z_loss(lt),
        "near_tie": near_tie_tokens(logits32, k),
    }


def route_backward(x, wg, bias, k, d_w=None, d_aux=0.0, d_z=0.0, noise=None, temperature=1.0):
    """Gradients of the router's losses, through the gate.

    "ops-transformer MoE operators" blog, 实现 (the gating operator carries
    the router's forward and its backward) and 坑3 (gradients reach the
    experts through the softmax). The pages print no backward; this is the
    chain rule of the forward in route(), for the scalar

        L = sum_{t,j} d_w[t, j] * w[t, j] + d_aux * aux + d_z * z

    (d_w: the upstream gradient of the renormalised top-k weights; aux, z:
    the load-balance loss and the z-loss). The top-k pick and the counts f_i
    are piecewise constant and pass no gradient; the fixed bias and the
    noise are inputs. Returns float64 d_logits [T, E] (the gradient with
    respect to the logits before the temperature), dx [T, d] and dwg [d, E].

      w_j = p_{i_j} / s, s = sum_j p_{i_j}:
          dL/dp_{i_j} = (d_w[t, j] - sum_m d_w[t, m] w_m) / s
      aux = E sum_i f_i P_i, P_i = mean_t p[t, i]:  dL/dp[t, i] += d_aux E f_i / T
      p = softmax(l / tau):  dL/dl = p (dL/dp - sum_e p_e dL/dp_e) / tau
      z = mean_t lse_t^2, lse_t = logsumexp(l_t / tau):
          dL/dl[t, e] += d_z (2 / T) lse_t p[t, e] / tau
      l = x Wg + b (+ noise):  dx = dL/dl Wg^T, dWg = x^T dL/dl
    """
    r = route(x, wg, bias, k, noise=noise, temperature=temperature)
    l64 = gate_logits(x, wg, bias)
    if noise is not None:
        l64 = l64 + np.asarray(noise, dtype=np.float64)
    out = route_backward_from(r["probs64"], r["topk_idx"], r["topk_w64"], l64, x, wg, d_w=d_w,
                              d_aux=d_aux, d_z=d_z, temperature=temperature)
    out["route"] = r
    return out


def route_backward_from(p, idx, w, logits, x, wg, d_w=None, d_aux=0.0, d_z=0.0, temperature=1.0):
    """route_backward's chain rule from a given forward: probabilities p
    [T, E], picks idx [T, k], renormalised weights w [T, k] and the logits
    before the temperature (used by the z-loss term only)."""
    p = np.asarray(p, dtype=np.float64)
    idx = np.asarray(idx)
    w = np.asarray(w, dtype=np.float64)
    T, E = p.shape
    k = idx.shape[1]
    dp = np.zeros((T, E))
    if d_w is not None:
        g = np.asarray(d_w, dtype=np.float64)
        s = np.take_along_axis(p, idx, axis=1).sum(axis=1)
        gw = (g * w).sum(axis=1)
        for j in range(k):
            dp[np.arange(T), idx[:, j]] += (g[:, j] - gw) / s
    if d_aux != 0.0:
        f = np.bincount(idx.reshape(-1), minlength=E).astype(np.float64) / (T * k)
        dp += d_aux * E * f[None, :] / T
    tau = float(temperature)
    dl = p * (dp - (p * dp).sum(axis=1, keepdims=True)) / tau
    if d_z != 0.0:
        lt = tempered_logits(logits, tau)
        m = lt.max(axis=1, keepdims=True)
        lse = m[:, 0] + np.log(np.exp(lt - m).sum(axis=1))
        dl += d_z * (2.0 / T) * lse[:, None] * p / tau
    x64 = np.asarray(x, dtype=np.float64)
    wg64 = np.asarray(wg, dtype=np.float64)
    return {"d_logits": dl, "dx": dl @ wg64.T, "dwg": x64.T @ dl}


# --------------------------------------------------------------------------
# router variants (training): jitter, logit noise, z-loss
# --------------------------------------------------------------------------
#
# The random numbers come from Philox4x32-10, the counter-based generator of
# Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2,
# 3" (SC 2011), written here from that definition: a 4 x 32-bit counter
# and a 2 x 32-bit key; each of the 10 rounds multiplies counter words 0 and
# 2 by fixed odd constants, keeps the high and low halves, and mixes them
# with words 1 and 3 and the key; the key advances by two Weyl constants
# between rounds.

_PHILOX_M = (0xD2511F53, 0xCD9E8D57)
_PHILOX_W = (0x9E3779B9, 0xBB67AE85)
_U32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """ctr: integer array [..., 4] of 32-bit words; key: (k0, k1).
    Returns uint32 [..., 4]."""
    c = np.asarray(ctr, dtype=np.uint64) & _U32
    c0, c1, c2, c3 = (c[..., i] for i in range(4))
    k0, k1 = np.uint64(key[0]) & _U32, np.uint64(key[1]) & _U32
    m0, m1 = np.uint64(_PHILOX_M[0]), np.uint64(_PHILOX_M[1])
    for _ in range(10):
        p0 = c0 * m0
        p1 = c2 * m1
        hi0, lo0 = p0 >> np.uint64(32), p0 & _U32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _U32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & _U32, lo1, (hi0 ^ c3 ^ k1) & _U32, lo0
        k0 = (k0 + np.uint64(_PHILOX_W[0])) & _U32
        k1 = (k1 + np.uint64(_PHILOX_W[1])) & _U32
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def _philox_words(n, stream, seed, per_call):
    """Word (n mod per_call) of Philox call floor(n / per_call) on counter
    (call low 32 bits, call high 32 bits, stream, 0), key (seed low, seed
    high), for every n in the integer array n; per_call is 4 or 2 (then the
    pair 2*(n mod 2), 2*(n mod 2)+1 is returned as two arrays)."""
    n = np.asarray(n, dtype=np.uint64)
    call = n // np.uint64(per_call)
    ctr = np.stack([call & _U32, call >> np.uint64(32), np.full_like(call, stream),
                    np.zeros_like(call)], axis=-1)
    out = philox4x32_10(ctr, (int(seed) & 0xFFFFFFFF, (int(seed) >> 32) & 0xFFFFFFFF))
    j = (n % np.uint64(per_call)).astype(np.int64)
    if per_call == 4:
        return np.take_along_axis(out, j[..., None], axis=-1)[..., 0]
    a = np.take_along_axis(out, (2 * j)[..., None], axis=-1)[..., 0]
    b = np.take_along_axis(out, (2 * j + 1)[..., None], axis=-1)[..., 0]
    return a, b


def jitter_multipliers(T, d, eps, seed):
    """Per-element router-input multipliers, uniform in [1 - eps, 1 + eps)
    (MegaBlocks page, section 5: the router input is multiplied by uniform
    noise in 1 +- eps during training). Element (t, i) = n = t*d + i uses
    Philox stream 0, word n mod 4 of call n / 4: u = (word >> 8) / 2^24, and
    m = (1 - eps) + (2 eps) * u, every operation in fp32 (returned fp32)."""
    n = np.arange(T * d, dtype=np.uint64)
    w = _philox_words(n, 0, seed, 4)
    u = ((w >> np.uint32(8)).astype(np.float64) * 2.0 ** -24).astype(np.float32)
    e32 = np.float32(eps)
    a = np.float32(1.0) - e32
    b = np.float32(2.0) * e32
    return (a + b * u).astype(np.float32).reshape(T, d)


def bf16_round(a32):
    """Round fp32 values to the nearest bf16 (ties to even), returned as fp32."""
    bits = np.asarray(a32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = ((bits + np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)) << np.uint64(16)
    return rounded.astype(np.uint32).view(np.float32)


def apply_jitter(x32, mult, bf16):
    """The router's input x * m, in fp32, rounded to bf16 for a bf16 layer
    (the router then reads a tensor of the layer's dtype)."""
    y = np.asarray(x32, dtype=np.float32) * np.asarray(mult, dtype=np.float32)
    return bf16_round(y) if bf16 else y


def logit_noise(T, E, std, seed):
    """Gaussian noise added to the router logits ("Integrating MoE into your
    model with Colossal-AI", step 2: NormalNoiseGenerator adds noise scaled by
    the number of experts; the scale is the std argument, 1/E in that
    reading). Logit (t, e) = n = t*E + e uses Philox stream 1, words
    2*(n mod 2) and 2*(n mod 2)+1 of call n / 2: u1 = ((w0 >> 8) + 1) / 2^24
    in (0, 1], u2 = (w1 >> 8) / 2^24, z = sqrt(-2 ln u1) cos(2 pi u2)
    (Box and Muller, 1958). Returned float64 [T, E]."""
    n = np.arange(T * E, dtype=np.uint64)
    w0, w1 = _philox_words(n, 1, seed, 2)
    u1 = ((w0 >> np.uint32(8)).astype(np.float64) + 1.0) * 2.0 ** -24
    u2 = (w1 >> np.uint32(8)).astype(np.float64) * 2.0 ** -24
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return (std * z).reshape(T, E)


def z_loss(logits):
    """Router z-loss: mean over tokens of the squared log-sum-exp of the
    logits the softmax sees (bias and noise included). The pages name the
    loss only (Colossal-AI's router_z_loss); this is the usual definition."""
    l = np.asarray(logits, dtype=np.float64)
    if l.shape[0] == 0:
        return 0.0
    m = l.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(l - m).sum(axis=1))
    return float(np.mean(lse ** 2))


# --------------------------------------------------------------------------
# permute
# --------------------------------------------------------------------------

def capacity(cf, k, T, E):
    """Expert capacity C = int(cf * (k * T / E)), or None when dropless.

    MegaBlocks page, sections 3 and 4.2 (world size 1). cf <= 0 means no
    capacity limit.
    """
    if cf is None or cf <= 0:
        return None
    return int(cf * (k * T / E))


def sort_end_bit(E):
    """Number of low key bits the sort needs: max(ceil(log2 E), 1).

    MegaBlocks page, section 4.1.
    """
    return max(int(math.ceil(math.log2(E))), 1) if E > 1 else 1


def permute(idx, E, cap=None):
    """Sorting metadata, capacity drop and the row map of the gathered layout.

    MegaBlocks page, sections 4.1 (stable sort of the flat top-k expert ids,
    histogram, inclusive cumsum = bins), 3/4.2 (capacity), 4.4/4.5 (an expert
    keeps the first C of its slots in sorted order; the rest are dropped).

    Layout of the gathered rows: the kept slots of expert 0, then of expert 1,
    ... each expert's slots in ascending flat-slot order, no padding. So expert
    e owns rows [seg_offsets[e], seg_offsets[e+1]).
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    S = T * k
    flat = idx.reshape(-1)
    if np.any((flat < 0) | (flat >= E)):
        raise ValueError("expert id out of range")
    mask = (1 << sort_end_bit(E)) - 1
    key = flat & mask
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    bins = np.cumsum(counts)
    sorted_slot = np.argsort(key, kind="stable")
    start = bins - counts                      # first sorted position of each expert
    rank = np.empty(S, dtype=np.int64)
    rank[sorted_slot] = np.arange(S) - start[flat[sorted_slot]]
    if cap is None:
        drop = np.zeros(S, dtype=bool)
        kept = counts.copy()
    else:
        drop = rank >= cap
        kept = np.minimum(counts, cap)
    seg_offsets = np.concatenate([[0], np.cumsum(kept)])
    slot_to_row = np.where(drop, -1, seg_offsets[flat] + rank)
    R = int(seg_offsets[-1])
    row_slot = np.empty(R, dtype=np.int64)
    keep = ~drop
    row_slot[slot_to_row[keep]] = np.nonzero(keep)[0]
    return {
        "counts": counts.astype(np.int32),
        "bins": bins.astype(np.int32),
        "sorted_slot": sorted_slot.astype(np.int32),
        "rank": rank.astype(np.int32),
        "drop": drop.astype(np.uint8),
        "kept_counts": kept.astype(np.int32),
        "seg_offsets": seg_offsets.astype(np.int32),
        "slot_to_row": slot_to_row.astype(np.int32),
        "row_slot": row_slot.astype(np.int32),
        "rows": R,
    }


def permute_binned(idx, E, cap=None):
    """The padded-binned layout of the pages' standard MoE path: expert e owns
    the C rows [e*C, (e+1)*C) of an [E, C, hs] bucket; its slot of rank r (in
    the stable expert order) sits in row e*C + r when r < C and is dropped
    otherwise; rows past an expert's kept slots are padding (row_slot -1,
    zero rows after the gather).

    MegaBlocks page, sections 4.3 (binned_gather into [E, C, hs]), 4.4 (the
    illustration's bucket[e, :len(rows)] = x[rows[:C]]), 4.5 (a short bin
    keeps zeros; slots of rank >= C have no row: dropped), 4.6 (capacity 0:
    C = the largest token count of the step, so nothing is dropped).

    cap None means that dynamic capacity. Everything but the rows is the
    permute() result for the same capacity; "bin" is C.
    """
    idx = np.asarray(idx, dtype=np.int64)
    dense = permute(idx, E, cap)
    counts = dense["counts"].astype(np.int64)
    C = int(counts.max()) if cap is None else int(cap)
    flat = idx.reshape(-1)
    rank = dense["rank"].astype(np.int64)
    drop = dense["drop"].astype(bool)
    kept = np.minimum(counts, C)
    seg_offsets = np.arange(E + 1, dtype=np.int64) * C
    slot_to_row = np.where(drop, -1, flat * C + rank)
    row_slot = np.full(E * C, -1, dtype=np.int64)
    keep = ~drop
    row_slot[slot_to_row[keep]] = np.nonzero(keep)[0]
    out = dict(dense)
    out.update({
        "kept_counts": kept.astype(np.int32),
        "seg_offsets": seg_offsets.astype(np.int32),
        "slot_to_row": slot_to_row.astype(np.int32),
        "row_slot": row_slot.astype(np.int32),
        "rows": E * C,
        "bin": C,
    })
    return out


def gather_binned(x, row_slot, k):
    """Bucket rows: x[row_slot[r] // k], or zeros where row_slot[r] < 0
    (padding; MegaBlocks page, section 4.5)."""
    x = np.asarray(x)
    rs = np.asarray(row_slot, dtype=np.int64)
    out = np.zeros((len(rs),) + x.shape[1:], dtype=x.dtype)
    live = rs >= 0
    out[live] = x[rs[live] // k]
    return out


def expert_ffn_binned(x_perm, kept_counts, bin_rows, w1, w3, w2, act):
    """The expert MLP of each bin's kept rows; padding rows stay zero (an
    expert applied to a zero row gives zero for both activations here, so
    this equals running it over the whole bucket, as the pages' bmm does)."""
    kept = np.asarray(kept_counts, dtype=np.int64)
    E = len(kept)
    y = np.zeros((E * bin_rows, np.asarray(w2[0]).shape[1]), dtype=np.float64)
    for e in range(E):
        a = e * bin_rows
        if kept[e] > 0:
            y[a:a + kept[e]] = _expert_mlp(x_perm[a:a + kept[e]], e, w1, w3, w2, act)
    return y


# --------------------------------------------------------------------------
# gather / expert FFN / combine
# --------------------------------------------------------------------------

def gather(x, row_slot, k):
    """x_perm[r] = x[row_slot[r] // k] (MegaBlocks page, section 4.3: the
    token of flat slot s is s // top_k)."""
    x = np.asarray(x)
    return x[np.asarray(row_slot, dtype=np.int64) // k]


def activation(z, act, z_up=None):
    """GELU (exact erf form) or SwiGLU's silu(z_gate) * z_up, float64."""
    z = np.asarray(z, dtype=np.float64)
    if act == "gelu":
        return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))
    if act == "swiglu":
        return (z / (1.0 + np.exp(-z))) * np.asarray(z_up, dtype=np.float64)
    raise ValueError(act)


def _expert_hidden(xe, e, w1, w3, act):
    xe = np.asarray(xe, dtype=np.float64)
    z1 = xe @ np.asarray(w1[e], dtype=np.float64)
    z3 = xe @ np.asarray(w3[e], dtype=np.float64) if act == "swiglu" else None
    return activation(z1, act, z3)


def _expert_mlp(xe, e, w1, w3, w2, act):
    return _expert_hidden(xe, e, w1, w3, act) @ np.asarray(w2[e], dtype=np.float64)


def expert_hidden(x_perm, seg_offsets, w1, w3, act):
    """The expert MLP's hidden rows h = act(x_perm W1[e]) (GELU) or
    silu(x_perm W_gate[e]) * (x_perm W_up[e]) (SwiGLU) over each expert's
    rows: the first bmm and the activation of the MegaBlocks page's section
    4.3. Returns float64 [R, F]."""
    seg = np.asarray(seg_offsets, dtype=np.int64)
    E = len(seg) - 1
    h = np.zeros((int(seg[-1]), np.asarray(w1[0]).shape[1]), dtype=np.float64)
    for e in range(E):
        a, b = int(seg[e]), int(seg[e + 1])
        if b > a:
            h[a:b] = _expert_hidden(x_perm[a:b], e, w1, w3, act)
    return h


def expert_ffn(x_perm, seg_offsets, w1, w3, w2, act):
    """Per-expert MLP over each expert's rows: bmm -> activation -> bmm.

    MegaBlocks page, section 4.3 (weights [E, hs, ffn]); the gated (SwiGLU)
    form follows the CANN operator list and Colossal-AI's gated-MLP option.
    w1 is W1 (GELU) or W_gate (SwiGLU), w3 is W_up (SwiGLU only), w2 is
    W2 / W_down. Returns float64 [R, d].
    """
    seg = np.asarray(seg_offsets, dtype=np.int64)
    E = len(seg) - 1
    y = np.zeros((int(seg[-1]), np.asarray(w2[0]).shape[1]), dtype=np.float64)
    for e in range(E):
        a, b = int(seg[e]), int(seg[e + 1])
        if b > a:
            y[a:b] = _expert_mlp(x_perm[a:b], e, w1, w3, w2, act)
    return y


def combine(y_perm, topk_w, slot_to_row, T, k):
    """out[t] = sum over j = 0..k-1 of w[t, j] * y_perm[row(t, j)], dropped
    slots skipped; a token with every slot dropped gets a zero row.

    ops-transformer blog, 原理 step 4 (weighted sum); MegaBlocks page,
    sections 4.3 and 5 (multiply by the router weight, sum over top-k).
    """
    y = np.asarray(y_perm, dtype=np.float64)
    w = np.asarray(topk_w, dtype=np.float64).reshape(T, k)
    rows = np.asarray(slot_to_row, dtype=np.int64).reshape(T, k)
    out = np.zeros((T, y.shape[1]), dtype=np.float64)
    for j in range(k):
        r = rows[:, j]
        m = r >= 0
        out[m] += w[m, j, None] * y[r[m]]
    return out


# --------------------------------------------------------------------------
# whole layer
# --------------------------------------------------------------------------

def forward(x, wg, bias, w1, w3, w2, k, act, cf=0.0, topk_idx=None, topk_w=None):
    """The whole MoE-layer forward. If topk_idx (and topk_w) are given, the
    permute/FFN/combine run on that routing instead of the oracle's own."""
    x = np.asarray(x)
    T = x.shape[0]
    E = np.asarray(wg).shape[1]
    r = route(x, wg, bias, k)
    idx = r["topk_idx"] if topk_idx is None else np.asarray(topk_idx)
    w = r["topk_w64"] if topk_w is None else np.asarray(topk_w, dtype=np.float64)
    pm = permute(idx, E, capacity(cf, k, T, E))
    xp = gather(x, pm["row_slot"], k)
    y = expert_ffn(xp, pm["seg_offsets"], w1, w3, w2, act)
    out = combine(y, w, pm["slot_to_row"], T, k)
    return {"route": r, "permute": pm, "x_perm": xp, "y_perm": y, "out": out}


# --------------------------------------------------------------------------
# expert-parallel dispatch
# --------------------------------------------------------------------------
#
# "MoE Router: who decides which expert a token goes to": the dispatch counts,
# for every chosen expert of every token, one send to the device holding that
# expert (device = expert / experts_per_device), then an all-to-all-v moves
# the rows; "ops-transformer MoE operators", 坑2: the tokens are computed on
# the cards that hold their experts and sent back; "Integrating MoE into your
# model with Colossal-AI", step 2: all-to-all to the expert's GPU, expert
# MLP, all-to-all back. Readings: experts are owned in contiguous blocks of
# E / world; each rank applies the capacity to its own tokens before sending
# (a dropped slot sends nothing); rows keep the permute's order (by expert,
# then arrival) on the way out and come back to the same places.

def ep_send_plan(idx, drop, E, world):
    """Rows this rank sends to each rank, their start in the expert-sorted
    gathered rows, and the per-expert counts each receiver needs (its slice
    of the kept counts). Counted slot by slot, as the page's dispatch loop
    does."""
    idx = np.asarray(idx, dtype=np.int64).reshape(-1)
    drop = np.asarray(drop, dtype=bool).reshape(-1)
    if E % world != 0:
        raise ValueError("E must be a multiple of world")
    e_loc = E // world
    send = np.zeros(world, dtype=np.int64)
    per_expert = np.zeros(E, dtype=np.int64)
    for s in range(len(idx)):
        if drop[s]:
            continue
        send[idx[s] // e_loc] += 1
        per_expert[idx[s]] += 1
    offsets = np.concatenate([[0], np.cumsum(send)])
    return {"send_rows": send, "send_offsets": offsets, "expert_counts": per_expert}


def ep_recv_plan(recv_counts):
    """recv_counts[src][e]: rows from rank src for this rank's local expert
    e. Rows arrive source-major (all of src 0's rows, in expert order, then
    src 1's). Returns the rows per source, where each source's rows start,
    the expert-major segment offsets (for expert e: src 0's rows, then src
    1's, ...) and the two row maps between the orders."""
    c = np.asarray(recv_counts, dtype=np.int64)
    world, e_loc = c.shape
    recv_rows = c.sum(axis=1)
    recv_offsets = np.concatenate([[0], np.cumsum(recv_rows)])
    # position of each received row: (src, e, i) in source-major order
    arrival = []
    for src in range(world):
        for e in range(e_loc):
            for i in range(c[src, e]):
                arrival.append((src, e, i))
    expert_major = sorted(range(len(arrival)), key=lambda q: (arrival[q][1], arrival[q][0], arrival[q][2]))
    local_to_recv = np.array(expert_major, dtype=np.int64)
    recv_to_local = np.empty_like(local_to_recv)
    recv_to_local[local_to_recv] = np.arange(len(local_to_recv))
    local_counts = c.sum(axis=0)
    local_seg = np.concatenate([[0], np.cumsum(local_counts)])
    return {"recv_rows": recv_rows, "recv_offsets": recv_offsets, "local_seg": local_seg,
            "local_to_recv": local_to_recv, "recv_to_local": recv_to_local}


def ep_forward(x_ranks, wg, bias, w1, w3, w2, k, act, cf=0.0):
    """The expert-parallel layer by plain message passing between the ranks'
    lists (no collective library): each rank routes, permutes (its own
    capacity) and gathers its own tokens; its rows for each destination rank
    are sent; each rank computes its experts on what it received and sends
    the outputs back, which land where the rows were; each rank combines.
    w1 / w3 / w2 hold all E experts (rank g uses its block). Returns each
    rank's output and route / permute results."""
    world = len(x_ranks)
    E = np.asarray(wg).shape[1]
    e_loc = E // world
    local = []
    sent = [[None] * world for _ in range(world)]   # sent[src][dst] = rows
    counts = [[None] * world for _ in range(world)]  # counts[src][dst] = per-local-expert counts
    for src, x in enumerate(x_ranks):
        x = np.asarray(x)
        T = x.shape[0]
        r = route(x, wg, bias, k)
        pm = permute(r["topk_idx"], E, capacity(cf, k, T, E))
        xp = gather(x, pm["row_slot"], k)
        plan = ep_send_plan(r["topk_idx"], pm["drop"], E, world)
        for dst in range(world):
            a, b = plan["send_offsets"][dst], plan["send_offsets"][dst + 1]
            sent[src][dst] = xp[a:b]
            counts[src][dst] = plan["expert_counts"][dst * e_loc:(dst + 1) * e_loc]
        local.append({"route": r, "permute": pm, "plan": plan, "T": T})
    back = [[None] * world for _ in range(world)]  # back[dst][src] = outputs of src's rows
    for dst in range(world):
        rp = ep_recv_plan(np.stack([counts[src][dst] for src in range(world)]))
        x_recv = np.concatenate([sent[src][dst] for src in range(world)], axis=0)
        x_loc = x_recv[rp["local_to_recv"]]
        y_loc = np.zeros((len(x_loc), np.asarray(w2[0]).shape[1]))
        for e in range(e_loc):
            a, b = rp["local_seg"][e], rp["local_seg"][e + 1]
            if b > a:
                y_loc[a:b] = _expert_mlp(x_loc[a:b], dst * e_loc + e, w1, w3, w2, act)
        y_recv = y_loc[rp["recv_to_local"]]
        for src in range(world):
            a, b = rp["recv_offsets"][src], rp["recv_offsets"][src + 1]
            back[dst][src] = y_recv[a:b]
    outs = []
    for src in range(world):
        st = local[src]
        y_perm = np.concatenate([back[dst][src] for dst in range(world)], axis=0)
        outs.append(combine(y_perm, st["route"]["topk_w64"], st["permute"]["slot_to_row"], st["T"], k))
    return {"out": outs, "local": local}


def forward_tokens(x, tokens, topk_idx, topk_w, slot_to_row, w1, w3, w2, act):
    """Layer output for a subset of tokens only, from a given routing and
    drop map (slot_to_row < 0 marks a dropped slot). Used to check full-size
    runs on sampled tokens: each sampled token's kept (token, expert) pairs
    go through that expert's MLP. Returns float64 [len(tokens), d]."""
    x = np.asarray(x)
    T = x.shape[0]
    idx = np.asarray(topk_idx).reshape(T, -1)
    k = idx.shape[1]
    w = np.asarray(topk_w, dtype=np.float64).reshape(T, k)
    rows = np.asarray(slot_to_row).reshape(T, k)
    tokens = np.asarray(tokens, dtype=np.int64)
    out = np.zeros((len(tokens), np.asarray(w2[0]).shape[1]), dtype=np.float64)
    pairs = [(i, int(t), j) for i, t in enumerate(tokens) for j in range(k) if rows[t, j] >= 0]
    for e in sorted({int(idx[t, j]) for _, t, j in pairs}):
        mine = [(i, t, j) for i, t, j in pairs if int(idx[t, j]) == e]
        y = _expert_mlp(x[[t for _, t, _ in mine]], e, w1, w3, w2, act)
        for (i, t, j), yr in zip(mine, y):
            out[i] += w[t, j] * yr
    return out
