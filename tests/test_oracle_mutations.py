"""Plant plausible mistakes in the CPU oracle and check that the pins catch
each one. The mistakes are planted in the oracle module only, on the CPU."""
import math

import numpy as np
import pytest
from scipy.special import erf

from oracle import moe_oracle as O
from tests.oracle_pins import ALL_PINS


def _ties_to_higher(logits32, k):
    l = np.asarray(logits32, dtype=np.float64)
    E = l.shape[1]
    order = E - 1 - np.argsort(-l[:, ::-1], axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def _no_renorm(probs, idx):
    return np.take_along_axis(np.asarray(probs, float), np.asarray(idx, np.int64), 1)


def _capacity_without_k(cf, k, T, E):
    return None if cf is None or cf <= 0 else int(cf * (T / E))


def _aux_over_tokens(probs, idx, E):
    p = np.asarray(probs, float)
    T, k = np.asarray(idx).shape
    f = np.bincount(np.asarray(idx).reshape(-1), minlength=E) / T
    return float(E * np.sum(f * p.mean(0)))


def _gelu_tanh(z, act, z_up=None):
    z = np.asarray(z, float)
    if act == "gelu":
        return 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))
    return (z / (1 + np.exp(-z))) * z_up


def _softmax_wrong_axis(l):
    l = np.asarray(l, float)
    e = np.exp(l - l.max(0, keepdims=True))
    return e / e.sum(0, keepdims=True)


def _gate_no_bias(x, wg, bias=None):
    return np.asarray(x, float) @ np.asarray(wg, float)


def _combine_swapped_weights(y_perm, topk_w, slot_to_row, T, k):
    w = np.asarray(topk_w, float).reshape(T, k)[:, ::-1]
    return _REAL["combine"](y_perm, w, slot_to_row, T, k)


def _gather_mod(x, row_slot, k):
    return np.asarray(x)[np.asarray(row_slot, np.int64) % np.asarray(x).shape[0]]


def _ffn_wrong_expert(x_perm, seg_offsets, w1, w3, w2, act):
    E = len(seg_offsets) - 1
    perm = [(e + 1) % E for e in range(E)]
    return _REAL["expert_ffn"](x_perm, seg_offsets, [w1[p] for p in perm],
                               None if w3 is None else [w3[p] for p in perm], w2, act)


def _permute_drop_gt(idx, E, cap=None):
    r = _REAL["permute"](idx, E, None if cap is None else cap + 1)
    return r


def _binned_bin_is_mean(idx, E, cap=None):
    if cap is None:
        flat = np.asarray(idx).reshape(-1)
        cap = int(math.ceil(len(flat) / E))
    return _REAL["permute_binned"](idx, E, cap)


def _binned_padding_repeats_row(x, row_slot, k):
    x = np.asarray(x)
    return x[np.abs(np.asarray(row_slot, np.int64)) // k]


def _philox_nine_rounds(ctr, key):
    c = np.asarray(ctr, dtype=np.uint64) & np.uint64(0xFFFFFFFF)
    c0, c1, c2, c3 = (c[..., i] for i in range(4))
    k0, k1 = np.uint64(key[0]), np.uint64(key[1])
    for _ in range(9):
        p0 = c0 * np.uint64(0xD2511F53)
        p1 = c2 * np.uint64(0xCD9E8D57)
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0) & np.uint64(0xFFFFFFFF), p1 & np.uint64(0xFFFFFFFF), \
            ((p0 >> np.uint64(32)) ^ c3 ^ k1) & np.uint64(0xFFFFFFFF), p0 & np.uint64(0xFFFFFFFF)
        k0 = (k0 + np.uint64(0x9E3779B9)) & np.uint64(0xFFFFFFFF)
        k1 = (k1 + np.uint64(0xBB67AE85)) & np.uint64(0xFFFFFFFF)
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def _z_loss_no_square(logits):
    l = np.asarray(logits, dtype=np.float64)
    m = l.max(axis=1, keepdims=True)
    return float(np.mean(m[:, 0] + np.log(np.exp(l - m).sum(axis=1))))


def _temperature_ignored(logits, temperature):
    return np.asarray(logits, dtype=np.float64)


def _jitter_half_width(T, d, eps, seed):
    return _REAL["jitter_multipliers"](T, d, eps / 2, seed)


def _backward_ignores_temperature(x, wg, bias, k, d_w=None, d_aux=0.0, d_z=0.0, noise=None,
                                  temperature=1.0):
    r = _REAL["route_backward"](x, wg, bias, k, d_w, d_aux, d_z, noise, temperature)
    return dict(r, d_logits=r["d_logits"] * temperature, dx=r["dx"] * temperature,
                dwg=r["dwg"] * temperature)


def _backward_drops_z(x, wg, bias, k, d_w=None, d_aux=0.0, d_z=0.0, noise=None, temperature=1.0):
    return _REAL["route_backward"](x, wg, bias, k, d_w, d_aux, 0.0, noise, temperature)


def _near_tie_next_column(logits32, k, eps=1e-3):
    l = np.sort(np.asarray(logits32, dtype=np.float64), axis=1)[:, ::-1]
    if k + 1 >= l.shape[1]:
        return np.zeros(l.shape[0], dtype=bool)
    return (l[:, k] - l[:, k + 1]) < eps


def _near_tie_sign(logits32, k, eps=1e-3):
    l = np.sort(np.asarray(logits32, dtype=np.float64), axis=1)[:, ::-1]
    if k >= l.shape[1]:
        return np.zeros(l.shape[0], dtype=bool)
    return (l[:, k] - l[:, k - 1]) < eps


def _near_tie_le(logits32, k, eps=1e-3):
    l = np.sort(np.asarray(logits32, dtype=np.float64), axis=1)[:, ::-1]
    if k >= l.shape[1]:
        return np.zeros(l.shape[0], dtype=bool)
    return (l[:, k - 1] - l[:, k]) <= eps


def _near_tie_unsorted(logits32, k, eps=1e-3):
    l = np.asarray(logits32, dtype=np.float64)
    if k >= l.shape[1]:
        return np.zeros(l.shape[0], dtype=bool)
    return np.abs(l[:, k - 1] - l[:, k]) < eps


def _ep_round_robin_owner(idx, drop, E, world):
    idx = np.asarray(idx, dtype=np.int64).reshape(-1)
    drop = np.asarray(drop, dtype=bool).reshape(-1)
    send = np.zeros(world, dtype=np.int64)
    for s in range(len(idx)):
        if not drop[s]:
            send[idx[s] % world] += 1
    per_expert = np.bincount(idx[~drop], minlength=E)
    return {"send_rows": send, "send_offsets": np.concatenate([[0], np.cumsum(send)]),
            "expert_counts": per_expert}


def _ep_recv_source_major(recv_counts):
    r = _REAL["ep_recv_plan"](recv_counts)
    n = len(r["local_to_recv"])
    return dict(r, local_to_recv=np.arange(n), recv_to_local=np.arange(n))


_REAL = {n: getattr(O, n) for n in ("combine", "expert_ffn", "permute", "permute_binned",
                                    "jitter_multipliers", "route_backward", "ep_recv_plan")}

MUTATIONS = {
    "topk_ties_to_higher_index": ("topk_select", _ties_to_higher),
    "no_renormalisation": ("renormalise", _no_renorm),
    "capacity_without_k": ("capacity", _capacity_without_k),
    "aux_f_over_tokens": ("aux_loss", _aux_over_tokens),
    "gelu_tanh_approximation": ("activation", _gelu_tanh),
    "softmax_wrong_axis": ("softmax_rows", _softmax_wrong_axis),
    "gate_drops_bias": ("gate_logits", _gate_no_bias),
    "combine_swaps_weights": ("combine", _combine_swapped_weights),
    "gather_wrong_token": ("gather", _gather_mod),
    "ffn_wrong_expert": ("expert_ffn", _ffn_wrong_expert),
    "drop_off_by_one": ("permute", _permute_drop_gt),
    "binned_dynamic_bin_is_mean_count": ("permute_binned", _binned_bin_is_mean),
    "binned_padding_not_zero": ("gather_binned", _binned_padding_repeats_row),
    "philox_nine_rounds": ("philox4x32_10", _philox_nine_rounds),
    "z_loss_without_square": ("z_loss", _z_loss_no_square),
    "jitter_half_width": ("jitter_multipliers", _jitter_half_width),
    "temperature_ignored": ("tempered_logits", _temperature_ignored),
    "backward_ignores_temperature": ("route_backward", _backward_ignores_temperature),
    "backward_drops_z_loss": ("route_backward", _backward_drops_z),
    "near_tie_next_column": ("near_tie_tokens", _near_tie_next_column),
    "near_tie_sign_slip": ("near_tie_tokens", _near_tie_sign),
    "near_tie_non_strict": ("near_tie_tokens", _near_tie_le),
    "near_tie_unsorted": ("near_tie_tokens", _near_tie_unsorted),
    "ep_round_robin_expert_owner": ("ep_send_plan", _ep_round_robin_owner),
    "ep_regroup_left_source_major": ("ep_recv_plan", _ep_recv_source_major),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(O, attr, bad)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(O)
        except (AssertionError, ValueError, IndexError, TypeError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
