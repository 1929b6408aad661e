"""Host model of the warp arg-max in router_select (router.cu).

Each top-k round there is two warp reductions: the largest order-preserving
32-bit key among the lanes' best untaken logits, then the lowest expert among
the lanes that hold that key. These tests pin that form to the comparison
rule the other routers use (a larger logit wins, equal logits go to the lower
expert; NaN is never selected) and to the key's properties, with lanes laid
out as in the kernel (lane l holds experts l + 32q).
"""
import struct

import numpy as np
import pytest

INT_MAX = 0x7FFFFFFF


def f32_bits(v):
    return struct.unpack("<I", struct.pack("<f", float(v)))[0]


def order_key(v):
    """The kernel's key: NaN -> 0, -0 -> +0, then sign-magnitude to offset binary."""
    if v != v:
        return 0
    u = 0 if v == 0.0 else f32_bits(v)
    return (~u & 0xFFFFFFFF) if (u & 0x80000000) else (u | 0x80000000)


def key_value(key):
    u = (key & 0x7FFFFFFF) if (key & 0x80000000) else (~key & 0xFFFFFFFF)
    return struct.unpack("<f", struct.pack("<I", u))[0]


def better(va, ea, vb, eb):
    return va > vb or (va == vb and ea < eb)


def lanes(vals, E):
    epl = max(1, (E + 31) // 32)
    v = np.full((32, epl), -np.inf, dtype=np.float32)
    for e in range(E):
        v[e % 32, e // 32] = vals[e]
    return v


def topk_by_comparison(v, E, k):
    """k rounds of a butterfly of better() over (value, expert) pairs."""
    taken = set()
    out = []
    for _ in range(k):
        bv, be = -np.inf, INT_MAX
        for e in range(E):
            x = v[e % 32, e // 32]
            if e not in taken and better(x, e, bv, be):
                bv, be = x, e
        out.append(be)
        if be < E:
            taken.add(be)
    return out


def topk_by_keys(v, E, k):
    """The kernel's form: per lane the best untaken key (q ascending, strict >),
    then max over lanes of the key and min over lanes holding it of the expert."""
    epl = v.shape[1]
    taken = [0] * 32
    out = []
    for _ in range(k):
        bk, be = [0] * 32, [INT_MAX] * 32
        for lane in range(32):
            for q in range(epl):
                e = lane + 32 * q
                key = order_key(v[lane, q])
                if e < E and not (taken[lane] >> q) & 1 and key > bk[lane]:
                    bk[lane], be[lane] = key, e
        wk = max(bk)
        e_sel = min(be[lane] if bk[lane] == wk else 0xFFFFFFFF for lane in range(32))
        out.append(e_sel)
        if e_sel < E:
            taken[e_sel % 32] |= 1 << (e_sel // 32)
    return out


def test_key_preserves_order_and_equality():
    rng = np.random.default_rng(7)
    special = [0.0, -0.0, 1e-45, -1e-45, 1e-30, -1e-30, 1.0, -1.0, 3.4e38, -3.4e38, np.inf, -np.inf]
    vals = np.concatenate([np.array(special, dtype=np.float32),
                           rng.standard_normal(400).astype(np.float32),
                           (rng.standard_normal(200) * 1e-38).astype(np.float32)])
    for a in vals:
        for b in vals[::7]:
            ka, kb = order_key(a), order_key(b)
            assert (ka > kb) == (a > b)
            assert (ka == kb) == (a == b)
            assert ka > 0 and kb > 0  # every number is above the "none" key
    for a in vals:
        if a == 0.0:
            assert key_value(order_key(a)) == 0.0
        else:
            assert f32_bits(key_value(order_key(a))) == f32_bits(a)


def test_nan_key_is_never_selected():
    assert order_key(float("nan")) == 0
    v = lanes(np.array([np.nan, 1.0, np.nan, -2.0], dtype=np.float32), 4)
    assert topk_by_keys(v, 4, 2) == [1, 3] == topk_by_comparison(v, 4, 2)


@pytest.mark.parametrize("seed", range(4))
def test_key_argmax_matches_comparison_butterfly(seed):
    rng = np.random.default_rng(100 + seed)
    pool = np.array([0.0, -0.0, 1.5, -1.5, 2.0, -np.inf, 3.25, 1e-30, -1e-30], dtype=np.float32)
    for _ in range(150):
        E = int(rng.integers(1, 257))
        k = int(rng.integers(1, min(8, E) + 1))
        vals = np.where(rng.random(E) < 0.5, rng.choice(pool, E),
                        rng.standard_normal(E).astype(np.float32)).astype(np.float32)
        v = lanes(vals, E)
        assert topk_by_keys(v, E, k) == topk_by_comparison(v, E, k)


def test_all_taken_gives_the_error_sentinel():
    v = lanes(np.array([1.0, 2.0], dtype=np.float32), 2)
    assert topk_by_keys(v, 2, 3)[-1] == INT_MAX == topk_by_comparison(v, 2, 3)[-1]
