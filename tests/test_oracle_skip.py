"""Pins of the oracle's expert skipping: slot s >= 1 is skipped when the
per-expert table value and the slot's Eq. 2 weight are both below their
thresholds; the top-1 expert is always kept; kept slots keep their weights.

Source: "ACE" (aimodeling.com), section "How ACE decides what to skip: GSP +
RCR" (two views must agree; the top-1 expert is always retained); Eq. 2 of
"Paper of the Week #3", section "The Receipt".
"""
import math

import numpy as np


def _z(rng, T, E, s=2.0):
    return rng.normal(0, s, (T, E)).astype(np.float32)


def test_no_threshold_is_the_fixed_route(orc):
    rng = np.random.default_rng(0)
    z = _z(rng, 50, 64)
    tab = rng.uniform(0, 1, 64).astype(np.float32)
    idx, w, k = orc.route_skip_f32(z, 6, 12, tab, 0.0, 0.0)  # nothing is below 0
    fi, fw = orc.route_f32(z, 6, 12)
    assert np.array_equal(idx, fi) and np.array_equal(w, fw) and (k == 6).all()


def test_both_views_low_everywhere_keeps_only_the_top1(orc):
    rng = np.random.default_rng(1)
    z = _z(rng, 40, 32)
    tab = np.zeros(32, np.float32)
    idx, w, k = orc.route_skip_f32(z, 5, 5, tab, 1.0, math.inf)
    fi, fw = orc.route_f32(z, 5, 5)
    assert (k == 1).all()
    assert np.array_equal(idx[:, 0], fi[:, 0]) and np.array_equal(w[:, 0], fw[:, 0])  # unchanged
    assert (idx[:, 1:] == orc.EMPTY_SLOT).all() and (w[:, 1:] == 0).all()


def test_one_view_alone_never_skips(orc):
    rng = np.random.default_rng(2)
    z = _z(rng, 40, 32)
    fi, fw = orc.route_f32(z, 5, 8)
    # every expert low, but no weight below 0
    idx, w, k = orc.route_skip_f32(z, 5, 8, np.zeros(32, np.float32), 1.0, 0.0)
    assert np.array_equal(idx, fi) and (k == 5).all()
    # every weight low, but no expert below -1
    idx, w, k = orc.route_skip_f32(z, 5, 8, np.zeros(32, np.float32), -1.0, math.inf)
    assert np.array_equal(idx, fi) and (k == 5).all()


def test_hand_case(orc):
    # p proportional to (8, 4, 2, 1): with k1 = k2 = 3, w = (8, 4, 2) / 14
    z = np.log(np.array([[8, 4, 2, 1]], np.float64)).astype(np.float32)
    tab = np.array([0.0, 0.5, 2.0, 0.0], np.float32)
    idx, w, k = orc.route_skip_f32(z, 3, 3, tab, 1.0, 0.3)
    # slot 1: expert 1, table 0.5 < 1 and w = 4/14 < 0.3: skipped; slot 2:
    # expert 2, table 2 >= 1: kept even though 2/14 < 0.3
    assert idx[0].tolist() == [0, orc.EMPTY_SLOT, 2] and k[0] == 2
    assert abs(w[0, 0] - 8 / 14) < 1e-6 and w[0, 1] == 0 and abs(w[0, 2] - 2 / 14) < 1e-6
    # weight threshold just below 4/14: slot 1 kept
    idx, _, k = orc.route_skip_f32(z, 3, 3, tab, 1.0, 0.28)
    assert idx[0].tolist() == [0, 1, 2] and k[0] == 3


def test_layer_is_the_fixed_layer_minus_the_skipped_slots(orc):
    rng = np.random.default_rng(3)
    d, E, I, k1, k2 = 32, 8, 16, 4, 6
    wg = rng.normal(0, 0.3, (E, I, d)).astype(np.float32)
    wu = rng.normal(0, 0.3, (E, I, d)).astype(np.float32)
    wd = rng.normal(0, 0.3, (E, d, I)).astype(np.float32)
    x = rng.normal(0, 1, (6, d)).astype(np.float32)
    z = _z(rng, 6, E, 1.0)
    tab = rng.uniform(0, 1, E).astype(np.float32)
    fetch = lambda e: (wg[e], wu[e], wd[e])
    idx, w, k = orc.route_skip_f32(z, k1, k2, tab, 0.6, 0.25)
    assert 0 < (k < k1).sum()  # some slots are skipped
    y = orc.layer_tokens_slots(x, idx, w, fetch)
    fi, fw = orc.route_f32(z, k1, k2)
    for t in range(6):
        ref = np.zeros(d, np.float64)
        for s in range(k1):
            if idx[t, s] == orc.EMPTY_SLOT:
                continue
            e = int(fi[t, s])
            h = wg[e].astype(np.float64) @ x[t]
            u = wu[e].astype(np.float64) @ x[t]
            ref += float(fw[t, s]) * (wd[e].astype(np.float64) @ (h / (1 + np.exp(-h)) * u))
        assert np.allclose(y[t], ref, rtol=1e-4, atol=1e-5)


def test_permute_skips_empty_slots_in_the_middle(orc):
    idx = np.array([[3, orc.EMPTY_SLOT, 1], [2, 0, orc.EMPTY_SLOT]], np.int32)
    off, ss, sp = orc.permute(idx, 4)
    assert list(off) == [0, 1, 2, 3, 4]
    assert list(ss) == [4, 2, 3, 0]
    assert sp[1] == -1 and sp[5] == -1
