"""Pins of the oracle's channel top-k inside the activated experts: each
token keeps the `keep` channels of its k1 experts with the largest
output-scaled score w_s * ||W_down[:, c]|| * |h_c|, and y sums only the kept
channels, exactly.

Source: "Channel Selection for Mixture-of-Experts Decoding Needs No
Calibration Data" (paperlayer.ai), section 2 "Background" (a channel owns a
gate row, an up row and a down column) and sections 5.2-5.3 (output-scaled
score, top-k across the token's experts, kept channels exact); Eq. 2 of
"Paper of the Week #3", section "The Receipt", for the weights w_s.
"""
import itertools

import numpy as np
import pytest


def _layer(rng, d, E, I, scale=0.3):
    wg = rng.normal(0, scale, (E, I, d)).astype(np.float32)
    wu = rng.normal(0, scale, (E, I, d)).astype(np.float32)
    wd = rng.normal(0, scale, (E, d, I)).astype(np.float32)
    return wg, wu, wd


def _run(orc, x, z, wg, wu, wd, k1, k2, keep, **kw):
    return orc.channel_topk_tokens(x, z, lambda e: (wg[e], wu[e], wd[e]),
                                   lambda e: orc.channel_norms(wd[e]), k1, k2, keep, **kw)


def test_norm_closed_forms(orc):
    d = 64
    wd = np.zeros((d, 4), np.float32)
    wd[:, 0] = 0.5                      # 0.5 * sqrt(64) = 4
    wd[:2, 1] = (3.0, 4.0)              # 5
    wd[:3, 2] = (1.0, -2.0, 2.0)        # 3
    n = orc.channel_norms(wd)
    assert list(n) == [4.0, 5.0, 3.0, 0.0]
    bits = (wd.view(np.uint32) >> 16).astype(np.uint16)  # the same values as bf16
    assert list(orc.channel_norms(bits)) == [4.0, 5.0, 3.0, 0.0]


def _closed_form_layer():
    """Two experts, d = 4, I = 3, x = e_0 so that g_c = W_g[c, 0], u_c =
    W_u[c, 0]; g = 40 makes silu(g) = 40 exactly in float32 and g = 0 makes
    it 0, so h is exact: expert 0 h = (40, -120, 0), expert 1 h = (80, 40, 20).
    Equal logits with k1 = k2 = 2 give w = (0.5, 0.5) exactly, slot 0 =
    expert 0 (ties go to the lower index)."""
    d, I = 4, 3
    wg = np.zeros((2, I, d), np.float32)
    wu = np.zeros((2, I, d), np.float32)
    wd = np.zeros((2, d, I), np.float32)
    wg[0, :, 0] = (40, 40, 0)
    wu[0, :, 0] = (1, -3, 5)
    wg[1, :, 0] = (40, 40, 40)
    wu[1, :, 0] = (2, 1, 0.5)
    wd[0, :, 0] = (3, 4, 0, 0)   # norm 5
    wd[0, :, 1] = (0, 0, 1, 0)   # norm 1
    wd[0, :, 2] = (2, 0, 0, 0)   # norm 2
    wd[1, :, 0] = (0, 1, 0, 0)   # norm 1
    wd[1, :, 1] = (0, 0, 0, 8)   # norm 8
    wd[1, :, 2] = (6, 8, 0, 0)   # norm 10
    x = np.array([[1, 0, 0, 0]], np.float32)
    z = np.zeros((1, 2), np.float32)
    return x, z, wg, wu, wd


def test_closed_form_scores_and_selection(orc):
    x, z, wg, wu, wd = _closed_form_layer()
    out = _run(orc, x, z, wg, wu, wd, 2, 2, 1)
    assert list(out["idx"][0]) == [0, 1] and list(out["w"][0]) == [0.5, 0.5]
    assert out["h"][0].tolist() == [[40, -120, 0], [80, 40, 20]]
    # 0.5 * (5*40, 1*120, 2*0) and 0.5 * (1*80, 8*40, 10*20)
    assert out["scores"][0].tolist() == [[100, 60, 0], [40, 160, 100]]
    # flat order q = s*I + c; the 100-100 tie goes to q = 0
    want = {1: [4], 2: [0, 4], 3: [0, 4, 5], 4: [0, 1, 4, 5], 5: [0, 1, 3, 4, 5],
            6: [0, 1, 2, 3, 4, 5]}
    for keep, kept in want.items():
        assert _run(orc, x, z, wg, wu, wd, 2, 2, keep)["kept"][0].tolist() == kept


def test_closed_form_output(orc):
    x, z, wg, wu, wd = _closed_form_layer()
    # keep 2: 0.5*40*(3,4,0,0) + 0.5*40*(0,0,0,8)
    assert _run(orc, x, z, wg, wu, wd, 2, 2, 2)["y"][0].tolist() == [60, 80, 0, 160]
    # keep 3 adds 0.5*20*(6,8,0,0)
    assert _run(orc, x, z, wg, wu, wd, 2, 2, 3)["y"][0].tolist() == [120, 160, 0, 160]
    # all six: the plain layer, 0.5*(o_0 + o_1)
    full = _run(orc, x, z, wg, wu, wd, 2, 2, 6)["y"][0]
    o0 = wd[0] @ np.array([40, -120, 0], np.float32)
    o1 = wd[1] @ np.array([80, 40, 20], np.float32)
    assert full.tolist() == (0.5 * (o0 + o1)).tolist()


def test_score_is_the_norm_of_the_channel_output(orc):
    # w_s * ||W_d[:, c]|| * |h_c| = ||w_s * h_c * W_d[:, c]||: the score is in
    # output units (section 5.2)
    rng = np.random.default_rng(0)
    d, E, I, k1, k2 = 48, 8, 24, 3, 5
    wg, wu, wd = _layer(rng, d, E, I)
    x = rng.normal(0, 1, (2, d)).astype(np.float32)
    z = rng.normal(0, 1, (2, E)).astype(np.float32)
    out = _run(orc, x, z, wg, wu, wd, k1, k2, 1)
    for t in range(2):
        for s in range(k1):
            e = int(out["idx"][t, s])
            contrib = (float(out["w"][t, s]) * out["h"][t, s].astype(np.float64)[None, :]
                       * wd[e].astype(np.float64))
            ref = np.sqrt((contrib * contrib).sum(axis=0))
            np.testing.assert_allclose(out["scores"][t, s], ref, rtol=4e-7, atol=0)


def test_keep_all_is_the_full_layer(orc):
    rng = np.random.default_rng(1)
    d, E, I, k1, k2 = 64, 8, 32, 3, 5
    wg, wu, wd = _layer(rng, d, E, I)
    x = rng.normal(0, 1, (4, d)).astype(np.float32)
    z = rng.normal(0, 1.5, (4, E)).astype(np.float32)
    out = _run(orc, x, z, wg, wu, wd, k1, k2, k1 * I)
    ref = orc.layer_tokens(x, z, lambda e: (wg[e], wu[e], wd[e]), k1, k2)
    assert np.array_equal(out["idx"], ref["idx"]) and np.array_equal(out["w"], ref["w"])
    scale = np.abs(ref["y"]).max()
    assert np.abs(out["y"] - ref["y"]).max() <= 2e-6 * scale


def test_nested_sets_and_one_channel_increments(orc):
    rng = np.random.default_rng(2)
    d, E, I, k1, k2 = 32, 6, 16, 2, 2
    wg, wu, wd = _layer(rng, d, E, I)
    x = rng.normal(0, 1, (1, d)).astype(np.float32)
    z = rng.normal(0, 1, (1, E)).astype(np.float32)
    prev = None
    for keep in range(1, k1 * I + 1):
        out = _run(orc, x, z, wg, wu, wd, k1, k2, keep)
        kept = set(out["kept"][0].tolist())
        assert len(kept) == keep
        if prev is not None:
            pk, py = prev
            added = kept - pk
            assert pk < kept and len(added) == 1
            s, c = divmod(added.pop(), I)
            e = int(out["idx"][0, s])
            step = float(out["w"][0, s]) * float(out["h"][0, s, c]) * wd[e][:, c].astype(np.float64)
            scale = np.abs(out["y"][0]).max() + np.abs(py).max()
            assert np.abs((out["y"][0] - py) - step).max() <= 1e-6 * scale
        prev = (kept, out["y"][0].astype(np.float64))


def test_doubling_a_down_column_doubles_its_score(orc):
    rng = np.random.default_rng(3)
    d, E, I, k1 = 32, 4, 8, 2
    wg, wu, wd = _layer(rng, d, E, I)
    x = rng.normal(0, 1, (1, d)).astype(np.float32)
    z = rng.normal(0, 1, (1, E)).astype(np.float32)
    a = _run(orc, x, z, wg, wu, wd, k1, k1, 1)
    e, c = int(a["idx"][0, 1]), 5
    wd2 = wd.copy()
    wd2[e][:, c] *= 2
    b = _run(orc, x, z, wg, wu, wd2, k1, k1, 1)
    want = a["scores"].copy()
    want[0, 1, c] *= 2
    assert np.array_equal(b["scores"], want)


def _brute_force_best(scores, keep):
    """Lexicographically smallest index tuple among the size-`keep` subsets
    with the largest float64 score sum."""
    best, best_sum = None, -1.0
    for comb in itertools.combinations(range(scores.size), keep):
        s = float(sum(float(scores[i]) for i in comb))
        if s > best_sum:
            best, best_sum = comb, s
    return list(best)


def test_selection_brute_force():
    import oracle
    rng = np.random.default_rng(4)
    for trial in range(40):
        # few distinct values, so that ties at the boundary are common
        sc = rng.integers(0, 4, size=9).astype(np.float32) * np.float32(0.75)
        for keep in range(1, 10):
            assert oracle.channel_select(sc, keep).tolist() == _brute_force_best(sc, keep)


def test_selection_boundary_invariants():
    import oracle
    rng = np.random.default_rng(5)
    sc = np.round(rng.exponential(1.0, 3000), 1).astype(np.float32)
    for keep in (1, 7, 300, 1499, 2999, 3000):
        kept = oracle.channel_select(sc, keep)
        assert kept.size == keep and np.all(np.diff(kept) > 0)
        mask = np.zeros(sc.size, bool)
        mask[kept] = True
        if keep < sc.size:
            lo, hi = sc[mask].min(), sc[~mask].max()
            assert lo >= hi
            if lo == hi:  # the tie at the boundary goes to the lower indices
                eq = np.nonzero(sc == lo)[0]
                assert np.all(mask[eq] == (eq < eq[mask[eq]].max() + 1))


def test_selection_rejects_bad_arguments():
    import oracle
    with pytest.raises(oracle.OracleError):
        oracle.channel_select(np.ones(4, np.float32), 0)
    with pytest.raises(oracle.OracleError):
        oracle.channel_select(np.ones(4, np.float32), 5)
    with pytest.raises(oracle.OracleError):
        oracle.channel_select(np.array([1, np.nan], np.float32), 1)
    with pytest.raises(oracle.OracleError):
        oracle.channel_select(np.array([1, -1], np.float32), 1)
