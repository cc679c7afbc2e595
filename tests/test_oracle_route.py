"""Pins of the CPU oracle's routing (exp_c, softmax, top-k, Eq. 2) against
facts that do not come from the oracle itself.

Eq. 2 and its special cases: "Paper of the Week #3 -- Half the FLOPs Is Not
Half the Time", section "The Receipt"; order of operations: the same page,
section "Ship It / Code of the Week".
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "eq2_closed_form.json")


def ulp32(v):
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 1e-300)))
    return np.exp2(e - 23)


# ---------------------------------------------------------------- exp_c
def test_exp_c_exhaustive_error_bound(orc):
    """Every float32 in [-87, -0]: within 2 ulp of the double exp, never subnormal."""
    worst, n, bad = orc.exp_c_sweep(1)
    assert n == 1118699521
    assert bad == 0
    assert worst <= 2.0, worst


def test_exp_c_special_values(orc):
    y = orc.exp_c(np.array([0.0, -0.0, -87.0, -87.0001, -np.inf, np.nan, -1e30], np.float32))
    assert y[0] == np.float32(1.0) and y[1] == np.float32(1.0)
    assert y[2] > 0 and np.isfinite(y[2])
    assert y[3] == 0 and y[4] == 0 and y[5] == 0 and y[6] == 0


def test_exp_c_against_numpy_expf_and_monotone(orc):
    rng = np.random.default_rng(1)
    x = np.sort(rng.uniform(-87, 0, 1_000_000).astype(np.float32))
    y = orc.exp_c(x)
    ref32 = np.exp(x)  # numpy's own float32 exp, an independent implementation
    assert np.all(np.abs(y.astype(np.float64) - ref32) <= 2 * ulp32(ref32) + 1 * ulp32(y))
    assert np.all(np.diff(y.astype(np.float64)) >= 0), "exp_c must be non-decreasing"


# ---------------------------------------------------------------- softmax
@pytest.mark.parametrize("E", [16, 32, 128, 512, 1024])
def test_softmax_uniform_is_exact(orc, E):
    p = orc.softmax_f32(np.full(E, 0.3, np.float32))
    assert np.all(p == np.float32(1.0 / E))


@pytest.mark.parametrize("E", [16, 100, 128, 512, 1000])
def test_softmax_sum_and_double_agreement(orc, E):
    rng = np.random.default_rng(E)
    for trial in range(20):
        z = (rng.standard_normal(E) * (0.5 + trial)).astype(np.float32)
        p = orc.softmax_f32(z)
        assert abs(float(p.astype(np.float64).sum()) - 1.0) <= E * 2.0 ** -23
        zd = z.astype(np.float64)
        ref = np.exp(zd - zd.max())
        ref /= ref.sum()
        big = ref > 1e-30
        rel = np.abs(p[big] - ref[big]) / ref[big]
        # exp_c (<= 2 ulp), the division and Z contribute a few ulp; rounding
        # z - max(z) to float32 adds |z - max| * 2^-24 after the exponential
        bound = 16 * 2.0 ** -24 + np.abs(zd - zd.max())[big] * 2.0 ** -24
        assert np.all(rel <= bound), (rel / bound).max()


def test_softmax_shift_invariance_in_double(orc):
    z = np.random.default_rng(3).standard_normal((4, 64))
    _, _, p1 = orc.route_f64(z, 2, 4)
    _, _, p2 = orc.route_f64(z + 17.25, 2, 4)
    assert np.allclose(p1, p2, rtol=1e-13, atol=0)


# ---------------------------------------------------------------- golden
def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_eq2_closed_form_cases(orc, case):
    p = [Fraction(s) for s in case["p"]]
    z64 = np.array([[math.log(float(v)) for v in p]])
    k1, k2 = case["k1"], case["k2"]
    w_exact = np.array([float(Fraction(s)) for s in case["w"]])
    idx64, w64, _ = orc.route_f64(z64, k1, k2)
    assert idx64[0].tolist() == case["idx"]
    assert np.allclose(w64[0], w_exact, rtol=1e-12, atol=0)
    idx32, w32 = orc.route_f32(z64.astype(np.float32), k1, k2)
    assert idx32[0].tolist() == case["idx"]
    assert np.allclose(w32[0], w_exact, rtol=2e-6, atol=0)


# ---------------------------------------------------------------- ties
@pytest.mark.parametrize("E,k1,k2", [(16, 2, 4), (16, 2, 2), (16, 2, 16), (128, 8, 16),
                                      (128, 4, 16), (128, 8, 8), (128, 4, 128), (512, 5, 20)])
def test_equal_logits_pick_lowest_indices(orc, E, k1, k2):
    z = np.zeros((3, E), np.float32)
    idx, w = orc.route_f32(z, k1, k2)
    assert np.all(idx == np.arange(k1)[None, :])
    K = min(k2, E)
    expect = np.float32(1.0 / K) if k2 < E else np.float32(1.0 / E)
    if K & (K - 1) == 0:  # power of two: exact
        assert np.all(w == expect)
    else:
        assert np.allclose(w, 1.0 / K, rtol=4 * 2.0 ** -23)


def test_duplicated_logits_tie_rule(orc):
    # two groups of equal logits; the lower index wins inside each group
    z = np.array([[0.0, 2.0, 1.0, 2.0, 1.0, 2.0, 0.0, 1.0]], np.float32)
    idx, _ = orc.route_f32(z, 5, 8)
    assert idx[0].tolist() == [1, 3, 5, 2, 4]


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("k", [2, 4])
def test_bruteforce_subsets_E16(orc, k):
    """The selected set is the max-mass k-subset (lexicographically lowest
    among equal masses), checked by enumerating all C(16, k) subsets."""
    rng = np.random.default_rng(100 + k)
    for trial in range(40):
        if trial % 4 == 3:  # inject exact duplicates
            z = rng.integers(-2, 3, 16).astype(np.float32)
        else:
            z = rng.standard_normal(16).astype(np.float32)
        idx, _ = orc.route_f32(z[None], k, k)
        p = orc.softmax_f32(z)
        best, best_mass = None, None
        for sub in itertools.combinations(range(16), k):
            mass = math.fsum(sorted(float(p[j]) for j in sub))
            if best_mass is None or mass > best_mass:
                best, best_mass = sub, mass
        assert sorted(idx[0].tolist()) == list(best)


# ---------------------------------------------------------------- Eq. 2
def _rand_logits(T, E, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal((T, E)) * scale).astype(np.float32)


@pytest.mark.parametrize("E,k", [(16, 2), (128, 8), (128, 4), (512, 10), (512, 5)])
def test_standard_renorm_sums_to_one(orc, E, k):
    z = _rand_logits(64, E, E + k)
    _, w = orc.route_f32(z, k, k)
    s = w.astype(np.float64).sum(axis=1)
    assert np.all(np.abs(s - 1.0) <= k * 2.0 ** -23)
    _, w64, _ = orc.route_f64(z.astype(np.float64), k, k)
    assert np.all(np.abs(w64.sum(axis=1) - 1.0) <= 1e-15 * k)


@pytest.mark.parametrize("E,k1,k2", [(16, 2, 16), (128, 8, 128), (128, 4, 200), (512, 5, 512)])
def test_no_renorm_returns_probabilities_bitwise(orc, E, k1, k2):
    z = _rand_logits(32, E, 7)
    idx, w = orc.route_f32(z, k1, k2)
    for t in range(z.shape[0]):
        p = orc.softmax_f32(z[t])
        assert np.array_equal(w[t], p[idx[t]])
    # and these probabilities are the softmax itself (double reference)
    zd = z.astype(np.float64)
    ref = np.exp(zd - zd.max(1, keepdims=True))
    ref /= ref.sum(1, keepdims=True)
    got = np.take_along_axis(ref, idx.astype(np.int64), 1)
    assert np.allclose(w, got, rtol=1e-5, atol=1e-12)


def test_mass_ratio_and_monotone_in_k2(orc):
    E, k1 = 128, 4
    z = _rand_logits(16, E, 11, scale=2.0).astype(np.float64)
    prev = None
    for k2 in [4, 6, 8, 16, 32, 64, 127, 128]:
        idx, w, p = orc.route_f64(z, k1, k2)
        ps = -np.sort(-p, axis=1)
        ratio = ps[:, :k1].sum(1) / ps[:, :min(k2, E)].sum(1)
        assert np.allclose(w.sum(1), ratio, rtol=1e-13)
        assert np.all(w.sum(1) <= 1.0 + 1e-15)
        if prev is not None:
            assert np.all(w.sum(1) <= prev + 1e-15)
            assert np.array_equal(idx, prev_idx), "k2 must not change which experts are selected"
        prev, prev_idx = w.sum(1), idx


def test_indices_independent_of_k2_float32(orc):
    z = _rand_logits(64, 128, 5)
    base, _ = orc.route_f32(z, 8, 8)
    for k2 in [16, 64, 128, 1000]:
        idx, _ = orc.route_f32(z, 8, k2)
        assert np.array_equal(idx, base)


def test_two_hot_closed_form(orc):
    # logits (a, a, 0, ..., 0): p_0 = p_1 = e^a / (2 e^a + E - 2)
    E, a = 16, 3.0
    z = np.zeros((1, E))
    z[0, :2] = a
    idx, w, p = orc.route_f64(z, 1, E)
    assert idx[0].tolist() == [0]
    assert abs(w[0, 0] - math.exp(a) / (2 * math.exp(a) + E - 2)) < 1e-15
    idx, w, _ = orc.route_f64(z, 1, 2)
    assert abs(w[0, 0] - 0.5) < 1e-15
    idx, w, _ = orc.route_f64(z, 2, 3)
    assert abs(w[0, 0] - math.exp(a) / (2 * math.exp(a) + 1)) < 1e-15


def test_bad_arguments(orc):
    z = _rand_logits(2, 16, 0)
    with pytest.raises(orc.OracleError):
        orc.route_f32(z, 4, 2)   # k2 < k1
    with pytest.raises(orc.OracleError):
        orc.route_f32(z, 17, 20)  # k1 > E
    with pytest.raises(orc.OracleError):
        orc.route_f32(z, 0, 2)


# ---------------------------------------------------------------- the page's router
def page_router_restated(logits64, k1, k2):
    """The page's router (softmax in float, topk of min(k2, E), slice k1,
    divide by the sum unless k2 >= E), restated with torch library calls in
    float64."""
    t = torch.from_numpy(logits64)
    E = t.shape[-1]
    probs = torch.softmax(t, dim=-1)
    vals, ix = torch.topk(probs, min(k2, E), dim=-1)
    scores = vals[:, :k1] if k2 >= E else vals[:, :k1] / vals.sum(-1, keepdim=True)
    return ix[:, :k1].numpy(), scores.numpy()


@pytest.mark.parametrize("E,k1,k2", [(16, 2, 4), (128, 8, 8), (128, 4, 16), (128, 4, 128),
                                      (512, 10, 10), (512, 5, 20)])
def test_against_page_router_library_topk(orc, E, k1, k2):
    z = _rand_logits(128, E, E * 31 + k1 * 7 + k2, scale=1.5)
    ix_ref, w_ref = page_router_restated(z.astype(np.float64), k1, k2)
    idx64, w64, _ = orc.route_f64(z.astype(np.float64), k1, k2)
    assert np.array_equal(idx64, ix_ref)
    assert np.allclose(w64, w_ref, rtol=1e-12, atol=0)
    idx32, w32 = orc.route_f32(z, k1, k2)
    assert np.array_equal(idx32, ix_ref)
    assert np.allclose(w32, w_ref, rtol=1e-6, atol=0)


def test_float32_canonical_vs_double_twin(orc):
    """Canonical float32 weights agree with the double twin to a few ulp;
    indices differ only where adjacent double probabilities are within 1e-6."""
    for E, k1, k2 in [(128, 8, 16), (128, 4, 128), (512, 10, 20), (1024, 8, 8)]:
        z = _rand_logits(256, E, E + k2, scale=1.0)
        i32, w32 = orc.route_f32(z, k1, k2)
        i64, w64, p64 = orc.route_f64(z.astype(np.float64), k1, k2)
        same = np.all(i32 == i64, axis=1)
        for t in np.where(~same)[0]:
            ps = np.sort(p64[t])[::-1]
            gaps = np.abs(np.diff(ps[:min(k2, E) + 1]))
            assert gaps.min() < 1e-6
        err = np.abs(w32[same].astype(np.float64) - w64[same])
        assert np.all(err <= 8 * ulp32(w64[same])), (E, k1, k2, (err / ulp32(w64[same])).max())
