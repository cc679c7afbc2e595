"""Pins of the oracle's variable-k (cascade) route: each token takes experts in
rank order until their probability mass reaches tau, at most kmax of them,
weighted by Eq. 2 with the fixed k2.

Source: the "cascade ... cover" arm of "Reading the MoE measurement defects"
(kozo-lab), sections 4 and 6.2-6.3; Eq. 2 of "Paper of the Week #3", section
"The Receipt".  The mass is read as the float32 rank-order partial sums (the
same sums as the top-k2 mass of Eq. 2).
"""
import math

import numpy as np
import pytest


@pytest.mark.parametrize("E", [16, 32, 64])
@pytest.mark.parametrize("tau", [0.01, 0.1, 0.25, 0.3, 0.5, 0.75, 1.0])
def test_uniform_logits_take_ceil_tau_E(orc, E, tau):
    # p = 1/E exactly (power-of-two E), so the mass after k experts is k/E
    # exactly and the first k with k/E >= tau is ceil(tau*E)
    z = np.zeros((3, E), np.float32)
    idx, w, k = orc.route_cascade_f32(z, E, E, tau)
    want = max(1, math.ceil(tau * E))
    assert (k == want).all()
    assert (idx[:, :want] == np.arange(want)).all()          # ties: lower index first
    assert (idx[:, want:] == orc.EMPTY_SLOT).all()
    assert (w[:, :want] == np.float32(1.0 / E)).all()         # k2 = E: no renormalisation
    assert (w[:, want:] == 0).all()


def test_two_hot_closed_form(orc):
    # z = (ln 3, 0, 0, 0): p = (1/2, 1/6, 1/6, 1/6); masses 1/2, 2/3, 5/6, 1
    z = np.array([[math.log(3.0), 0, 0, 0]], np.float32)
    for tau, want in [(0.4, 1), (0.5, 1), (0.6, 2), (0.7, 3), (0.8, 3), (0.9, 4)]:
        _, _, k = orc.route_cascade_f32(z, 4, 4, tau)
        assert k[0] == want, (tau, k[0])


def test_tau_at_or_below_the_top_probability_takes_one(orc):
    rng = np.random.default_rng(0)
    z = rng.normal(0, 2.0, (64, 40)).astype(np.float32)
    p = np.stack([orc.softmax_f32(r) for r in z])
    for t in range(64):
        _, _, k = orc.route_cascade_f32(z[t:t + 1], 8, 16, float(p[t].max()))
        assert k[0] == 1
    _, _, k = orc.route_cascade_f32(z, 8, 16, 0.0)
    assert (k == 1).all()


def test_unreachable_tau_takes_kmax(orc):
    rng = np.random.default_rng(1)
    z = rng.normal(0, 1.0, (32, 24)).astype(np.float32)
    _, _, k = orc.route_cascade_f32(z, 6, 10, 1.5)
    assert (k == 6).all()


def test_minimal_and_equal_to_fixed_route_on_the_prefix(orc):
    rng = np.random.default_rng(2)
    E, kmax, k2 = 48, 10, 16
    z = rng.normal(0, 1.5, (200, E)).astype(np.float32)
    p = np.stack([orc.softmax_f32(r) for r in z])
    for tau in (0.2, 0.5, 0.8, 0.95):
        idx, w, k = orc.route_cascade_f32(z, kmax, k2, tau)
        fidx, fw = orc.route_f32(z, kmax, k2)
        for t in range(z.shape[0]):
            kt = int(k[t])
            assert 1 <= kt <= kmax
            # the taken prefix is the fixed route's, weights bit for bit
            assert (idx[t, :kt] == fidx[t, :kt]).all()
            assert (w[t, :kt] == fw[t, :kt]).all()
            assert (idx[t, kt:] == orc.EMPTY_SLOT).all() and (w[t, kt:] == 0).all()
            # brute force in the library: rank with a stable sort (p desc, index asc),
            # float32 prefix sums in rank order; k is the first prefix reaching tau
            order = np.lexsort((np.arange(E), -p[t]))
            mass = np.cumsum(p[t, order].astype(np.float32), dtype=np.float32)
            reach = np.nonzero(mass[:kmax] >= np.float32(tau))[0]
            want = int(reach[0]) + 1 if reach.size else kmax
            assert kt == want, (t, tau, kt, want)


def test_k_is_monotone_in_tau(orc):
    rng = np.random.default_rng(3)
    z = rng.normal(0, 1.0, (100, 32)).astype(np.float32)
    prev = None
    for tau in np.linspace(0.0, 1.0, 21):
        _, _, k = orc.route_cascade_f32(z, 12, 12, float(tau))
        if prev is not None:
            assert (k >= prev).all()
        prev = k


def test_permute_skips_empty_slots(orc):
    idx = np.array([[3, 1, orc.EMPTY_SLOT], [1, orc.EMPTY_SLOT, orc.EMPTY_SLOT], [0, 3, 2]],
                   np.int32)
    off, ss, sp = orc.permute(idx, 4)
    assert list(off) == [0, 1, 3, 4, 6]
    assert list(ss) == [6, 1, 3, 8, 0, 7]
    assert sp[2] == -1 and sp[4] == -1 and sp[5] == -1
    for i, s in enumerate(ss):
        assert sp[s] == i


def test_cascade_layer_sums_only_the_taken_experts(orc):
    rng = np.random.default_rng(4)
    d, E, I = 32, 8, 8
    x = rng.normal(0, 1, (5, d)).astype(np.float32)
    z = rng.normal(0, 2, (5, E)).astype(np.float32)
    wg = rng.normal(0, 0.3, (E, I, d)).astype(np.float32)
    wu = rng.normal(0, 0.3, (E, I, d)).astype(np.float32)
    wd = rng.normal(0, 0.3, (E, d, I)).astype(np.float32)
    out = orc.layer_tokens_cascade(x, z, lambda e: (wg[e], wu[e], wd[e]), 4, 6, 0.6)
    for t in range(5):
        kt = int(out["k"][t])
        ref = np.zeros(d, np.float64)
        for s in range(kt):
            e = int(out["idx"][t, s])
            h = wg[e].astype(np.float64) @ x[t]
            u = wu[e].astype(np.float64) @ x[t]
            hh = h / (1 + np.exp(-h)) * u
            ref += float(out["w"][t, s]) * (wd[e].astype(np.float64) @ hh)
        assert np.allclose(out["y"][t], ref, rtol=1e-4, atol=1e-5)
