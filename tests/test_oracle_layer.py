"""Pins of the CPU oracle's logits, SwiGLU expert, combine, permutation and
whole layer against library routines, closed forms and invariants.

Expert structure: "Channel Selection for Mixture-of-Experts Decoding Needs No
Calibration Data", section 2 "Background" (a routed expert is a gated MLP;
channel c owns gate row c, up row c and down column c).  Weights of the
combine: Eq. 2 of "Paper of the Week #3", section "The Receipt".
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from routed_expert_layer_route_b200 import synth


def swiglu_f64(x, wg, wu, wd):
    """Library routines in float64: F.linear + F.silu."""
    x = torch.as_tensor(x, dtype=torch.float64)
    g = F.linear(x, torch.as_tensor(wg, dtype=torch.float64))
    u = F.linear(x, torch.as_tensor(wu, dtype=torch.float64))
    return F.linear(F.silu(g) * u, torch.as_tensor(wd, dtype=torch.float64)).numpy()


def bf16_round(a):
    return torch.as_tensor(a, dtype=torch.float32).to(torch.bfloat16)


# ---------------------------------------------------------------- logits
def test_logits_exact_on_representable_inputs(orc):
    rng = np.random.default_rng(0)
    T, d, E = 5, 64, 16
    # small multiples of 1/8: every product and partial sum is exact in float32
    x = (rng.integers(-16, 17, (T, d)) / 8.0).astype(np.float32)
    wr = (rng.integers(-16, 17, (E, d)) / 8.0).astype(np.float32)
    z = orc.logits(x, wr)
    assert np.array_equal(z.astype(np.float64), x.astype(np.float64) @ wr.T.astype(np.float64))
    b = (rng.integers(-8, 9, E) / 4.0).astype(np.float32)
    zb = orc.logits(x, wr, b)
    assert np.array_equal(zb - z, np.broadcast_to(b, z.shape))


def test_logits_bf16_widening_matches_library(orc):
    layer = synth.make_layer(8, 256, 32, 16, seed=3)
    z = orc.logits(synth.to_numpy(layer.x), synth.to_numpy(layer.w_router))
    ref = layer.x.double() @ layer.w_router.double().T
    assert np.allclose(z, ref.numpy(), rtol=0, atol=1e-5)


# ---------------------------------------------------------------- expert
def test_expert_single_channel_closed_form(orc):
    rng = np.random.default_rng(1)
    d = 64
    x = rng.standard_normal(d).astype(np.float32)
    wg = rng.standard_normal((1, d)).astype(np.float32) * 0.1
    wu = rng.standard_normal((1, d)).astype(np.float32) * 0.1
    wd = rng.standard_normal((d, 1)).astype(np.float32)
    h, o = orc.expert(x, wg, wu, wd)
    g = float(wg[0].astype(np.float64) @ x)
    u = float(wu[0].astype(np.float64) @ x)
    hh = g / (1 + np.exp(-g)) * u
    assert abs(h[0] - hh) <= 1e-5 * max(1.0, abs(hh))
    assert np.allclose(o, wd[:, 0] * hh, rtol=1e-5, atol=1e-6)


def test_expert_zero_weights_give_zero(orc):
    d, I = 64, 32
    x = np.random.default_rng(2).standard_normal(d).astype(np.float32)
    z = np.zeros((I, d), np.float32)
    h, o = orc.expert(x, z, z, np.zeros((d, I), np.float32))
    assert np.all(h == 0) and np.all(o == 0)


@pytest.mark.parametrize("dtype", ["float32", "bfloat16"])
def test_expert_against_library_f64(orc, dtype):
    layer = synth.make_layer(3, 256, 4, 96, seed=5, dtype=synth.torch_dtype(dtype))
    for t in range(3):
        for e in range(4):
            xf = layer.x[t].float().numpy()
            _, o = orc.expert(xf, synth.to_numpy(layer.w_gate[e]), synth.to_numpy(layer.w_up[e]),
                              synth.to_numpy(layer.w_down[e]))
            ref = swiglu_f64(layer.x[t].double().numpy(), layer.w_gate[e].double().numpy(),
                             layer.w_up[e].double().numpy(), layer.w_down[e].double().numpy())
            assert np.allclose(o, ref, rtol=1e-4, atol=2e-6), np.abs(o - ref).max()


def test_expert_linear_in_down_and_not_transposed(orc):
    rng = np.random.default_rng(6)
    d, I = 64, 32
    x = rng.standard_normal(d).astype(np.float32)
    wg = (rng.standard_normal((I, d)) * 0.1).astype(np.float32)
    wu = (rng.standard_normal((I, d)) * 0.1).astype(np.float32)
    wd = (rng.standard_normal((d, I)) * 0.1).astype(np.float32)
    h, o = orc.expert(x, wg, wu, wd)
    _, o2 = orc.expert(x, wg, wu, 2 * wd)
    assert np.array_equal(o2, 2 * o)
    # a unit down matrix picks channels: o_j = h_{perm j}
    eye = np.zeros((d, I), np.float32)
    perm = rng.permutation(I)
    for j in range(I):
        eye[j, perm[j]] = 1.0
    _, o3 = orc.expert(x, wg, wu, eye)
    assert np.array_equal(o3[:I], h[perm]) and np.all(o3[I:] == 0)
    # swapping gate and up changes the output (the gate is the silu side)
    _, o4 = orc.expert(x, wu, wg, wd)
    assert not np.allclose(o4, o)


def test_expert_thread_count_does_not_matter(orc):
    layer = synth.make_layer(1, 128, 2, 64, seed=7)
    xf = layer.x[0].float().numpy()
    args = (synth.to_numpy(layer.w_gate[1]), synth.to_numpy(layer.w_up[1]), synth.to_numpy(layer.w_down[1]))
    _, a = orc.expert(xf, *args, par=True)
    _, b = orc.expert(xf, *args, par=False)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- combine
def test_combine_single_slot_is_scaled_output(orc):
    o = np.random.default_rng(8).standard_normal((1, 64)).astype(np.float32)
    w = np.array([0.37], np.float32)
    assert np.array_equal(orc.combine(o, w), (w[0] * o[0]).astype(np.float32))


def test_combine_order_only_changes_rounding(orc):
    rng = np.random.default_rng(9)
    o = rng.standard_normal((8, 256)).astype(np.float32)
    w = rng.uniform(0, 1, 8).astype(np.float32)
    y = orc.combine(o, w)
    perm = rng.permutation(8)
    y2 = orc.combine(o[perm], w[perm])
    ref = (w.astype(np.float64)[:, None] * o).sum(0)
    assert np.allclose(y, ref, atol=1e-5) and np.allclose(y2, ref, atol=1e-5)


# ---------------------------------------------------------------- permutation
@pytest.mark.parametrize("T,k1,E", [(1, 8, 128), (4, 2, 16), (64, 8, 128), (4096, 8, 128),
                                     (64, 10, 512), (33, 3, 7)])
def test_permute_properties_and_bruteforce(orc, T, k1, E):
    rng = np.random.default_rng(T * 100 + k1)
    idx = np.stack([rng.choice(E, k1, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, sorted_slot, slot_pos = orc.permute(idx, E)
    counts = np.bincount(idx.ravel(), minlength=E)
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert offsets[-1] == T * k1
    assert np.array_equal(sorted_slot, np.argsort(idx.ravel(), kind="stable"))
    assert np.array_equal(sorted_slot[slot_pos], np.arange(T * k1))
    for e in range(E):
        seg = sorted_slot[offsets[e]:offsets[e + 1]]
        assert np.all(idx.ravel()[seg] == e) and np.all(np.diff(seg) > 0)


def test_permute_empty_and_bad(orc):
    offsets, ss, sp = orc.permute(np.zeros((0, 4), np.int32), 8)
    assert np.all(offsets == 0) and ss.size == 0 and sp.size == 0
    with pytest.raises(orc.OracleError):
        orc.permute(np.array([[0, 9]], np.int32), 8)


# ---------------------------------------------------------------- whole layer
def test_layer_identical_experts_scale_by_weight_sum(orc):
    """All experts equal: y = (sum_s w_s) * FFN(x) and sum_s w_s = M(k1)/M(k2)."""
    T, d, E, I = 6, 64, 16, 32
    base = synth.make_layer(T, d, 1, I, seed=10, dtype=torch.float32)
    wr = synth.make_layer(T, d, E, 1, seed=11, dtype=torch.float32).w_router.numpy() * 40
    wg = np.repeat(base.w_gate.numpy(), E, 0)
    wu = np.repeat(base.w_up.numpy(), E, 0)
    wd = np.repeat(base.w_down.numpy(), E, 0)
    x = base.x.numpy()
    ffn = swiglu_f64(x.astype(np.float64), base.w_gate[0].double().numpy(),
                     base.w_up[0].double().numpy(), base.w_down[0].double().numpy())
    for k1, k2 in [(2, 2), (2, 4), (2, 16), (4, 8)]:
        out = orc.layer(x, wr, None, wg, wu, wd, k1, k2)
        _, _, p = orc.route_f64(out["z"].astype(np.float64), k1, k2)
        ps = -np.sort(-p, axis=1)
        ratio = ps[:, :k1].sum(1) / (ps[:, :min(k2, E)].sum(1) if k2 < E else 1.0)
        assert np.allclose(out["y"], ratio[:, None] * ffn, rtol=1e-4, atol=1e-6)
        if k1 == k2:
            assert np.allclose(out["y"], ffn, rtol=1e-4, atol=1e-6)


def test_layer_single_expert_is_swiglu_mlp(orc):
    layer = synth.make_layer(5, 128, 1, 64, seed=12, dtype=torch.float32)
    out = orc.layer(layer.x.numpy(), layer.w_router.numpy(), None, layer.w_gate.numpy(),
                    layer.w_up.numpy(), layer.w_down.numpy(), 1, 1)
    assert np.all(out["w"] == 1.0) and np.all(out["idx"] == 0)
    ref = swiglu_f64(layer.x.double().numpy(), layer.w_gate[0].double().numpy(),
                     layer.w_up[0].double().numpy(), layer.w_down[0].double().numpy())
    assert np.allclose(out["y"], ref, rtol=1e-4, atol=1e-6)


def test_layer_zero_experts_give_zero(orc):
    layer = synth.make_layer(3, 64, 16, 32, seed=13, dtype=torch.float32)
    zg = np.zeros_like(layer.w_gate.numpy())
    out = orc.layer(layer.x.numpy(), layer.w_router.numpy(), None, zg, zg,
                    np.zeros_like(layer.w_down.numpy()), 2, 4)
    assert np.all(out["y"] == 0)


def test_layer_brute_force_sum_over_selected(orc):
    """y equals the Eq. 2 weighted sum of per-expert library SwiGLU outputs,
    with the selection re-derived in double precision."""
    layer = synth.make_layer(4, 64, 16, 32, seed=0, dtype=torch.float32)
    for k1, k2 in [(2, 2), (2, 4), (2, 16)]:
        out = orc.layer(layer.x.numpy(), layer.w_router.numpy(), None, layer.w_gate.numpy(),
                        layer.w_up.numpy(), layer.w_down.numpy(), k1, k2)
        z = layer.x.double() @ layer.w_router.double().T
        p = torch.softmax(z, -1).numpy()
        for t in range(4):
            order = sorted(range(16), key=lambda j: (-p[t, j], j))
            sel = order[:k1]
            mass = sum(p[t, j] for j in order[:min(k2, 16)]) if k2 < 16 else 1.0
            ref = sum(p[t, e] / mass * swiglu_f64(layer.x[t].double().numpy(),
                                                   layer.w_gate[e].double().numpy(),
                                                   layer.w_up[e].double().numpy(),
                                                   layer.w_down[e].double().numpy())
                      for e in sel)
            assert out["idx"][t].tolist() == sel
            assert np.allclose(out["y"][t], ref, rtol=1e-4, atol=1e-6)


def test_layer_routes_from_given_logits(orc):
    layer = synth.make_layer(4, 64, 16, 32, seed=14, dtype=torch.float32)
    z = np.random.default_rng(0).standard_normal((4, 16)).astype(np.float32)
    out = orc.layer(layer.x.numpy(), layer.w_router.numpy(), None, layer.w_gate.numpy(),
                    layer.w_up.numpy(), layer.w_down.numpy(), 2, 4, logits_in=z)
    idx, w = orc.route_f32(z, 2, 4)
    assert np.array_equal(out["idx"], idx) and np.array_equal(out["w"], w)
    assert np.array_equal(out["z"], z)


def test_layer_tokens_matches_layer(orc):
    layer = synth.make_layer(6, 128, 16, 64, seed=15)
    args = [synth.to_numpy(t) for t in (layer.x, layer.w_router, layer.w_gate, layer.w_up, layer.w_down)]
    full = orc.layer(args[0], args[1], None, args[2], args[3], args[4], 4, 8)
    sub = orc.layer_tokens(args[0][[1, 4]], full["z"][[1, 4]],
                           lambda e: (args[2][e], args[3][e], args[4][e]), 4, 8)
    assert np.array_equal(sub["y"], full["y"][[1, 4]])


def test_seeded_inputs_reproducible():
    a = synth.make_layer(2, 64, 16, 32, seed=0, layer=3)
    b = synth.make_layer(2, 64, 16, 32, seed=0, layer=3)
    c = synth.make_layer(2, 64, 16, 32, seed=0, layer=4)
    for f in ("x", "w_router", "w_gate", "w_up", "w_down"):
        assert torch.equal(getattr(a, f), getattr(b, f))
        assert not torch.equal(getattr(a, f), getattr(c, f))
    rms = a.x.float().pow(2).mean(-1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-2)
