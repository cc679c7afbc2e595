"""GPU parity of the channel top-k layer (moe_layer_channel_topk) and the
down-column norms (moe_channel_norms) against the oracle.

Source: "Channel Selection for Mixture-of-Experts Decoding Needs No
Calibration Data" (paperlayer.ai), section 2 "Background" and sections
5.2-5.3; Eq. 2 of "Paper of the Week #3", section "The Receipt".

What is compared, and how:
  * logits within the usual bound, routing bit for bit (the oracle routes
    the GPU's logits);
  * h (every channel of the token's experts) within float32 tolerance of the
    oracle's h (summation order and the exp differ);
  * the scores bit for bit against (w_s * n) * |h| recomputed in float32
    from the GPU's own w, norms and h (the one float32 formula both sides
    take the selection from);
  * the kept set bit for bit against the oracle's selection on the GPU's
    scores;
  * y within the layer tolerance against the oracle's y over that kept set;
  * and end to end with nothing taken from the GPU but its logits: the oracle
    computes its own down-column norms, h, scores and kept set; that kept set
    must equal the GPU's except for swaps between channels whose oracle
    scores lie within SWAP_REL of the keep-th best oracle score (float32
    rounding of h can only reorder such near-ties); with no swap, y within
    the layer tolerance of the oracle's own y.
"""
import numpy as np
import pytest
import torch

import oracle
from routed_expert_layer_route_b200 import moe, synth

from parity import assert_close_layer, logits_bound

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
# relative width of the score band around the keep-th best oracle score in
# which the two kept sets may differ: h agrees to ~1e-6 relative (float32
# sums in another order), so scores that far apart are never reordered
SWAP_REL = 1e-4


@pytest.mark.parametrize("E,d,I", [(8, 256, 96), (4, 64, 16), (3, 6144, 32), (16, 2048, 768)])
def test_channel_norms_both_layouts(E, d, I):
    L = synth.make_layer(1, d, E, I, seed=E + d, device=DEV)
    n_hf = moe.moe_channel_norms(L.w_down)
    n_cm = moe.moe_channel_norms(moe.moe_pack_w_down(L.w_down), channel_major=True)
    torch.cuda.synchronize()
    wd = synth.to_numpy(L.w_down)
    ref = np.stack([oracle.channel_norms(wd[e]) for e in range(E)])
    np.testing.assert_allclose(n_hf.cpu().numpy(), ref, rtol=2e-6 * np.sqrt(d), atol=0)
    np.testing.assert_allclose(n_cm.cpu().numpy(), ref, rtol=2e-6 * np.sqrt(d), atol=0)


def _run(L, k1, k2, keep, w_down_cm=None, norms=None, y_dtype=torch.float32):
    T, d = L.x.shape
    E, I, _ = L.w_gate.shape
    if w_down_cm is None:
        w_down_cm = moe.moe_pack_w_down(L.w_down)
    if norms is None:
        norms = moe.moe_channel_norms(w_down_cm, channel_major=True)
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    y = torch.empty(T, d, dtype=y_dtype, device=DEV)
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    z = torch.empty(T, E, dtype=torch.float32, device=DEV)
    h = torch.empty(T, k1, I, dtype=torch.float32, device=DEV)
    sc = torch.empty(T, k1, I, dtype=torch.float32, device=DEV)
    kept = torch.full((T, keep), -1, dtype=torch.int32, device=DEV)
    moe.moe_layer_channel_topk(L.x, L.w_router, L.bias, L.w_gate, L.w_up, w_down_cm, norms, k1, k2,
                               keep, y, ws, topk_idx_out=idx, topk_w_out=w, logits_out=z,
                               h_out=h, scores_out=sc, kept_out=kept)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    return dict(y=y.float().cpu().numpy(), idx=idx.cpu().numpy(), w=w.cpu().numpy(),
                z=z.cpu().numpy(), h=h.cpu().numpy(), scores=sc.cpu().numpy(),
                kept=kept.cpu().numpy(), norms=norms.cpu().numpy())


def _check(L, k1, k2, keep, g, tokens=None):
    T = L.x.shape[0]
    E, I, _ = L.w_gate.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    xs = synth.to_numpy(L.x[torch.as_tensor(tokens, device=DEV)])
    z_or = oracle.logits(xs, synth.to_numpy(L.w_router), synth.to_numpy(L.bias))
    assert np.abs(g["z"][tokens] - z_or).max() <= logits_bound(L.x, L.w_router)

    def fetch(e):
        return (synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]), synth.to_numpy(L.w_down[e]))

    ref = oracle.channel_topk_tokens(xs, g["z"][tokens], fetch, lambda e: g["norms"][e], k1, k2,
                                     keep, kept_in=g["kept"][tokens])
    assert np.array_equal(g["idx"][tokens], ref["idx"])
    assert np.array_equal(g["w"][tokens], ref["w"])
    hg = g["h"][tokens]
    np.testing.assert_allclose(hg, ref["h"], rtol=1e-3, atol=1e-4 * np.abs(ref["h"]).max())
    for i, t in enumerate(tokens):
        nrm = g["norms"][g["idx"][t]]                      # [k1 x I] of the slots' experts
        want = oracle.channel_scores(g["h"][t], g["w"][t], nrm)
        assert np.array_equal(g["scores"][t], want), "score formula"
        assert np.array_equal(g["kept"][t], oracle.channel_select(g["scores"][t], keep)), "kept set"
    assert_close_layer(g["y"][tokens], ref["y"], "channel top-k layer")
    _check_own_selection(L, k1, k2, keep, g, tokens, xs, fetch)
    return ref


def _check_own_selection(L, k1, k2, keep, g, tokens, xs, fetch):
    """The oracle's own kept set (own norms, h and scores) against the GPU's."""
    wd = {}

    def own_norms(e):
        if e not in wd:
            wd[e] = oracle.channel_norms(synth.to_numpy(L.w_down[e]))
        return wd[e]

    own = oracle.channel_topk_tokens(xs, g["z"][tokens], fetch, own_norms, k1, k2, keep)
    swaps = 0
    for i, t in enumerate(tokens):
        sc = own["scores"][i].ravel().astype(np.float64)
        kth = np.sort(sc)[::-1][keep - 1]
        a, b = set(own["kept"][i].tolist()), set(g["kept"][t].tolist())
        diff = sorted(a ^ b)
        assert len(a - b) == len(b - a)
        for q in diff:
            assert abs(sc[q] - kth) <= SWAP_REL * kth, \
                "token %d channel %d: score %.9g vs keep-th %.9g" % (t, q, sc[q], kth)
        swaps += len(a - b)
        if not diff:
            assert_close_layer(g["y"][t], own["y"][i], "channel top-k, oracle's own kept set")
    print("channel top-k own selection: %d near-tie swaps over %d tokens" % (swaps, len(tokens)))
    return swaps


@pytest.mark.parametrize("T,d,E,I,k1,k2,keeps", [
    (1, 256, 16, 64, 4, 8, [1, 37, 128, 256]),
    (3, 512, 32, 96, 6, 6, [100, 576]),
    (1, 64, 8, 32, 2, 3, [5, 64]),          # d = 64: 64 rows side by side in k_ctk_down
    (2, 1536, 16, 48, 3, 16, [77]),         # d = 1536: 192 vectors per row, two rows side by side
    (1, 6144, 8, 64, 2, 2, [50, 128]),      # d = 6144: two vectors per thread
])
def test_layer_channel_topk_small(T, d, E, I, k1, k2, keeps):
    L = synth.make_layer(T, d, E, I, seed=T * 7 + d, device=DEV, bias="normal")
    wdc = moe.moe_pack_w_down(L.w_down)
    norms = moe.moe_channel_norms(wdc, channel_major=True)
    for keep in keeps:
        _check(L, k1, k2, keep, _run(L, k1, k2, keep, wdc, norms))


@pytest.mark.parametrize("k1,k2,frac", [(8, 16, 0.25), (8, 8, 0.5), (4, 16, 0.125), (8, 16, 1.0)])
def test_layer_channel_topk_decode_b1(k1, k2, frac):
    T, d, E, I = 1, 2048, 128, 768
    L = synth.make_layer(T, d, E, I, seed=11, device=DEV)
    keep = int(frac * k1 * I)
    g = _run(L, k1, k2, keep, y_dtype=torch.bfloat16)
    _check(L, k1, k2, keep, g)


def test_layer_channel_topk_large_shape():
    # d = 4096, I = 1024, k1 = 10: 10240 channels per token
    T, d, E, I, k1, k2 = 1, 4096, 32, 1024, 10, 10
    L = synth.make_layer(T, d, E, I, seed=5, device=DEV)
    g = _run(L, k1, k2, 2048)
    _check(L, k1, k2, 2048, g)


def test_keep_all_matches_the_decode_layer():
    T, d, E, I, k1, k2 = 1, 2048, 64, 256, 4, 16
    L = synth.make_layer(T, d, E, I, seed=2, device=DEV)
    wdc = moe.moe_pack_w_down(L.w_down)
    g = _run(L, k1, k2, k1 * I, wdc)
    assert np.array_equal(g["kept"][0], np.arange(k1 * I))
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    y = torch.empty(T, d, dtype=torch.float32, device=DEV)
    moe.moe_layer(L.x, L.w_router, L.bias, L.w_gate, L.w_up, wdc, k1, k2, y, ws,
                  flags=moe.MOE_WDOWN_CHANNEL_MAJOR)
    torch.cuda.synchronize()
    assert_close_layer(g["y"], y.cpu().numpy(), "keep-all vs decode layer")


def test_ties_go_to_the_lower_flat_index():
    # zero router: equal logits, w = 1/k1 exactly (k1 = k2 = 4); every expert
    # the same weights with identical rows: every channel scores the same
    T, d, E, I, k1 = 1, 256, 8, 64, 4
    L = synth.make_layer(T, d, E, I, seed=3, device=DEV)
    L.w_router.zero_()
    L.w_gate.copy_(L.w_gate[:1, :1].clone().expand(E, I, d))
    L.w_up.copy_(L.w_up[:1, :1].clone().expand(E, I, d))
    L.w_down.copy_(L.w_down[:1, :, :1].clone().expand(E, d, I))
    for keep in (1, 13, 200):
        g = _run(L, k1, k1, keep)
        assert np.all(g["scores"] == g["scores"].flat[0])
        assert np.array_equal(g["kept"][0], np.arange(keep))
        _check(L, k1, k1, keep, g)


def test_channel_topk_argument_checks():
    T, d, E, I, k1 = 1, 256, 16, 64, 4
    L = synth.make_layer(T, d, E, I, seed=1, device=DEV)
    for keep, status in ((0, moe.MOE_ERR_INVALID_ARG), (k1 * I + 1, moe.MOE_ERR_INVALID_ARG)):
        with pytest.raises(moe.MoeError) as ei:
            _run(L, k1, k1, keep)
        assert ei.value.status == status
    big = synth.make_layer(T, d, 64, 2064, seed=1, device=DEV)  # 8 * 2064 > 16384 channels
    with pytest.raises(moe.MoeError) as ei:
        _run(big, 8, 8, 100)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("T,d,E,I,k1,k2,keep", [
    (1, 64, 1024, 16, 32, 64, 1),        # the widest route (1024 experts), smallest experts
    (1, 64, 1024, 16, 32, 2000, 512),    # k2 > E: no renormalisation, every channel kept
    (2, 128, 64, 512, 32, 32, 16384),    # the most channels a token may have (32 x 512)
])
def test_layer_channel_topk_edge_shapes(T, d, E, I, k1, k2, keep):
    L = synth.make_layer(T, d, E, I, seed=E + I, device=DEV, bias="normal")
    _check(L, k1, k2, keep, _run(L, k1, k2, keep))
