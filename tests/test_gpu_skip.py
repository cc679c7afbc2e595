"""GPU parity of expert skipping (top-1 kept) against the oracle: routing bit
for bit on the same logits, and the layer on the one-token decode path and on
the tensor-core grouped path, where skipped slots sit between kept ones.

Source: "ACE" (aimodeling.com), section "How ACE decides what to skip: GSP +
RCR"; Eq. 2 of "Paper of the Week #3", section "The Receipt".
"""
import math

import numpy as np
import pytest
import torch

import oracle
from routed_expert_layer_route_b200 import moe, synth

from parity import assert_close_layer, logits_bound

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _table(E, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.rand(E, generator=g, dtype=torch.float32)


@pytest.mark.parametrize("T,E,k1,k2", [(64, 16, 4, 8), (64, 128, 8, 16), (33, 256, 8, 8),
                                       (9, 1024, 10, 20)])
@pytest.mark.parametrize("th_e,th_w", [(0.0, 0.0), (0.5, 0.1), (0.7, 0.3), (2.0, math.inf)])
def test_route_skip_bit_exact(T, E, k1, k2, th_e, th_w):
    rng = np.random.default_rng(T + E)
    z = rng.normal(0, 2.0, (T, E)).astype(np.float32)
    tab = _table(E, E)
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    cnt = torch.empty(T, dtype=torch.int32, device=DEV)
    moe.moe_route_skip(None, None, None, torch.from_numpy(z).to(DEV), k1, k2, tab.to(DEV), th_e,
                       th_w, idx, w, cnt)
    torch.cuda.synchronize()
    ri, rw, rk = oracle.route_skip_f32(z, k1, k2, tab.numpy(), th_e, th_w)
    assert np.array_equal(cnt.cpu().numpy(), rk)
    assert np.array_equal(idx.cpu().numpy(), ri)
    assert np.array_equal(w.cpu().numpy(), rw)


def _run(L, k1, k2, tab, th_e, th_w, flags, w_down=None):
    T, d = L.x.shape
    E, I, _ = L.w_gate.shape
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    y = torch.empty(T, d, dtype=torch.float32, device=DEV)
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    cnt = torch.empty(T, dtype=torch.int32, device=DEV)
    z = torch.empty(T, E, dtype=torch.float32, device=DEV)
    moe.moe_layer_skip(L.x, L.w_router, L.bias, L.w_gate, L.w_up,
                       L.w_down if w_down is None else w_down, k1, k2, tab, th_e, th_w, y, ws,
                       topk_idx_out=idx, topk_w_out=w, topk_count_out=cnt, logits_out=z,
                       flags=flags)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    return y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(), cnt.cpu().numpy(), z.cpu().numpy()


def _check(L, k1, k2, tab, th_e, th_w, out, tokens):
    y, idx, w, cnt, z = out
    tokens = np.asarray(tokens)
    xs = synth.to_numpy(L.x[torch.as_tensor(tokens, device=DEV)])
    z_or = oracle.logits(xs, synth.to_numpy(L.w_router), synth.to_numpy(L.bias))
    assert np.abs(z[tokens] - z_or).max() <= logits_bound(L.x, L.w_router)
    ri, rw, rk = oracle.route_skip_f32(z[tokens], k1, k2, tab.cpu().numpy(), th_e, th_w)
    assert np.array_equal(idx[tokens], ri) and np.array_equal(w[tokens], rw)
    assert np.array_equal(cnt[tokens], rk)

    def fetch(e):
        return (synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]), synth.to_numpy(L.w_down[e]))

    ref = oracle.layer_tokens_slots(xs, ri, rw, fetch)
    assert_close_layer(y[tokens], ref, "skip layer")
    return rk


def _peaky(T, d, E, I, seed, bias=None):
    L = synth.make_layer(T, d, E, I, seed=seed, device=DEV, bias=bias)
    L.w_router = (L.w_router.float() * (1.5 / (0.02 * d ** 0.5))).to(torch.bfloat16)
    return L


@pytest.mark.parametrize("th_e,th_w", [(0.5, 0.1), (0.8, 0.2)])
def test_layer_skip_grouped_all_tokens(th_e, th_w):
    T, d, E, I, k1, k2 = 48, 256, 16, 128, 4, 8
    L = _peaky(T, d, E, I, seed=21, bias="normal")
    tab = _table(E, 3).to(DEV)
    out = _run(L, k1, k2, tab, th_e, th_w, moe.MOE_PATH_GROUPED)
    k = _check(L, k1, k2, tab, th_e, th_w, out, list(range(T)))
    idx = out[1]
    # skipped slots between kept ones occur
    assert any(idx[t, s] == moe.MOE_EMPTY_SLOT and idx[t, s + 1] != moe.MOE_EMPTY_SLOT
               for t in range(T) for s in range(1, k1 - 1))
    assert k.min() < k1


def test_layer_skip_decode_one_token():
    d, E, I, k1, k2 = 256, 16, 64, 6, 8
    hits = 0
    for seed in range(6):
        L = _peaky(1, d, E, I, seed=40 + seed)
        tab = _table(E, seed).to(DEV)
        out = _run(L, k1, k2, tab, 0.6, 0.15, moe.MOE_WDOWN_CHANNEL_MAJOR,
                   w_down=moe.moe_pack_w_down(L.w_down))
        k = _check(L, k1, k2, tab, 0.6, 0.15, out, [0])
        hits += int(k[0] < k1)
    assert hits > 0


def test_layer_skip_decode_few_tokens():
    # the few-token decode kernel: skipped slots between kept ones
    d, E, I, k1, k2 = 256, 16, 64, 6, 8
    hits = 0
    for T, seed in ((2, 60), (4, 61), (7, 62)):
        L = _peaky(T, d, E, I, seed=seed)
        tab = _table(E, seed).to(DEV)
        out = _run(L, k1, k2, tab, 0.6, 0.15, moe.MOE_WDOWN_CHANNEL_MAJOR,
                   w_down=moe.moe_pack_w_down(L.w_down))
        k = _check(L, k1, k2, tab, 0.6, 0.15, out, list(range(T)))
        hits += int((k < k1).sum())
    assert hits > 0


def test_layer_skip_full_size_decode_and_batch():
    tab = _table(128, 11).to(DEV)
    L1 = _peaky(1, 2048, 128, 768, seed=0)
    out = _run(L1, 8, 16, tab, 0.5, 0.12, moe.MOE_WDOWN_CHANNEL_MAJOR,
               w_down=moe.moe_pack_w_down(L1.w_down))
    _check(L1, 8, 16, tab, 0.5, 0.12, out, [0])
    L = _peaky(64, 2048, 128, 768, seed=1, bias="normal")
    out = _run(L, 8, 16, tab, 0.5, 0.12, moe.MOE_PATH_AUTO)
    _check(L, 8, 16, tab, 0.5, 0.12, out, [0, 7, 31, 63])


def test_skip_argument_checks():
    L = synth.make_layer(1, 256, 16, 64, seed=1, device=DEV)
    tab = _table(16, 0).to(DEV)
    wdc = moe.moe_pack_w_down(L.w_down)
    for t, th_e, th_w in ((None, 0.5, 0.5), (tab, math.nan, 0.5), (tab, 0.5, math.nan)):
        with pytest.raises(moe.MoeError) as ei:
            _run(L, 4, 8, t, th_e, th_w, moe.MOE_WDOWN_CHANNEL_MAJOR, w_down=wdc)
        assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    L2 = synth.make_layer(4, 192, 16, 96, seed=1, device=DEV)  # d, I not multiples of 128
    with pytest.raises(moe.MoeError) as ei:
        _run(L2, 4, 8, tab, 0.5, 0.5, moe.MOE_PATH_AUTO)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE


def test_layer_skip_edge_shapes():
    # 32 slots of 1024 experts on the decode path; every slot but the first skipped
    d, E, I, k1, k2 = 64, 1024, 16, 32, 32
    L = _peaky(1, d, E, I, seed=77)
    tab = torch.zeros(E, dtype=torch.float32, device=DEV)
    out = _run(L, k1, k2, tab, 1.0, math.inf, moe.MOE_WDOWN_CHANNEL_MAJOR,
               w_down=moe.moe_pack_w_down(L.w_down))
    k = _check(L, k1, k2, tab, 1.0, math.inf, out, [0])
    assert k[0] == 1
