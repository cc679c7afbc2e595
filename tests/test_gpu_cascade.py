"""GPU parity of the variable-k (cascade) route and layer against the oracle:
each token takes experts in rank order until their probability mass reaches
tau (at most k1), weighted by Eq. 2 with the fixed k2.

Source: the "cascade ... cover" arm of "Reading the MoE measurement defects"
(kozo-lab), sections 4 and 6.2-6.3; Eq. 2 of "Paper of the Week #3", section
"The Receipt".
"""
import numpy as np
import pytest
import torch

import oracle
from routed_expert_layer_route_b200 import moe, synth

from parity import assert_close_layer, logits_bound

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.mark.parametrize("T,E,k1,k2", [(64, 16, 4, 8), (64, 128, 8, 16), (33, 128, 8, 128),
                                       (16, 512, 10, 20), (9, 40, 6, 1000)])
@pytest.mark.parametrize("tau", [0.0, 0.3, 0.7, 0.9, 1.5])
def test_route_cascade_bit_exact(T, E, k1, k2, tau):
    rng = np.random.default_rng(T + E + k1)
    z = rng.normal(0, 2.0, (T, E)).astype(np.float32)
    zg = torch.from_numpy(z).to(DEV)
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    cnt = torch.empty(T, dtype=torch.int32, device=DEV)
    moe.moe_route_cascade(None, None, None, zg, k1, k2, tau, idx, w, cnt)
    torch.cuda.synchronize()
    ri, rw, rk = oracle.route_cascade_f32(z, k1, k2, tau)
    assert np.array_equal(cnt.cpu().numpy(), rk)
    assert np.array_equal(idx.cpu().numpy(), ri)
    assert np.array_equal(w.cpu().numpy(), rw)


@pytest.mark.parametrize("T,k1,E,chunked", [(40, 8, 32, False), (1500, 8, 128, True)])
def test_permute_with_empty_slots(T, k1, E, chunked):
    rng = np.random.default_rng(5)
    z = rng.normal(0, 2.5, (T, E)).astype(np.float32)
    ri, _, rk = oracle.route_cascade_f32(z, k1, k1, 0.6)
    assert rk.min() < k1  # some slots are empty
    off, ss, sp = oracle.permute(ri, E)
    ti = torch.from_numpy(ri).to(DEV)
    g_off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    g_ss = torch.full((T * k1,), -7, dtype=torch.int32, device=DEV)
    g_sp = torch.full((T * k1,), -7, dtype=torch.int32, device=DEV)
    ws = moe.workspace(T, 64, E, 16, k1, device=DEV) if chunked else None
    moe.moe_permute(ti, E, g_off, g_ss, g_sp, ws=ws)
    torch.cuda.synchronize()
    if ws is not None:
        assert moe.moe_read_device_status(ws) == 0
    n = int(off[-1])
    assert np.array_equal(g_off.cpu().numpy(), off)
    assert np.array_equal(g_ss.cpu().numpy()[:n], ss)
    valid = ri.ravel() != oracle.EMPTY_SLOT
    assert np.array_equal(g_sp.cpu().numpy()[valid], sp[valid])


def _peaky_layer(T, d, E, I, seed, bias=None):
    """A layer whose router logits spread (std ~1.5), so the cascade's k varies."""
    L = synth.make_layer(T, d, E, I, seed=seed, device=DEV, bias=bias)
    L.w_router = (L.w_router.float() * (1.5 / (0.02 * d ** 0.5))).to(torch.bfloat16)
    return L


def _run_cascade(L, k1, k2, tau, flags, w_down=None):
    T, d = L.x.shape
    E, I, _ = L.w_gate.shape
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    y = torch.empty(T, d, dtype=torch.float32, device=DEV)
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    cnt = torch.empty(T, dtype=torch.int32, device=DEV)
    z = torch.empty(T, E, dtype=torch.float32, device=DEV)
    moe.moe_layer_cascade(L.x, L.w_router, L.bias, L.w_gate, L.w_up,
                          L.w_down if w_down is None else w_down, k1, k2, tau, y, ws,
                          topk_idx_out=idx, topk_w_out=w, topk_count_out=cnt, logits_out=z,
                          flags=flags)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    return y, idx, w, cnt, z


def _check_against_oracle(L, k1, k2, tau, y, idx, w, cnt, z, tokens):
    tokens = np.asarray(tokens)
    zn = z.cpu().numpy()[tokens]
    xs = synth.to_numpy(L.x[torch.as_tensor(tokens, device=DEV)])
    z_or = oracle.logits(xs, synth.to_numpy(L.w_router), synth.to_numpy(L.bias))
    assert np.abs(zn - z_or).max() <= logits_bound(L.x, L.w_router)

    def fetch(e):
        return (synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]), synth.to_numpy(L.w_down[e]))

    ref = oracle.layer_tokens_cascade(xs, zn, fetch, k1, k2, tau)
    assert np.array_equal(cnt.cpu().numpy()[tokens], ref["k"])
    assert np.array_equal(idx.cpu().numpy()[tokens], ref["idx"])
    assert np.array_equal(w.cpu().numpy()[tokens], ref["w"])
    assert_close_layer(y.cpu().numpy()[tokens], ref["y"], "cascade layer")
    return ref["k"]


@pytest.mark.parametrize("tau", [0.3, 0.6, 0.9])
def test_layer_cascade_grouped_all_tokens(tau):
    T, d, E, I, k1, k2 = 48, 256, 16, 128, 4, 8
    L = _peaky_layer(T, d, E, I, seed=21, bias="normal")
    y, idx, w, cnt, z = _run_cascade(L, k1, k2, tau, moe.MOE_PATH_GROUPED)
    k = _check_against_oracle(L, k1, k2, tau, y, idx, w, cnt, z, list(range(T)))
    if tau < 0.9:
        assert k.min() < k1  # the cascade stops early for some tokens


@pytest.mark.parametrize("tau", [0.2, 0.5, 0.8, 0.99])
def test_layer_cascade_decode_one_token(tau):
    d, E, I, k1, k2 = 256, 16, 64, 6, 8
    for seed in range(3):
        L = _peaky_layer(1, d, E, I, seed=30 + seed)
        wdc = moe.moe_pack_w_down(L.w_down)
        y, idx, w, cnt, z = _run_cascade(L, k1, k2, tau, moe.MOE_WDOWN_CHANNEL_MAJOR, w_down=wdc)
        _check_against_oracle(L, k1, k2, tau, y, idx, w, cnt, z, [0])


@pytest.mark.parametrize("tau", [0.3, 0.7])
def test_layer_cascade_decode_few_tokens(tau):
    # the few-token decode kernel: each token's k_t slots, empty slots skipped
    # in the union of the routed experts
    d, E, I, k1, k2 = 256, 16, 64, 6, 8
    ks = []
    for T, seed in ((2, 50), (5, 51), (8, 52)):
        L = _peaky_layer(T, d, E, I, seed=seed, bias="normal")
        wdc = moe.moe_pack_w_down(L.w_down)
        y, idx, w, cnt, z = _run_cascade(L, k1, k2, tau, moe.MOE_WDOWN_CHANNEL_MAJOR, w_down=wdc)
        ks.append(_check_against_oracle(L, k1, k2, tau, y, idx, w, cnt, z, list(range(T))))
    assert np.concatenate(ks).min() < k1  # the cascade stops early for some tokens


@pytest.mark.parametrize("tau", [0.5, 0.9])
def test_layer_cascade_full_size_decode_and_batch(tau):
    L1 = _peaky_layer(1, 2048, 128, 768, seed=0)
    y, idx, w, cnt, z = _run_cascade(L1, 8, 16, tau, moe.MOE_WDOWN_CHANNEL_MAJOR,
                                     w_down=moe.moe_pack_w_down(L1.w_down))
    _check_against_oracle(L1, 8, 16, tau, y, idx, w, cnt, z, [0])
    L = _peaky_layer(64, 2048, 128, 768, seed=1, bias="normal")
    y, idx, w, cnt, z = _run_cascade(L, 8, 16, tau, moe.MOE_PATH_AUTO)
    _check_against_oracle(L, 8, 16, tau, y, idx, w, cnt, z, [0, 7, 31, 63])


def test_cascade_rejects_the_streaming_path():
    L = synth.make_layer(4, 192, 16, 96, seed=1, device=DEV)  # d, I not multiples of 128
    with pytest.raises(moe.MoeError) as ei:
        _run_cascade(L, 4, 8, 0.5, moe.MOE_PATH_AUTO)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE
