"""GPU routing parity: the device exponential, the float32 softmax / top-k /
Eq. 2 weights and the permutation, compared bit for bit with the oracle.

Eq. 2: "Paper of the Week #3 -- Half the FLOPs Is Not Half the Time",
section "The Receipt"; order of operations: its "Code of the Week" section.
"""
import numpy as np
import pytest
import torch

import oracle
from routed_expert_layer_route_b200 import moe, synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def gpu_exp(x_np):
    x = torch.from_numpy(x_np).to(DEV)
    y = torch.empty_like(x)
    moe.moe_test_exp_c(x, y)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def test_device_exp_matches_oracle_bitwise():
    # every 5th float32 in [-87, -0], plus the values around -87, 0 and beyond
    lo = np.float32(-0.0).view(np.uint32)
    hi = np.float32(-87.0).view(np.uint32)
    for start in range(int(lo), int(hi) + 1, 1 << 26):
        bits = np.arange(start, min(start + (1 << 26), int(hi) + 1), 5, dtype=np.uint64)
        x = bits.astype(np.uint32).view(np.float32)
        assert np.array_equal(gpu_exp(x).view(np.uint32), oracle.exp_c(x).view(np.uint32))
    edge = np.array([0.0, -0.0, -87.0, -87.00001, -88.0, -1e30, -np.inf, np.nan, 1.0, 88.0, 88.5,
                     -0.34657359, 0.34657359, -1e-30], np.float32)
    rnd = np.random.default_rng(0).uniform(-100, 0, 1 << 20).astype(np.float32)
    for x in (edge, rnd):
        assert np.array_equal(gpu_exp(x).view(np.uint32), oracle.exp_c(x).view(np.uint32))


def route_gpu(z_np, k1, k2):
    z = torch.from_numpy(np.ascontiguousarray(z_np, np.float32)).to(DEV)
    T = z.shape[0]
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    moe.moe_route(None, None, None, z, k1, k2, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


CASES = [
    (4, 16, 2, 2), (4, 16, 2, 4), (4, 16, 2, 16),
    (1, 128, 8, 8), (1, 128, 8, 16), (1, 128, 8, 128), (1, 128, 4, 4), (1, 128, 4, 16),
    (1, 128, 4, 128), (32, 128, 8, 8), (32, 128, 4, 16), (4096, 128, 8, 16), (4096, 128, 4, 16),
    (64, 512, 10, 10), (64, 512, 5, 20), (7, 1024, 8, 8), (5, 1000, 32, 999), (3, 33, 3, 2000),
    (9, 1, 1, 1), (2, 128, 32, 64),
]


@pytest.mark.parametrize("T,E,k1,k2", CASES)
@pytest.mark.parametrize("scale", [1.0, 30.0])
def test_route_bit_exact(T, E, k1, k2, scale):
    z = synth.make_logits(T, E, seed=T * 7 + E, scale=scale).numpy()
    idx, w = route_gpu(z, k1, k2)
    ri, rw = oracle.route_f32(z, k1, k2)
    assert np.array_equal(idx, ri)
    assert np.array_equal(w.view(np.uint32), rw.view(np.uint32))


@pytest.mark.parametrize("E,k1,k2", [(16, 2, 4), (128, 8, 16), (128, 4, 128), (512, 5, 20)])
def test_route_ties_bit_exact(E, k1, k2):
    rng = np.random.default_rng(E + k1)
    T = 64
    z = np.zeros((T, E), np.float32)
    z[1] = 1.0                                                   # all equal
    z[2:20] = rng.integers(-2, 3, (18, E)).astype(np.float32)    # many exact duplicates
    base = rng.standard_normal(E).astype(np.float32)
    for t in range(20, T):                                       # ulp-adjacent near ties
        z[t] = base
        j = rng.integers(0, E, 4)
        z[t, j] = np.nextafter(z[t, j], np.float32(np.inf))
    idx, w = route_gpu(z, k1, k2)
    ri, rw = oracle.route_f32(z, k1, k2)
    assert np.array_equal(idx, ri)
    assert np.array_equal(w.view(np.uint32), rw.view(np.uint32))


@pytest.mark.parametrize("T,d,E,bias", [(1, 2048, 128, None), (8, 2048, 128, "normal"),
                                         (33, 512, 64, None), (64, 4096, 512, None),
                                         (3, 64, 16, "zipf")])
def test_route_from_hidden_states(T, d, E, bias):
    L = synth.make_layer(T, d, E, 16, seed=1, device=DEV, bias=bias)
    z = torch.empty(T, E, dtype=torch.float32, device=DEV)
    idx = torch.empty(T, 4, dtype=torch.int32, device=DEV)
    w = torch.empty(T, 4, dtype=torch.float32, device=DEV)
    moe.moe_route(L.x, L.w_router, L.bias, z, 4, 8, idx, w)
    torch.cuda.synchronize()
    zn = z.cpu().numpy()
    z_or = oracle.logits(synth.to_numpy(L.x), synth.to_numpy(L.w_router), synth.to_numpy(L.bias))
    bound = 1e-4 * np.sqrt(d) * float(L.x.abs().max()) * float(L.w_router.abs().max())
    assert np.abs(zn - z_or).max() <= bound
    ri, rw = oracle.route_f32(zn, 4, 8)
    assert np.array_equal(idx.cpu().numpy(), ri)
    assert np.array_equal(w.cpu().numpy(), rw)
    # routing without a logits output goes through the workspace
    ws = moe.workspace(T, d, E, 16, 4, device=DEV)
    idx2 = torch.empty_like(idx)
    w2 = torch.empty_like(w)
    moe.moe_route(L.x, L.w_router, L.bias, None, 4, 8, idx2, w2, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(w, w2)


@pytest.mark.parametrize("T,k1,E", [(1, 8, 128), (4, 2, 16), (64, 8, 128), (4096, 8, 128),
                                     (4096, 4, 128), (64, 10, 512), (33, 3, 7), (100, 8, 1024),
                                     (1, 1, 1), (2000, 32, 64)])
def test_permute_exact(T, k1, E):
    rng = np.random.default_rng(T + k1 + E)
    idx = np.stack([rng.choice(E, k1, replace=False) for _ in range(T)]).astype(np.int32)
    off, ss, sp = oracle.permute(idx, E)
    ti = torch.from_numpy(idx).to(DEV)
    g_off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    g_ss = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    g_sp = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    moe.moe_permute(ti, E, g_off, g_ss, g_sp)
    torch.cuda.synchronize()
    assert np.array_equal(g_off.cpu().numpy(), off)
    assert np.array_equal(g_ss.cpu().numpy(), ss)
    assert np.array_equal(g_sp.cpu().numpy(), sp)
    if T * k1 > 4096:  # with a workspace: the chunked two-kernel sort
        ws = moe.workspace(T, 64, E, 16, k1, device=DEV)
        for t in (g_off, g_ss, g_sp):
            t.fill_(-7)
        moe.moe_permute(ti, E, g_off, g_ss, g_sp, ws=ws)
        torch.cuda.synchronize()
        assert moe.moe_read_device_status(ws) == 0
        assert np.array_equal(g_off.cpu().numpy(), off)
        assert np.array_equal(g_ss.cpu().numpy(), ss)
        assert np.array_equal(g_sp.cpu().numpy(), sp)


def test_permute_chunked_bad_expert_sets_device_status():
    E, T, k1 = 64, 1024, 8
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(E, k1, replace=False) for _ in range(T)]).astype(np.int32)
    idx[5, 3] = 99
    idx[700, 0] = -2
    ws = moe.workspace(T, 64, E, 16, k1, device=DEV)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    ss = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    sp = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    moe.moe_permute(torch.from_numpy(idx).to(DEV), E, off, ss, sp, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_CHECK
    assert int(off[-1]) == T * k1 - 2  # the two bad slots are dropped
    good = np.sort(ss.cpu().numpy()[: T * k1 - 2])
    assert np.array_equal(good, np.setdiff1d(np.arange(T * k1), [5 * k1 + 3, 700 * k1]))


def test_permute_bad_expert_sets_device_status():
    E, T, k1 = 16, 4, 2
    idx = torch.tensor([[0, 1], [2, 99], [3, 4], [5, -1]], dtype=torch.int32, device=DEV)
    ws = moe.workspace(T, 64, E, 16, k1, device=DEV)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    ss = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    sp = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    moe.moe_permute(idx, E, off, ss, sp, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_CHECK
    assert moe.moe_read_device_status(ws) == 0  # reading clears it
    assert int(off[-1]) == 6                    # the two bad slots are dropped
