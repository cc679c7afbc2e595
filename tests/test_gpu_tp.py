"""GPU parity of the channel-split tensor-parallel layer: the G shards of a
layer run one after another on one GPU (each exactly what rank g runs), every
shard routes bit-identically, and the sum of their float32 partials -- what
the all-reduce forms across ranks -- matches the oracle's whole layer.

Source: "Channel Selection for Mixture-of-Experts Decoding Needs No
Calibration Data" (paperlayer.ai), section 2 "Background"; Eq. 2 of "Paper of
the Week #3", section "The Receipt".
"""
import numpy as np
import pytest
import torch

import oracle
from routed_expert_layer_route_b200 import moe, synth, tp

from parity import assert_close_layer, logits_bound

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _shards_sum(L, k1, k2, world, channel_major):
    T, d = L.x.shape
    E = L.w_gate.shape[0]
    total = torch.zeros(T, d, dtype=torch.float32, device=DEV)
    routes = []
    for r in range(world):
        sh = tp.ChannelSplitLayer(L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, r, world,
                                  channel_major=channel_major)
        ws = moe.workspace(T, d, E, sh.I_shard, k1, device=DEV)
        part = torch.empty(T, d, dtype=torch.float32, device=DEV)
        idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
        w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
        z = torch.empty(T, E, dtype=torch.float32, device=DEV)
        sh.partial(L.x, k1, k2, part, ws, topk_idx_out=idx, topk_w_out=w, logits_out=z)
        torch.cuda.synchronize()
        assert moe.moe_read_device_status(ws) == 0
        total += part
        routes.append((idx.cpu().numpy(), w.cpu().numpy(), z.cpu().numpy()))
    torch.cuda.synchronize()
    return total.cpu().numpy(), routes


@pytest.mark.parametrize("T,world,channel_major,bias", [
    (1, 2, True, None), (1, 4, True, None), (1, 8, True, None),   # decode path per shard
    (8, 2, False, "normal"),                                      # grouped GEMMs (I/G = 384)
    (8, 4, False, "normal"),                                      # streaming kernel (I/G = 192)
])
def test_channel_split_sums_to_the_layer(T, world, channel_major, bias):
    d, E, I, k1, k2 = 2048, 128, 768, 8, 16
    L = synth.make_layer(T, d, E, I, seed=4, device=DEV, bias=bias)
    y, routes = _shards_sum(L, k1, k2, world, channel_major)
    idx0, w0, z0 = routes[0]
    for idx, w, z in routes[1:]:  # every rank routes the same way, bit for bit
        assert np.array_equal(idx, idx0) and np.array_equal(w, w0) and np.array_equal(z, z0)
    z_or = oracle.logits(synth.to_numpy(L.x), synth.to_numpy(L.w_router), synth.to_numpy(L.bias))
    assert np.abs(z0 - z_or).max() <= logits_bound(L.x, L.w_router)

    def fetch(e):
        return (synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]), synth.to_numpy(L.w_down[e]))

    ref = oracle.layer_tokens(synth.to_numpy(L.x), z0, fetch, k1, k2)
    assert np.array_equal(idx0, ref["idx"]) and np.array_equal(w0, ref["w"])
    assert_close_layer(y, ref["y"], "channel-split sum of %d shards" % world)


def test_forward_without_a_group_is_the_partial():
    T, d, E, I, k1, k2 = 1, 2048, 64, 256, 4, 16
    L = synth.make_layer(T, d, E, I, seed=6, device=DEV)
    sh = tp.ChannelSplitLayer(L.w_router, L.bias, L.w_gate, L.w_up, L.w_down, 0, 1,
                              channel_major=True)
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    y = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    sh.forward(L.x, k1, k2, y, ws)
    full = torch.empty(T, d, dtype=torch.float32, device=DEV)
    moe.moe_layer(L.x, L.w_router, L.bias, L.w_gate, L.w_up, moe.moe_pack_w_down(L.w_down), k1,
                  k2, full, moe.workspace(T, d, E, I, k1, device=DEV),
                  flags=moe.MOE_WDOWN_CHANNEL_MAJOR)
    torch.cuda.synchronize()
    assert_close_layer(y.float().cpu().numpy(), full.cpu().numpy(), "world 1 forward")
