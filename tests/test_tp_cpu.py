"""Host logic of the channel-split tensor-parallel layer on CPU: the channel
ranges, the weight shards, and two gloo ranks whose oracle partials summed by
an all-reduce give the whole layer.

Source: "Channel Selection for Mixture-of-Experts Decoding Needs No
Calibration Data" (paperlayer.ai), section 2 "Background" (a channel owns a
gate row, an up row and a down column, so the layer splits over channels).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_channel_ranges_cover_the_channels_once():
    from routed_expert_layer_route_b200 import tp
    for I, world in ((768, 1), (768, 2), (768, 4), (768, 8), (1024, 8), (96, 2)):
        seen = np.zeros(I, int)
        for r in range(world):
            lo, hi = tp.channel_range(I, world, r)
            assert (hi - lo) % tp.CHANNEL_ALIGN == 0 and hi - lo == I // world
            seen[lo:hi] += 1
        assert (seen == 1).all()
    for I, world, rank in ((768, 5, 0), (96, 4, 0), (768, 2, 2), (768, 0, 0)):
        with pytest.raises(ValueError):
            tp.channel_range(I, world, rank)


def test_shards_are_the_channel_slices():
    from routed_expert_layer_route_b200 import synth, tp
    L = synth.make_layer(2, 64, 4, 64, seed=3, device="cpu")
    parts = [tp.shard_weights(L.w_gate, L.w_up, L.w_down, r, 4) for r in range(4)]
    assert torch.equal(torch.cat([p[0] for p in parts], dim=1), L.w_gate)
    assert torch.equal(torch.cat([p[1] for p in parts], dim=1), L.w_up)
    assert torch.equal(torch.cat([p[2] for p in parts], dim=2), L.w_down)
    assert all(p[2].is_contiguous() for p in parts)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from routed_expert_layer_route_b200 import synth, tp
        T, d, E, I, k1, k2 = 3, 64, 8, 64, 3, 5
        L = synth.make_layer(T, d, E, I, seed=9, device="cpu", bias="normal")
        wg, wu, wd = tp.shard_weights(L.w_gate, L.w_up, L.w_down, rank, world)
        args = [synth.to_numpy(t) for t in (L.x, L.w_router, L.bias)]
        part = oracle.layer(*args, synth.to_numpy(wg), synth.to_numpy(wu), synth.to_numpy(wd),
                            k1, k2)
        y = torch.from_numpy(part["y"].copy())
        dist.all_reduce(y)
        full = oracle.layer(*args, synth.to_numpy(L.w_gate), synth.to_numpy(L.w_up),
                            synth.to_numpy(L.w_down), k1, k2)
        q.put((rank, part["idx"].tolist(), float(np.abs(y.numpy() - full["y"]).max()),
               float(np.abs(full["y"]).max()), full["idx"].tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_sum_their_shards_to_the_layer():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, idx, err, scale, full_idx = q.get(timeout=120)
        out[r] = (idx, err, scale, full_idx)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        idx, err, scale, full_idx = out[r]
        assert idx == full_idx          # every rank routes like the whole layer
        assert err <= 1e-5 * scale      # the summed partials are the layer
