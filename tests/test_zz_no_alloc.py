"""moe_expert_ffn_noalloc: the expert-FFN step for callers that cannot give
the library device scratch memory (for example a plugin inside an engine
that owns the whole device memory pool, or a service that forbids
allocations after start-up).  Its scratch is a fixed array inside libmoe.so.

Checked against moe_expert_ffn (the workspace entry point) on the same
routed inputs, within the layer tolerance the other tests use (max-abs 2e-2,
relative L2 5e-3), over calls made back to back so that whatever one call
leaves in the shared array cannot disturb the next; every routed slot of the
one-token and the three-token case is also checked against the CPU oracle's
expert on the bf16-rounded inputs, and the array's device status word must
read OK after the calls.  This file is collected last so a
stop-at-first-failure run has already run every other test."""
import numpy as np
import pytest
import torch

import oracle
from routed_expert_layer_route_b200 import moe, synth

from parity import assert_close_layer

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def routed_case(T, d, E, I, k1, k2, seed, bias):
    L = synth.make_layer(T, d, E, I, seed=seed, device=DEV, bias=bias)
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    z = torch.empty(T, E, dtype=torch.float32, device=DEV)
    moe.moe_route(L.x, L.w_router, L.bias, z, k1, k2, idx, w)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    ss = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    sp = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    moe.moe_permute(idx, E, off, ss, sp)
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    ref = torch.empty(T * k1, d, dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn(L.x, off, ss, L.w_gate, L.w_up, L.w_down, k1, ref, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    L.idx = idx
    return L, off, ss, k1, ref


def assert_slots_match_oracle(L, ss, k1, out):
    """Every routed slot's expert output against the oracle's expert (float32
    on the bf16-rounded token and weights)."""
    ssn, idxn, on = ss.cpu().numpy(), L.idx.cpu().numpy().ravel(), out.cpu().numpy()
    xn = synth.to_numpy(L.x)
    xf = (xn.astype(np.uint32) << 16).view(np.float32)
    for p in range(ssn.size):
        slot = int(ssn[p])
        t, e = slot // k1, int(idxn[slot])
        _, o = oracle.expert(xf[t], synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]),
                             synth.to_numpy(L.w_down[e]))
        assert_close_layer(on[p], o, "noalloc slot %d vs oracle" % p)


def test_noalloc_matches_workspace_entry_on_calls_in_a_row():
    cases = [routed_case(1, 2048, 128, 768, 8, 8, 0, None),
             routed_case(8, 512, 64, 256, 4, 16, 1, "normal"),
             routed_case(3, 256, 16, 96, 2, 4, 2, None)]
    outs = []
    for L, off, ss, k1, ref in cases + cases[:1]:   # four calls back to back, no sync between
        out = torch.full_like(ref, float("nan"))
        moe.moe_expert_ffn_noalloc(L.x, off, ss, L.w_gate, L.w_up, L.w_down, k1, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert moe.moe_noalloc_read_status() == 0
    for (L, off, ss, k1, ref), out in zip(cases + cases[:1], outs):
        got, want = out.cpu().numpy(), ref.cpu().numpy()
        assert np.isfinite(got).all()
        assert_close_layer(got, want, "noalloc")
    for i in (0, 2, 3):  # the one-token case (twice) and the three-token case
        L, off, ss, k1, _ = (cases + cases[:1])[i]
        assert_slots_match_oracle(L, ss, k1, outs[i])


def test_noalloc_rejects_shapes_beyond_its_scratch():
    T, d, E, I, k1 = 128, 512, 64, 1024, 8   # T*k1*I = 1048576 > 1047424
    L = synth.make_layer(1, d, E, 16, seed=3, device=DEV)
    x = torch.zeros(T, d, dtype=torch.bfloat16, device=DEV)
    wg = torch.zeros(E, I, d, dtype=torch.bfloat16, device=DEV)
    wd = torch.zeros(E, d, I, dtype=torch.bfloat16, device=DEV)
    off = torch.zeros(E + 1, dtype=torch.int32, device=DEV)
    ss = torch.zeros(T * k1, dtype=torch.int32, device=DEV)
    out = torch.empty(T * k1, d, dtype=torch.float32, device=DEV)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_expert_ffn_noalloc(x, off, ss, wg, wg, wd, k1, out)
    assert ei.value.status == moe.MOE_ERR_SCRATCH_LIMIT
    del L
