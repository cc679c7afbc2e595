"""GPU parity of the whole layer and of its expert-FFN / combine steps
against the CPU oracle, at small sizes (every token checked) and at the
method's full workload sizes (sampled tokens).

Expert structure: "Channel Selection for Mixture-of-Experts Decoding Needs No
Calibration Data", section 2 "Background"; weights: Eq. 2 of "Paper of the
Week #3", section "The Receipt".
"""
import numpy as np
import pytest
import torch

import oracle
from routed_expert_layer_route_b200 import moe, synth

from parity import (assert_close_layer, check_layer_full, check_layer_sampled, run_layer,
                    tile_boundary_tokens)

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _free():
    yield
    torch.cuda.empty_cache()


SMALL = [
    # T, d, E, I, k1, k2, bias
    (1, 64, 16, 32, 2, 2, None),
    (4, 64, 16, 32, 2, 4, None),
    (4, 64, 16, 32, 2, 16, None),
    (1, 256, 16, 64, 2, 4, None),
    (2, 256, 64, 96, 8, 16, "normal"),
    (7, 512, 64, 256, 4, 16, "normal"),
    (33, 256, 32, 80, 3, 5, None),
    (64, 1024, 64, 128, 8, 64, "zipf"),
    (5, 128, 1, 48, 1, 1, None),
    (3, 192, 20, 32, 20, 20, None),      # k1 = E: every expert runs
    (17, 320, 40, 112, 6, 1000, None),   # k2 > E: no renormalisation
]


CM = moe.MOE_WDOWN_CHANNEL_MAJOR


@pytest.mark.parametrize("T,d,E,I,k1,k2,bias", SMALL)
def test_layer_small_all_tokens(T, d, E, I, k1, k2, bias):
    L = synth.make_layer(T, d, E, I, seed=T + d + E, device=DEV, bias=bias)
    check_layer_full(L, k1, k2)
    if T <= 8:  # the single-pass decode path on the channel-major down matrix
        wdc = moe.moe_pack_w_down(L.w_down)
        check_layer_full(L, k1, k2, flags=CM, w_down=wdc)
        check_layer_full(L, k1, k2, flags=moe.MOE_PATH_DECODE | CM, w_down=wdc)


@pytest.mark.parametrize("E,d,I", [(16, 64, 32), (3, 2048, 768), (2, 320, 112), (1, 4096, 1024)])
def test_pack_w_down_is_the_transpose(E, d, I):
    wd = synth.normal((E, d, I), 1.0, synth.make_generator(DEV, 5), DEV, torch.bfloat16)
    wdc = moe.moe_pack_w_down(wd)
    torch.cuda.synchronize()
    assert torch.equal(wdc, wd.transpose(1, 2).contiguous())


@pytest.mark.parametrize("d,E,I,k1,k2", [(64, 16, 32, 2, 4), (256, 64, 96, 8, 16),
                                          (1024, 40, 112, 6, 1000), (192, 20, 32, 20, 20),
                                          (512, 128, 256, 32, 64),
                                          # many experts: 128 router CTAs of 8 rows, the
                                          # widest warp router; E not a power of two
                                          (256, 1024, 32, 8, 16), (512, 1000, 48, 6, 40),
                                          (4096, 300, 64, 4, 12)])
def test_decode_path_single_token(d, E, I, k1, k2):
    L = synth.make_layer(1, d, E, I, seed=d + E + k1, device=DEV, bias="normal")
    wdc = moe.moe_pack_w_down(L.w_down)
    check_layer_full(L, k1, k2, flags=CM, w_down=wdc)


# the few-token decode kernel: (tokens the partials cover, row vectors per lane)
# = (2, 1), (4, 1), (8, 1), (2, 2), (4, 2); one to three channels per stage;
# experts shared by several tokens (E small) and none shared (E large)
FEW = [
    # T, d, E, I, k1, k2, bias
    (2, 256, 64, 96, 8, 16, "normal"),
    (2, 5632, 16, 32, 2, 4, None),        # one channel per stage, two row vectors per lane
    (3, 512, 128, 256, 4, 16, None),
    (4, 4096, 300, 64, 4, 12, "normal"),  # E not a power of two, two row vectors per lane
    (5, 1024, 40, 112, 6, 1000, None),    # k2 > E
    (6, 256, 1024, 32, 8, 16, "normal"),  # seven router rows per CTA, the widest router
    (7, 2816, 64, 128, 8, 8, None),       # the widest d with one row vector per lane
    (8, 128, 8, 16, 8, 8, None),          # k1 = E: all eight tokens on every expert
    (8, 2048, 128, 768, 8, 16, "zipf"),
    (8, 512, 200, 48, 8, 1000, None),     # T*k1 = 64 slots, short experts: several per CTA
]


@pytest.mark.parametrize("T,d,E,I,k1,k2,bias", FEW)
def test_decode_path_few_tokens(T, d, E, I, k1, k2, bias):
    L = synth.make_layer(T, d, E, I, seed=T * 7 + d + E, device=DEV, bias=bias)
    wdc = moe.moe_pack_w_down(L.w_down)
    check_layer_full(L, k1, k2, flags=CM, w_down=wdc)
    check_layer_full(L, k1, k2, flags=moe.MOE_PATH_DECODE | CM, w_down=wdc)
    # bf16 output: the float32 result rounded (up to one step: the sums' order varies)
    y32, *_ = run_layer(L, k1, k2, flags=CM, w_down=wdc)
    y16, *_ = run_layer(L, k1, k2, flags=CM, w_down=wdc, y_dtype=torch.bfloat16)
    assert torch.allclose(y32.to(torch.bfloat16).float(), y16.float(), rtol=2 ** -7, atol=1e-6)


@pytest.mark.parametrize("T,E,k1,k2,group", [(4, 128, 8, 16, 2), (8, 64, 6, 20, 3),
                                             (2, 128, 32, 127, 128), (5, 16, 4, 8, 16)])
def test_decode_few_tokens_route_ties(T, E, k1, k2, group):
    """Equal logits on the few-token path: repeated router rows give bit-equal
    logits; the rank order falls back to the lower expert index."""
    d, I = 256, 32
    L = synth.make_layer(T, d, E, I, seed=E + k1 + group + T, device=DEV)
    L.w_router = L.w_router[torch.arange(E, device=DEV) // group * group].contiguous()
    wdc = moe.moe_pack_w_down(L.w_down)
    _, idx, _, z = run_layer(L, k1, k2, flags=CM, w_down=wdc)
    zn = z.cpu().numpy()
    for g0 in range(0, E, group):
        assert np.all(zn[:, g0:g0 + group] == zn[:, g0:g0 + 1])
    check_layer_full(L, k1, k2, flags=CM, w_down=wdc)


@pytest.mark.parametrize("E,k1,k2,group", [(128, 8, 16, 2), (128, 4, 128, 4), (128, 32, 127, 128),
                                           (64, 6, 20, 3), (16, 4, 8, 16), (100, 5, 9, 7),
                                           (512, 10, 20, 4)])
def test_decode_route_ties(E, k1, k2, group):
    """Equal logits on the one-token path: router rows repeated in runs of
    `group` give bit-equal logits, so the rank order must fall back to the
    lower expert index (the tie rule of the page's router, restated in the
    oracle).  group = E: every logit equal, p = 1/E."""
    d, I = 256, 32
    L = synth.make_layer(1, d, E, I, seed=E + k1 + group, device=DEV)
    L.w_router = L.w_router[torch.arange(E, device=DEV) // group * group].contiguous()
    wdc = moe.moe_pack_w_down(L.w_down)
    _, idx, _, z = run_layer(L, k1, k2, flags=CM, w_down=wdc)
    zn = z.cpu().numpy()[0]
    for g0 in range(0, E, group):  # the repeated rows give bit-equal logits
        assert np.all(zn[g0:g0 + group] == zn[g0])
    check_layer_full(L, k1, k2, flags=CM, w_down=wdc)


def test_channel_major_down_token_limits():
    # nine tokens, or eight with more than one row vector per lane per token
    # partial (d > 2816), or more than 64 routed slots: no decode kernel
    for T, d, k1 in ((9, 256, 2), (8, 4096, 2), (5, 256, 16)):
        L = synth.make_layer(T, d, 16, 32, seed=7, device=DEV)
        wdc = moe.moe_pack_w_down(L.w_down)
        with pytest.raises(moe.MoeError) as ei:
            run_layer(L, k1, 16, flags=CM, w_down=wdc)
        assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE
    L = synth.make_layer(2, 256, 16, 32, seed=7, device=DEV)
    with pytest.raises(moe.MoeError) as ei:  # the decode path needs the channel-major matrix
        run_layer(L, 2, 4, flags=moe.MOE_PATH_DECODE)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("packed", [False, True], ids=["stream", "decode"])
def test_layer_bf16_output_is_rounded_f32_output(packed):
    T = 1 if packed else 9
    L = synth.make_layer(T, 512, 32, 64, seed=2, device=DEV)
    kw = dict(flags=CM, w_down=moe.moe_pack_w_down(L.w_down)) if packed else {}
    y32, *_ = run_layer(L, 4, 8, y_dtype=torch.float32, **kw)
    y16, *_ = run_layer(L, 4, 8, y_dtype=torch.bfloat16, **kw)
    if not packed:  # deterministic path: exactly the rounded float32 output
        assert torch.equal(y32.to(torch.bfloat16), y16)
    else:  # float32 sums in a timing-dependent order: equal up to one bf16 rounding step
        assert torch.allclose(y32.to(torch.bfloat16).float(), y16.float(), rtol=2 ** -7, atol=1e-6)


def test_layer_deterministic_and_workspace_reuse():
    L = synth.make_layer(8, 512, 32, 64, seed=3, device=DEV, bias="normal")
    big = moe.workspace(64, 2048, 128, 768, 8, device=DEV)   # larger than needed
    st = moe.MOE_PATH_STREAM
    a, ia, wa, _ = run_layer(L, 4, 16, ws=big, flags=st)
    b, ib, wb, _ = run_layer(L, 4, 16, ws=big, flags=st)
    c, ic, wc, _ = run_layer(L, 4, 16, flags=st)
    assert torch.equal(a, b) and torch.equal(a, c)
    assert torch.equal(ia, ic) and torch.equal(wa, wc)
    # the one-token decode path routes identically and agrees to float32 rounding
    L1 = synth.make_layer(1, 512, 32, 64, seed=3, device=DEV, bias="normal")
    s_y, s_i, s_w, _ = run_layer(L1, 4, 16, ws=big, flags=st)
    d_y, d_i, d_w, _ = run_layer(L1, 4, 16, ws=big, flags=CM, w_down=moe.moe_pack_w_down(L1.w_down))
    assert torch.equal(d_i, s_i) and torch.equal(d_w, s_w)
    assert torch.allclose(d_y, s_y, rtol=1e-5, atol=1e-6)
    # the few-token decode path on the same workspace after the calls above
    # (the decode accumulator sits at one place for every batch size)
    wdc = moe.moe_pack_w_down(L.w_down)
    for _ in range(2):
        m_y, m_i, m_w, _ = run_layer(L, 4, 16, ws=big, flags=CM, w_down=wdc)
        assert torch.equal(m_i, ia) and torch.equal(m_w, wa)
        assert torch.allclose(m_y, a, rtol=1e-5, atol=1e-6)
        run_layer(L1, 4, 16, ws=big, flags=st)


def test_indices_do_not_depend_on_k2():
    L = synth.make_layer(16, 256, 64, 32, seed=4, device=DEV)
    base = run_layer(L, 4, 4)[1]
    for k2 in (8, 16, 64, 500):
        assert torch.equal(run_layer(L, 4, k2)[1], base)


def test_expert_ffn_and_combine_steps():
    T, d, E, I, k1, k2 = 12, 384, 24, 96, 3, 6
    L = synth.make_layer(T, d, E, I, seed=5, device=DEV, bias="normal")
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    z = torch.empty(T, E, dtype=torch.float32, device=DEV)
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    moe.moe_route(L.x, L.w_router, L.bias, z, k1, k2, idx, w)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    ss = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    sp = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    moe.moe_permute(idx, E, off, ss, sp)
    out = torch.empty(T * k1, d, dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn(L.x, off, ss, L.w_gate, L.w_up, L.w_down, k1, out, ws)
    y = torch.empty(T, d, dtype=torch.float32, device=DEV)
    moe.moe_combine(out, sp, w, y)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    # per-slot expert outputs against the oracle expert
    ssn, idxn, on = ss.cpu().numpy(), idx.cpu().numpy(), out.cpu().numpy()
    xn = synth.to_numpy(L.x)
    xf = (xn.astype(np.uint32) << 16).view(np.float32)
    for p in range(T * k1):
        slot = int(ssn[p])
        t, e = slot // k1, int(idxn.ravel()[slot])
        _, o = oracle.expert(xf[t], synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]),
                             synth.to_numpy(L.w_down[e]))
        assert_close_layer(on[p], o, "slot %d" % p)
        assert np.abs(on[p] - o).max() <= 1e-4 * max(1.0, np.abs(o).max())
    # combine against the oracle combine of the GPU's own expert outputs
    spn, wn = sp.cpu().numpy(), w.cpu().numpy()
    for t in range(T):
        ref = oracle.combine(on[spn[t * k1:(t + 1) * k1]], wn[t])
        assert np.allclose(y[t].cpu().numpy(), ref, rtol=0, atol=1e-6)
    # and the whole layer gives the same y
    y2, *_ = run_layer(L, k1, k2)
    assert torch.allclose(y, y2, rtol=0, atol=1e-6)


def test_zero_tokens_is_a_noop():
    L = synth.make_layer(0, 256, 16, 32, seed=6, device=DEV)
    ws = moe.workspace(1, 256, 16, 32, 2, device=DEV)
    y = torch.empty(0, 256, device=DEV)
    moe.moe_layer(L.x, L.w_router, None, L.w_gate, L.w_up, L.w_down, 2, 4, y, ws)
    torch.cuda.synchronize()


# ------------------------------------------------------------------ full sizes
# the method's workloads: d=2048, E=128, I=768 (decode / prefill) and
# d=4096, E=512, I=1024 (large), bf16, launched exactly as the benchmark does
@pytest.mark.parametrize("k1,k2", [(8, 8), (8, 16), (8, 128), (4, 4), (4, 16), (4, 128)])
def test_decode_b1_full_size(k1, k2):
    for layer in range(2):
        L = synth.make_layer(1, 2048, 128, 768, seed=0, layer=layer, device=DEV)
        check_layer_sampled(L, k1, k2, [0])
        check_layer_sampled(L, k1, k2, [0], flags=CM, w_down=moe.moe_pack_w_down(L.w_down))


@pytest.mark.parametrize("T", [8, 32])
@pytest.mark.parametrize("k1,k2", [(8, 8), (4, 16)])
def test_decode_small_batch_full_size(T, k1, k2):
    L = synth.make_layer(T, 2048, 128, 768, seed=0, layer=1, device=DEV, bias="normal")
    tokens = list(range(T)) if T == 8 else [0, 5, 17, 31]
    check_layer_sampled(L, k1, k2, tokens)  # AUTO: the tensor-core path
    check_layer_sampled(L, k1, k2, tokens, flags=moe.MOE_PATH_STREAM)
    if T <= 8:  # the few-token decode kernel
        check_layer_sampled(L, k1, k2, tokens, flags=CM, w_down=moe.moe_pack_w_down(L.w_down))


@pytest.mark.parametrize("T", [1, 64])
@pytest.mark.parametrize("k1,k2", [(10, 10), (5, 20)])
def test_large_full_size(T, k1, k2):
    # every token of the batch, each routed expert's weights fetched once
    L = synth.make_layer(T, 4096, 512, 1024, seed=0, layer=0, device=DEV)
    check_layer_sampled(L, k1, k2, list(range(T)), by_expert=True)
    if T == 1:
        check_layer_sampled(L, k1, k2, [0], flags=CM, w_down=moe.moe_pack_w_down(L.w_down))


@pytest.mark.parametrize("k1,k2", [(8, 16), (4, 16)])
def test_prefill_full_size_sampled(k1, k2):
    # AUTO runs the tensor-core grouped GEMMs at this batch size; 256 tokens:
    # every token of the busiest expert's last, partial token tile, the tokens
    # at the 128- and 256-row token-tile boundaries of the experts, the first
    # and last token, the rest drawn at random
    L = synth.make_layer(4096, 2048, 128, 768, seed=0, layer=0, device=DEV, bias="zipf")

    def pick(idx):
        return sorted(set(tile_boundary_tokens(idx, 128, 254, seed=k1)) | {0, 4095})

    idx = check_layer_sampled(L, k1, k2, pick, by_expert=True)
    # Zipf bias: the most popular expert gets many more tokens than the least
    counts = np.bincount(idx.ravel(), minlength=128)
    assert counts.max() > 4 * max(1, np.median(counts))
    # the streaming path on the same layer (float32 h: tight), 64 of its tokens
    check_layer_sampled(L, k1, k2, lambda i: tile_boundary_tokens(i, 128, 64, seed=k1 + 1),
                        flags=moe.MOE_PATH_STREAM, by_expert=True)


# ------------------------------------------------------------------ tensor-core grouped path
GROUPED = moe.MOE_PATH_GROUPED
GSMALL = [
    # T, d, E, I, k1, k2, bias
    (1, 128, 8, 128, 2, 4, None),
    (16, 128, 16, 128, 4, 8, None),
    (64, 256, 16, 256, 4, 16, "normal"),
    (300, 256, 4, 128, 2, 4, None),      # > 256 slots per expert: several token tiles
    (200, 512, 32, 384, 8, 8, "zipf"),   # ragged tiles, experts without tokens
    (37, 384, 64, 128, 3, 1000, None),
    (130, 128, 2, 256, 2, 2, None),      # k1 = E: every token in every expert
    (256, 256, 128, 128, 4, 16, "normal"),  # router logits on the tensor cores too
    (300, 128, 256, 128, 6, 6, None),    # two 128-expert logit tiles, ragged token tile
    # I a multiple of 256: the gate/up GEMM runs on CTA pairs (256-row tiles)
    (600, 256, 4, 512, 2, 4, None),      # 300 slots per expert: a full and a ragged token tile
    (77, 256, 16, 768, 5, 9, "zipf"),    # three 256-row tiles, tiles of a few tokens
    (9, 128, 8, 256, 1, 2, None),        # token tiles of one to a few tokens (N = 16)
    (520, 384, 2, 256, 1, 2, "normal"),  # k1 = 1: token tiles of 256 exactly and a remainder
]


@pytest.fixture(params=["pair", "single"])
def gemm_kernels(request):
    """Run a grouped-path test with the CTA-pair gate/up GEMM (where I allows
    it) and again with the single-CTA one."""
    moe.moe_test_set_grouped_single(1 if request.param == "single" else 0)
    yield request.param
    moe.moe_test_set_grouped_single(0)


def test_pair_kernels_launchable():
    # a B200 holds many clusters of two of these CTAs; the pair kernel is the default
    assert moe.moe_test_grouped_pairs(1) >= 1
    assert moe.moe_test_grouped_pairs(2) == -1


@pytest.mark.parametrize("T,d,E,I,k1,k2,bias", GSMALL)
def test_layer_grouped_all_tokens(T, d, E, I, k1, k2, bias, gemm_kernels):
    L = synth.make_layer(T, d, E, I, seed=T + d + E + 1, device=DEV, bias=bias)
    check_layer_full(L, k1, k2, flags=GROUPED, tight=False)


@pytest.mark.parametrize("T,d,E,I,k1", [(48, 256, 8, 128, 2), (520, 128, 4, 256, 2),
                                       (300, 256, 6, 512, 3)])
def test_expert_ffn_grouped_per_slot(T, d, E, I, k1, gemm_kernels):
    L = synth.make_layer(T, d, E, I, seed=11, device=DEV, bias="normal")
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    idx = torch.empty(T, k1, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k1, dtype=torch.float32, device=DEV)
    z = torch.empty(T, E, dtype=torch.float32, device=DEV)
    moe.moe_route(L.x, L.w_router, L.bias, z, k1, k1, idx, w)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    ss = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    sp = torch.empty(T * k1, dtype=torch.int32, device=DEV)
    moe.moe_permute(idx, E, off, ss, sp)
    out = torch.full((T * k1, d), float("nan"), dtype=torch.float32, device=DEV)
    moe.moe_expert_ffn(L.x, off, ss, L.w_gate, L.w_up, L.w_down, k1, out, ws, flags=GROUPED)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
    ssn, idxn, on = ss.cpu().numpy(), idx.cpu().numpy(), out.cpu().numpy()
    xf = (synth.to_numpy(L.x).astype(np.uint32) << 16).view(np.float32)
    experts = {}
    ref = np.empty_like(on)
    for p in range(T * k1):
        slot = int(ssn[p])
        t, e = slot // k1, int(idxn.ravel()[slot])
        if e not in experts:
            experts[e] = (synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]),
                          synth.to_numpy(L.w_down[e]))
        ref[p] = oracle.expert(xf[t], *experts[e])[1]
    assert_close_layer(on, ref, "grouped expert outputs")


def test_grouped_rejects_partial_tiles():
    L = synth.make_layer(8, 192, 8, 128, seed=1, device=DEV)   # d not a multiple of 128
    with pytest.raises(moe.MoeError) as ei:
        run_layer(L, 2, 4, flags=GROUPED)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE
