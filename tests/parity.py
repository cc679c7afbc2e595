"""Helpers shared by the GPU parity tests: run the C-ABI path on seeded
inputs and compare with the CPU oracle.

Tolerances (layer output, float32 accumulation on bf16-rounded inputs):
max-abs error 2e-2 and relative L2 error 5e-3 against the oracle.  Routing
indices and weights are compared bit for bit, the oracle routing the GPU's
own float32 logits (so a near-tie at the k1 boundary cannot turn a
last-bit logit difference into an O(1) output difference); the logits
themselves are checked separately against the oracle's.
"""
import numpy as np
import torch

import oracle
from routed_expert_layer_route_b200 import moe, synth

MAX_ABS = 2e-2
REL_L2 = 5e-3


def takes_grouped_path(T, d, I, flags):
    """The path moe_layer takes rounds h to bf16 (the tensor-core grouped
    GEMMs): explicitly, or by AUTO for two or more tokens with d and I
    multiples of 128 (the rule in include/moe.h)."""
    path = flags & moe.MOE_PATH_MASK
    if path == moe.MOE_PATH_GROUPED:
        return True
    return (path == moe.MOE_PATH_AUTO and not (flags & moe.MOE_WDOWN_CHANNEL_MAJOR)
            and T >= 2 and d % 128 == 0 and I % 128 == 0)


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def assert_close_layer(y_gpu, y_ref, what=""):
    err = float(np.abs(y_gpu - y_ref).max()) if y_ref.size else 0.0
    rel = rel_l2(y_gpu, y_ref) if y_ref.size else 0.0
    assert err <= MAX_ABS and rel <= REL_L2, "%s max-abs %.3g rel-L2 %.3g" % (what, err, rel)
    return err, rel


def logits_bound(x, w):
    d = x.shape[-1]
    return 1e-4 * np.sqrt(d) * float(x.abs().max()) * float(w.abs().max())


def run_layer(L, k1, k2, y_dtype=torch.float32, flags=moe.MOE_PATH_AUTO, ws=None, w_down=None):
    """moe_layer on the GPU; w_down overrides L.w_down (e.g. the channel-major
    copy, with flags | MOE_WDOWN_CHANNEL_MAJOR)."""
    T, d = L.x.shape
    E, I, _ = L.w_gate.shape
    dev = L.x.device
    if ws is None:
        ws = moe.workspace(T, d, E, I, k1, device=dev)
    y = torch.empty(T, d, device=dev, dtype=y_dtype)
    idx = torch.empty(T, k1, device=dev, dtype=torch.int32)
    w = torch.empty(T, k1, device=dev, dtype=torch.float32)
    z = torch.empty(T, E, device=dev, dtype=torch.float32)
    moe.moe_layer(L.x, L.w_router, L.bias, L.w_gate, L.w_up,
                  L.w_down if w_down is None else w_down, k1, k2, y, ws,
                  topk_idx_out=idx, topk_w_out=w, logits_out=z, flags=flags)
    torch.cuda.synchronize()
    status = moe.moe_read_device_status(ws)
    assert status == 0, moe.status_string(status)
    return y, idx, w, z


def check_layer_full(L, k1, k2, flags=moe.MOE_PATH_AUTO, tight=None, w_down=None):
    """Whole-layer parity against oracle.layer (all tokens, all weights on host).
    tight (default: unless the path rounds h to bf16): float32 output within
    1e-4 relative, i.e. only the summation order differs from the oracle."""
    T, d = L.x.shape
    if tight is None:
        tight = not takes_grouped_path(T, d, L.w_gate.shape[1], flags)
    y, idx, w, z = run_layer(L, k1, k2, flags=flags, w_down=w_down)
    zn = z.cpu().numpy()
    # logits against the oracle's own
    z_or = oracle.logits(synth.to_numpy(L.x), synth.to_numpy(L.w_router), synth.to_numpy(L.bias))
    assert np.abs(zn - z_or).max() <= logits_bound(L.x, L.w_router)
    ref = oracle.layer(synth.to_numpy(L.x), synth.to_numpy(L.w_router), synth.to_numpy(L.bias),
                       synth.to_numpy(L.w_gate), synth.to_numpy(L.w_up), synth.to_numpy(L.w_down),
                       k1, k2, logits_in=zn)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert np.array_equal(w.cpu().numpy(), ref["w"])
    yy = y.cpu().numpy()
    err, rel = assert_close_layer(yy, ref["y"], "layer")
    if tight:
        # float32 output: only summation order differs from the oracle
        assert rel <= 1e-4, rel
    return yy, ref


def check_layer_sampled(L, k1, k2, tokens, flags=moe.MOE_PATH_AUTO, w_down=None, tight=None,
                        by_expert=False):
    """Parity on sampled tokens; expert weights are fetched to the host only
    for the experts those tokens use.  tokens: a list, or a function of the
    GPU's routing [T x k1] returning the list.  by_expert: fetch each expert
    once and drop it after use (oracle_layer_by_expert), for many tokens of a
    large layer.  tight as for check_layer_full."""
    T, d = L.x.shape
    if tight is None:
        tight = not takes_grouped_path(T, d, L.w_gate.shape[1], flags)
    y, idx, w, z = run_layer(L, k1, k2, flags=flags, w_down=w_down)
    if callable(tokens):
        tokens = tokens(idx.cpu().numpy())
    tokens = np.asarray(tokens)
    zn = z.cpu().numpy()[tokens]
    xs = synth.to_numpy(L.x[torch.as_tensor(tokens, device=L.x.device)])
    # logits of the sampled tokens against the oracle's own
    z_or = oracle.logits(xs, synth.to_numpy(L.w_router), synth.to_numpy(L.bias))
    assert np.abs(zn - z_or).max() <= logits_bound(L.x, L.w_router)

    def fetch(e):
        return (synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]), synth.to_numpy(L.w_down[e]))

    if by_expert:
        ref = oracle_layer_by_expert(L, tokens, zn, k1, k2)
    else:
        ref = oracle.layer_tokens(xs, zn, fetch, k1, k2)
    assert np.array_equal(idx.cpu().numpy()[tokens], ref["idx"])
    assert np.array_equal(w.cpu().numpy()[tokens], ref["w"])
    yy = y.cpu().numpy()[tokens]
    err, rel = assert_close_layer(yy, ref["y"], "sampled layer")
    if tight:
        assert rel <= 1e-4, rel
    return idx.cpu().numpy()


def oracle_layer_by_expert(L, tokens, z_rows, k1, k2):
    """oracle.layer_tokens for many sampled tokens of a large layer, with
    each routed expert's weights brought to the host once and dropped after
    use (the same oracle steps: route the given float32 logits, every routed
    slot through oracle.expert, oracle.combine in slot order)."""
    idx, w = oracle.route_f32(z_rows, k1, k2)
    xs = synth.to_numpy(L.x[torch.as_tensor(np.asarray(tokens), device=L.x.device)])
    xf = (xs.astype(np.uint32) << 16).view(np.float32)
    n, d = xf.shape
    o = np.empty((n, k1, d), np.float32)
    for e in np.unique(idx):
        e = int(e)
        wg, wu, wd = (synth.to_numpy(L.w_gate[e]), synth.to_numpy(L.w_up[e]),
                      synth.to_numpy(L.w_down[e]))
        for t, s in zip(*np.nonzero(idx == e)):
            o[t, s] = oracle.expert(xf[t], wg, wu, wd)[1]
    y = np.stack([oracle.combine(o[t], w[t]) for t in range(n)]) if n else np.empty((0, d))
    return {"y": y, "idx": idx, "w": w}


def tile_boundary_tokens(idx, E, n, seed, tile=256, half=128):
    """Up to n tokens of a routed batch that exercise the grouped GEMMs' token
    tiles: the routed tokens (in the stable expert order the permutation
    builds) at positions 0, half-1, half, tile-1, tile, ... of every expert
    and every token of the busiest expert's last, partial tile; the rest
    drawn at random (seeded).  idx: [T x k1] routing of the batch."""
    T, k1 = idx.shape
    flat = idx.ravel()
    order = np.argsort(flat, kind="stable")   # slots in expert order, stable by slot
    counts = np.bincount(flat, minlength=E)
    offs = np.concatenate([[0], np.cumsum(counts)])
    pick = []
    busiest = int(np.argmax(counts))
    c = int(counts[busiest])
    last0 = (c - 1) // tile * tile if c else 0
    pick += [int(order[offs[busiest] + j]) // k1 for j in range(last0, c)]
    for e in np.argsort(-counts, kind="stable"):
        for j in range(0, int(counts[e]), half):
            for q in (j - 1, j):
                if 0 <= q < counts[e]:
                    pick.append(int(order[offs[e] + q]) // k1)
    seen, out = set(), []
    for t in pick:
        if t not in seen and len(out) < n:
            seen.add(t)
            out.append(t)
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(T), np.asarray(out, np.int64))
    extra = rng.choice(rest, size=min(len(rest), n - len(out)), replace=False)
    return sorted(out + [int(t) for t in extra])
