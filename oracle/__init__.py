"""Python wrapper (ctypes + numpy) around the plain C oracle in oracle.c.

TEST INFRASTRUCTURE ONLY.  The test-suite, the smoke check and the CPU-baseline
leg of the benchmark are the only callers.  Nothing in the GPU product path
imports this package, and this package imports nothing from the product.

Array conventions
-----------------
* float32 numpy arrays are passed as float32 (dtype code 0);
* numpy ``uint16`` arrays are read as bfloat16 bit patterns (dtype code 1) and
  widened exactly to float32 inside the C code.

What each function computes, and which passage it follows, is documented in
oracle.c next to the C function of the same name.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    """Load (building first if needed) liboracle.so."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        vp = ctypes.c_void_p
        ci = ctypes.c_int
        L.oracle_exp_c.argtypes = [ctypes.c_float]
        L.oracle_exp_c.restype = ctypes.c_float
        L.oracle_exp_c_array.argtypes = [f32p, f32p, ctypes.c_int64]
        L.oracle_exp_c_array.restype = None
        L.oracle_exp_c_sweep.argtypes = [ctypes.c_uint32, i64p, i64p]
        L.oracle_exp_c_sweep.restype = ctypes.c_double
        L.oracle_softmax_f32.argtypes = [f32p, ci, f32p]
        L.oracle_softmax_f32.restype = None
        L.oracle_route_f32.argtypes = [f32p, ci, ci, ci, ci, i32p, f32p]
        L.oracle_route_f32.restype = ci
        L.oracle_route_cascade_f32.argtypes = [f32p, ci, ci, ci, ci, ctypes.c_float, i32p, f32p,
                                               i32p]
        L.oracle_route_cascade_f32.restype = ci
        L.oracle_route_f64.argtypes = [f64p, ci, ci, ci, ci, i32p, f64p, f64p]
        L.oracle_route_f64.restype = ci
        L.oracle_logits.argtypes = [vp, ci, vp, ci, f32p, ci, ci, ci, f32p]
        L.oracle_logits.restype = None
        L.oracle_expert.argtypes = [f32p, vp, vp, vp, ci, ci, ci, f32p, f32p, ci]
        L.oracle_expert.restype = None
        L.oracle_combine.argtypes = [f32p, f32p, ci, ci, f32p]
        L.oracle_combine.restype = None
        L.oracle_permute.argtypes = [i32p, ci, ci, ci, i32p, i32p, i32p]
        L.oracle_permute.restype = ci
        L.oracle_layer.argtypes = [vp, ci, vp, f32p, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci,
                                   f32p, f32p, i32p, f32p, f32p]
        L.oracle_layer.restype = ci
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = ci
        _lib = L
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _wcode(a):
    """(contiguous array, dtype code) for a weight/activation array."""
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a), 1
    return _f32(a), 0


class OracleError(RuntimeError):
    pass


def num_threads():
    return lib().oracle_num_threads()


def exp_c(x):
    x = _f32(x)
    y = np.empty_like(x)
    lib().oracle_exp_c_array(_ptr(x, ctypes.c_float), _ptr(y, ctypes.c_float), x.size)
    return y


def exp_c_sweep(stride=1):
    """(max ulp error vs double exp, values checked, non-normal results) over
    every stride-th float32 in [-87, -0]."""
    n = ctypes.c_int64(0)
    bad = ctypes.c_int64(0)
    worst = lib().oracle_exp_c_sweep(stride, ctypes.byref(n), ctypes.byref(bad))
    return worst, n.value, bad.value


def softmax_f32(z):
    z = _f32(z)
    assert z.ndim == 1
    p = np.empty_like(z)
    lib().oracle_softmax_f32(_ptr(z, ctypes.c_float), z.size, _ptr(p, ctypes.c_float))
    return p


def route_f32(logits, k1, k2):
    z = _f32(logits)
    T, E = z.shape
    idx = np.empty((T, k1), np.int32)
    w = np.empty((T, k1), np.float32)
    rc = lib().oracle_route_f32(_ptr(z, ctypes.c_float), T, E, k1, k2, _ptr(idx, ctypes.c_int32),
                                _ptr(w, ctypes.c_float))
    if rc != 0:
        raise OracleError("oracle_route_f32: bad arguments (T=%d E=%d k1=%d k2=%d)" % (T, E, k1, k2))
    return idx, w


EMPTY_SLOT = 0x7fffffff  # an unused slot of a variable-k (cascade) route


def route_cascade_f32(logits, kmax, k2, tau):
    """Variable k per token: returns (idx [T x kmax], w [T x kmax], k [T]);
    slots s >= k[t] hold EMPTY_SLOT and weight 0."""
    z = _f32(logits)
    T, E = z.shape
    idx = np.empty((T, kmax), np.int32)
    w = np.empty((T, kmax), np.float32)
    k = np.empty(T, np.int32)
    rc = lib().oracle_route_cascade_f32(_ptr(z, ctypes.c_float), T, E, kmax, k2, ctypes.c_float(tau),
                                        _ptr(idx, ctypes.c_int32), _ptr(w, ctypes.c_float),
                                        _ptr(k, ctypes.c_int32))
    if rc != 0:
        raise OracleError("oracle_route_cascade_f32: bad arguments (T=%d E=%d kmax=%d k2=%d)"
                          % (T, E, kmax, k2))
    return idx, w, k


def layer_tokens_cascade(xrows, z_rows, fetch_expert, kmax, k2, tau):
    """layer_tokens with the variable-k route: each token sums only its k[t]
    experts.  Returns dict(y, idx, w, k)."""
    idx, w, k = route_cascade_f32(z_rows, kmax, k2, tau)
    n = idx.shape[0]
    xa, xc = _wcode(xrows)
    d = xa.shape[1]
    xf_all = (xa.astype(np.uint32) << 16).view(np.float32) if xc == 1 else xa
    y = np.empty((n, d), np.float32)
    cache = {}
    for t in range(n):
        kt = int(k[t])
        o = np.empty((kt, d), np.float32)
        for s in range(kt):
            e = int(idx[t, s])
            if e not in cache:
                cache[e] = fetch_expert(e)
            _, o[s] = expert(xf_all[t], *cache[e], par=True)
        y[t] = combine(o, w[t, :kt])
    return {"y": y, "idx": idx, "w": w, "k": k}


def route_f64(logits, k1, k2):
    z = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = z.shape
    idx = np.empty((T, k1), np.int32)
    w = np.empty((T, k1), np.float64)
    p = np.empty((T, E), np.float64)
    rc = lib().oracle_route_f64(_ptr(z, ctypes.c_double), T, E, k1, k2, _ptr(idx, ctypes.c_int32),
                                _ptr(w, ctypes.c_double), _ptr(p, ctypes.c_double))
    if rc != 0:
        raise OracleError("oracle_route_f64: bad arguments (T=%d E=%d k1=%d k2=%d)" % (T, E, k1, k2))
    return idx, w, p


def logits(x, wr, bias=None):
    xa, xc = _wcode(x)
    wa, wc = _wcode(wr)
    T, d = xa.shape
    E = wa.shape[0]
    assert wa.shape == (E, d)
    z = np.empty((T, E), np.float32)
    b = None if bias is None else _f32(bias)
    lib().oracle_logits(xa.ctypes.data, xc, wa.ctypes.data, wc,
                        None if b is None else _ptr(b, ctypes.c_float), T, d, E,
                        _ptr(z, ctypes.c_float))
    return z


def expert(xf, wg, wu, wd, par=True):
    """One token (float32 [d]) through one expert; returns (h [I], o [d])."""
    xf = _f32(xf)
    ga, gc = _wcode(wg)
    ua, uc = _wcode(wu)
    da, dc = _wcode(wd)
    assert gc == uc == dc
    I, d = ga.shape
    assert xf.shape == (d,) and ua.shape == (I, d) and da.shape == (d, I)
    h = np.empty(I, np.float32)
    o = np.empty(d, np.float32)
    lib().oracle_expert(_ptr(xf, ctypes.c_float), ga.ctypes.data, ua.ctypes.data, da.ctypes.data, gc,
                        d, I, _ptr(h, ctypes.c_float), _ptr(o, ctypes.c_float), 1 if par else 0)
    return h, o


def combine(o, w):
    o = _f32(o)
    w = _f32(w)
    k1, d = o.shape
    assert w.shape == (k1,)
    y = np.empty(d, np.float32)
    lib().oracle_combine(_ptr(o, ctypes.c_float), _ptr(w, ctypes.c_float), k1, d,
                         _ptr(y, ctypes.c_float))
    return y


def permute(idx, E):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k1 = idx.shape
    n = T * k1
    offsets = np.empty(E + 1, np.int32)
    sorted_slot = np.empty(max(n, 1), np.int32)
    slot_pos = np.empty(max(n, 1), np.int32)
    rc = lib().oracle_permute(_ptr(idx, ctypes.c_int32), T, k1, E, _ptr(offsets, ctypes.c_int32),
                              _ptr(sorted_slot, ctypes.c_int32), _ptr(slot_pos, ctypes.c_int32))
    if rc != 0:
        raise OracleError("oracle_permute: expert index out of range")
    # slots holding EMPTY_SLOT are not placed (slot_pos -1)
    return offsets, sorted_slot[:int(offsets[E])], slot_pos[:n]


def layer(x, wr, bias, wg, wu, wd, k1, k2, logits_in=None):
    """Whole layer in float32; returns dict(y, idx, w, z)."""
    xa, xc = _wcode(x)
    wra, wrc = _wcode(wr)
    ga, gc = _wcode(wg)
    ua, uc = _wcode(wu)
    da, dc = _wcode(wd)
    assert wrc == gc == uc == dc
    T, d = xa.shape
    E, I, _ = ga.shape
    assert wra.shape == (E, d) and ua.shape == (E, I, d) and da.shape == (E, d, I)
    y = np.empty((T, d), np.float32)
    idx = np.empty((T, k1), np.int32)
    w = np.empty((T, k1), np.float32)
    z = np.empty((T, E), np.float32)
    b = None if bias is None else _f32(bias)
    zin = None if logits_in is None else _f32(logits_in)
    rc = lib().oracle_layer(xa.ctypes.data, xc, wra.ctypes.data,
                            None if b is None else _ptr(b, ctypes.c_float),
                            ga.ctypes.data, ua.ctypes.data, da.ctypes.data, gc, T, d, E, I, k1, k2,
                            None if zin is None else _ptr(zin, ctypes.c_float),
                            _ptr(y, ctypes.c_float), _ptr(idx, ctypes.c_int32),
                            _ptr(w, ctypes.c_float), _ptr(z, ctypes.c_float))
    if rc != 0:
        raise OracleError("oracle_layer: bad arguments")
    return {"y": y, "idx": idx, "w": w, "z": z}


def layer_tokens(xrows, z_rows, fetch_expert, k1, k2):
    """Layer output for a few tokens whose weights are fetched per expert.

    xrows  [n x d] float32 or bf16 bits (uint16), the sampled tokens
    z_rows [n x E] float32 logits to route on
    fetch_expert(e) -> (wg [I x d], wu [I x d], wd [d x I]) for expert e
    Returns dict(y [n x d] float32, idx, w).  Used where the full weight
    set does not fit in host memory: only the selected experts are fetched.
    """
    idx, w = route_f32(z_rows, k1, k2)
    n = idx.shape[0]
    xa, xc = _wcode(xrows)
    d = xa.shape[1]
    if xc == 1:
        xf_all = (xa.astype(np.uint32) << 16).view(np.float32)
    else:
        xf_all = xa
    y = np.empty((n, d), np.float32)
    cache = {}
    for t in range(n):
        o = np.empty((k1, d), np.float32)
        for s in range(k1):
            e = int(idx[t, s])
            if e not in cache:
                cache[e] = fetch_expert(e)
            wg, wu, wd = cache[e]
            _, o[s] = expert(xf_all[t], wg, wu, wd, par=True)
        y[t] = combine(o, w[t])
    return {"y": y, "idx": idx, "w": w}


# ---------------------------------------------------------------------------
# Channel top-k inside the activated experts ("Channel Selection for
# Mixture-of-Experts Decoding Needs No Calibration Data", paperlayer.ai):
# section 2 "Background" (channel c of a routed expert owns gate row c, up
# row c and down column c), section 5.2 "Output-scaled scoring and exact
# top-k computation" (score = router weight x down-column norm x activation
# magnitude, in output units, so that channels of different experts compare
# and the best ones are taken across a token's experts), section 5.3 (kept
# channels are computed exactly).  The ternary sketch that screens channels
# and the low-rank recovery of skipped ones are not part of this oracle: h is
# computed exactly for every channel and skipped channels add nothing.


def _widen(a):
    a, code = _wcode(a)
    return (a.astype(np.uint32) << 16).view(np.float32) if code == 1 else a


def channel_norms(wd):
    """Down-column norms of one expert: wd [d x I] (bf16 bits or float32) ->
    float32 [I], n_c = sqrt(sum_r wd[r, c]^2) in float64, rounded once."""
    w = _widen(wd).astype(np.float64)
    return np.sqrt((w * w).sum(axis=0)).astype(np.float32)


def channel_scores(h, w, norms):
    """Output-scaled channel scores of one token: h [k x I] float32 channel
    activations of its k slots, w [k] float32 Eq. 2 weights, norms [k x I]
    float32 down-column norms of each slot's expert.  score = (w_s * n) * |h|,
    two float32 products in that order, each rounded once."""
    h = _f32(h)
    wn = np.asarray(w, np.float32)[:, None] * _f32(norms)
    return (wn * np.abs(h)).astype(np.float32)


def channel_select(scores, keep):
    """The `keep` best channels of one token over all its slots: flat indices
    q = s*I + c (ascending) of the largest float32 scores, equal scores going
    to the lower flat index (slot rank first, then channel).  Scores must be
    finite and non-negative."""
    s = np.asarray(scores, np.float32).ravel()
    if not 1 <= keep <= s.size:
        raise OracleError("channel_select: keep=%d outside [1, %d]" % (keep, s.size))
    if not np.isfinite(s).all() or (s < 0).any():
        raise OracleError("channel_select: scores must be finite and non-negative")
    order = np.lexsort((np.arange(s.size), -s.astype(np.float64)))
    return np.sort(order[:keep]).astype(np.int32)


def channel_topk_tokens(xrows, z_rows, fetch_expert, fetch_norms, k1, k2, keep, scores_in=None,
                        kept_in=None):
    """Layer output with channel top-k for a few tokens.

    xrows [n x d] float32 or bf16 bits, z_rows [n x E] float32 logits to route
    on, fetch_expert(e) -> (wg [I x d], wu [I x d], wd [d x I]),
    fetch_norms(e) -> float32 [I] down-column norms, keep channels per token.
    Per token: route (Eq. 2), h [k1 x I] for every channel of its k1 experts
    (oracle_expert), scores (channel_scores), the kept set (channel_select on
    scores_in[t] when given, else on its own scores; kept_in[t] overrides
    both), and y = sum over kept (s, c) of w_s * h[s, c] * wd_s[:, c],
    accumulated in float64.  Returns dict(y [n x d] float32, idx, w, h,
    norms, scores, kept [n x keep])."""
    idx, w = route_f32(z_rows, k1, k2)
    n = idx.shape[0]
    xf_all = _widen(xrows)
    d = xf_all.shape[1]
    cache, ncache = {}, {}
    hs, ns, ss, ks = [], [], [], []
    y = np.empty((n, d), np.float32)
    for t in range(n):
        h = []
        nrm = []
        for s in range(k1):
            e = int(idx[t, s])
            if e not in cache:
                cache[e] = fetch_expert(e)
                ncache[e] = _f32(fetch_norms(e))
            h.append(expert(xf_all[t], *cache[e], par=True)[0])
            nrm.append(ncache[e])
        h = np.stack(h)
        nrm = np.stack(nrm)
        I = h.shape[1]
        sc = channel_scores(h, w[t], nrm)
        if kept_in is not None:
            kept = np.asarray(kept_in[t], np.int32)
        else:
            kept = channel_select(sc if scores_in is None else scores_in[t], keep)
        acc = np.zeros(d, np.float64)
        slot, ch = np.divmod(kept, I)
        for s in range(k1):
            cs = ch[slot == s]
            if cs.size:
                wd = _widen(cache[int(idx[t, s])][2]).astype(np.float64)
                coef = float(w[t, s]) * h[s, cs].astype(np.float64)
                acc += wd[:, cs] @ coef
        y[t] = acc
        hs.append(h)
        ns.append(nrm)
        ss.append(sc)
        ks.append(kept)
    return {"y": y, "idx": idx, "w": w, "h": np.stack(hs), "norms": np.stack(ns),
            "scores": np.stack(ss), "kept": np.stack(ks)}


# ---------------------------------------------------------------------------
# Expert skipping with the top-1 expert always kept (the shell of "ACE",
# aimodeling.com, section "How ACE decides what to skip: GSP + RCR": a slot is
# skipped only when two independent views both call it low-contribution, and
# the top-1 expert is always retained).  Reading taken here: the first view is
# a per-expert scalar looked up at inference (the page's offline statistic;
# the caller supplies the table), the second is the slot's Eq. 2 weight (the
# token's router-conditioned view); kept slots keep their Eq. 2 weights.


def route_skip_f32(logits, k1, k2, table, th_e, th_w):
    """route_f32, then slot s >= 1 of each token becomes EMPTY_SLOT (weight 0)
    when table[e_s] < th_e and w_s < th_w (float32 comparisons).  Returns
    (idx, w, count of kept slots per token)."""
    idx, w = route_f32(logits, k1, k2)
    tab = np.asarray(table, np.float32)
    low = (tab[idx] < np.float32(th_e)) & (w < np.float32(th_w))
    low[:, 0] = False  # the top-1 expert is always kept
    idx = np.where(low, np.int32(EMPTY_SLOT), idx).astype(np.int32)
    w = np.where(low, np.float32(0.0), w).astype(np.float32)
    return idx, w, (~low).sum(axis=1).astype(np.int32)


def layer_tokens_slots(xrows, idx, w, fetch_expert):
    """Layer output for a few tokens from given routing outputs: y[t] sums
    w[t, s] * FFN_{idx[t, s]}(x_t) over the slots that are not EMPTY_SLOT, in
    slot order (oracle_expert, oracle_combine)."""
    xf_all = _widen(xrows)
    n, d = xf_all.shape
    y = np.empty((n, d), np.float32)
    cache = {}
    for t in range(n):
        slots = [s for s in range(idx.shape[1]) if idx[t, s] != EMPTY_SLOT]
        o = np.empty((len(slots), d), np.float32)
        for i, s in enumerate(slots):
            e = int(idx[t, s])
            if e not in cache:
                cache[e] = fetch_expert(e)
            _, o[i] = expert(xf_all[t], *cache[e], par=True)
        y[t] = combine(o, w[t, slots]) if slots else 0.0
    return y
