"""ctypes binding of libmoe.so.  Argument marshalling only: every step of the
layer runs in the library's CUDA kernels.  The call names are those of
include/moe.h; arguments are torch tensors on the current CUDA device (or
None where the C call takes NULL).  A non-OK status raises MoeError.

There is no fallback: if libmoe.so is missing or fails to load, every call
raises.  With MOE_LIB_VARIANT=checks in the environment the checked build
libmoe_checks.so is loaded instead (the same calls; kernels also verify the
index tables they otherwise trust).
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_VARIANT = os.environ.get("MOE_LIB_VARIANT", "")
if LIB_VARIANT not in ("", "checks"):
    raise RuntimeError("MOE_LIB_VARIANT must be unset or 'checks', not %r" % LIB_VARIANT)
LIB_PATH = os.path.join(HERE, "libmoe_checks.so" if LIB_VARIANT == "checks" else "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_WORKSPACE_TOO_SMALL = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_DEVICE_CHECK = -6
MOE_ERR_SCRATCH_LIMIT = -7

MOE_DTYPE_F32 = 0
MOE_DTYPE_BF16 = 1

MOE_PATH_AUTO = 0
MOE_PATH_STREAM = 1
MOE_PATH_GROUPED = 2
MOE_PATH_DECODE = 3
MOE_PATH_MASK = 0xFF
MOE_WDOWN_CHANNEL_MAJOR = 0x100
MOE_EMPTY_SLOT = 0x7FFFFFFF

# every symbol include/*.h declares, with (restype, argtypes)
_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_f = ctypes.c_float
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_version": (_i, []),
    "moe_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "moe_workspace_init": (_i, [_vp, _sz, _vp]),
    "moe_read_device_status": (_i, [_vp, ctypes.POINTER(_i), _vp]),
    "moe_route": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_ffn": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _sz,
                            _vp]),
    "moe_combine": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _i, _vp]),
    "moe_layer": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp,
                       _vp, _i, _vp, _sz, _vp]),
    "moe_route_cascade": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _sz,
                               _vp]),
    "moe_layer_cascade": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _i,
                               _vp, _vp, _vp, _vp, _i, _vp, _sz, _vp]),
    "moe_route_skip": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _f, _f, _vp, _vp, _vp,
                            _vp, _sz, _vp]),
    "moe_layer_skip": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _f, _f, _vp,
                            _i, _vp, _vp, _vp, _vp, _i, _vp, _sz, _vp]),
    "moe_expert_ffn_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "moe_noalloc_read_status": (_i, [ctypes.POINTER(_i), _vp]),
    "moe_pack_w_down": (_i, [_vp, _vp, _i, _i, _i, _vp]),
    "moe_channel_norms": (_i, [_vp, _i, _i, _i, _i, _vp, _vp]),
    "moe_layer_channel_topk": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                    _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_test_exp_c": (_i, [_vp, _vp, ctypes.c_int64, _vp]),
    "moe_test_num_sms": (_i, []),
    "moe_test_set_grouped_single": (_i, [_i]),
    "moe_test_grouped_pairs": (_i, [_i]),
    "moe_test_set_wait_limit_ns": (_i, [ctypes.c_uint64]),
    "moe_test_wait_never_set": (_i, [_vp, _sz, _i, _vp]),
    "moe_test_expert_stream": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _i, _vp,
                                    _sz, _vp]),
    "moe_test_expert_grouped": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
}

_lib = None


class MoeError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (where, status_string(status), status))


def lib():
    """Load libmoe.so (raises if it is missing: there is no CPU fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("%s not built; run python -m routed_expert_layer_route_b200.build%s"
                               % (LIB_PATH, " --checks" if LIB_VARIANT else ""))
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status):
    return lib().moe_status_string(int(status)).decode()


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc, where):
    if rc != MOE_OK:
        raise MoeError(rc, where)


def moe_version():
    return lib().moe_version()


def moe_workspace_size(T, d, E, I, k1):
    return lib().moe_workspace_size(T, d, E, I, k1)


def moe_workspace_init(ws, stream=None):
    _check(lib().moe_workspace_init(_p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_workspace_init")


def moe_read_device_status(ws, stream=None):
    v = ctypes.c_int(0)
    _check(lib().moe_read_device_status(_p(ws), ctypes.byref(v), _stream(stream)),
           "moe_read_device_status")
    return v.value


def workspace(T, d, E, I, k1, device=None, stream=None):
    """Allocate (torch) and initialise a workspace for these shapes.  The
    zeroing is enqueued on `stream` (default: the current stream): give the
    stream the layer calls will run on, or order the two streams yourself."""
    n = moe_workspace_size(T, d, E, I, k1)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))
    moe_workspace_init(ws, stream)
    return ws


def _ws_args(ws):
    if ws is None:
        return None, 0
    return _p(ws), ws.numel() * ws.element_size()


def moe_route(x, w_router, bias, logits, k1, k2, topk_idx, topk_w, ws=None, stream=None, T=None,
              d=None, E=None):
    """x None: route the given float32 logits [T x E]; else compute them."""
    if x is not None:
        T, d = x.shape
        E = w_router.shape[0]
    else:
        T, E = logits.shape
        d = d or 0
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_route(_p(x), _p(w_router), _p(bias), _p(logits), T, d, E, k1, k2,
                           _p(topk_idx), _p(topk_w), wsp, wsn, _stream(stream)), "moe_route")


def moe_permute(topk_idx, E, expert_offsets, sorted_slot, slot_pos, ws=None, stream=None):
    T, k1 = topk_idx.shape
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_permute(_p(topk_idx), T, k1, E, _p(expert_offsets), _p(sorted_slot),
                             _p(slot_pos), wsp, wsn, _stream(stream)), "moe_permute")


def moe_expert_ffn(x, expert_offsets, sorted_slot, w_gate, w_up, w_down, k1, out, ws,
                   flags=MOE_PATH_AUTO, stream=None):
    T, d = x.shape
    E, I, _ = w_gate.shape
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_expert_ffn(_p(x), _p(expert_offsets), _p(sorted_slot), _p(w_gate), _p(w_up),
                                _p(w_down), T, d, E, I, k1, _p(out), flags, wsp, wsn,
                                _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_noalloc(x, expert_offsets, sorted_slot, w_gate, w_up, w_down, k1, out,
                           stream=None):
    """moe_expert_ffn for callers that cannot provide device scratch memory:
    the library uses a fixed array of its own instead of a workspace (limit
    T * k1 * I <= 1047424; calls that overlap on the GPU share that array and
    race, so keep them on one stream)."""
    T, d = x.shape
    E, I, _ = w_gate.shape
    _check(lib().moe_expert_ffn_noalloc(_p(x), _p(expert_offsets), _p(sorted_slot), _p(w_gate),
                                        _p(w_up), _p(w_down), T, d, E, I, k1, _p(out),
                                        _stream(stream)), "moe_expert_ffn_noalloc")


def moe_noalloc_read_status(stream=None):
    """The device status of moe_expert_ffn_noalloc calls on the current device
    since the last read (0 = OK); reading clears it.  Synchronises the stream."""
    v = ctypes.c_int(0)
    _check(lib().moe_noalloc_read_status(ctypes.byref(v), _stream(stream)),
           "moe_noalloc_read_status")
    return v.value


def moe_pack_w_down(w_down, w_down_cm=None, stream=None):
    """Channel-major copy [E x I x d] of a down matrix [E x d x I] (bf16)."""
    E, d, I = w_down.shape
    if w_down_cm is None:
        w_down_cm = torch.empty((E, I, d), dtype=w_down.dtype, device=w_down.device)
    _check(lib().moe_pack_w_down(_p(w_down), _p(w_down_cm), E, d, I, _stream(stream)),
           "moe_pack_w_down")
    return w_down_cm


def moe_route_skip(x, w_router, bias, logits, k1, k2, expert_score, theta_expert, theta_weight,
                   topk_idx, topk_w, topk_count=None, ws=None, stream=None):
    """Routing with expert skipping (top-1 kept); x None routes the given logits."""
    if x is not None:
        T, d = x.shape
        E = w_router.shape[0]
    else:
        T, E = logits.shape
        d = 0
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_route_skip(_p(x), _p(w_router), _p(bias), _p(logits), T, d, E, k1, k2,
                                _p(expert_score), float(theta_expert), float(theta_weight),
                                _p(topk_idx), _p(topk_w), _p(topk_count), wsp, wsn,
                                _stream(stream)), "moe_route_skip")


def moe_layer_skip(x, w_router, bias, w_gate, w_up, w_down, k1, k2, expert_score, theta_expert,
                   theta_weight, y, ws, topk_idx_out=None, topk_w_out=None, topk_count_out=None,
                   logits_out=None, flags=MOE_PATH_AUTO, stream=None):
    """moe_layer with expert skipping (top-1 kept)."""
    T, d = x.shape
    E, I, _ = w_gate.shape
    y_dtype = MOE_DTYPE_BF16 if y.dtype == torch.bfloat16 else MOE_DTYPE_F32
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_layer_skip(_p(x), _p(w_router), _p(bias), _p(w_gate), _p(w_up), _p(w_down),
                                T, d, E, I, k1, k2, _p(expert_score), float(theta_expert),
                                float(theta_weight), _p(y), y_dtype, _p(topk_idx_out),
                                _p(topk_w_out), _p(topk_count_out), _p(logits_out), flags, wsp,
                                wsn, _stream(stream)), "moe_layer_skip")


def moe_channel_norms(w_down, channel_major=False, norms=None, stream=None):
    """float32 [E x I] down-column norms of w_down: [E x d x I] (HF layout) or,
    with channel_major, [E x I x d] (moe_pack_w_down's output)."""
    if channel_major:
        E, I, d = w_down.shape
    else:
        E, d, I = w_down.shape
    if norms is None:
        norms = torch.empty((E, I), dtype=torch.float32, device=w_down.device)
    _check(lib().moe_channel_norms(_p(w_down), E, d, I,
                                   MOE_WDOWN_CHANNEL_MAJOR if channel_major else 0, _p(norms),
                                   _stream(stream)), "moe_channel_norms")
    return norms


def moe_layer_channel_topk(x, w_router, bias, w_gate, w_up, w_down_cm, norms, k1, k2, keep, y, ws,
                           topk_idx_out=None, topk_w_out=None, logits_out=None, h_out=None,
                           scores_out=None, kept_out=None, stream=None):
    """The layer with channel top-k: each token keeps the `keep` channels of
    its k1 experts with the largest w * ||down column|| * |h| (w_down_cm
    channel-major, norms from moe_channel_norms)."""
    T, d = x.shape
    E, I, _ = w_gate.shape
    y_dtype = MOE_DTYPE_BF16 if y.dtype == torch.bfloat16 else MOE_DTYPE_F32
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_layer_channel_topk(_p(x), _p(w_router), _p(bias), _p(w_gate), _p(w_up),
                                        _p(w_down_cm), _p(norms), T, d, E, I, k1, k2, int(keep),
                                        _p(y), y_dtype, _p(topk_idx_out), _p(topk_w_out),
                                        _p(logits_out), _p(h_out), _p(scores_out), _p(kept_out),
                                        wsp, wsn, _stream(stream)), "moe_layer_channel_topk")


def moe_combine(expert_out, slot_pos, topk_w, y, stream=None):
    T, k1 = topk_w.shape
    d = y.shape[1]
    y_dtype = MOE_DTYPE_BF16 if y.dtype == torch.bfloat16 else MOE_DTYPE_F32
    _check(lib().moe_combine(_p(expert_out), _p(slot_pos), _p(topk_w), T, d, k1, _p(y), y_dtype,
                             _stream(stream)), "moe_combine")


def moe_layer(x, w_router, bias, w_gate, w_up, w_down, k1, k2, y, ws, topk_idx_out=None,
              topk_w_out=None, logits_out=None, flags=MOE_PATH_AUTO, stream=None):
    """w_down: [E x d x I], or the channel-major [E x I x d] copy from
    moe_pack_w_down together with flags | MOE_WDOWN_CHANNEL_MAJOR."""
    T, d = x.shape
    E, I, _ = w_gate.shape
    y_dtype = MOE_DTYPE_BF16 if y.dtype == torch.bfloat16 else MOE_DTYPE_F32
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_layer(_p(x), _p(w_router), _p(bias), _p(w_gate), _p(w_up), _p(w_down), T, d,
                           E, I, k1, k2, _p(y), y_dtype, _p(topk_idx_out), _p(topk_w_out),
                           _p(logits_out), flags, wsp, wsn, _stream(stream)), "moe_layer")


def moe_test_exp_c(x, y, stream=None):
    _check(lib().moe_test_exp_c(_p(x), _p(y), x.numel(), _stream(stream)), "moe_test_exp_c")


def moe_test_num_sms():
    return lib().moe_test_num_sms()


def moe_test_set_grouped_single(single):
    _check(lib().moe_test_set_grouped_single(int(single)), "moe_test_set_grouped_single")


def moe_test_grouped_pairs(which):
    return lib().moe_test_grouped_pairs(int(which))


def moe_test_set_wait_limit_ns(ns):
    _check(lib().moe_test_set_wait_limit_ns(int(ns)), "moe_test_set_wait_limit_ns")


def moe_test_wait_never_set(ws, which, stream=None):
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_test_wait_never_set(wsp, wsn, int(which), _stream(stream)),
           "moe_test_wait_never_set")


def moe_test_expert_stream(x, w_gate, w_up, w_down, k1, k2, y, ws, flags=MOE_PATH_AUTO,
                           stream=None):
    T, d = x.shape
    E, I, _ = w_gate.shape
    y_dtype = MOE_DTYPE_BF16 if y.dtype == torch.bfloat16 else MOE_DTYPE_F32
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_test_expert_stream(_p(x), _p(w_gate), _p(w_up), _p(w_down), T, d, E, I, k1,
                                        k2, _p(y), y_dtype, flags, wsp, wsn, _stream(stream)),
           "moe_test_expert_stream")


def moe_test_expert_grouped(x, w_gate, w_up, w_down, k1, which, ws, stream=None):
    """Kernels of the grouped expert FFN alone (which, a bit set: 4 token-row
    gather, 1 gate/up GEMM, 2 down GEMM) on the routing tables a previous
    moe_layer call left in ws."""
    T, d = x.shape
    E, I, _ = w_gate.shape
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_test_expert_grouped(_p(x), _p(w_gate), _p(w_up), _p(w_down), T, d, E, I, k1,
                                         which, wsp, wsn, _stream(stream)),
           "moe_test_expert_grouped")


def moe_route_cascade(x, w_router, bias, logits, k1, k2, tau, topk_idx, topk_w, topk_count=None,
                      ws=None, stream=None):
    """Variable-k route (k_t <= k1 per token covering mass tau); unused slots
    hold MOE_EMPTY_SLOT with weight 0."""
    if x is None:
        T, E = logits.shape
        d = 0
    else:
        T, d = x.shape
        E = w_router.shape[0]
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_route_cascade(_p(x), _p(w_router), _p(bias), _p(logits), T, d, E, k1, k2,
                                   float(tau), _p(topk_idx), _p(topk_w), _p(topk_count), wsp, wsn,
                                   _stream(stream)), "moe_route_cascade")


def moe_layer_cascade(x, w_router, bias, w_gate, w_up, w_down, k1, k2, tau, y, ws,
                      topk_idx_out=None, topk_w_out=None, topk_count_out=None, logits_out=None,
                      flags=MOE_PATH_AUTO, stream=None):
    """moe_layer with the variable-k route."""
    T, d = x.shape
    E, I, _ = w_gate.shape
    y_dtype = MOE_DTYPE_BF16 if y.dtype == torch.bfloat16 else MOE_DTYPE_F32
    wsp, wsn = _ws_args(ws)
    _check(lib().moe_layer_cascade(_p(x), _p(w_router), _p(bias), _p(w_gate), _p(w_up), _p(w_down),
                                   T, d, E, I, k1, k2, float(tau), _p(y), y_dtype, _p(topk_idx_out),
                                   _p(topk_w_out), _p(topk_count_out), _p(logits_out), flags, wsp,
                                   wsn, _stream(stream)), "moe_layer_cascade")
