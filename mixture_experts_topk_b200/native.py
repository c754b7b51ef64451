"""ctypes binding of the C ABI in include/moe_b200.h.

Argument marshalling only: every step of the layer runs in the CUDA library
(libmoe_b200.so, built in-tree).  torch provides device memory and the
current stream.  There is no fallback: if the library is missing, importing
it raises.
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
                3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT",
                6: "MOE_ERR_DEVICE_BOUNDS"}

EXPORTED = (
    "moe_last_error", "moe_init", "moe_destroy", "moe_weights_size", "moe_workspace_size",
    "moe_workspace_view_get", "moe_pack_weights", "moe_route", "moe_dispatch", "moe_gate_up",
    "moe_down", "moe_combine", "moe_forward", "moe_forward_routed", "moe_workspace_init",
    "moe_get_status", "moe_dispatch_noalloc", "moe_set_tile_config", "moe_set_launch_options", "moe_set_gemm_options", "moe_set_wait_limit", "moe_set_picker_params",
    "moe_get_picker_params", "moe_set_gate_up_model", "moe_get_gate_up_model", "moe_set_gate_up_tile",
)


class MoeError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class moe_config(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("I", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int),
                ("score", ctypes.c_int), ("fmt", ctypes.c_int), ("has_bias", ctypes.c_int),
                ("max_T", ctypes.c_int), ("hidden_global_scale", ctypes.c_float),
                ("act", ctypes.c_int), ("act_alpha", ctypes.c_float), ("act_limit", ctypes.c_float)]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("gate_q", "gate_s", "gate_g", "up_q", "up_s", "up_g", "down_q", "down_s", "down_g")]


VIEW_FIELDS = ("status", "ids", "w", "counts", "offsets", "num_tiles", "tile_ptr", "pick", "tiles", "perm", "inv",
               "x_global", "xq", "xs", "hq", "hs", "o", "logits", "o_exp")


class moe_workspace_view(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in VIEW_FIELDS]


_lib = None


def load(path=LIB_PATH):
    """Load the CUDA library (raises OSError when it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"{path} not found: build it with __graft_entry__.build()")
        L = ctypes.CDLL(path)
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        S = ctypes.c_size_t
        sigs = {
            "moe_last_error": (ctypes.c_char_p, []),
            "moe_init": (I, [ctypes.POINTER(moe_config), ctypes.POINTER(P)]),
            "moe_destroy": (I, [P]),
            "moe_weights_size": (I, [P, ctypes.POINTER(S)]),
            "moe_workspace_size": (I, [P, ctypes.POINTER(S)]),
            "moe_workspace_view_get": (I, [P, P, ctypes.POINTER(moe_workspace_view)]),
            "moe_pack_weights": (I, [P, ctypes.POINTER(moe_weights), P, P]),
            "moe_route": (I, [P, P, I, P, P, P, P, P, P]),
            "moe_dispatch": (I, [P, P, P, I, P, P]),
            "moe_gate_up": (I, [P, P, I, P, P]),
            "moe_down": (I, [P, P, P, I, P, P]),
            "moe_combine": (I, [P, I, P, P, P]),
            "moe_forward": (I, [P, P, I, P, P, P, P, P, P]),
            "moe_forward_routed": (I, [P, P, I, P, P, P, P, P, P]),
            "moe_workspace_init": (I, [P, P, P]),
            "moe_get_status": (I, [P, P, P]),
            "moe_dispatch_noalloc": (I, [P, P, P, I] + [P] * 10),
            "moe_set_tile_config": (I, [P, I]),
            "moe_set_launch_options": (I, [P, I]),
            "moe_set_gemm_options": (I, [P, I]),
            "moe_set_wait_limit": (I, [P, ctypes.c_longlong]),
            "moe_set_picker_params": (I, [P, P]),
            "moe_get_picker_params": (I, [P, P]),
            "moe_set_gate_up_model": (I, [P, P]),
            "moe_set_gate_up_tile": (I, [P, I]),
            "moe_get_gate_up_model": (I, [P, P]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(st):
    if st != MOE_OK:
        raise MoeError(st, load().moe_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------ same names as the C ABI
def moe_init(wl, max_T):
    cfg = moe_config(wl.H, wl.I, wl.E, wl.k, wl.score, wl.fmt, int(wl.has_bias), int(max_T),
                     float(wl.hidden_global_scale), int(wl.act), float(wl.act_alpha), float(wl.act_limit))
    h = ctypes.c_void_p()
    _check(load().moe_init(ctypes.byref(cfg), ctypes.byref(h)))
    return h


def moe_destroy(h):
    _check(load().moe_destroy(h))


def moe_weights_size(h):
    n = ctypes.c_size_t()
    _check(load().moe_weights_size(h, ctypes.byref(n)))
    return n.value


def moe_workspace_size(h):
    n = ctypes.c_size_t()
    _check(load().moe_workspace_size(h, ctypes.byref(n)))
    return n.value


def moe_workspace_view_get(h, ws):
    v = moe_workspace_view()
    _check(load().moe_workspace_view_get(h, _ptr(ws), ctypes.byref(v)))
    return {n: getattr(v, n) for n in VIEW_FIELDS}


def moe_pack_weights(h, weights, packed, stream=None):
    src = moe_weights(*[weights[n].data_ptr() if weights.get(n) is not None else None for n in
                        ("gate_q", "gate_s", "gate_g", "up_q", "up_s", "up_g", "down_q", "down_s", "down_g")])
    _check(load().moe_pack_weights(h, ctypes.byref(src), _ptr(packed), _stream(stream)))


def moe_route(h, x, T, wr, bias, ids, w, ws, stream=None):
    _check(load().moe_route(h, _ptr(x), T, _ptr(wr), _ptr(bias), _ptr(ids), _ptr(w), _ptr(ws), _stream(stream)))


def moe_dispatch(h, x, ids, T, ws, stream=None):
    _check(load().moe_dispatch(h, _ptr(x), _ptr(ids), T, _ptr(ws), _stream(stream)))


def moe_gate_up(h, packed, T, ws, stream=None):
    _check(load().moe_gate_up(h, _ptr(packed), T, _ptr(ws), _stream(stream)))


def moe_down(h, packed, w, T, ws, stream=None):
    _check(load().moe_down(h, _ptr(packed), _ptr(w), T, _ptr(ws), _stream(stream)))


def moe_combine(h, T, y, ws, stream=None):
    _check(load().moe_combine(h, T, _ptr(y), _ptr(ws), _stream(stream)))


def moe_forward(h, x, T, wr, bias, packed, y, ws, stream=None):
    _check(load().moe_forward(h, _ptr(x), T, _ptr(wr), _ptr(bias), _ptr(packed), _ptr(y), _ptr(ws),
                              _stream(stream)))


def moe_forward_routed(h, x, T, ids, w, packed, y, ws, stream=None):
    _check(load().moe_forward_routed(h, _ptr(x), T, _ptr(ids), _ptr(w), _ptr(packed), _ptr(y), _ptr(ws),
                                     _stream(stream)))


def moe_dispatch_noalloc(h, x, ids, T, counts, offsets, num_tiles, tiles, perm, inv, xq, xs, status,
                         stream=None):
    """moe_dispatch with caller-given outputs and no workspace (for callers that
    cannot allocate device memory; the scratch is inside the library)."""
    _check(load().moe_dispatch_noalloc(h, _ptr(x), _ptr(ids), T, _ptr(counts), _ptr(offsets), _ptr(num_tiles),
                                       _ptr(tiles), _ptr(perm), _ptr(inv), _ptr(xq), _ptr(xs), _ptr(status),
                                       _stream(stream)))


def moe_set_tile_config(h, down_bn):
    _check(load().moe_set_tile_config(h, int(down_bn)))


def moe_set_launch_options(h, pdl):
    _check(load().moe_set_launch_options(h, int(pdl)))


def moe_set_gemm_options(h, cta_pairs):
    _check(load().moe_set_gemm_options(h, int(cta_pairs)))


def moe_set_wait_limit(h, cycles):
    _check(load().moe_set_wait_limit(h, int(cycles)))


def moe_set_picker_params(h, alpha, beta, bw, gamma):
    arr = (ctypes.c_longlong * 4)(alpha, beta, bw, gamma)
    _check(load().moe_set_picker_params(h, arr))


def moe_get_picker_params(h):
    """-> (alpha, beta, bw, gamma, num_sms)"""
    arr = (ctypes.c_longlong * 5)()
    _check(load().moe_get_picker_params(h, arr))
    return tuple(arr)


def moe_set_gate_up_tile(h, bn):
    _check(load().moe_set_gate_up_tile(h, bn))


def moe_set_gate_up_model(h, *params):
    """params: a_0, b_0, a_1, b_1, a_2, b_2 (ps per unit: kb a + b of each mode)"""
    arr = (ctypes.c_longlong * 6)(*params)
    _check(load().moe_set_gate_up_model(h, arr))


def moe_get_gate_up_model(h):
    """(a_0, b_0, a_1, b_1, a_2, b_2, nb, kb, num_sms, allowed-mode mask)"""
    arr = (ctypes.c_longlong * 10)()
    _check(load().moe_get_gate_up_model(h, arr))
    return tuple(arr)


def moe_workspace_init(h, ws, stream=None):
    _check(load().moe_workspace_init(h, _ptr(ws), _stream(stream)))


def moe_get_status(h, ws, stream=None):
    """Returns the status code (0 = OK) and clears it; does not raise."""
    st = load().moe_get_status(h, _ptr(ws), _stream(stream))
    return st, (load().moe_last_error().decode() if st else "")


# ------------------------------------------------------------ device buffers
class Layer:
    """One layer's handle, packed weights and one workspace, all in torch memory."""

    def __init__(self, wl, weights, max_T, device="cuda"):
        self.wl = wl
        self.max_T = max_T
        self.h = moe_init(wl, max_T)
        self.packed = torch.empty(moe_weights_size(self.h), dtype=torch.uint8, device=device)
        self.ws = torch.empty(moe_workspace_size(self.h), dtype=torch.uint8, device=device)
        moe_workspace_init(self.h, self.ws)
        dev = {n: (v.to(device) if v is not None else None) for n, v in weights.items()
               if n.endswith(("_q", "_s", "_g"))}
        moe_pack_weights(self.h, dev, self.packed)
        torch.cuda.synchronize()
        self.view = moe_workspace_view_get(self.h, self.ws)

    def region(self, name, dtype, count):
        """A torch tensor aliasing `count` elements of a workspace region."""
        off = self.view[name] - self.ws.data_ptr()
        nbytes = count * torch.empty(0, dtype=dtype).element_size()
        return self.ws[off:off + nbytes].view(dtype)

    def forward(self, x, wr, bias, y=None, stream=None):
        T = x.shape[0]
        if y is None:
            y = torch.empty(T, self.wl.H, dtype=torch.bfloat16, device=x.device)
        moe_forward(self.h, x, T, wr, bias, self.packed, y, self.ws, stream)
        return y

    def status(self):
        return moe_get_status(self.h, self.ws)

    def close(self):
        if self.h is not None:
            moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
