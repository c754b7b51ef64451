"""Python access to the CPU oracle (moe_oracle.c) through ctypes.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  Nothing on the CUDA path imports it, and
it imports nothing from the CUDA path.  Inputs and outputs are numpy arrays.
"""
import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.c")
LIB = os.path.join(HERE, "libmoe_oracle.so")

FMT_FP8_ROW, FMT_FP8_BLOCK128, FMT_NVFP4, FMT_MX32 = 0, 1, 2, 3
SCORE_SOFTMAX, SCORE_SIGMOID = 0, 1
TILE_M = 128


def build(force=False):
    """Compile the oracle with gcc (plain C + OpenMP)."""
    hdr = os.path.join(HERE, "moe_oracle.h")
    if not force and os.path.exists(LIB) and \
            os.path.getmtime(LIB) >= max(os.path.getmtime(SRC), os.path.getmtime(hdr)):
        return LIB
    cmd = ["gcc", "-O2", "-fopenmp", "-mfma", "-ffp-contract=off", "-fno-math-errno",
           "-Wall", "-shared", "-fPIC", SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


_lib = None


class _Proj(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("s", ctypes.c_void_p), ("g", ctypes.c_void_p)]


class _Layer(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("I", ctypes.c_int), ("E", ctypes.c_int),
                ("k", ctypes.c_int), ("score", ctypes.c_int), ("fmt", ctypes.c_int),
                ("hidden_global", ctypes.c_float),
                ("gate", _Proj), ("up", _Proj), ("down", _Proj),
                ("expert_slot", ctypes.c_void_p),
                ("act", ctypes.c_int), ("act_alpha", ctypes.c_double), ("act_limit", ctypes.c_double),
                ("hidden_rule", ctypes.c_int)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        P, I, I64, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        sig = {
            "orc_e4m3_value": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e4m3_encode": (ctypes.c_uint8, [F]),
            "orc_e2m1_value": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e2m1_encode": (ctypes.c_uint8, [F]),
            "orc_e4m3_encode_n": (None, [P, I64, P]),
            "orc_e2m1_encode_n": (None, [P, I64, P]),
            "orc_router_logits": (None, [P, I, I, P, P, I, P]),
            "orc_router_logits_f64": (None, [P, I, I, P, P, I, P]),
            "orc_topk": (None, [P, I, I, I, I, P, P]),
            "orc_dispatch": (None, [P, I, I, I, P, P, P, P]),
            "orc_schedule": (I, [P, I, P, P]),
            "orc_quant_rows": (None, [I, P, I, I, F, P, P]),
            "orc_nvfp4_global": (F, [P, I64]),
            "orc_weight_row": (None, [P, P, I, I, I, I, P]),
            "orc_expert_rows": (None, [P, I, I, P, P, F, P, P, P, P]),
            "orc_down_rows": (None, [P, I, I, P, P, P]),
            "orc_moe_forward": (I, [P, P, I, P, P, I, P, P, P, P]),
            "orc_num_threads": (I, []),
            "orc_pick_down_tile": (I, [P, I, I, I, I, I64, I64, I64, I64, P]),
            "orc_pick_split": (I, [P, I, I, I, I64, I]),
            "orc_pick_gu_mode": (I, [P, I, I, I, I, I, P]),
            "orc_glu": (ctypes.c_double, [I, ctypes.c_double, ctypes.c_double, ctypes.c_double, ctypes.c_double]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads():
    return lib().orc_num_threads()


# ---------------------------------------------------------------- codecs
def e4m3_value(code):
    return lib().orc_e4m3_value(int(code))


def e2m1_value(code):
    return lib().orc_e2m1_value(int(code))


def e4m3_encode(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(x), x.size, _p(out))
    return out


def e2m1_encode(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e2m1_encode_n(_p(x), x.size, _p(out))
    return out


# ---------------------------------------------------------------- router
def router_logits(x_bf16_bits, wr, bias=None):
    """x: [T,H] uint16 (bf16 bits); wr: [E,H] fp32; bias: [E] fp32 or None -> [T,E] fp32."""
    x = _c(x_bf16_bits, np.uint16)
    wr = _c(wr, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float32)
    lib().orc_router_logits(_p(x), T, H, _p(wr), _p(b), E, _p(out))
    return out


def router_logits_f64(x_bf16_bits, wr, bias=None):
    x = _c(x_bf16_bits, np.uint16)
    wr = _c(wr, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float64)
    lib().orc_router_logits_f64(_p(x), T, H, _p(wr), _p(b), E, _p(out))
    return out


def topk(logits, k, score):
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lib().orc_topk(_p(lg), T, E, k, score, _p(ids), _p(w))
    return ids, w


# ---------------------------------------------------------------- dispatch
def dispatch(ids, E):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    lib().orc_dispatch(_p(ids), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv))
    return counts, offsets, perm, inv


def schedule(offsets):
    offsets = _c(offsets, np.int32)
    E = offsets.size - 1
    cap = int(offsets[-1]) // TILE_M + E + 1
    te = np.empty(cap, np.int32)
    tr = np.empty(cap, np.int32)
    n = lib().orc_schedule(_p(offsets), E, _p(te), _p(tr))
    return te[:n].copy(), tr[:n].copy()


# ---------------------------------------------------------------- tile choice
def pick_down_tile(counts, H, I, num_sms, alpha, beta, bw, gamma):
    """Down GEMM tile choice from the expert histogram -> (candidate, [cost per candidate])."""
    counts = _c(counts, np.int32)
    costs = np.empty(3, np.int64)
    c = lib().orc_pick_down_tile(_p(counts), counts.size, H, I, num_sms, alpha, beta, bw, gamma, _p(costs))
    return c, costs


ACT_SWIGLU, ACT_SWIGLU_BOUNDED, ACT_SWIGLU_OAI, ACT_GEGLU, ACT_REGLU, ACT_RELU2 = range(6)


def glu(act, g, u, alpha=0.0, limit=0.0):
    """Gated activation act(g, u) in fp64 (scalars or arrays)."""
    f = np.vectorize(lambda a, b: lib().orc_glu(act, float(alpha), float(limit), float(a), float(b)))
    return f(np.asarray(g, np.float64), np.asarray(u, np.float64))


def pick_split(counts, split_nb, split_kb, o_rows, num_sms):
    """K split S of the FP8_ROW down GEMM from the expert histogram (1 = none)."""
    counts = _c(counts, np.int32)
    return lib().orc_pick_split(_p(counts), counts.size, split_nb, split_kb, o_rows, num_sms)


# ---------------------------------------------------------------- quantisers
def pick_gu_mode(counts, nb, kb, num_sms, ps, allow=7):
    """Gated FP8_ROW gate/up mode: 0 single CTAs on 256-wide tiles, 1 CTA
    pairs, 2 single CTAs on 128-wide tiles (moe_oracle.h)."""
    c = _c(counts, np.int32)
    p = _c(ps, np.int64)
    assert p.size == 6
    return int(lib().orc_pick_gu_mode(_p(c), c.size, nb, kb, num_sms, allow, _p(p)))


def code_bytes(fmt, K):
    return K // 2 if fmt == FMT_NVFP4 else K


def scale_shape(fmt, rows, K):
    if fmt == FMT_FP8_ROW:
        return (rows,), np.float32
    if fmt == FMT_FP8_BLOCK128:
        return (rows, K // 128), np.float32
    if fmt == FMT_MX32:
        return (rows, K // 32), np.uint8
    return (rows, K // 16), np.uint8


HIDDEN_LAYER, HIDDEN_PER_TOKEN = 0, 1


def hidden_fmt(fmt, rule=HIDDEN_LAYER):
    """Format of the requantised hidden: MX32 for FP8_ROW, otherwise the layer's
    own; with the per-token reading (FP8 formats) one fp32 scale per row."""
    if rule == HIDDEN_PER_TOKEN and fmt != FMT_NVFP4:
        return FMT_FP8_ROW
    return FMT_MX32 if fmt == FMT_FP8_ROW else fmt


def quant_rows(fmt, x, g=0.0):
    """fp32 rows [R,K] -> (codes, scales) in the layer's activation format."""
    x = _c(x, np.float32)
    R, K = x.shape
    codes = np.empty((R, code_bytes(fmt, K)), np.uint8)
    shp, dt = scale_shape(fmt, R, K)
    scales = np.empty(shp, dt)
    lib().orc_quant_rows(fmt, _p(x), R, K, float(g), _p(codes), _p(scales))
    return codes, scales


def nvfp4_global(x):
    x = _c(x, np.float32)
    return lib().orc_nvfp4_global(_p(x), x.size)


# ---------------------------------------------------------------- layer
class Layer:
    """Holds numpy copies of the quantised weights and the ctypes struct over them."""

    def __init__(self, wl, weights, expert_slot=None, hidden_rule=HIDDEN_LAYER):
        self.wl = wl
        self.hidden_rule = hidden_rule
        self._keep = {}
        st = _Layer()
        st.H, st.I, st.E, st.k = wl.H, wl.I, wl.E, wl.k
        st.score, st.fmt = wl.score, wl.fmt
        st.hidden_global = float(wl.hidden_global_scale)
        st.act, st.act_alpha, st.act_limit = wl.act, float(wl.act_alpha), float(wl.act_limit)
        st.hidden_rule = hidden_rule
        for p in ("gate", "up", "down"):
            if weights.get(p + "_q") is None:      # ReLU^2 experts have no gate
                setattr(st, p, _Proj(None, None, None))
                continue
            q = _c(weights[p + "_q"], np.uint8)
            s = np.ascontiguousarray(weights[p + "_s"])
            g = None if wl.fmt != FMT_NVFP4 else _c(weights[p + "_g"], np.float32)
            self._keep[p] = (q, s, g)
            setattr(st, p, _Proj(q.ctypes.data, s.ctypes.data, None if g is None else g.ctypes.data))
        if expert_slot is not None:
            es = _c(expert_slot, np.int32)
            self._keep["slot"] = es
            st.expert_slot = es.ctypes.data
        else:
            st.expert_slot = None
        self.st = st

    def ref(self):
        return ctypes.byref(self.st)

    def weight_row(self, proj, e, n):
        wl = self.wl
        N, K = (wl.I, wl.H) if proj in ("gate", "up") else (wl.H, wl.I)
        out = np.empty(K, np.float64)
        lib().orc_weight_row(self.ref(), ctypes.byref(getattr(self.st, proj)), N, K, e, n, _p(out))
        return out

    def expert_rows(self, e, a_codes, a_scales, x_global=0.0):
        wl = self.wl
        a_codes = _c(a_codes, np.uint8)
        a_scales = np.ascontiguousarray(a_scales)
        R = a_codes.shape[0]
        h = np.empty((R, wl.I), np.float64)
        hq = np.empty((R, code_bytes(wl.fmt, wl.I)), np.uint8)
        shp, dt = scale_shape(hidden_fmt(wl.fmt, self.hidden_rule), R, wl.I)
        hs = np.empty(shp, dt)
        o = np.empty((R, wl.H), np.float64)
        lib().orc_expert_rows(self.ref(), e, R, _p(a_codes), _p(a_scales), float(x_global),
                              _p(h), _p(hq), _p(hs), _p(o))
        return h, hq, hs, o

    def down_rows(self, e, h_codes, h_scales):
        wl = self.wl
        h_codes = _c(h_codes, np.uint8)
        h_scales = np.ascontiguousarray(h_scales)
        R = h_codes.shape[0]
        o = np.empty((R, wl.H), np.float64)
        lib().orc_down_rows(self.ref(), e, R, _p(h_codes), _p(h_scales), _p(o))
        return o

    def forward(self, x_bf16_bits, wr, bias, sel=None):
        """Routing for all tokens and fp64 Y for the tokens in sel (default: all)."""
        wl = self.wl
        x = _c(x_bf16_bits, np.uint16)
        T = x.shape[0]
        sel = np.arange(T, dtype=np.int32) if sel is None else _c(sel, np.int32)
        wr = _c(wr, np.float32)
        b = None if bias is None else _c(bias, np.float32)
        ids = np.empty((T, wl.k), np.int32)
        w = np.empty((T, wl.k), np.float64)
        y = np.empty((sel.size, wl.H), np.float64)
        rc = lib().orc_moe_forward(self.ref(), _p(x), T, _p(wr), _p(b), sel.size, _p(sel),
                                   _p(ids), _p(w), _p(y))
        if rc != 0:
            raise ValueError("oracle: a selected token needs an expert whose weights were not provided")
        return ids, w, y
