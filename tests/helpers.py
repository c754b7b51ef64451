"""Shared helpers of the tests: tolerance, bf16 bits, oracle intermediates in slot order."""
import numpy as np
import torch

import oracle
from mixture_experts_topk_b200 import workloads as W


def tolerance_violations(y_gpu, y_ref):
    """Elements outside |gpu - ref| <= 2e-2 |ref| + 2e-3 rms(ref) (rms over the whole output)."""
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    bad = np.abs(y_gpu - y_ref) > 2e-2 * np.abs(y_ref) + 2e-3 * rms
    return int(bad.sum())


def bits(x_bf16):
    return x_bf16.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def x_global(wl, x_bf16):
    if wl.fmt != W.FMT_NVFP4:
        return 0.0
    return oracle.nvfp4_global(x_bf16.float().numpy())


def slot_order_reference(wl, L, x_bf16, ids, w, with_ffn=True):
    """The oracle's intermediates for every assignment, in the dispatch slot order.

    Returns dict with counts, offsets, perm, inv, xq/xs (quantised X per slot),
    hq/hs (requantised hidden per slot), o (fp64 down output times routing weight).
    """
    T = x_bf16.shape[0]
    counts, offsets, perm, inv = oracle.dispatch(ids, wl.E)
    xf = x_bf16.float().numpy()
    g = x_global(wl, x_bf16)
    xq_tok, xs_tok = oracle.quant_rows(wl.fmt, xf, g)
    A = T * wl.k
    tok = perm // wl.k
    xq = xq_tok[tok]
    xs = xs_tok[tok]
    hq = np.zeros((A, oracle.code_bytes(wl.fmt, wl.I)), np.uint8)
    shp, dt = oracle.scale_shape(oracle.hidden_fmt(wl.fmt), A, wl.I)
    hs = np.zeros(shp, dt)
    h = np.zeros((A, wl.I), np.float64)
    o = np.zeros((A, wl.H), np.float64)
    for e in range(wl.E if with_ffn else 0):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        he, hqe, hse, oe = L.expert_rows(e, xq[a:b], xs[a:b], g)
        h[a:b], hq[a:b], hs[a:b], o[a:b] = he, hqe, hse, oe
    wflat = np.asarray(w, np.float64).reshape(-1)
    o_w = o * wflat[perm][:, None]
    return dict(counts=counts, offsets=offsets, perm=perm, inv=inv, xq=xq, xs=xs, h=h, hq=hq, hs=hs,
                o=o, o_w=o_w, x_global=g)
