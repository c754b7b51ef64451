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


def fp8_values(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def abs_down_weights(wl, weights, slot):
    """|W_down| of the expert in weight slot `slot`, dequantised with torch's fp8 conversion ([H, I] fp64)."""
    q = np.asarray(weights["down_q"][slot])
    if wl.fmt == W.FMT_NVFP4:
        sb = np.repeat(fp8_values(np.asarray(weights["down_s"][slot])), 16, axis=1)
        return np.abs(e2m1_values(q)) * sb * float(np.asarray(weights["down_g"])[slot])
    s = np.asarray(weights["down_s"][slot], np.float64)
    v = np.abs(fp8_values(q))
    if wl.fmt == W.FMT_FP8_ROW:
        return v * s[:, None]
    return v * np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)


def deviation_bound_rows(wl, weights, slot_of, rows, n_out):
    """sum over rows (out_index, expert, weight, h_gpu [I], h_ref [I]) of
    |weight| * |W_down[e]| @ |h_gpu - h_ref|, per output row ([n_out, H])."""
    extra = np.zeros((n_out, wl.H))
    cache = {}
    for i, e, wj, v_gpu, v_ref in rows:
        dv = np.abs(np.asarray(v_gpu, np.float64) - np.asarray(v_ref, np.float64))
        if not dv.any():
            continue
        if e not in cache:
            cache[e] = abs_down_weights(wl, weights, slot_of(e))
        extra[i] += abs(float(wj)) * (cache[e] @ dv)
    return extra


def hidden_values(codes, scales, I):
    """FP8 hidden codes x their (row, 128-column) scales -> fp64 values."""
    return fp8_values(codes) * np.repeat(np.asarray(scales, np.float64).reshape(-1), 128)[:I]


def hidden_deviation_bound(wl, L, ids, w, ref, hq_gpu, hs_gpu, tokens=None, values=None):
    """Largest change of Y that differences between the GPU's and the oracle's
    requantised hidden can cause, per output element:
        sum_j |w_j| sum_n |h_gpu[slot(t,j), n] - h_ref[slot(t,j), n]| |W_down[e_j][m, n]|
    h values are code value x block scale.  A hidden code that rounds the other
    way at a rounding boundary (fp32 vs fp64 accumulation) moves its whole
    output row by about one e4m3 step times the weights; this bound lets the
    end-to-end check tell such moves from real errors.  (FP8 formats only.)"""
    T = ids.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    nb = wl.I // 128
    extra = np.zeros((len(tokens), wl.H))
    wd_abs = {}
    for i, t in enumerate(tokens):
        for j in range(wl.k):
            e = int(ids[t, j])
            r = int(ref["inv"][t * wl.k + j])
            if values is not None:
                v_gpu, v_ref = values[0][r], values[1][r]
            else:
                v_gpu = fp8_values(hq_gpu[r]) * np.repeat(hs_gpu[r].reshape(nb).astype(np.float64), 128)
                v_ref = fp8_values(ref["hq"][r]) * np.repeat(ref["hs"][r].reshape(nb).astype(np.float64), 128)
            dv = np.abs(v_gpu - v_ref)
            if not dv.any():
                continue
            if e not in wd_abs:
                wd_abs[e] = np.abs(np.stack([L.weight_row("down", e, m) for m in range(wl.H)]))
            extra[i] += abs(float(w[t, j])) * (wd_abs[e] @ dv)
    return extra


def tolerance_violations_with_bound(y_gpu, y_ref, extra):
    """Elements outside 2e-2 |ref| + 2e-3 rms(ref) + extra, and outside the plain tolerance."""
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    tol = 2e-2 * np.abs(y_ref) + 2e-3 * rms
    err = np.abs(y_gpu - y_ref)
    # bf16 output: the bound gets the final rounding of the moved value too
    slack = extra * (1 + 2.0 ** -8)
    return int((err > tol + slack).sum()), int((err > tol).sum())


# ------------------------------------------------------------------ NVFP4 layout
E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def sf_offset(row, c, sf_cols):
    """Byte of scale factor (row, column c) in the chunked layout the tensor cores
    read: per 128-row tile and 4 columns, 512 B, row r at (r%32)*16 + (r//32)*4 + c%4."""
    row = np.asarray(row, np.int64)
    c = np.asarray(c, np.int64)
    r = row % 128
    return ((row // 128) * (sf_cols // 4) + c // 4) * 512 + (r % 32) * 16 + (r // 32) * 4 + c % 4


def padded_rows(slots, ids_flat, perm, offsets, tile_ptr):
    """128-padded row of each assignment slot: tile_ptr[e]*128 + slot - offsets[e]."""
    slots = np.asarray(slots, np.int64)
    e = ids_flat[perm[slots]]
    return tile_ptr[e].astype(np.int64) * 128 + slots - offsets[e]


def gather_sf(buf, rows, sf_cols):
    """Row-major [len(rows), sf_cols] scale factors out of the chunked layout."""
    rows = np.asarray(rows, np.int64)
    cols = np.arange(sf_cols)
    return buf[sf_offset(rows[:, None], cols[None, :], sf_cols)]


def scatter_sf(buf, rows, sf_rm, sf_cols):
    rows = np.asarray(rows, np.int64)
    cols = np.arange(sf_cols)
    buf[sf_offset(rows[:, None], cols[None, :], sf_cols)] = sf_rm


def e2m1_values(packed):
    p = np.ascontiguousarray(packed, np.uint8)
    nib = np.stack([p & 15, p >> 4], axis=-1).reshape(*p.shape[:-1], p.shape[-1] * 2)
    mag = E2M1_MAG[nib & 7]
    return np.where(nib & 8, -mag, mag)


def nvfp4_hidden_values(codes, sf_rm, g):
    return e2m1_values(codes) * np.repeat(fp8_values(sf_rm), 16, axis=-1) * float(g)


def mx_hidden_values(codes, sf_rm):
    """MX32 hidden: e4m3 code x 2^(scale code - 127) per 32 columns."""
    return fp8_values(codes) * np.repeat(np.exp2(np.asarray(sf_rm, np.float64) - 127), 32, axis=-1)


def hidden_padded(wl):
    """The hidden sits in 128-padded rows with chunked block scales (FP8_ROW, NVFP4)."""
    return wl.fmt != W.FMT_FP8_BLOCK128


def hidden_sf_cols(wl):
    return wl.I // 32 if wl.fmt == W.FMT_FP8_ROW else wl.I // 16


def hidden_code_bytes(wl):
    return wl.I // 2 if wl.fmt == W.FMT_NVFP4 else wl.I


def hidden_values_of(wl, codes, scales):
    """fp64 values of hidden rows given their codes and row-major scales, any format."""
    if wl.fmt == W.FMT_FP8_ROW:
        return mx_hidden_values(codes, scales)
    if wl.fmt == W.FMT_NVFP4:
        return nvfp4_hidden_values(codes, scales, wl.hidden_global_scale)
    nb = wl.I // 128
    return fp8_values(codes) * np.repeat(np.asarray(scales, np.float64).reshape(-1, nb), 128, axis=1)
