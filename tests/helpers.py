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
    # rows in expert order, so that one |W_down| is held at a time
    cur_e, cur_w = None, None
    for i, e, wj, v_gpu, v_ref in sorted(rows, key=lambda r: r[1]):
        dv = np.abs(np.asarray(v_gpu, np.float64) - np.asarray(v_ref, np.float64))
        if not dv.any():
            continue
        if e != cur_e:
            cur_e, cur_w = e, abs_down_weights(wl, weights, slot_of(e))
        extra[i] += abs(float(wj)) * (cur_w @ dv)
    return extra


def hidden_values(codes, scales, I):
    """FP8 hidden codes x their (row, 128-column) scales -> fp64 values."""
    return fp8_values(codes) * np.repeat(np.asarray(scales, np.float64).reshape(-1), 128)[:I]


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


# ------------------------------------------------------------------ end-to-end checks
def sample_tokens(T, k, offsets, perm, seed, n_random=16, all_up_to=128):
    """Tokens whose outputs an end-to-end check compares: every token when T is
    small, else the tokens owning the first and the last slot of every 128-row
    tile of every expert (so the ragged last tile of each expert, both halves
    of every CTA pair, the half-empty pair of an odd tile count, and through
    whole output rows every column block and every K-split copy), plus tokens 0
    and T-1 and n_random seeded random tokens."""
    if T <= all_up_to:
        return np.arange(T, dtype=np.int32)
    sel = {0, T - 1}
    E = len(offsets) - 1
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        for r0 in range(a, b, 128):
            r1 = min(r0 + 128, b) - 1
            sel.add(int(perm[r0]) // k)
            sel.add(int(perm[r1]) // k)
    rng = np.random.default_rng(seed)
    sel.update(int(t) for t in rng.choice(T, size=min(n_random, T), replace=False))
    return np.array(sorted(sel), np.int32)


def gpu_hidden_rows(layer, wl, slots, ids_flat, perm, offsets):
    """(codes, row-major scales) of the GPU's requantised hidden for the given
    assignment slots, gathered on the device (any format)."""
    slots = np.asarray(slots, np.int64)
    A_max = layer.max_T * wl.k
    if not hidden_padded(wl):
        n = A_max + 128
        idx = torch.from_numpy(slots).cuda()
        hq = layer.region("hq", torch.uint8, n * wl.I).view(n, wl.I)[idx].cpu().numpy()
        hs = layer.region("hs", torch.float32, n * (wl.I // 128)).view(n, wl.I // 128)[idx].cpu().numpy()
        return hq, hs
    tile_ptr = layer.region("tile_ptr", torch.int32, wl.E + 1).cpu().numpy()
    prow = padded_rows(slots, ids_flat, perm, offsets, tile_ptr)
    n = A_max + 128 * wl.E
    cb, sc = hidden_code_bytes(wl), hidden_sf_cols(wl)
    hq = layer.region("hq", torch.uint8, n * cb).view(n, cb)[torch.from_numpy(prow).cuda()].cpu().numpy()
    off = torch.from_numpy(sf_offset(prow[:, None], np.arange(sc)[None, :], sc)).cuda()
    hs = layer.region("hs", torch.uint8, n * sc)[off].cpu().numpy()
    return hq, hs


def parity_report(case, checked, plain, max_ratio, bounded_ok=True, extra=None):
    """One line per end-to-end check: elements compared, elements outside the
    plain tolerance |gpu - ref| <= 2e-2 |ref| + 2e-3 rms(ref), and the largest
    |gpu - ref| / (2e-2 |ref| + 2e-3 rms(ref)).  Printed, and appended as JSON
    to the file named by MOE_PARITY_REPORT when that is set."""
    import json
    import os
    rec = {"case": case, "elements": int(checked), "outside_plain": int(plain),
           "max_ratio": float(max_ratio), "within_bound": bool(bounded_ok)}
    if extra:
        rec.update(extra)
    line = json.dumps(rec)
    print("PARITY", line)
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(line + "\n")
    return rec


def check_layer_output(case, wl, layer, L, x, ids, w, sel, y_gpu_sel, y_ref, weights, slot_of):
    """Y of the sampled tokens against the oracle.

    Every element must satisfy |gpu - ref| <= 2e-2 |ref| + 2e-3 rms(ref) (rms
    over the compared rows), or, for the few that do not, stay inside that
    tolerance widened by the exact bound on what the GPU's hidden codes that
    rounded the other way can move the output (deviation_bound_rows).  At most
    1e-3 of the elements (2 at least) may need the widening.  The bound is only
    computed for the tokens that need it.  Returns the report record."""
    y_gpu_sel = np.asarray(y_gpu_sel, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    tol = 2e-2 * np.abs(y_ref) + 2e-3 * rms
    err = np.abs(y_gpu_sel - y_ref)
    outside = err > tol
    plain = int(outside.sum())
    max_ratio = float(np.max(err / np.where(tol > 0, tol, np.inf))) if y_ref.size else 0.0
    bounded_ok = True
    if plain:
        need = np.nonzero(outside.any(axis=1))[0]
        T, k = ids.shape
        counts, offsets, perm, inv = oracle.dispatch(ids, wl.E)
        fp4 = wl.fmt == W.FMT_NVFP4
        g_x = oracle.nvfp4_global(x.float().cpu().numpy()) if fp4 else 0.0
        toks = np.asarray(sel)[need]
        xq_tok, xs_tok = oracle.quant_rows(wl.fmt, x[torch.from_numpy(toks).long().to(x.device)].float().cpu().numpy(),
                                           g_x)
        slots = np.array([int(inv[t * k + j]) for t in toks for j in range(k)], np.int64)
        hq_g, hs_g = gpu_hidden_rows(layer, wl, slots, ids.reshape(-1), perm, offsets)
        v_gpu_all = hidden_values_of(wl, hq_g, hs_g)
        rows = []
        by_e = {}
        for i, t in enumerate(toks):
            for j in range(k):
                by_e.setdefault(int(ids[t, j]), []).append((i, j))
        for e, lst in by_e.items():
            ii = np.array([i for i, _ in lst])
            _, hq_r, hs_r, _ = L.expert_rows(e, xq_tok[ii], xs_tok[ii], g_x)
            v_ref = hidden_values_of(wl, hq_r, hs_r)
            for r, (i, j) in enumerate(lst):
                rows.append((i, e, w[toks[i], j], v_gpu_all[i * k + j], v_ref[r]))
        extra = deviation_bound_rows(wl, weights, slot_of, rows, len(toks))
        slack = extra * (1 + 2.0 ** -8)
        bounded_ok = bool(np.all(err[need] <= tol[need] + slack))
    rec = parity_report(case, y_ref.size, plain, max_ratio, bounded_ok, {"tokens": int(len(sel))})
    assert bounded_ok, f"{case}: an element lies outside the tolerance widened by the hidden-flip bound"
    assert plain <= max(2, 1e-3 * y_ref.size), f"{case}: {plain} elements outside the plain tolerance"
    return rec
