"""Layer-level pins of the CPU oracle.

- one expert, top-1: the layer is a dense SwiGLU MLP, computed here with torch
  fp64 matmuls and torch's SiLU on operands dequantised by torch's own fp8
  conversion (and a literal E2M1 table), not by the oracle's decoder;
- all logits equal: experts 0..k-1 with weight 1/k, so Y is the mean of those
  experts' outputs;
- sigmoid scores with zero router weights: the selection is the k largest
  biases and the weights are sigmoid(b)/sum, a closed form;
- permuting the tokens permutes routing and output.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_topk_b200 import synth, workloads as W

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def fp8_val(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def e2m1_val(packed):
    p = np.ascontiguousarray(packed, np.uint8)
    lo, hi = p & 15, p >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(*p.shape[:-1], p.shape[-1] * 2)
    mag = E2M1_MAG[nib & 7]
    return np.where(nib & 8, -mag, mag)


def deq_weight(wl, d, p, e):
    q = d[p + "_q"][e].numpy()
    s = d[p + "_s"][e].numpy()
    if wl.fmt == W.FMT_FP8_ROW:
        return fp8_val(q) * s.astype(np.float64)[:, None]
    if wl.fmt == W.FMT_FP8_BLOCK128:
        return fp8_val(q) * np.kron(s.astype(np.float64), np.ones((128, 128)))
    v = e2m1_val(q)
    sb = np.repeat(fp8_val(s), 16, axis=1)
    return v * sb * float(d[p + "_g"][e])


def deq_act(wl, codes, scales, g=0.0):
    if wl.fmt == oracle.FMT_MX32:
        return fp8_val(codes) * np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=1)
    if wl.fmt == W.FMT_FP8_ROW:
        return fp8_val(codes) * scales.astype(np.float64)[:, None]
    if wl.fmt == W.FMT_FP8_BLOCK128:
        return fp8_val(codes) * np.repeat(scales.astype(np.float64), 128, axis=1)
    return e2m1_val(codes) * np.repeat(fp8_val(scales), 16, axis=1) * g


def bf16_bits(x):
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


FMTS = [W.FMT_FP8_ROW, W.FMT_FP8_BLOCK128, W.FMT_NVFP4]


@pytest.mark.parametrize("fmt", FMTS)
def test_single_expert_is_dense_swiglu_mlp(fmt):
    wl = W.custom(H=256, I=384, E=1, k=1, fmt=fmt)
    d = synth.layer(wl, seed=5)
    L = oracle.Layer(wl, d)
    x = synth.tokens(wl, 6, seed=5)
    xf = x.to(torch.float32).numpy()
    g_x = oracle.nvfp4_global(xf) if fmt == W.FMT_NVFP4 else 0.0
    codes, scales = oracle.quant_rows(fmt, xf, g_x)
    h, hq, hs, o = L.expert_rows(0, codes, scales, g_x)

    a = torch.from_numpy(deq_act(wl, codes, scales, g_x))
    wg = torch.from_numpy(deq_weight(wl, d, "gate", 0))
    wu = torch.from_numpy(deq_weight(wl, d, "up", 0))
    wd = torch.from_numpy(deq_weight(wl, d, "down", 0))
    h_ref = torch.nn.functional.silu(a @ wg.T) * (a @ wu.T)
    np.testing.assert_allclose(h, h_ref.numpy(), rtol=1e-12, atol=1e-12)
    # the requantised hidden is what the down projection sees
    hfmt = oracle.hidden_fmt(fmt)
    hq2, hs2 = oracle.quant_rows(hfmt, h_ref.numpy().astype(np.float32), wl.hidden_global_scale)
    assert (hq2 == hq).mean() > 0.999
    hwl = W.custom(H=wl.H, I=wl.I, E=1, k=1, fmt=hfmt)
    o_ref = torch.from_numpy(deq_act(hwl, hq, hs, wl.hidden_global_scale)) @ wd.T
    np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-12, atol=1e-12)

    # the whole layer with one expert and top-1 is the same MLP with weight 1
    ids, w, y = L.forward(bf16_bits(x), d["wr"].numpy(), None)
    assert (ids == 0).all() and (w == 1.0).all()
    np.testing.assert_allclose(y, o_ref.numpy(), rtol=1e-12, atol=1e-12)


def _torch_glu(act, g, u, alpha, limit):
    """The gated activations written with torch fp64 library routines."""
    F = torch.nn.functional
    if act == W.ACT_SWIGLU:
        return F.silu(g) * u
    if act == W.ACT_SWIGLU_BOUNDED:
        return F.silu(torch.clamp(g, max=limit)) * torch.clamp(u, -limit, limit)
    if act == W.ACT_SWIGLU_OAI:
        gc = torch.clamp(g, max=limit)
        return gc * torch.sigmoid(alpha * gc) * (torch.clamp(u, -limit, limit) + 1.0)
    if act == W.ACT_GEGLU:
        return F.gelu(g, approximate="none") * u
    if act == W.ACT_RELU2:
        return F.relu(u) ** 2
    return F.relu(g) * u


ACTS = [(W.ACT_SWIGLU, 0.0, 0.0), (W.ACT_SWIGLU_BOUNDED, 0.0, 0.25), (W.ACT_SWIGLU_OAI, 1.702, 0.3),
        (W.ACT_GEGLU, 0.0, 0.0), (W.ACT_REGLU, 0.0, 0.0), (W.ACT_RELU2, 0.0, 0.0)]


@pytest.mark.parametrize("act,alpha,limit", ACTS)
@pytest.mark.parametrize("fmt", FMTS)
def test_single_expert_is_the_dense_gated_mlp_of_each_activation(fmt, act, alpha, limit):
    """E = 1, top-1 with each gated activation: the hidden equals the dense MLP
    written with torch fp64 routines (the limits are chosen inside the range of
    the pre-activations, so the clamps bind on part of the elements)."""
    wl = W.custom(H=256, I=256, E=1, k=1, fmt=fmt, act=act, act_alpha=alpha, act_limit=limit)
    d = synth.layer(wl, seed=8)
    L = oracle.Layer(wl, d)
    x = synth.tokens(wl, 5, seed=8)
    xf = x.to(torch.float32).numpy()
    g_x = oracle.nvfp4_global(xf) if fmt == W.FMT_NVFP4 else 0.0
    codes, scales = oracle.quant_rows(fmt, xf, g_x)
    h, hq, hs, o = L.expert_rows(0, codes, scales, g_x)
    a = torch.from_numpy(deq_act(wl, codes, scales, g_x))
    u = a @ torch.from_numpy(deq_weight(wl, d, "up", 0)).T
    g = u if act == W.ACT_RELU2 else a @ torch.from_numpy(deq_weight(wl, d, "gate", 0)).T
    if act == W.ACT_RELU2:
        assert d["gate_q"] is None
    if limit > 0.0:
        assert (g > limit).any() and (u.abs() > limit).any()
    h_ref = _torch_glu(act, g, u, alpha, limit)
    np.testing.assert_allclose(h, h_ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("fmt", FMTS)
def test_equal_logits_average_the_first_k_experts(fmt):
    wl = W.custom(H=256, I=256, E=5, k=3, fmt=fmt)
    d = synth.layer(wl, seed=6)
    L = oracle.Layer(wl, d)
    x = synth.tokens(wl, 4, seed=6)
    wr0 = np.zeros((wl.E, wl.H), np.float32)
    ids, w, y = L.forward(bf16_bits(x), wr0, None)
    assert (ids == np.arange(3)).all()
    np.testing.assert_allclose(w, 1.0 / 3.0, rtol=1e-15)
    xf = x.to(torch.float32).numpy()
    g_x = oracle.nvfp4_global(xf) if fmt == W.FMT_NVFP4 else 0.0
    codes, scales = oracle.quant_rows(fmt, xf, g_x)
    outs = [L.expert_rows(e, codes, scales, g_x)[3] for e in range(3)]
    np.testing.assert_allclose(y, sum(outs) / 3.0, rtol=1e-12, atol=1e-12)


def test_sigmoid_scores_with_bias_only_closed_form():
    wl = W.custom(H=256, I=128, E=6, k=2, score=W.SCORE_SIGMOID)
    d = synth.layer(wl, seed=7)
    L = oracle.Layer(wl, d)
    x = synth.tokens(wl, 3, seed=7)
    bias = np.float32([0.5, -1.0, 2.0, 2.0, 0.25, -3.0])
    ids, w, _ = L.forward(bf16_bits(x), np.zeros((6, 256), np.float32), bias)
    assert (ids == [2, 3]).all()          # tie at 2.0 -> lower id first
    np.testing.assert_allclose(w, 0.5, rtol=1e-15)
    bias[3] = 1.0
    ids, w, _ = L.forward(bf16_bits(x), np.zeros((6, 256), np.float32), bias)
    s2, s1 = 1 / (1 + math.exp(-2.0)), 1 / (1 + math.exp(-1.0))
    assert (ids == [2, 3]).all()
    np.testing.assert_allclose(w, np.broadcast_to([s2 / (s1 + s2), s1 / (s1 + s2)], w.shape), rtol=1e-14)


@pytest.mark.parametrize("fmt", FMTS)
def test_token_permutation_equivariance(fmt):
    wl = W.custom(H=256, I=128, E=8, k=2, fmt=fmt)
    d = synth.layer(wl, seed=8)
    L = oracle.Layer(wl, d)
    x = synth.tokens(wl, 9, seed=8)
    xb = bf16_bits(x)
    ids, w, y = L.forward(xb, d["wr"].numpy(), None)
    p = np.random.default_rng(8).permutation(9)
    ids2, w2, y2 = L.forward(np.ascontiguousarray(xb[p]), d["wr"].numpy(), None)
    assert (ids2 == ids[p]).all()
    assert (w2 == w[p]).all()
    assert (y2 == y[p]).all()


def test_counts_sum_to_assignments_on_skewed_workload():
    wl = W.custom(H=256, I=128, E=64, k=8, zipf_s=1.2)
    d = synth.layer(wl, seed=9)
    x = synth.tokens(wl, 200, seed=9)
    lg = oracle.router_logits(bf16_bits(x), d["wr"].numpy(), d["bias"].numpy())
    ids, _ = oracle.topk(lg, wl.k, wl.score)
    counts, offsets, perm, inv = oracle.dispatch(ids, wl.E)
    assert counts.sum() == 200 * 8 and offsets[-1] == 200 * 8
    assert (counts == 0).sum() > 0          # the Zipf bias leaves experts empty
    assert all(len(set(r)) == wl.k for r in ids)   # distinct experts per token


def test_subset_forward_matches_full_forward():
    wl = W.custom(H=256, I=128, E=8, k=2)
    d = synth.layer(wl, seed=10)
    x = synth.tokens(wl, 12, seed=10)
    L = oracle.Layer(wl, d)
    ids, w, y = L.forward(bf16_bits(x), d["wr"].numpy(), None)
    sel = np.int32([11, 3, 4])
    used = sorted(set(ids[sel].reshape(-1)))
    slot = np.full(wl.E, -1, np.int32)
    slot[used] = np.arange(len(used))
    sub = {k_: (v[used] if k_.endswith(("_q", "_s", "_g")) else v) for k_, v in d.items()}
    Ls = oracle.Layer(wl, sub, expert_slot=slot)
    ids2, w2, y2 = Ls.forward(bf16_bits(x), d["wr"].numpy(), None, sel=sel)
    assert (ids2 == ids).all()
    assert (y2 == y[sel]).all()


@pytest.mark.parametrize("fmt", [W.FMT_FP8_ROW, W.FMT_FP8_BLOCK128])
def test_per_token_hidden_reading_is_the_row_rule_on_the_dense_mlp(fmt):
    """The oracle-only per-token hidden (one fp32 scale per hidden row, the
    FP8_ROW rule of X): with one expert and top-1, its codes and scales are
    those of the row rule applied to the torch fp64 SwiGLU rounded to fp32,
    and the output is their dequantised values through W_down."""
    wl = W.custom(H=256, I=384, E=1, k=1, fmt=fmt)
    d = synth.layer(wl, seed=15)
    L = oracle.Layer(wl, d, hidden_rule=oracle.HIDDEN_PER_TOKEN)
    x = synth.tokens(wl, 7, seed=15)
    xf = x.to(torch.float32).numpy()
    codes, scales = oracle.quant_rows(fmt, xf)
    h, hq, hs, o = L.expert_rows(0, codes, scales)
    assert hs.shape == (7,) and hs.dtype == np.float32
    a = torch.from_numpy(deq_act(wl, codes, scales))
    h_ref = torch.nn.functional.silu(a @ torch.from_numpy(deq_weight(wl, d, "gate", 0)).T) * \
        (a @ torch.from_numpy(deq_weight(wl, d, "up", 0)).T)
    np.testing.assert_allclose(h, h_ref.numpy(), rtol=1e-12, atol=1e-12)
    hf = h_ref.numpy().astype(np.float32)
    s_ref = np.abs(hf).max(axis=1) / np.float32(448.0)     # fp32 division, as the row rule
    assert (hs == s_ref).all()
    hq2, hs2 = oracle.quant_rows(W.FMT_FP8_ROW, hf)
    assert (hs2 == hs).all()
    assert (hq2 == hq).mean() > 0.999
    o_ref = (fp8_val(hq) * hs.astype(np.float64)[:, None]) @ deq_weight(wl, d, "down", 0).T
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)


# the FP8_ROW workloads at a few tokens each (only the experts those tokens use
# are drawn)
READING_CASES = [("tiny", 16), ("qwen3.5-35b-a3b", 6), ("mixtral-8x7b", 1)]


@pytest.mark.parametrize("name,T", READING_CASES)
def test_block_scaled_hidden_distance_from_per_token_reading(name, T):
    """How far the layer's block-scaled hidden (MX32, a power-of-two scale per
    32 columns) moves Y from the literal per-token reading of "activations
    dynamically quantised per token".  Both round the same fp32 hidden to e4m3,
    on different grids, so each hidden value moves by at most the sum of the
    two half steps, and Y by at most sum_j |w_j| |W_down| |dh|; the measured
    distance (elements outside the benchmark spec's tolerance when the per-token Y
    is taken as the reference, the largest ratio to it, the relative rms) is
    reported, and must stay inside that bound."""
    wl = W.WORKLOADS[name]
    x = synth.tokens(wl, T, seed=2)
    wr, bias = synth.router(wl, seed=2)
    lg = oracle.router_logits(bf16_bits(x), wr.numpy(), None if bias is None else bias.numpy())
    ids, w = oracle.topk(lg, wl.k, wl.score)
    used = sorted(set(ids.reshape(-1).tolist()))
    slot = np.full(wl.E, -1, np.int32)
    slot[used] = np.arange(len(used))
    de = synth.experts(wl, seed=2, experts_subset=used)
    sub = {k_: v[used] for k_, v in de.items() if v is not None}
    b = None if bias is None else bias.numpy()
    L_mx = oracle.Layer(wl, sub, expert_slot=slot)
    L_pt = oracle.Layer(wl, sub, expert_slot=slot, hidden_rule=oracle.HIDDEN_PER_TOKEN)
    _, _, y_mx = L_mx.forward(bf16_bits(x), wr.numpy(), b)
    _, _, y_pt = L_pt.forward(bf16_bits(x), wr.numpy(), b)
    rms = float(np.sqrt(np.mean(y_pt ** 2)))
    tol = 2e-2 * np.abs(y_pt) + 2e-3 * rms
    err = np.abs(y_mx - y_pt)
    # the bound: per (t, j), |dh| <= half an e4m3 step of each grid at h
    xq, xs = oracle.quant_rows(wl.fmt, x.to(torch.float32).numpy())
    bound = np.zeros_like(y_pt)
    for e in used:
        rows = [(t, j) for t in range(T) for j in range(wl.k) if ids[t, j] == e]
        tt = np.array([t for t, _ in rows])
        h, hq_mx, hs_mx, _ = L_mx.expert_rows(e, xq[tt], xs[tt])
        _, hq_pt, hs_pt, _ = L_pt.expert_rows(e, xq[tt], xs[tt])
        v_mx = fp8_val(hq_mx) * np.repeat(np.exp2(hs_mx.astype(np.float64) - 127), 32, axis=1)
        v_pt = fp8_val(hq_pt) * hs_pt.astype(np.float64)[:, None]
        hf = h.astype(np.float32).astype(np.float64)
        # half a step of e4m3 at |v| (2^-4 relative, or the subnormal step 2^-10 of the scale)
        step_mx = np.maximum(np.abs(hf) * 2.0 ** -4, np.repeat(np.exp2(hs_mx.astype(np.float64) - 127), 32, axis=1)
                             * 2.0 ** -10)
        step_pt = np.maximum(np.abs(hf) * 2.0 ** -4, hs_pt.astype(np.float64)[:, None] * 2.0 ** -10)
        assert np.all(np.abs(v_mx - v_pt) <= step_mx + step_pt + 1e-300)
        wd = np.abs(deq_weight(wl, sub, "down", int(slot[e])))
        dh = np.abs(v_mx - v_pt)
        for r, (t, j) in enumerate(rows):
            bound[t] += abs(w[t, j]) * (wd @ dh[r])
    assert np.all(err <= bound * (1 + 1e-9) + 1e-300)
    rec = {"case": f"{name} T={T}", "elements": int(y_pt.size), "outside_tolerance": int((err > tol).sum()),
           "max_ratio": float(np.max(err / tol)), "rel_rms": float(np.sqrt(np.mean(err ** 2))) / rms}
    print("HIDDEN_READING", rec)
