"""Parity of the CUDA path with the CPU oracle, step by step and end to end.

Bit-exact: router ids, dispatch counts/offsets/perm/inv/tile table, quantised
X codes and scales.  Floating point: routing weights within 2e-6 (fp32 vs
fp64), the hidden codes within one code step on at most 1e-3 of the
elements, the layer output within |gpu - ref| <= 2e-2 |ref| + 2e-3 rms(ref).
All calls go through the C ABI (mixture_experts_topk_b200.native).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_topk_b200 import native, synth, workloads as W
from helpers import (bits, check_layer_output, fp8_values, gather_sf, hidden_code_bytes, hidden_padded,
                     hidden_sf_cols, hidden_values_of, padded_rows, scatter_sf, slot_order_reference,
                     tolerance_violations)

pytestmark = pytest.mark.gpu

# small shapes spanning several tiles and ragged tails, plus the named workloads at small T
CASES = {
    "tiny": (W.WORKLOADS["tiny"], 16),
    "row-ragged": (W.custom(H=512, I=384, E=8, k=2), 300),
    "row-skew-e64": (W.custom(H=256, I=256, E=64, k=8, zipf_s=1.2), 100),
    "block128-ragged": (W.custom(H=512, I=384, E=8, k=2, score=W.SCORE_SIGMOID, fmt=W.FMT_FP8_BLOCK128), 300),
    "t1": (W.custom(H=256, I=128, E=8, k=2), 1),
    "row-split-t3": (W.custom(H=512, I=2048, E=8, k=2), 3),
    # K = 2048: the down GEMM stores full 32-row groups as TMA boxes, here with a
    # 4-way K split (rows per expert 52, 44, 48, 48: one full group and a ragged one)
    "row-split-boxes-t96": (W.custom(H=512, I=2048, E=4, k=2), 96),
    # T k >= 512 E: the gate/up GEMM runs on CTA pairs (odd row-tile counts included)
    "row-pairs-t2100": (W.custom(H=512, I=256, E=8, k=2), 2100),
    # K = I = 2304 > 2048 as well: the down GEMM also runs on CTA pairs
    "row-pairs-deepk-t2100": (W.custom(H=512, I=2304, E=8, k=2), 2100),
    # above 4 x 148 tokens the quantisation runs one warp per token
    "row-t700": (W.custom(H=256, I=128, E=8, k=2), 700),
    "block128-t700": (W.custom(H=256, I=128, E=8, k=2, score=W.SCORE_SIGMOID, fmt=W.FMT_FP8_BLOCK128), 700),
    "nvfp4-ragged": (W.custom(H=512, I=512, E=8, k=2, fmt=W.FMT_NVFP4), 300),
    "nvfp4-skew-e32": (W.custom(H=256, I=256, E=32, k=4, fmt=W.FMT_NVFP4, zipf_s=1.0), 50),
    # above 128 tokens with more than 8 experts the router runs on the tensor cores
    "row-skew-e64-t300": (W.custom(H=512, I=256, E=64, k=8, zipf_s=1.2), 300),
    "block128-e48-t260": (W.custom(H=512, I=256, E=48, k=6, score=W.SCORE_SIGMOID, fmt=W.FMT_FP8_BLOCK128), 260),
    # H = 1024: two 512-column slices of the combine per token group
    "row-h1024": (W.custom(H=1024, I=256, E=8, k=2), 300),
}


def nvfp4(wl):
    return wl.fmt == W.FMT_NVFP4


def gpu_slot_rows(layer, wl, ids, T):
    """Row of each assignment slot in the GPU's X/hidden buffers (padded for NVFP4)."""
    A = T * wl.k
    if not nvfp4(wl):
        return np.arange(A)
    counts, offsets, perm, inv = oracle.dispatch(ids, wl.E)
    tile_ptr = layer.region("tile_ptr", torch.int32, wl.E + 1).cpu().numpy()
    return padded_rows(np.arange(A), ids.reshape(-1), perm, offsets, tile_ptr)


def slot_rows(layer, wl, ids, T, padded):
    A = T * wl.k
    if not padded:
        return np.arange(A)
    counts, offsets, perm, inv = oracle.dispatch(ids, wl.E)
    tile_ptr = layer.region("tile_ptr", torch.int32, wl.E + 1).cpu().numpy()
    return padded_rows(np.arange(A), ids.reshape(-1), perm, offsets, tile_ptr)


def gpu_rows(layer, wl, name, nbytes_per_row, padded=None):
    padded = nvfp4(wl) if padded is None else padded
    v = layer.view[name] - layer.ws.data_ptr()
    n = layer.max_T * wl.k + (128 * wl.E if padded else 0)
    return layer.ws[v:v + n * nbytes_per_row].cpu().numpy().reshape(n, nbytes_per_row)


def gpu_hidden(layer, wl, ids, T):
    """(codes, row-major scales) of the GPU's hidden in slot order, any format."""
    A = T * wl.k
    if not hidden_padded(wl):
        hq = layer.region("hq", torch.uint8, A * wl.I).cpu().numpy().reshape(A, wl.I)
        hs = layer.region("hs", torch.float32, A * wl.I // 128).cpu().numpy().reshape(A, -1)
        return hq, hs
    rows = slot_rows(layer, wl, ids, T, True)
    hq = gpu_rows(layer, wl, "hq", hidden_code_bytes(wl), True)[rows]
    hs = gather_sf(gpu_rows(layer, wl, "hs", hidden_sf_cols(wl), True).reshape(-1), rows, hidden_sf_cols(wl))
    return hq, hs


def inject_hidden(layer, wl, ids, T, hq, hs):
    """Write oracle hidden codes/scales (slot order) into the GPU's hidden buffers."""
    A = T * wl.k
    if not hidden_padded(wl):
        layer.region("hq", torch.uint8, A * wl.I).copy_(torch.from_numpy(hq.reshape(-1)).cuda())
        layer.region("hs", torch.float32, A * wl.I // 128).copy_(torch.from_numpy(hs.reshape(-1)).cuda())
        return
    rows = slot_rows(layer, wl, ids, T, True)
    n_rows = layer.max_T * wl.k + 128 * wl.E
    hq_all = np.zeros((n_rows, hidden_code_bytes(wl)), np.uint8)
    hq_all[rows] = hq
    sf_all = np.zeros(n_rows * hidden_sf_cols(wl), np.uint8)
    scatter_sf(sf_all, rows, hs, hidden_sf_cols(wl))
    layer.region("hq", torch.uint8, hq_all.size).copy_(torch.from_numpy(hq_all.reshape(-1)).cuda())
    layer.region("hs", torch.uint8, sf_all.size).copy_(torch.from_numpy(sf_all).cuda())


def expected_split(wl, max_T, counts, sms):
    """The down GEMM's K split the oracle's rule gives for this workspace."""
    if wl.fmt != W.FMT_FP8_ROW:
        return 1
    A_max = max_T * wl.k
    return oracle.pick_split(counts, wl.H // 256, wl.I // 128, A_max + 7 * min(A_max, 256), sms)


def build_case(name, seed=0):
    wl, T = CASES[name]
    d = synth.layer(wl, seed=seed)
    x = synth.tokens(wl, T, seed=seed)
    return wl, T, d, x


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    native.load()


def run_route(layer, x, d):
    T = x.shape[0]
    wl = layer.wl
    ids = torch.empty(T, wl.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.k, dtype=torch.float32, device="cuda")
    bias = d["bias"].cuda() if d["bias"] is not None else None
    native.moe_route(layer.h, x.cuda(), T, d["wr"].cuda(), bias, ids, w, layer.ws)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_router_ids_bit_exact(name):
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    ids, w = run_route(layer, x, d)
    lg = oracle.router_logits(bits(x), d["wr"].numpy(), None if d["bias"] is None else d["bias"].numpy())
    ids_ref, w_ref = oracle.topk(lg, wl.k, wl.score)
    assert (ids == ids_ref).all()
    np.testing.assert_allclose(w, w_ref, rtol=0, atol=2e-6)
    assert layer.status()[0] == 0


@pytest.mark.parametrize("H,E,k,score,T", [(7168, 256, 8, W.SCORE_SIGMOID, 20), (2048, 256, 8, W.SCORE_SOFTMAX, 64),
                                           (4096, 8, 2, W.SCORE_SOFTMAX, 33), (4096, 8, 2, W.SCORE_SOFTMAX, 1),
                                           (2048, 250, 8, W.SCORE_SOFTMAX, 127), (256, 32, 4, W.SCORE_SIGMOID, 5),
                                           (256, 3, 2, W.SCORE_SOFTMAX, 7),
                                           (2048, 256, 8, W.SCORE_SOFTMAX, 129), (4096, 8, 2, W.SCORE_SOFTMAX, 150),
                                           (512, 40, 4, W.SCORE_SIGMOID, 200), (6144, 256, 8, W.SCORE_SOFTMAX, 257),
                                           # enough 128-token tiles for 128-expert tensor-core tiles
                                           (256, 256, 8, W.SCORE_SOFTMAX, 4864), (512, 200, 6, W.SCORE_SIGMOID, 9600)])
def test_router_named_shapes_bit_exact(H, E, k, score, T):
    """Both logits kernels (small batches, and the tiled one above 128 tokens)
    give the oracle's fp32 logits bit for bit, and its ids."""
    wl = W.custom(H=H, I=128, E=E, k=k, score=score, router_init="uniform", zipf_s=1.0)
    wr, bias = synth.router(wl, seed=3)
    x = synth.tokens(wl, T, seed=3)
    h = native.moe_init(wl, T)
    ws = torch.empty(native.moe_workspace_size(h), dtype=torch.uint8, device="cuda")
    native.moe_workspace_init(h, ws)
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    native.moe_route(h, x.cuda(), T, wr.cuda(), bias.cuda(), ids, w, ws)
    torch.cuda.synchronize()
    lg_ref = oracle.router_logits(bits(x), wr.numpy(), bias.numpy())
    off = native.moe_workspace_view_get(h, ws)["logits"] - ws.data_ptr()
    lg = ws[off:off + T * E * 4].view(torch.float32).cpu().numpy().reshape(T, E)
    ids_ref, w_ref = oracle.topk(lg_ref, k, score)
    assert (ids.cpu().numpy() == ids_ref).all()
    np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=0, atol=2e-6)
    same = lg.view(np.uint32) == lg_ref.astype(np.float32).view(np.uint32)
    if not router_uses_filter(T, E):
        assert same.all()
    else:
        # the selected experts' logits are canonical; every other logit is
        # canonical or within the certified distance of it
        assert same[np.arange(T)[:, None], ids_ref].all()
        D = router_filter_bound(x, wr.numpy(), bias.numpy(), lg)
        assert np.all(same | (np.abs(lg.astype(np.float64) - lg_ref.astype(np.float64)) <= D))
    native.moe_destroy(h)


def router_uses_filter(T, E):
    """Batches above 128 tokens with more than 8 experts route through the
    integer tensor-core pass and the certified candidate filter."""
    return T > 128 and E > 8


def router_filter_bound(x_bf16, wr, bias, l_stored):
    """The distance the filter certifies between a stored approximate logit
    and the canonical one, restated from its definition: fixed-point rows
    rounded at half of 2^(e - 14) (e the smallest integer with max|row| <=
    2^e), the canonical chain's gamma(H/32 + 6) (sum|x w| + |b|) with
    sum|x w| <= min(sum|x| max|w|, max|x| sum|w|), and the fp32 evaluation
    of the approximation (2^-23 (|l| + |b|) + 2^-126)."""
    x = x_bf16.float().numpy().astype(np.float64)
    w = np.asarray(wr, np.float64)
    H = x.shape[1]

    def expo(a):
        m = np.abs(a).max(axis=1)
        return np.where(m > 0, np.frexp(m)[1], 0)

    ex, ew = expo(x), expo(w)
    qw = np.rint(w * np.exp2(14.0 - ew)[:, None])
    sx, mx = np.abs(x).sum(1), np.abs(x).max(1)
    sw, mw = np.abs(w).sum(1), np.abs(w).max(1)
    swq = np.abs(qw).sum(1) * np.exp2(ew - 14.0)
    n = H // 32 + 6
    gamma = n * 2.0 ** -24 / (1 - n * 2.0 ** -24)
    dfix = np.exp2(ew - 15.0)[None, :] * sx[:, None] + np.exp2(ex - 15.0)[:, None] * swq[None, :]
    sxw = np.minimum(sx[:, None] * mw[None, :], mx[:, None] * sw[None, :])
    b = np.zeros(w.shape[0]) if bias is None else np.abs(np.asarray(bias, np.float64))
    dst = (np.abs(l_stored.astype(np.float64)) + b[None, :]) * 2.0 ** -23 + 2.0 ** -126
    return (dfix + gamma * (sxw + b[None, :]) + dst) * (1 + 2.0 ** -20)


@pytest.mark.parametrize("T", [129, 300])
def test_router_filter_keeps_exact_and_near_ties(T):
    """Batches on the tensor-core router with experts whose canonical logits
    tie exactly (duplicated router rows: the lower id must come first) or
    differ in their last bits (a row with one element nudged by one ulp): the
    ids are the oracle's, bit for bit."""
    wl = W.custom(H=2048, I=128, E=64, k=8, router_init="uniform")
    wr, _ = synth.router(wl, seed=4)
    wr = wr.clone()
    x = synth.tokens(wl, T, seed=4)
    # nine experts made strong for every token (the batch's mean direction adds
    # about sqrt(H / T) to their logits), so the top 8 is cut inside them and
    # the tie groups below land on both sides of the cut
    boost = x.float().mean(0)
    for e in (3, 5, 9, 10, 11, 12, 17, 40, 41):
        wr[e] += boost / boost.norm()
    wr[5] = wr[3]                                    # exact tie with expert 3
    wr[17] = wr[9]                                   # exact tie with expert 9
    wr[10] = wr[9]
    wr[10, 100] = torch.nextafter(wr[10, 100], torch.tensor(1.0))   # a near tie
    wr[41] = wr[40]
    wr[41, 7] = torch.nextafter(wr[41, 7], torch.tensor(-1.0))
    h = native.moe_init(wl, T)
    ws = torch.empty(native.moe_workspace_size(h), dtype=torch.uint8, device="cuda")
    native.moe_workspace_init(h, ws)
    ids = torch.empty(T, 8, dtype=torch.int32, device="cuda")
    w = torch.empty(T, 8, dtype=torch.float32, device="cuda")
    native.moe_route(h, x.cuda(), T, wr.cuda(), None, ids, w, ws)
    torch.cuda.synchronize()
    lg_ref = oracle.router_logits(bits(x), wr.numpy(), None)
    ids_ref, w_ref = oracle.topk(lg_ref, 8, wl.score)
    assert ((ids_ref == 3).any(1) & (ids_ref == 5).any(1)).any(), "the exact tie reaches the top k"
    assert ((ids_ref == 9).any(1) & ~(ids_ref == 17).any(1)).any(), "an exact tie is cut by k"
    assert (ids.cpu().numpy() == ids_ref).all()
    np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=0, atol=2e-6)
    native.moe_destroy(h)


def test_router_equal_logits_tie_break():
    wl = W.custom(H=256, I=128, E=16, k=4)
    h = native.moe_init(wl, 8)
    ws = torch.empty(native.moe_workspace_size(h), dtype=torch.uint8, device="cuda")
    native.moe_workspace_init(h, ws)
    x = synth.tokens(wl, 8, seed=1).cuda()
    wr = torch.zeros(16, 256, device="cuda")
    ids = torch.empty(8, 4, dtype=torch.int32, device="cuda")
    w = torch.empty(8, 4, dtype=torch.float32, device="cuda")
    native.moe_route(h, x, 8, wr, None, ids, w, ws)
    torch.cuda.synchronize()
    assert (ids.cpu().numpy() == np.arange(4)).all()
    assert np.allclose(w.cpu().numpy(), 0.25, atol=0)
    native.moe_destroy(h)


@pytest.mark.parametrize("name", list(CASES))
def test_dispatch_bit_exact(name):
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    L = oracle.Layer(wl, d)
    ids, w, _ = L.forward(bits(x), d["wr"].numpy(), None if d["bias"] is None else d["bias"].numpy(),
                          sel=np.zeros(0, np.int32))
    ref = slot_order_reference(wl, L, x, ids, w, with_ffn=False)
    native.moe_dispatch(layer.h, x.cuda(), torch.from_numpy(ids).cuda(), T, layer.ws)
    torch.cuda.synchronize()
    A = T * wl.k
    E = wl.E
    counts, offsets, perm, inv = oracle.dispatch(ids, E)
    assert (layer.region("counts", torch.int32, E).cpu().numpy() == counts).all()
    assert (layer.region("offsets", torch.int32, E + 1).cpu().numpy() == offsets).all()
    assert (layer.region("perm", torch.int32, A).cpu().numpy() == perm).all()
    assert (layer.region("inv", torch.int32, A).cpu().numpy() == inv).all()
    te, tr = oracle.schedule(offsets)
    nt = int(layer.region("num_tiles", torch.int32, 1).cpu().numpy()[0])
    assert nt == te.size
    tiles = layer.region("tiles", torch.int32, 2 * nt).cpu().numpy().reshape(nt, 2)
    assert (tiles[:, 0] == te).all() and (tiles[:, 1] == tr).all()
    tile_ptr = layer.region("tile_ptr", torch.int32, E + 1).cpu().numpy()
    assert (tile_ptr == np.searchsorted(te, np.arange(E + 1), side="left")).all()
    a, b, bw, g, sms = native.moe_get_picker_params(layer.h)
    want, _ = oracle.pick_down_tile(counts, wl.H, wl.I, sms, a, b, bw, g)
    pick = layer.region("pick", torch.int32, 3).cpu().numpy()
    assert int(pick[0]) == want
    assert int(pick[1]) == expected_split(wl, T, counts, sms)
    model = native.moe_get_gate_up_model(layer.h)
    nb, kb, sms, allow = model[6:]
    if wl.fmt == W.FMT_FP8_ROW and wl.act != W.ACT_RELU2:
        assert (nb, kb, allow) == (2 * wl.I // 256, wl.H // 128, 7)
        assert int(pick[2]) == oracle.pick_gu_mode(counts, nb, kb, sms, list(model[:6]), allow)
    else:
        assert nb == 0 and int(pick[2]) == 0
    rows = gpu_slot_rows(layer, wl, ids, T)
    if nvfp4(wl):
        xq = gpu_rows(layer, wl, "xq", wl.H // 2)[rows]
        xs = gather_sf(gpu_rows(layer, wl, "xs", wl.H // 16).reshape(-1), rows, wl.H // 16)
        amax = layer.region("x_global", torch.int32, 1).view(torch.float32).item()
        assert amax == float(x.float().abs().max())
    else:
        xq = layer.region("xq", torch.uint8, A * wl.H).cpu().numpy().reshape(A, wl.H)
        if wl.fmt == W.FMT_FP8_ROW:
            xs = layer.region("xs", torch.float32, A).cpu().numpy()
        else:
            xs = layer.region("xs", torch.float32, A * wl.H // 128).cpu().numpy().reshape(A, -1)
    assert (xq == ref["xq"]).all()
    assert (xs == ref["xs"]).all()
    assert layer.status()[0] == 0


def _dispatch_and_reference(name):
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    L = oracle.Layer(wl, d)
    bias = None if d["bias"] is None else d["bias"].numpy()
    ids, w, _ = L.forward(bits(x), d["wr"].numpy(), bias, sel=np.zeros(0, np.int32))
    ref = slot_order_reference(wl, L, x, ids, w)
    native.moe_dispatch(layer.h, x.cuda(), torch.from_numpy(ids).cuda(), T, layer.ws)
    return wl, T, d, x, layer, ids, w, ref


@pytest.mark.parametrize("name", list(CASES))
def test_gate_up_hidden_matches_oracle(name):
    wl, T, d, x, layer, ids, w, ref = _dispatch_and_reference(name)
    native.moe_gate_up(layer.h, layer.packed, T, layer.ws)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    hq, hs = gpu_hidden(layer, wl, ids, T)
    if wl.fmt == W.FMT_FP8_BLOCK128:
        np.testing.assert_allclose(hs, ref["hs"], rtol=1e-4, atol=0)
    else:
        assert (hs != ref["hs"]).mean() <= 1e-3      # block scale codes
    v_gpu = hidden_values_of(wl, hq, hs)
    v_ref = hidden_values_of(wl, ref["hq"], ref["hs"])
    # codes (and for the block-scaled formats the scale codes) decide the values;
    # fp32 block scales (FP8_BLOCK128) differ in their last bits, so compare codes
    mism = (hq != ref["hq"]) if wl.fmt == W.FMT_FP8_BLOCK128 else (v_gpu != v_ref)
    assert mism.mean() <= 2e-3, f"{mism.mean():.2e} of the hidden codes differ"
    # a differing value is one rounding step away (a flip at a rounding boundary):
    # an e4m3 step is at most 1/8 of the value (+ the subnormal step), an e2m1
    # step at most 2 x the block scale
    if nvfp4(wl):
        step = np.repeat(fp8_values(ref["hs"]), 16, axis=1) * wl.hidden_global_scale * 2.0
        assert np.all(np.abs(v_gpu - v_ref) <= step * 1.0001)
    else:
        unit = np.abs(hidden_values_of(wl, np.full_like(ref["hq"], 0x01), ref["hs"]))   # 2^-9 x scale
        assert np.all(np.abs(v_gpu - v_ref) <= np.abs(v_ref) * 0.125 + unit * 1.0001 + 1e-30)


# the FP8_BLOCK128 down GEMM has three tile widths (0 = picked from the
# histogram), the FP8_ROW one two (128: two accumulators in TMEM), NVFP4 one
DOWN_WIDTHS = {W.FMT_FP8_BLOCK128: (0, 64, 128, 256), W.FMT_FP8_ROW: (0, 128), W.FMT_NVFP4: (0,)}
DOWN_CASES = [(n, bn) for n in CASES for bn in DOWN_WIDTHS[CASES[n][0].fmt]]


@pytest.mark.parametrize("name,down_bn", DOWN_CASES, ids=[f"{n}-bn{b}" for n, b in DOWN_CASES])
def test_down_matches_oracle_on_oracle_hidden(name, down_bn):
    wl, T, d, x, layer, ids, w, ref = _dispatch_and_reference(name)
    native.moe_set_tile_config(layer.h, down_bn)
    A = T * wl.k
    torch.cuda.synchronize()
    inject_hidden(layer, wl, ids, T, ref["hq"], ref["hs"])
    w_dev = torch.from_numpy(w.astype(np.float32)).cuda()
    native.moe_down(layer.h, layer.packed, w_dev, T, layer.ws)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    S = int(layer.region("pick", torch.int32, 2).cpu().numpy()[1])
    if name == "row-split-t3":
        assert S == 4                     # 10 units, s_max = 16 K-blocks / 4
    o = decode_o(layer, wl, S, A).sum(axis=0)
    assert tolerance_violations(o, ref["o_w"]) == 0


def decode_o(layer, wl, S, A):
    """The down GEMM's weighted rows [S, A, H]: fp16 values times 2^(e - 15),
    one exponent e per 32 columns (the layout moe_b200.h documents)."""
    q = layer.region("o", torch.float16, S * A * wl.H).float().cpu().numpy().reshape(S, A, wl.H // 32, 32)
    e = layer.region("o_exp", torch.int8, S * A * wl.H // 32).cpu().numpy().reshape(S, A, wl.H // 32, 1)
    return (q.astype(np.float64) * np.exp2(e.astype(np.float64) - 15)).reshape(S, A, wl.H)


# the gated activation variants, on each format; the limits bind on part of the
# pre-activations, and T = 300 over 8 experts exercises the row and the sparse
# gate/up epilogues
ACT_CASES = {
    "row-bounded": (W.custom(H=512, I=384, E=8, k=2, act=W.ACT_SWIGLU_BOUNDED, act_limit=0.25), 300),
    "row-oai": (W.custom(H=512, I=384, E=8, k=2, act=W.ACT_SWIGLU_OAI, act_alpha=1.702, act_limit=0.3), 300),
    "row-geglu": (W.custom(H=512, I=384, E=8, k=2, act=W.ACT_GEGLU), 300),
    "row-reglu": (W.custom(H=512, I=384, E=8, k=2, act=W.ACT_REGLU), 300),
    "block128-oai": (W.custom(H=512, I=384, E=8, k=2, score=W.SCORE_SIGMOID, fmt=W.FMT_FP8_BLOCK128,
                              act=W.ACT_SWIGLU_OAI, act_alpha=1.702, act_limit=0.3), 300),
    "block128-geglu": (W.custom(H=512, I=384, E=8, k=2, score=W.SCORE_SIGMOID, fmt=W.FMT_FP8_BLOCK128,
                                act=W.ACT_GEGLU), 300),
    "nvfp4-bounded": (W.custom(H=512, I=512, E=8, k=2, fmt=W.FMT_NVFP4, act=W.ACT_SWIGLU_BOUNDED,
                               act_limit=0.25), 300),
    "nvfp4-reglu": (W.custom(H=512, I=512, E=8, k=2, fmt=W.FMT_NVFP4, act=W.ACT_REGLU), 300),
    # ReLU^2 experts: up and down only
    "row-relu2": (W.custom(H=512, I=512, E=8, k=2, act=W.ACT_RELU2), 300),
    "row-relu2-t3": (W.custom(H=512, I=512, E=8, k=2, act=W.ACT_RELU2), 3),
    "block128-relu2": (W.custom(H=512, I=512, E=8, k=2, score=W.SCORE_SIGMOID, fmt=W.FMT_FP8_BLOCK128,
                                act=W.ACT_RELU2), 300),
    "nvfp4-relu2": (W.custom(H=512, I=512, E=8, k=2, fmt=W.FMT_NVFP4, act=W.ACT_RELU2), 300),
}


@pytest.mark.parametrize("name", list(ACT_CASES))
def test_forward_end_to_end_activation_variants(name):
    wl, T = ACT_CASES[name]
    d = synth.layer(wl, seed=0)
    x = synth.tokens(wl, T, seed=0)
    check_forward(name, wl, T, d, x)


@pytest.mark.parametrize("name", list(CASES))
def test_forward_end_to_end(name):
    """Y of every token within 2e-2 |ref| + 2e-3 rms(ref); the few elements
    outside it must lie inside it widened by the bound on what hidden codes
    that rounded the other way can move, and are counted in the report (see
    helpers.check_layer_output)."""
    wl, T, d, x = build_case(name)
    check_forward(name, wl, T, d, x)


def numpy_weights(d):
    return {k_: (None if v is None else v.numpy()) for k_, v in d.items() if k_.endswith(("_q", "_s", "_g"))}


def check_forward(case, wl, T, d, x):
    layer = native.Layer(wl, d, max_T=T)
    bias = d["bias"].cuda() if d["bias"] is not None else None
    y = layer.forward(x.cuda(), d["wr"].cuda(), bias)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    L = oracle.Layer(wl, d)
    ids, w, y_ref = L.forward(bits(x), d["wr"].numpy(), None if d["bias"] is None else d["bias"].numpy())
    assert (layer.region("ids", torch.int32, T * wl.k).cpu().numpy().reshape(T, wl.k) == ids).all()
    check_layer_output(case, wl, layer, L, x, ids, w, np.arange(T), y.float().cpu().numpy(), y_ref,
                       numpy_weights(d), lambda e: e)


# moe_forward_routed on every format, and for FP8_ROW on both down GEMM paths
# it can take with a caller's routing weights: the chained one (launched with
# programmatic dependent launch, waiting per expert for the gate/up parts) on
# single CTAs with shallow and deep K splits, and on CTA pairs
ROUTED_CASES = ["row-ragged", "row-split-boxes-t96", "row-pairs-deepk-t2100", "block128-ragged", "nvfp4-ragged",
                "nvfp4-skew-e32"]


@pytest.mark.parametrize("name", ROUTED_CASES)
def test_forward_routed(name):
    """The layer with routing given by the caller (LightMoE README, "MoE
    inference": __call__(x, top_k_ids, top_k_weights)).  Given the router's
    own ids and weights it returns moe_forward's bits; given the oracle's ids
    and (fp32) weights, its Y matches the oracle's."""
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    xc, wr = x.cuda(), d["wr"].cuda()
    bias = d["bias"].cuda() if d["bias"] is not None else None
    native.moe_set_launch_options(layer.h, 1)
    y_fwd = layer.forward(xc, wr, bias).clone()
    ids_g = layer.region("ids", torch.int32, T * wl.k).clone()
    w_g = layer.region("w", torch.float32, T * wl.k).clone()
    y_r = torch.empty_like(y_fwd)
    native.moe_forward_routed(layer.h, xc, T, ids_g, w_g, layer.packed, y_r, layer.ws)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    assert torch.equal(y_fwd, y_r)

    L = oracle.Layer(wl, d)
    ids, w, y_ref = L.forward(bits(x), d["wr"].numpy(), None if d["bias"] is None else d["bias"].numpy())
    y_r.zero_()
    native.moe_forward_routed(layer.h, xc, T, torch.from_numpy(ids).cuda(),
                              torch.from_numpy(w.astype(np.float32)).cuda(), layer.packed, y_r, layer.ws)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    check_layer_output(f"routed {name}", wl, layer, L, x, ids, w, np.arange(T), y_r.float().cpu().numpy(), y_ref,
                       numpy_weights(d), lambda e: e)


@pytest.mark.parametrize("name", ["row-ragged", "nvfp4-ragged"])
def test_forward_routed_reports_out_of_range_ids(name):
    """Caller-given expert ids outside [0, E) are skipped (no slot, no rows)
    and reported as MOE_ERR_DEVICE_BOUNDS by moe_get_status; the tokens that
    do not use them keep the output of the clean routing up to the tolerance."""
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    L = oracle.Layer(wl, d)
    ids, w, y_ref = L.forward(bits(x), d["wr"].numpy(), None if d["bias"] is None else d["bias"].numpy())
    bad = ids.copy()
    bad[5, 1] = wl.E
    bad[7, 0] = -1
    y = torch.empty(T, wl.H, dtype=torch.bfloat16, device="cuda")
    native.moe_forward_routed(layer.h, x.cuda(), T, torch.from_numpy(bad).cuda(),
                              torch.from_numpy(w.astype(np.float32)).cuda(), layer.packed, y, layer.ws)
    st, _ = layer.status()
    assert st == 6                          # MOE_ERR_DEVICE_BOUNDS
    keep = np.setdiff1d(np.arange(T), [5, 7])
    yk = y.float().cpu().numpy()[keep]
    assert np.isfinite(yk).all()
    assert tolerance_violations(yk, y_ref[keep]) <= 1e-3 * yk.size
    assert layer.status()[0] == 0           # the status word was cleared by the read


def test_forward_twice_same_bits():
    wl, T, d, x = build_case("row-ragged")
    layer = native.Layer(wl, d, max_T=T)
    y1 = layer.forward(x.cuda(), d["wr"].cuda(), None).clone()
    y2 = layer.forward(x.cuda(), d["wr"].cuda(), None)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("name", ["row-skew-e64", "row-pairs-t2100", "row-split-boxes-t96", "block128-ragged", "nvfp4-ragged"])
def test_launch_modes_same_bits(name):
    """Programmatic dependent launch on or off, direct calls or a replayed CUDA
    graph of the call: the same kernels on the same data give the same bits."""
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    xc, wr = x.cuda(), d["wr"].cuda()
    bias = d["bias"].cuda() if d["bias"] is not None else None
    native.moe_set_launch_options(layer.h, 0)
    y_plain = layer.forward(xc, wr, bias).clone()
    native.moe_set_launch_options(layer.h, 1)
    y_pdl = layer.forward(xc, wr, bias).clone()
    y = torch.empty(T, wl.H, dtype=torch.bfloat16, device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        native.moe_forward(layer.h, xc, T, wr, bias, layer.packed, y, layer.ws)
    y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    assert torch.equal(y_plain, y_pdl)
    assert torch.equal(y_plain, y)
    del g


@pytest.mark.parametrize("name", ["row-pairs-t2100", "row-pairs-deepk-t2100"])
def test_cta_pairs_match_single_ctas(name):
    """The GEMMs on CTA pairs (M = 256 MMAs over two row tiles; the gate/up GEMM,
    and with K > 2048 the down GEMM too) give the hidden codes and the layer
    output of the single-CTA kernels, up to the fp32 summation order inside
    the tensor core.  The gate/up modes are forced both through the options
    and through the cost model's parameters; either way the dispatch writes
    the mode the kernel then runs."""
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    xc, wr = x.cuda(), d["wr"].cuda()
    n_hq = (T * wl.k + 128 * wl.E) * wl.I

    def run(mode=None, params=None):
        if mode is not None:
            native.moe_set_gemm_options(layer.h, mode)
        if params is not None:
            native.moe_set_gate_up_model(layer.h, *params)
        y = layer.forward(xc, wr, None).clone()
        torch.cuda.synchronize()
        assert layer.status()[0] == 0
        return y, layer.region("hq", torch.uint8, n_hq).clone(), int(layer.region("pick", torch.int32, 3)[2])

    big = 10 ** 12
    default = native.moe_get_gate_up_model(layer.h)[:6]
    y_pair, hq_pair, pk_pair = run(2)
    y_single, hq_single, pk_single = run(0, (0, 0, big, big, big, big))
    assert (pk_pair, pk_single) == (1, 0)
    # the options back to the default; the model's parameters force each mode
    y_p1, hq_p1, pk1 = run(1, (big, big, 0, 0, big, big))
    y_p0, hq_p0, pk0 = run(None, (0, 0, big, big, big, big))
    assert (pk1, pk0) == (1, 0)
    assert torch.equal(hq_p1, hq_pair) and torch.equal(y_p1, y_pair)
    assert torch.equal(hq_p0, hq_single) and torch.equal(y_p0, y_single)
    native.moe_set_gate_up_model(layer.h, *default)
    assert (hq_pair != hq_single).float().mean().item() <= 1e-3
    assert tolerance_violations(y_pair.float().cpu().numpy(), y_single.float().cpu().numpy()) == 0
    with pytest.raises(native.MoeError):
        native.moe_set_gemm_options(layer.h, 3)
    with pytest.raises(native.MoeError):
        native.moe_set_gate_up_model(layer.h, -1, 0, 0, 0, 0, 0)
    # pairs forced on and 128-wide tiles forced on contradict each other
    native.moe_set_gemm_options(layer.h, 2)
    with pytest.raises(native.MoeError):
        native.moe_set_gate_up_tile(layer.h, 128)
    native.moe_set_gemm_options(layer.h, 1)


@pytest.mark.parametrize("name", ["row-ragged", "row-t700", "row-split-boxes-t96", "row-skew-e64"])
def test_gate_up_tile_widths_agree(name):
    """The gated FP8_ROW gate/up GEMM on 128-wide tiles (64 gate + 64 up
    columns) and on 256-wide tiles: the same hidden codes and scales up to the
    fp32 summation order inside the tensor core, and outputs within the
    tolerance of each other.  The oracle parity tests run whichever width the
    dispatch picks."""
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    xc, wr = x.cuda(), d["wr"].cuda()
    bias = None if d["bias"] is None else d["bias"].cuda()
    n_hq = (T * wl.k + 128 * wl.E) * wl.I
    n_hs = (T * wl.k + 128 * wl.E) * wl.I // 32
    out = {}
    for bn, mode in ((128, 2), (256, 0)):
        native.moe_set_gemm_options(layer.h, 0)
        native.moe_set_gate_up_tile(layer.h, bn)
        y = layer.forward(xc, wr, bias).clone()
        torch.cuda.synchronize()
        assert layer.status()[0] == 0
        assert int(layer.region("pick", torch.int32, 3)[2]) == mode
        out[bn] = (y, layer.region("hq", torch.uint8, n_hq).clone(), layer.region("hs", torch.uint8, n_hs).clone())
    (y1, hq1, hs1), (y2, hq2, hs2) = out[128], out[256]
    assert (hq1 != hq2).float().mean().item() <= 1e-3
    assert (hs1 != hs2).float().mean().item() <= 1e-3
    assert tolerance_violations(y1.float().cpu().numpy(), y2.float().cpu().numpy()) == 0
    native.moe_set_gate_up_tile(layer.h, 0)
    with pytest.raises(native.MoeError):
        native.moe_set_gate_up_tile(layer.h, 64)


@pytest.mark.parametrize("name", ["row-ragged", "row-t700", "row-split-boxes-t96", "row-pairs-deepk-t2100"])
def test_down_tile_widths_agree(name):
    """The FP8_ROW down GEMM on 128-wide tiles (two accumulators) and on its
    default tiles, through the whole layer (chained behind the gate/up GEMM
    for T k <= 4096, with a K split at T = 96, deep K at I = 2304): the same
    fp16 rows up to the fp32 summation order inside the tensor core."""
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    xc, wr = x.cuda(), d["wr"].cuda()
    ys = {}
    for bn in (128, 0):
        native.moe_set_tile_config(layer.h, bn)
        ys[bn] = layer.forward(xc, wr, None).clone()
        torch.cuda.synchronize()
        assert layer.status()[0] == 0
    assert tolerance_violations(ys[128].float().cpu().numpy(), ys[0].float().cpu().numpy()) == 0
    assert (ys[128] != ys[0]).float().mean().item() <= 1e-3


def test_gate_up_tile_width_needs_a_gated_fp8_row_layer():
    wl, T, d, x = build_case("block128-ragged")
    layer = native.Layer(wl, d, max_T=T)
    with pytest.raises(native.MoeError):
        native.moe_set_gate_up_tile(layer.h, 128)
    native.moe_set_gate_up_tile(layer.h, 256)


def bf16_bits_rne(a):
    """float32 -> bfloat16 bits, round to nearest even (finite values)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


@pytest.mark.parametrize("name", ["row-h1024", "row-ragged", "row-split-boxes-t96", "block128-ragged", "nvfp4-ragged"])
def test_combine_adds_rows_in_fixed_order(name):
    """Y is, bit for bit, bf16 of the fp32 sum of each token's k weighted rows
    (and their K-split copies) in (j, s) order, from the fp16 rows and block
    exponents the down GEMM wrote."""
    wl, T, d, x = build_case(name)
    layer = native.Layer(wl, d, max_T=T)
    bias = None if d["bias"] is None else d["bias"].cuda()
    y = layer.forward(x.cuda(), d["wr"].cuda(), bias)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    A = T * wl.k
    S = int(layer.region("pick", torch.int32, 3).cpu().numpy()[1]) if wl.fmt == W.FMT_FP8_ROW else 1
    rows = decode_o(layer, wl, S, A).astype(np.float32)          # exact: fp16 x a power of two
    inv = layer.region("inv", torch.int32, A).cpu().numpy().reshape(T, wl.k)
    acc = np.zeros((T, wl.H), np.float32)
    for j in range(wl.k):
        for sp in range(S):
            ok = inv[:, j] >= 0
            acc[ok] = acc[ok] + rows[sp, inv[ok, j]]
    want = bf16_bits_rne(acc).reshape(T, wl.H)
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    assert (got == want).all(), f"{(got != want).sum()} of {got.size} differ"


def test_empty_batch():
    wl, T, d, x = build_case("tiny")
    layer = native.Layer(wl, d, max_T=T)
    y = torch.empty(0, wl.H, dtype=torch.bfloat16, device="cuda")
    native.moe_forward(layer.h, x[:0].cuda(), 0, d["wr"].cuda(), None, layer.packed, y, layer.ws)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0


@pytest.mark.parametrize("fmt", [W.FMT_FP8_ROW, W.FMT_FP8_BLOCK128, W.FMT_NVFP4])
def test_workspace_regions_hold_the_documented_layouts(fmt):
    """The workspace regions of xq/xs/hq/hs are at least as large as the row
    layouts moe_b200.h documents (slot order with 128 spare rows, or rows
    padded to 128 per expert; the scale bytes per row of each format).  The
    hidden is read through those layouts, and compared with the oracle's, by
    test_gate_up_hidden_matches_oracle."""
    wl = W.custom(H=512, I=384 if fmt != W.FMT_NVFP4 else 512, E=8, k=2, fmt=fmt,
                  score=W.SCORE_SIGMOID if fmt == W.FMT_FP8_BLOCK128 else W.SCORE_SOFTMAX)
    max_T = 300
    h = native.moe_init(wl, max_T)
    size = native.moe_workspace_size(h)
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    v = native.moe_workspace_view_get(h, ws)
    A, H, I, E = max_T * wl.k, wl.H, wl.I, wl.E
    slot_rows, padded_rows_ = A + 128, A + 128 * E
    if fmt == W.FMT_FP8_ROW:
        xq, xs = slot_rows * H, slot_rows * 4
        hq, hs = padded_rows_ * I, padded_rows_ * (I // 32)
    elif fmt == W.FMT_FP8_BLOCK128:
        xq, xs = slot_rows * H, slot_rows * (H // 128) * 4
        hq, hs = slot_rows * I, slot_rows * (I // 128) * 4
    else:
        xq, xs = padded_rows_ * H // 2, padded_rows_ * (H // 16)
        hq, hs = padded_rows_ * I // 2, padded_rows_ * (I // 16)
    assert v["xs"] - v["xq"] >= xq
    assert v["hq"] - v["xs"] >= xs
    assert v["hs"] - v["hq"] >= hq
    assert v["o"] - v["hs"] >= hs
    assert v["o_exp"] - v["o"] >= A * H * 2                 # fp16 rows
    assert ws.data_ptr() + size - v["o_exp"] >= A * H // 32  # one exponent byte per 32 columns
    native.moe_destroy(h)
