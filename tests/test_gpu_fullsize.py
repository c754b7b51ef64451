"""Parity at the workloads' own sizes, in the launch configuration bench.py times.

For every token: router ids bit-exact and weights within 2e-6, dispatch
(counts, offsets, perm, inv) bit-exact.  For a seeded sample of tokens: Y
against the oracle within 2e-2 |ref| + 2e-3 rms(ref), widened only by the
bound on what hidden codes that rounded the other way can move (see
helpers.deviation_bound_rows); rms is taken over the sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_topk_b200 import native, synth, workloads as W
from helpers import (bits, deviation_bound_rows, gather_sf, hidden_code_bytes, hidden_padded, hidden_sf_cols,
                     hidden_values_of, padded_rows, tolerance_violations_with_bound)

pytestmark = pytest.mark.gpu

CASES = [("mixtral-8x7b", 1, None), ("mixtral-8x7b", 32, None), ("mixtral-8x7b", 4096, 6),
         ("qwen3.5-35b-a3b", 64, 16), ("qwen3.5-35b-a3b", 8192, 8),
         ("deepseek-v3", 16, 6), ("deepseek-v3", 4096, 4), ("glm-5.2", 8192, 4)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    native.load()


@pytest.mark.parametrize("name,T,n_sample", CASES, ids=[f"{n}-T{t}" for n, t, _ in CASES])
def test_full_size_layer(name, T, n_sample):
    wl = W.WORKLOADS[name]
    seed = 1
    d = synth.layer(wl, seed=seed, device="cuda")
    x = synth.tokens(wl, T, seed=seed, device="cuda")
    layer = native.Layer(wl, d, max_T=T)
    y = layer.forward(x, d["wr"], d["bias"])
    torch.cuda.synchronize()
    st, msg = layer.status()
    assert st == 0, msg
    A = T * wl.k

    xb = bits(x.cpu())
    wr = d["wr"].cpu().numpy()
    bias = None if d["bias"] is None else d["bias"].cpu().numpy()
    ids, w = oracle.topk(oracle.router_logits(xb, wr, bias), wl.k, wl.score)
    ids_gpu = layer.region("ids", torch.int32, A).cpu().numpy().reshape(T, wl.k)
    assert (ids_gpu == ids).all()
    w_gpu = layer.region("w", torch.float32, A).cpu().numpy().reshape(T, wl.k)
    np.testing.assert_allclose(w_gpu, w, rtol=0, atol=2e-6)
    counts, offsets, perm, inv = oracle.dispatch(ids, wl.E)
    assert (layer.region("offsets", torch.int32, wl.E + 1).cpu().numpy() == offsets).all()
    assert (layer.region("perm", torch.int32, A).cpu().numpy() == perm).all()
    inv_gpu = layer.region("inv", torch.int32, A).cpu().numpy()
    assert (inv_gpu == inv).all()

    rng = np.random.default_rng(T)
    sel = np.arange(T) if n_sample is None else np.unique(np.concatenate(
        [[0, T - 1], rng.choice(T, size=n_sample - 2, replace=False)])).astype(np.int32)
    used = sorted(set(ids[sel].reshape(-1).tolist()))
    slot = np.full(wl.E, -1, np.int32)
    slot[used] = np.arange(len(used))
    sub = {k_: d[k_][used].cpu().numpy() for k_ in d if k_.endswith(("_q", "_s", "_g"))}
    L = oracle.Layer(wl, sub, expert_slot=slot)
    _, _, y_ref = L.forward(xb, wr, bias, sel=sel)

    # the hidden of every sampled (token, slot): oracle vs GPU, for the bound
    fp4 = wl.fmt == W.FMT_NVFP4
    x_sel = x[torch.from_numpy(sel).long().to(x.device)].float().cpu().numpy()
    g_x = oracle.nvfp4_global(x.float().cpu().numpy()) if fp4 else 0.0
    xq_tok, xs_tok = oracle.quant_rows(wl.fmt, x_sel, g_x)
    padded = hidden_padded(wl)
    if padded:
        tile_ptr = layer.region("tile_ptr", torch.int32, wl.E + 1).cpu().numpy()
        n_rows = A + 128 * wl.E
        off = layer.view["hq"] - layer.ws.data_ptr()
        hq_all = layer.ws[off:off + n_rows * hidden_code_bytes(wl)].view(n_rows, hidden_code_bytes(wl))
        off = layer.view["hs"] - layer.ws.data_ptr()
        hsf_all = layer.ws[off:off + n_rows * hidden_sf_cols(wl)].cpu().numpy()
    else:
        hq_gpu = layer.region("hq", torch.uint8, A * wl.I).view(A, wl.I)
        hs_gpu = layer.region("hs", torch.float32, A * wl.I // 128).view(A, wl.I // 128)
    rows = []
    for i, t in enumerate(sel):
        for j in range(wl.k):
            e = int(ids[t, j])
            _, hq_r, hs_r, _ = L.expert_rows(e, xq_tok[i:i + 1], xs_tok[i:i + 1], g_x)
            r = int(inv[t * wl.k + j])
            if padded:
                prow = int(padded_rows([r], ids.reshape(-1), perm, offsets, tile_ptr)[0])
                v_gpu = hidden_values_of(wl, hq_all[prow].cpu().numpy()[None],
                                         gather_sf(hsf_all, [prow], hidden_sf_cols(wl)))[0]
            else:
                v_gpu = hidden_values_of(wl, hq_gpu[r].cpu().numpy()[None], hs_gpu[r].cpu().numpy()[None])[0]
            v_ref = hidden_values_of(wl, hq_r, hs_r)[0]
            rows.append((i, e, w[t, j], v_gpu, v_ref))
    extra = deviation_bound_rows(wl, sub, lambda e: int(slot[e]), rows, len(sel))
    y_gpu = y[torch.from_numpy(sel).long().cuda()].float().cpu().numpy()
    bad, plain = tolerance_violations_with_bound(y_gpu, y_ref, extra)
    assert bad == 0
    assert plain <= max(2, 1e-3 * y_ref.size), f"{plain} elements outside the plain tolerance"
    layer.close()
