"""Parity at the workloads' own sizes, in the launch configuration bench.py times.

Every (workload, T) point of the benchmark: the tiny layer, the Mixtral-8x7B
sweep T in {1, 32, 128, 512, 4096}, Qwen3.5-35B-A3B T in {64, 8192},
DeepSeek-V3 T in {16, 4096} and GLM-5.2 T = 8192.

For every token: router ids bit-exact and weights within 2e-6, dispatch
(counts, offsets, perm, inv) bit-exact.  Y is compared for every token when
T <= 128, else for the tokens owning the first and the last slot of every
128-row tile of every expert (helpers.sample_tokens) plus seeded random ones,
within 2e-2 |ref| + 2e-3 rms(ref) per element (rms over the compared rows).
Elements outside it must stay inside it widened by the exact bound on what
hidden codes that rounded the other way can move them, and may be at most
1e-3 of the elements; each case reports how many there were
(helpers.check_layer_output).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_topk_b200 import native, synth, workloads as W
from helpers import bits, check_layer_output, sample_tokens

pytestmark = pytest.mark.gpu

CASES = [("tiny", 16), ("mixtral-8x7b", 1), ("mixtral-8x7b", 32), ("mixtral-8x7b", 128), ("mixtral-8x7b", 512),
         ("mixtral-8x7b", 4096), ("qwen3.5-35b-a3b", 64), ("qwen3.5-35b-a3b", 8192), ("deepseek-v3", 16),
         ("deepseek-v3", 4096), ("glm-5.2", 8192)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    native.load()


@pytest.mark.parametrize("name,T", CASES, ids=[f"{n}-T{t}" for n, t in CASES])
def test_full_size_layer(name, T):
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
    assert (layer.region("counts", torch.int32, wl.E).cpu().numpy() == counts).all()
    assert (layer.region("offsets", torch.int32, wl.E + 1).cpu().numpy() == offsets).all()
    assert (layer.region("perm", torch.int32, A).cpu().numpy() == perm).all()
    assert (layer.region("inv", torch.int32, A).cpu().numpy() == inv).all()

    sel = sample_tokens(T, wl.k, offsets, perm, seed=T)
    used = sorted(set(ids[sel].reshape(-1).tolist()))
    slot = np.full(wl.E, -1, np.int32)
    slot[used] = np.arange(len(used))
    sub = {k_: d[k_][used].cpu().numpy() for k_ in d if k_.endswith(("_q", "_s", "_g")) and d[k_] is not None}
    L = oracle.Layer(wl, sub, expert_slot=slot)
    _, _, y_ref = L.forward(xb, wr, bias, sel=sel)
    y_gpu = y[torch.from_numpy(sel).long().cuda()].float().cpu().numpy()
    check_layer_output(f"{name} T={T}", wl, layer, L, x, ids, w, sel, y_gpu, y_ref, sub, lambda e: int(slot[e]))
    layer.close()
