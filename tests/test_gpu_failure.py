"""Failure detection on the GPU without a fault.

The GEMM kernels' waits on another role or CTA are given 64 SM cycles, far
less than one copy takes, so they run out.  Each kernel then records
MOE_ERR_DEVICE_TIMEOUT and the role in the workspace status word, waits for its
own copies and MMAs in flight (a fixed limit), frees its TMEM and returns.  The
host reads the status; the same context then runs the layer again with the
default limit and gets the same bits as before the failure.
"""
import pytest
import torch

from mixture_experts_topk_b200 import native, synth, workloads as W

pytestmark = pytest.mark.gpu

MOE_ERR_DEVICE_TIMEOUT = 5

CASES = {
    "fp8-row": W.custom(H=512, I=256, E=8, k=2),
    # K = I > 2048: the down GEMM's deep-K variant (4 stages, rows stored from registers)
    "fp8-row-deep-k": W.custom(H=512, I=2304, E=8, k=2),
    # both GEMMs on CTA pairs (the down GEMM's pairs wait on each other's copies too)
    "fp8-row-deep-k-pairs": W.custom(H=512, I=2304, E=8, k=2),
    # the gate/up GEMM on CTA pairs (waits on the other CTA's copies)
    "fp8-row-pairs": W.custom(H=512, I=256, E=8, k=2),
    # the gate/up GEMM on 128-wide tiles (8 of 16 epilogue warps working)
    "fp8-row-narrow": W.custom(H=512, I=256, E=8, k=2),
    "fp8-block128": W.custom(H=512, I=256, E=8, k=2, score=W.SCORE_SIGMOID, fmt=W.FMT_FP8_BLOCK128),
    "nvfp4": W.custom(H=512, I=256, E=8, k=2, fmt=W.FMT_NVFP4),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    native.load()


@pytest.mark.parametrize("name", list(CASES))
def test_wait_timeout_is_reported_and_the_context_stays_usable(name):
    wl = CASES[name]
    T = 2100 if name.endswith("pairs") else 200
    d = synth.layer(wl, seed=5)
    layer = native.Layer(wl, d, max_T=T)
    if name.endswith("pairs"):
        # the cost model's parameters chosen so that the gate/up kernel runs as pairs
        native.moe_set_gate_up_model(layer.h, 10 ** 12, 10 ** 12, 0, 0, 10 ** 12, 10 ** 12)
    if name.endswith("narrow"):
        native.moe_set_gate_up_tile(layer.h, 128)
    x, wr = synth.tokens(wl, T, seed=5).cuda(), d["wr"].cuda()
    y_ref = layer.forward(x, wr, None).clone()
    if name.endswith("pairs"):
        assert int(layer.region("pick", torch.int32, 3)[2]) == 1
    if name.endswith("narrow"):
        assert int(layer.region("pick", torch.int32, 3)[2]) == 2
    torch.cuda.synchronize()
    assert layer.status()[0] == 0

    with pytest.raises(native.MoeError):
        native.moe_set_wait_limit(layer.h, 0)
    native.moe_set_wait_limit(layer.h, 64)
    layer.forward(x, wr, None)
    torch.cuda.synchronize()
    st, msg = layer.status()
    assert st == MOE_ERR_DEVICE_TIMEOUT and "GEMM" in msg, (st, msg)
    assert layer.status()[0] == 0          # reading the status cleared it

    native.moe_set_wait_limit(layer.h, 2_000_000_000)
    y = layer.forward(x, wr, None)
    torch.cuda.synchronize()
    assert layer.status()[0] == 0
    assert torch.equal(y, y_ref)
    layer.close()
