"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device
memory (their host framework owns every allocation and hands the layer only
its input and output buffers).  Its scratch is an array inside the library.

Checked through the C ABI against moe_dispatch (the workspace entry point) on
two calls in a row with different batches, bit for bit (integers, codes and
scales are exact in both), so the second call shows that what the first call
left in the shared array does not leak into its result.  This file is named
to be collected last.
"""
import numpy as np
import pytest
import torch

from mixture_experts_topk_b200 import native, synth, workloads as W

pytestmark = pytest.mark.gpu


def _noalloc_outputs(wl, T):
    A = T * wl.k
    dev = "cuda"
    scale_cols = 1 if wl.fmt == W.FMT_FP8_ROW else wl.H // 128
    return dict(counts=torch.empty(wl.E, dtype=torch.int32, device=dev),
                offsets=torch.empty(wl.E + 1, dtype=torch.int32, device=dev),
                num_tiles=torch.empty(1, dtype=torch.int32, device=dev),
                tiles=torch.empty((A // 128 + wl.E + 1) * 2, dtype=torch.int32, device=dev),
                perm=torch.empty(A, dtype=torch.int32, device=dev),
                inv=torch.empty(A, dtype=torch.int32, device=dev),
                xq=torch.empty(A * wl.H, dtype=torch.uint8, device=dev),
                xs=torch.empty(A * scale_cols, dtype=torch.float32, device=dev),
                status=torch.full((2,), 7, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("fmt", [W.FMT_FP8_ROW, W.FMT_FP8_BLOCK128])
def test_noalloc_dispatch_matches_workspace_dispatch_twice(fmt):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wl = W.custom(H=512, I=128, E=64, k=8, fmt=fmt, zipf_s=1.2)
    max_T = 300
    h = native.moe_init(wl, max_T)
    ws = torch.empty(native.moe_workspace_size(h), dtype=torch.uint8, device="cuda")
    native.moe_workspace_init(h, ws)
    view = native.moe_workspace_view_get(h, ws)

    def region(name, dtype, count):
        off = view[name] - ws.data_ptr()
        n = count * torch.empty(0, dtype=dtype).element_size()
        return ws[off:off + n].view(dtype)

    for call, (T, seed) in enumerate([(300, 11), (170, 12)]):
        d_router = synth.router(wl, seed=seed)
        x = synth.tokens(wl, T, seed=seed).cuda()
        ids = torch.empty(T, wl.k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, wl.k, dtype=torch.float32, device="cuda")
        native.moe_route(h, x, T, d_router[0].cuda(), d_router[1].cuda(), ids, w, ws)
        native.moe_dispatch(h, x, ids, T, ws)
        out = _noalloc_outputs(wl, T)
        native.moe_dispatch_noalloc(h, x, ids, T, out["counts"], out["offsets"], out["num_tiles"], out["tiles"],
                                    out["perm"], out["inv"], out["xq"], out["xs"], out["status"])
        torch.cuda.synchronize()
        A = T * wl.k
        assert out["status"].cpu().tolist() == [0, 0]
        assert torch.equal(out["counts"], region("counts", torch.int32, wl.E))
        assert torch.equal(out["offsets"], region("offsets", torch.int32, wl.E + 1))
        nt = int(region("num_tiles", torch.int32, 1).item())
        assert int(out["num_tiles"].item()) == nt
        assert torch.equal(out["tiles"][:2 * nt], region("tiles", torch.int32, 2 * nt))
        assert torch.equal(out["perm"], region("perm", torch.int32, A))
        assert torch.equal(out["inv"], region("inv", torch.int32, A))
        assert torch.equal(out["xq"], region("xq", torch.uint8, A * wl.H))
        assert torch.equal(out["xs"], region("xs", torch.float32, out["xs"].numel()))
        assert int(out["counts"].sum().item()) == A, f"call {call}"
    native.moe_destroy(h)


@pytest.mark.parametrize("E,k,T,seed", [(64, 8, 40, 21),     # one chunk: moe_dispatch's single-CTA kernel
                                        (8, 2, 500, 22),     # few experts, one chunk, one CTA per token
                                        (8, 2, 700, 24),     # few experts, two chunks, chunked quantisation
                                        (64, 8, 0, 23)])     # empty batch
def test_noalloc_dispatch_matches_workspace_dispatch_other_paths(E, k, T, seed):
    """moe_dispatch takes other kernels for a single chunk of assignments and
    for batches of at most 4 tokens per SM; the results must still agree bit
    for bit with this entry point, which always runs the chunked kernels."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    wl = W.custom(H=256, I=128, E=E, k=k)
    h = native.moe_init(wl, max(T, 1))
    ws = torch.empty(native.moe_workspace_size(h), dtype=torch.uint8, device="cuda")
    native.moe_workspace_init(h, ws)
    view = native.moe_workspace_view_get(h, ws)

    def region(name, dtype, count):
        off = view[name] - ws.data_ptr()
        n = count * torch.empty(0, dtype=dtype).element_size()
        return ws[off:off + n].view(dtype)

    d_router = synth.router(wl, seed=seed)
    x = synth.tokens(wl, T, seed=seed).cuda()
    ids = torch.empty(T, wl.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.k, dtype=torch.float32, device="cuda")
    if T > 0:
        native.moe_route(h, x, T, d_router[0].cuda(), None, ids, w, ws)
    native.moe_dispatch(h, x, ids, T, ws)
    out = _noalloc_outputs(wl, T)
    native.moe_dispatch_noalloc(h, x, ids, T, out["counts"], out["offsets"], out["num_tiles"], out["tiles"],
                                out["perm"], out["inv"], out["xq"], out["xs"], out["status"])
    torch.cuda.synchronize()
    A = T * wl.k
    assert out["status"].cpu().tolist() == [0, 0]
    assert torch.equal(out["counts"], region("counts", torch.int32, wl.E))
    assert torch.equal(out["offsets"], region("offsets", torch.int32, wl.E + 1))
    nt = int(region("num_tiles", torch.int32, 1).item())
    assert int(out["num_tiles"].item()) == nt
    assert torch.equal(out["tiles"][:2 * nt], region("tiles", torch.int32, 2 * nt))
    assert torch.equal(out["perm"], region("perm", torch.int32, A))
    assert torch.equal(out["inv"], region("inv", torch.int32, A))
    assert torch.equal(out["xq"], region("xq", torch.uint8, A * wl.H))
    assert torch.equal(out["xs"], region("xs", torch.float32, out["xs"].numel()))
    assert int(out["counts"].sum().item()) == A
    native.moe_destroy(h)


@pytest.mark.parametrize("E,k", [(256, 8), (8, 2)])
def test_noalloc_rejects_more_assignments_than_its_scratch(E, k):
    """More than 131072 assignments are refused before anything is launched,
    also with few experts, where the per-chunk counts alone would still fit."""
    native.load()
    wl = W.custom(H=256, I=128, E=E, k=k)
    h = native.moe_init(wl, 16)
    too_many = 131072 // k + 1
    with pytest.raises(native.MoeError) as ei:
        native.moe_dispatch_noalloc(h, None, None, too_many, *[None] * 9)
    assert ei.value.status == 2
    with pytest.raises(native.MoeError) as ei:
        native.moe_dispatch_noalloc(h, None, None, 70000, *[None] * 9)
    assert ei.value.status == 2
    native.moe_destroy(h)
