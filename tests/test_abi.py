"""The C ABI library: it builds for sm_100a here, loads, and exports every entry
point include/moe_b200.h declares.  No compute call is made (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|moe_status)\s+(moe_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from mixture_experts_topk_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for must in ("moe_init", "moe_route", "moe_dispatch", "moe_forward", "moe_destroy"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol(lib):
    from mixture_experts_topk_b200 import native
    assert set(declared_entry_points()) <= set(native.EXPORTED)


def test_init_rejects_bad_shapes_without_a_gpu(lib):
    from mixture_experts_topk_b200 import native, workloads as W
    native.load()
    bad = [W.custom(H=200, I=128, E=8, k=2), W.custom(H=256, I=100, E=8, k=2),
           W.custom(H=256, I=128, E=300, k=2), W.custom(H=256, I=128, E=8, k=9)]
    for wl in bad:
        with pytest.raises(native.MoeError) as ei:
            native.moe_init(wl, 16)
        assert ei.value.status == 2
    with pytest.raises(native.MoeError) as ei:
        native.moe_init(W.custom(H=256, I=128, E=8, k=8), 131072 // 8 + 1)
    assert ei.value.status == 2


def test_init_rejects_bad_activation_settings_without_a_gpu(lib):
    from mixture_experts_topk_b200 import native, workloads as W
    native.load()
    bad = [W.custom(H=256, I=128, E=8, k=2, act=7),
           W.custom(H=256, I=128, E=8, k=2, act=W.ACT_SWIGLU_BOUNDED, act_limit=0.0),
           W.custom(H=256, I=128, E=8, k=2, act=W.ACT_SWIGLU_OAI, act_alpha=0.0, act_limit=7.0),
           W.custom(H=256, I=128, E=8, k=2, act=W.ACT_SWIGLU_OAI, act_alpha=1.702, act_limit=-1.0)]
    for wl in bad:
        with pytest.raises(native.MoeError) as ei:
            native.moe_init(wl, 16)
        assert ei.value.status == 1
    # ReLU^2 experts tile the up projection alone, 256 rows at a time
    with pytest.raises(native.MoeError) as ei:
        native.moe_init(W.custom(H=256, I=384, E=8, k=2, act=W.ACT_RELU2), 16)
    assert ei.value.status == 2


def test_graft_build_compiles_everything():
    import __graft_entry__
    __graft_entry__.build()
    assert os.path.exists(os.path.join(ROOT, "mixture_experts_topk_b200", "libmoe_b200.so"))
    assert os.path.exists(os.path.join(ROOT, "oracle", "libmoe_oracle.so"))
