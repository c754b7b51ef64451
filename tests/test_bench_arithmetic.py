"""The benchmark's algorithmic work (the numerators of every roofline
fraction it reports), checked against figures worked out by hand."""
import dataclasses
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from mixture_experts_topk_b200 import workloads as W  # noqa: E402


@pytest.fixture(scope="module")
def bench():
    import bench as b
    return b


def test_fp8_row_work_by_hand(bench):
    # H 256, I 128, E 4, k 2, T 3; experts 0, 2, 3 touched.
    # FLOPs: 2 A (gate + up + down) H I = 2 * 6 * 3 * 256 * 128 = 1,179,648;
    # router 2 T E H = 6,144.  Bytes per touched expert: 3 H I codes = 98,304
    # plus fp32 row scales for 2I gate/up rows and H down rows = 4 * 512;
    # plus Wr (4 * 256 * 4 = 4,096) and X in / Y out in bf16 (2 * 3 * 256 * 2).
    wl = W.custom(H=256, I=128, E=4, k=2)
    fl_t, fl_r, byts, touched = bench.algorithmic_work(wl, 3, np.array([2, 0, 3, 1]))
    assert (fl_t, fl_r, touched) == (1_179_648, 6_144, 3)
    assert byts == 3 * (98_304 + 2_048) + 4_096 + 3_072


def test_fp8_block128_work_by_hand(bench):
    # H 256, I 256: codes 3 * 65,536; one fp32 scale per 128 x 128 block of each
    # of the three matrices (2 x 2 blocks each) = 4 * 12 = 48 bytes
    wl = W.custom(H=256, I=256, E=2, k=1, fmt=W.FMT_FP8_BLOCK128, score=W.SCORE_SIGMOID)
    fl_t, fl_r, byts, touched = bench.algorithmic_work(wl, 5, np.array([5, 0]))
    assert touched == 1
    assert fl_t == 2 * 5 * 3 * 256 * 256 and fl_r == 2 * 5 * 2 * 256
    assert byts == (196_608 + 48) + 2 * 256 * 4 + 2 * 5 * 256 * 2


def test_nvfp4_work_by_hand(bench):
    # half a byte per weight plus one e4m3 scale per 16 weights:
    # 3 * 256 * 256 * (1/2 + 1/16) = 110,592 bytes per touched expert
    wl = W.custom(H=256, I=256, E=8, k=2, fmt=W.FMT_NVFP4)
    fl_t, fl_r, byts, touched = bench.algorithmic_work(wl, 4, np.array([1, 1, 0, 0, 2, 0, 4, 0]))
    assert touched == 4
    assert byts == 4 * 110_592 + 8 * 256 * 4 + 2 * 4 * 256 * 2
    assert fl_t == 2 * 8 * 3 * 256 * 256


def test_relu2_experts_have_two_matrices(bench):
    # no gate: 2 A H I FLOPs per matrix for up and down only; FP8_ROW scales for
    # I up rows and H down rows
    wl = dataclasses.replace(W.custom(H=256, I=256, E=2, k=1), act=bench.ACTS["relu2"][0])
    assert bench.n_proj(wl) == 2
    fl_t, _, byts, _ = bench.algorithmic_work(wl, 2, np.array([1, 1]))
    assert fl_t == 2 * 2 * 2 * 256 * 256
    assert byts == 2 * (2 * 65_536 + 4 * (256 + 256)) + 2 * 256 * 4 + 2 * 2 * 256 * 2


def test_traffic_record_hash_ignores_comments_and_layout(bench, tmp_path, monkeypatch):
    """The committed DRAM counters stay valid across comment or layout edits of
    the GEMM sources and are dropped when the code itself changes."""
    import shutil
    src = os.path.join(bench.ROOT, "mixture_experts_topk_b200", "csrc")
    root = tmp_path / "repo"
    (root / "mixture_experts_topk_b200" / "csrc").mkdir(parents=True)
    for f in ("gemm.cuh", "gemm_mx.cuh", "common.cuh"):
        shutil.copy(os.path.join(src, f), root / "mixture_experts_topk_b200" / "csrc" / f)
    monkeypatch.setattr(bench, "ROOT", str(root))
    h0 = bench.kernel_sources_hash()
    g = root / "mixture_experts_topk_b200" / "csrc" / "gemm.cuh"
    text = g.read_text()
    g.write_text("// a new comment line\n/* and a block\n   comment */\n" + text.replace("\n", "\n  ", 5))
    assert bench.kernel_sources_hash() == h0
    g.write_text(text.replace("GEMM_BK = 128", "GEMM_BK = 64", 1))
    assert bench.kernel_sources_hash() != h0
