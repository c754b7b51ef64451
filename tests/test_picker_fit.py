"""The down-tile cost model's fit against the committed B200 sweep: the table
parses, the installed parameters give the picks and regrets the table states,
and refitting the table gives back the installed parameters."""
import os

import pytest

from mixture_experts_topk_b200 import picker_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SWEEP = os.path.join(ROOT, "profiles", "down_tile_sweep.md")
INSTALLED = (334419, 2114, 38684, 17030139)   # the values moe_init sets


@pytest.fixture(scope="module")
def rows():
    return picker_fit.read_table(SWEEP)


def test_sweep_table_parses(rows):
    assert len(rows) == 24   # 8 workloads x 3 tile widths
    assert {r["bn"] for r in rows} == {64, 128, 256}


def test_model_time_by_hand():
    # Qwen3.5 T = 64, BN = 128: tiles 47 * 16 = 752 -> 6 waves of 148;
    # t_mma = 6 * 4 * (alpha + 128 beta); active CTAs 148;
    # t_load = 47 * 2048 * 512 * 1e6 / (148 * bw); time = gamma + max of the two
    a, b, bw, g = INSTALLED
    t_mma = 6 * 4 * (a + 128 * b)
    t_load = 47 * 2048 * 512 * 1e6 / (148 * bw)
    assert picker_fit.model_ps(INSTALLED, 2048, 512, 47, 47, 128) == pytest.approx(g + max(t_mma, t_load))


def test_installed_parameters_give_the_stated_picks_and_regrets(rows):
    reg = picker_fit.regret(rows, INSTALLED)
    picks = {w: bn for w, (bn, _) in reg.items()}
    assert picks == {"deepseek-v3 T=16": 256, "deepseek-v3 T=4096": 256, "mixtral-8x7b T=1": 64,
                     "mixtral-8x7b T=32": 256, "mixtral-8x7b T=4096": 256, "mixtral-8x7b T=512": 256,
                     "qwen3.5-35b-a3b T=64": 256, "qwen3.5-35b-a3b T=8192": 256}
    mean = sum(r for _, r in reg.values()) / len(reg)
    assert mean == pytest.approx(0.036, abs=0.0006)


def test_refit_reproduces_the_installed_parameters(rows):
    p = picker_fit.fit(rows)
    for got, want in zip(p, INSTALLED):
        assert got == pytest.approx(want, rel=0.02)
