"""The down-tile cost model's fit against the committed B200 sweep: the table
parses, the installed parameters give the picks and regrets the table states,
and refitting the table gives back the installed parameters.  The gate/up
CTA-mode sweep tool restates the dispatch's pair rule; it is checked against
the oracle's rule."""
import os

import numpy as np
import pytest

import oracle

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


def test_mode_sweep_rule_is_the_oracle_rule():
    """The sweep tool's restatement of the gate/up mode rule (on m-tile
    counts) picks what the oracle's rule picks on the histograms themselves."""
    from mixture_experts_topk_b200 import gate_up_mode_sweep as gs
    rng = np.random.default_rng(3)
    for trial in range(400):
        E = int(rng.choice([8, 32, 64, 256]))
        counts = rng.integers(0, int(rng.choice([3, 200, 1500])), size=E).astype(np.int32)
        nb, kb = int(rng.choice([1, 4, 16, 112])), int(rng.choice([2, 16, 32]))
        ps = [int(v) for v in rng.integers(1, 10 ** 6, size=6)]
        allow = int(rng.integers(0, 8))
        mt = (counts + 127) // 128
        want = oracle.pick_gu_mode(counts, nb, kb, 148, ps, allow)
        assert gs.pick(int(mt.sum()), int((mt % 2).sum()), nb, kb, ps, allow) == want, (trial, E, nb, kb, ps)


def test_mode_sweep_table_reader(tmp_path):
    from mixture_experts_topk_b200 import gate_up_mode_sweep as gs
    f = tmp_path / "t.md"
    f.write_text(gs.HEADER + "\n| tiny T=16 | 8 | 8 | 1 | 2 | 0.0086 | 0.0120 | 0.0070 |\n"
                 "| mixtral-8x7b T=4096 | 67 | 3 | 112 | 32 | 0.9292 | 0.9248 | 1.1 |\n")
    rows = gs.read_table(str(f))
    assert [r["workload"] for r in rows] == ["tiny T=16", "mixtral-8x7b T=4096"]
    # tiny: one wave in every mode -> the cheapest unit, narrow (2 x 334000);
    # Mixtral-8x7B T = 4096: pairs (53 waves of 16.0 us against 51 of 16.9 and
    # 102 of 10.7)
    res = gs.evaluate(rows, gs.INSTALLED)
    assert [p for _, p, _ in res] == [2, 1]
    assert all(rg == 0.0 for _, _, rg in res)
