"""Fit the four parameters of the down GEMM tile-choice cost model to a sweep.

The sweep is a list of measurements (H, I, m_tiles, touched experts, tile width
BN, measured down GEMM ms), e.g. the table in profiles/down_tile_sweep.md,
taken with `bench.py --down-bn BN` on every workload.  The fit minimises the
squared log error of the model time; the result is what moe_init installs
(moe_set_picker_params changes it at run time).

    python -m mixture_experts_topk_b200.picker_fit profiles/down_tile_sweep.md
"""
import math
import re
import sys

import numpy as np
from scipy.optimize import minimize

NUM_SMS = 148


def model_ps(p, H, I, m_tiles, touched, bn, num_sms=NUM_SMS):
    alpha, beta, bw, gamma = p
    tiles = m_tiles * (H // bn)
    waves = -(-tiles // num_sms)
    t_mma = waves * (I // 128) * (alpha + beta * bn)
    active = min(tiles, num_sms)
    t_load = touched * H * I * 1e6 / (active * bw) if active else 0.0
    return gamma + max(t_mma, t_load)


def read_table(path):
    rows = []
    for line in open(path):
        m = re.match(r"\|\s*([\w.\-]+ T=\d+)\s*\|\s*(\d+)\s*\|\s*(\d+)\s*\|\s*(\d+)\s*\|\s*(\d+)\s*\|\s*(\d+)\s*\|\s*([\d.]+)\s*\|", line)
        if m:
            rows.append(dict(workload=m.group(1), H=int(m.group(2)), I=int(m.group(3)), m_tiles=int(m.group(4)),
                             touched=int(m.group(5)), bn=int(m.group(6)), down_ms=float(m.group(7))))
    return rows


def fit(rows, start=(240000, 2200, 60000, 5000)):
    def loss(q):
        p = np.exp(q)
        return sum((math.log(model_ps(p, r["H"], r["I"], r["m_tiles"], r["touched"], r["bn"])) -
                    math.log(r["down_ms"] * 1e9)) ** 2 for r in rows)
    res = minimize(loss, np.log(np.array(start, float)), method="Nelder-Mead",
                   options={"maxiter": 4000, "xatol": 1e-6, "fatol": 1e-9})
    return [int(round(v)) for v in np.exp(res.x)]


def regret(rows, p):
    by = {}
    for r in rows:
        by.setdefault(r["workload"], []).append(r)
    out = {}
    for w, rs in by.items():
        pick = min(rs, key=lambda r: (model_ps(p, r["H"], r["I"], r["m_tiles"], r["touched"], r["bn"]), -r["bn"]))
        best = min(r["down_ms"] for r in rs)
        out[w] = (pick["bn"], pick["down_ms"] / best - 1.0)
    return out


if __name__ == "__main__":
    rows = read_table(sys.argv[1])
    p = fit(rows)
    print("alpha_ps, beta_ps, bw_cta, gamma_ps =", p)
    for w, (bn, rg) in regret(rows, p).items():
        print(f"{w:28s} pick BN={bn:3d} regret {100 * rg:.1f}%")
