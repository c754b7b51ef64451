"""Measure and evaluate the gate/up GEMM's mode choice.

The gated FP8_ROW gate/up GEMM is launched as 2-CTA clusters that run one of
three modes: 0 single CTAs on 256-wide tiles, 1 CTA pairs (M = 256 over two
row tiles of one expert), 2 single CTAs on 128-wide tiles.  The dispatch picks
the mode from the expert histogram with the wave cost model that
moe_set_gate_up_model documents (RaMP abstract: the configuration comes from
the runtime histogram through a cost model of CTA waves).

    python -m mixture_experts_topk_b200.gate_up_mode_sweep run        # on a GPU: markdown rows
    python -m mixture_experts_topk_b200.gate_up_mode_sweep evaluate profiles/gate_up_mode_sweep.md

`run` times the kernel with the mode forced each way (through the cost
parameters) in short interleaved segments, so that the modes see the same
power-capped clock, and prints one markdown row per (workload, T) with the
medians.  `evaluate` reads such a table and reports the mode the model picks
under the parameters the library installs, and its regret against the
fastest measured mode.
"""
import re
import sys

import numpy as np

NUM_SMS = 148
BIG = 10 ** 12
# the parameters moe_init installs (a_0, b_0, a_1, b_1, a_2, b_2)
INSTALLED = (527000, 0, 493000, 200000, 334000, 0)

CASES = [("tiny", 16), ("mixtral-8x7b", 1), ("mixtral-8x7b", 32), ("mixtral-8x7b", 128),
         ("qwen3.5-35b-a3b", 64), ("mixtral-8x7b", 512), ("mixtral-8x7b", 1024), ("mixtral-8x7b", 2048),
         ("mixtral-8x7b", 3072), ("mixtral-8x7b", 4096), ("qwen3.5-35b-a3b", 256), ("qwen3.5-35b-a3b", 2048),
         ("qwen3.5-35b-a3b", 4096), ("qwen3.5-35b-a3b", 8192), ("wide-e64", 64), ("wide-e64", 2048),
         ("wide-e64", 8192), ("deep-i4096", 16), ("deep-i4096", 1024), ("deep-i4096", 4096)]

HEADER = ("| workload | m_tiles | odd | n_blocks | k_blocks | wide ms | pairs ms | narrow ms |\n"
          "|---|---|---|---|---|---|---|---|")

FORCE = ((0, 0, BIG, BIG, BIG, BIG), (BIG, BIG, 0, 0, BIG, BIG), (BIG, BIG, BIG, BIG, 0, 0))


def pick(m_tiles, n_odd, nb, kb, ps, allow=7, num_sms=NUM_SMS):
    """The mode the dispatch writes: the same integer rule."""
    if nb == 0 or m_tiles == 0:
        return 0
    units = (m_tiles * nb, (m_tiles + n_odd) // 2 * nb, 2 * m_tiles * nb)
    slots = (num_sms, num_sms // 2, num_sms)
    best, best_c = -1, 0
    for m in range(3):
        if not (allow >> m) & 1:
            continue
        c = -(-units[m] // slots[m]) * (kb * ps[2 * m] + ps[2 * m + 1])
        if best < 0 or c < best_c:
            best, best_c = m, c
    return max(best, 0)


def run(reps=12, seg=4):
    import torch

    from . import native, synth, workloads as W
    native.load()
    extra = {"wide-e64": W.custom(name="wide-e64", H=4096, I=2048, E=64, k=4, zipf_s=0.5),
             "deep-i4096": W.custom(name="deep-i4096", H=2048, I=4096, E=32, k=2)}
    print(HEADER)
    cache = {}
    for name, T in CASES:
        wl = extra.get(name) or W.WORKLOADS[name]
        if name not in cache:
            cache.clear()
            torch.cuda.empty_cache()
            cache[name] = synth.layer(wl, seed=0, device="cuda")
        d = cache[name]
        layer = native.Layer(wl, d, max_T=T)
        x = synth.tokens(wl, T, seed=0, device="cuda")
        default = native.moe_get_gate_up_model(layer.h)[:6]
        layer.forward(x, d["wr"], d["bias"])
        torch.cuda.synchronize()
        counts = layer.region("counts", torch.int32, wl.E).cpu().numpy()
        mt = (counts + 127) // 128
        n = seg if T >= 512 else 12 * seg
        times = {0: [], 1: [], 2: []}
        for _ in range(reps if T >= 512 else 2 * reps):
            for mode in range(3):
                native.moe_set_gate_up_model(layer.h, *FORCE[mode])
                layer.forward(x, d["wr"], d["bias"])   # the dispatch writes the forced mode
                for _ in range(2):
                    native.moe_gate_up(layer.h, layer.packed, T, layer.ws)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(n):
                    native.moe_gate_up(layer.h, layer.packed, T, layer.ws)
                e1.record()
                torch.cuda.synchronize()
                assert int(layer.region("pick", torch.int32, 3)[2]) == mode
                times[mode].append(e0.elapsed_time(e1) / n)
        native.moe_set_gate_up_model(layer.h, *default)
        st, msg = layer.status()
        assert st == 0, msg
        layer.close()
        print(f"| {name} T={T} | {int(mt.sum())} | {int((mt % 2).sum())} | {2 * wl.I // 256} | {wl.H // 128} "
              f"| {np.median(times[0]):.4f} | {np.median(times[1]):.4f} | {np.median(times[2]):.4f} |", flush=True)


def read_table(path):
    rows = []
    pat = r"\|\s*([\w.\-]+ T=\d+)\s*\|" + r"\s*(\d+)\s*\|" * 4 + r"\s*([\d.]+)\s*\|" * 3
    for line in open(path):
        m = re.match(pat, line)
        if m:
            rows.append(dict(workload=m.group(1), m_tiles=int(m.group(2)), odd=int(m.group(3)), nb=int(m.group(4)),
                             kb=int(m.group(5)), ms=(float(m.group(6)), float(m.group(7)), float(m.group(8)))))
    return rows


def evaluate(rows, ps):
    out = []
    for r in rows:
        p = pick(r["m_tiles"], r["odd"], r["nb"], r["kb"], ps)
        out.append((r["workload"], p, r["ms"][p] / min(r["ms"]) - 1.0))
    return out


if __name__ == "__main__":
    if sys.argv[1] == "run":
        run()
    else:
        ps = INSTALLED if len(sys.argv) < 4 else tuple(int(v) for v in sys.argv[3].split(","))
        res = evaluate(read_table(sys.argv[2]), ps)
        names = ("wide", "pairs", "narrow")
        for w, p, rg in res:
            print(f"{w:28s} pick {names[p]:6s} regret {100 * rg:.1f}%")
        rgs = [rg for _, _, rg in res]
        print(f"mean regret {100 * np.mean(rgs):.2f}%, max {100 * max(rgs):.1f}%")
