"""Plain layer calls of one named workload with fewer experts, for profiler
captures that must stay small on the device (a few GB): the same H, I, k,
score, format and router initialisation, E experts instead of the workload's.

    python -m mixture_experts_topk_b200.profile_case --workload deepseek-v3 --experts 64 --tokens 1024 --calls 4

Each call is `moe_forward` on the same seeded inputs, synchronised, with the
status checked; nothing is timed here (profile the process, e.g. with ncu)."""
import argparse
import dataclasses

import torch

from . import native, synth
from .workloads import WORKLOADS


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", required=True, choices=sorted(WORKLOADS))
    ap.add_argument("--experts", type=int, required=True)
    ap.add_argument("--tokens", type=int, required=True)
    ap.add_argument("--calls", type=int, default=4)
    a = ap.parse_args(argv)
    wl = dataclasses.replace(WORKLOADS[a.workload], name=f"{a.workload}-e{a.experts}", E=a.experts)
    if a.experts < wl.k:
        raise SystemExit("--experts must be at least the workload's k")
    d = synth.layer(wl, seed=0, device="cuda")
    layer = native.Layer(wl, d, max_T=a.tokens)
    x = synth.tokens(wl, a.tokens, seed=0, device="cuda")
    for _ in range(a.calls):
        layer.forward(x, d["wr"], d["bias"])
        torch.cuda.synchronize()
        st, msg = layer.status()
        if st != 0:
            raise SystemExit(f"layer status {st}: {msg}")
    print(f"{wl.name} T={a.tokens}: {a.calls} calls ok")


if __name__ == "__main__":
    main()
