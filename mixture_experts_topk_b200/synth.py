"""Seeded synthetic inputs for the routed MoE FFN layer.

This module draws random numbers and nothing else of the layer: it never
routes, dispatches, multiplies or requantises an activation.  It is the only
code shared by the CUDA path's tests/bench and by the oracle.

Recipe (every tensor has its own seed derived from (seed, tensor tag)):
  X        ~ N(0, 1), rounded to bf16
  Wr       ~ N(0, 1/H) ("normal") or U(-sqrt(3/H), +sqrt(3/H)) ("uniform"); fp32
  bias[e]  = -s * ln(r_e), r a seeded permutation of 1..E, so exp(bias) is Zipf(s)
  W_gate, W_up ~ N(0, 1/H), W_down ~ N(0, 1/I), then quantised OFFLINE (weights
  reach the layer already quantised, as a checkpoint would hold them):
    FP8_ROW       s_n = amax_n/448 per output channel, code = e4m3(w/s_n)
    FP8_BLOCK128  the same per 128x128 block
    NVFP4         g = amax/(448*6) per (expert, projection); 16-wide blocks along
                  K with e4m3 block scale of amax_blk/(6 g); e2m1 code nearest.
  The fp8 conversions are torch's own (float8_e4m3fn); the e2m1 code is the
  nearest grid value found by torch.bucketize.
"""
import hashlib
import math

import torch

from .workloads import ACT_RELU2, FMT_FP8_BLOCK128, FMT_FP8_ROW, FMT_NVFP4

E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _seed(seed, tag):
    h = hashlib.sha256(f"{seed}:{tag}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed, tag, device):
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, tag))
    return g


def tokens(wl, T, seed=0, device="cpu"):
    """X [T, H] bf16 ~ N(0, 1)."""
    g = _gen(seed, f"X:{T}", device)
    return torch.randn(T, wl.H, generator=g, device=device).to(torch.bfloat16)


def router(wl, seed=0, device="cpu"):
    """(Wr [E, H] fp32, bias [E] fp32 or None)."""
    g = _gen(seed, "Wr", device)
    if wl.router_init == "uniform":
        a = math.sqrt(3.0 / wl.H)
        wr = (torch.rand(wl.E, wl.H, generator=g, device=device) * 2.0 - 1.0) * a
    else:
        wr = torch.randn(wl.E, wl.H, generator=g, device=device) / math.sqrt(wl.H)
    bias = None
    if wl.has_bias:
        gb = _gen(seed, "bias", "cpu")
        r = torch.randperm(wl.E, generator=gb).to(torch.float64) + 1.0
        bias = (-wl.zipf_s * torch.log(r)).to(torch.float32).to(device)
    return wr.contiguous(), bias


def _fp8(x):
    return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def _fp8_value(code):
    return code.view(torch.float8_e4m3fn).to(torch.float32)


def _quant_fp8_row(w):
    s = w.abs().amax(dim=1) / 448.0
    s = torch.where(s > 0, s, torch.ones_like(s))
    return _fp8(w / s[:, None]), s.to(torch.float32)


def _quant_fp8_block(w):
    n, k = w.shape
    wb = w.view(n // 128, 128, k // 128, 128)
    s = wb.abs().amax(dim=(1, 3)) / 448.0
    s = torch.where(s > 0, s, torch.ones_like(s))
    q = _fp8(wb / s[:, None, :, None]).view(n, k)
    return q, s.to(torch.float32)


def _quant_nvfp4(w):
    n, k = w.shape
    amax = w.abs().max()
    g = (amax / (448.0 * 6.0)).to(torch.float32)
    wb = w.view(n, k // 16, 16)
    sb_code = _fp8(wb.abs().amax(dim=2) / 6.0 / g)
    sb = _fp8_value(sb_code)
    denom = (sb * g)[:, :, None]
    v = torch.where(denom > 0, wb / denom, torch.zeros_like(wb))
    grid = torch.tensor(E2M1_GRID, device=w.device)
    mids = (grid[1:] + grid[:-1]) / 2
    mag = torch.bucketize(v.abs().clamp(max=6.0), mids)
    code = (mag | ((v < 0).to(mag.dtype) << 3)).to(torch.uint8).view(n, k)
    packed = code[:, 0::2] | (code[:, 1::2] << 4)
    return packed.contiguous(), sb_code.contiguous(), g.reshape(1)


def _quant(w, fmt):
    if fmt == FMT_FP8_ROW:
        return _quant_fp8_row(w) + (None,)
    if fmt == FMT_FP8_BLOCK128:
        return _quant_fp8_block(w) + (None,)
    if fmt == FMT_NVFP4:
        return _quant_nvfp4(w)
    raise ValueError(fmt)


def experts(wl, seed=0, device="cpu", experts_subset=None):
    """Quantised expert weights in the plain layout the layer takes.

    Returns a dict with, for p in (gate, up, down):
      p_q      codes: [E, N, K] uint8 (fp8) or [E, N, K/2] uint8 (e2m1, low nibble first)
      p_s      scales: [E, N] fp32 (FP8_ROW), [E, N/128, K/128] fp32 (FP8_BLOCK128),
               [E, N, K/16] uint8 e4m3 codes (NVFP4)
      p_g      [E] fp32 NVFP4 global scale (absent otherwise)
    gate/up: N = I, K = H; down: N = H, K = I.  experts_subset draws only those
    experts (the others are left zero), for sampled checks of huge layers.
    ReLU^2 experts have no gate: gate_q / gate_s / gate_g are None.
    """
    E = wl.E
    shapes = {"gate": (wl.I, wl.H), "up": (wl.I, wl.H), "down": (wl.H, wl.I)}
    if wl.act == ACT_RELU2:
        del shapes["gate"]
    out = {}
    for p, (n, k) in shapes.items():
        kq = k // 2 if wl.fmt == FMT_NVFP4 else k
        out[p + "_q"] = torch.zeros(E, n, kq, dtype=torch.uint8, device=device)
        if wl.fmt == FMT_FP8_ROW:
            out[p + "_s"] = torch.zeros(E, n, dtype=torch.float32, device=device)
        elif wl.fmt == FMT_FP8_BLOCK128:
            out[p + "_s"] = torch.zeros(E, n // 128, k // 128, dtype=torch.float32, device=device)
        else:
            out[p + "_s"] = torch.zeros(E, n, k // 16, dtype=torch.uint8, device=device)
            out[p + "_g"] = torch.zeros(E, dtype=torch.float32, device=device)
    todo = range(E) if experts_subset is None else sorted(set(int(e) for e in experts_subset))
    for e in todo:
        for p, (n, k) in shapes.items():
            g = _gen(seed, f"W:{p}:{e}", device)
            w = torch.randn(n, k, generator=g, device=device) / math.sqrt(k)
            q, s, gg = _quant(w, wl.fmt)
            out[p + "_q"][e].copy_(q)
            out[p + "_s"][e].copy_(s)
            if gg is not None:
                out[p + "_g"][e] = gg[0]
    if wl.act == ACT_RELU2:
        out.update(gate_q=None, gate_s=None, gate_g=None)
    return out


def layer(wl, seed=0, device="cpu", experts_subset=None):
    wr, bias = router(wl, seed, device)
    d = experts(wl, seed, device, experts_subset)
    d["wr"] = wr
    d["bias"] = bias
    return d
