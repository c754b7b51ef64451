"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against a library routine (torch's fp8
conversion, Python's stable sort, torch fp64 matmul + SiLU), brute force on
tiny inputs, a hand-derived closed form, or an invariant of the layer.  The
pages print no worked numeric example, so no value here comes from them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_topk_b200 import synth, workloads as W

E2M1_MAG = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # OCP FP4 E2M1 magnitudes in code order


def bf16_bits(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def torch_e4m3(x):
    x = np.clip(np.asarray(x, np.float32), -448.0, 448.0)
    return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def torch_e4m3_value(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


# ------------------------------------------------------------------ codecs
def test_e4m3_values_match_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch_e4m3_value(codes)
    ours = np.array([oracle.e4m3_value(c) for c in codes])
    assert (np.isnan(ours) == np.isnan(ref)).all()
    ok = ~np.isnan(ref)
    assert (ours[ok] == ref[ok]).all()
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_matches_torch_on_bit_sweep_and_ties():
    bits = np.arange(0, 2 ** 32, 509, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    vals = torch_e4m3_value(np.arange(127, dtype=np.uint8))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)            # exact ties
    near = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)),
                           np.nextafter(mids, np.float32(0)), vals.astype(np.float32),
                           np.float32([448.0, 464.0, 480.0, 1e30, 3.4e38, 0.0])])
    x = np.concatenate([x, near, -near])
    assert (oracle.e4m3_encode(x) == torch_e4m3(x)).all()


def _brute_e2m1(x):
    a = min(abs(float(x)), 6.0)
    c = min(range(8), key=lambda c: (abs(E2M1_MAG[c] - a), c & 1))   # nearest, tie -> even code
    return c | (8 if math.copysign(1.0, float(x)) < 0 else 0)


def test_e2m1_values_and_encode_by_brute_force():
    for c in range(16):
        v = E2M1_MAG[c & 7] * (-1.0 if c & 8 else 1.0)
        assert oracle.e2m1_value(c) == v
    grid = np.arange(-8.0, 8.0, 1.0 / 64, dtype=np.float32)
    mids = np.float32([(a + b) / 2 for a, b in zip(E2M1_MAG[:-1], E2M1_MAG[1:])])
    extra = np.concatenate([mids, np.nextafter(mids, np.float32(9)), np.nextafter(mids, np.float32(0)),
                            np.float32([1e-30, 7.0, 1e9])])
    rng = np.random.default_rng(0)
    x = np.concatenate([grid, extra, -extra, rng.normal(0, 3, 5000).astype(np.float32)])
    got = oracle.e2m1_encode(x)
    want = np.array([_brute_e2m1(v) for v in x], np.uint8)
    assert (got == want).all()
    # hand-checked ties: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    hand = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in hand.items():
        assert oracle.e2m1_encode(np.float32([v]))[0] == c


# ------------------------------------------------------------------ router
def test_router_canonical_order_within_fp64_bound():
    rng = np.random.default_rng(1)
    for H, E, T in [(256, 8, 5), (1024, 16, 7), (7168, 4, 3)]:
        x = bf16_bits(rng.normal(size=(T, H)))
        wr = rng.normal(0, 1 / math.sqrt(H), size=(E, H)).astype(np.float32)
        bias = rng.normal(size=E).astype(np.float32)
        l32 = oracle.router_logits(x, wr, bias).astype(np.float64)
        l64 = oracle.router_logits_f64(x, wr, bias)
        xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
        absdot = np.abs(xf) @ np.abs(wr.astype(np.float64)).T
        bound = (H / 32 + 7) * 2.0 ** -24 * (absdot + np.abs(bias)[None, :])
        assert (np.abs(l32 - l64) <= bound).all()


def test_router_chain_and_lane_assignment_closed_form():
    # lane 0's chain sees 2^24 first, so its later +1 terms round away (ties to
    # even); lane 1 sums eight ones exactly; the tree adds 2^24 + 8 exactly.
    H = 512
    w = np.zeros((1, H), np.float32)
    w[0, 0] = 2.0 ** 24
    w[0, 1:8] = 1.0           # lane 0, i=0, j=1..7
    w[0, 256] = 1.0           # lane 0, i=1, j=0
    w[0, 8:16] = 1.0          # lane 1
    x = bf16_bits(np.ones((1, H)))
    assert oracle.router_logits(x, w)[0, 0] == np.float32(2.0 ** 24 + 8)


def test_router_pairwise_tree_shape_closed_form():
    # partials p0=2^24, p2=1, p3=1: ((p0+p1)+(p2+p3)) = 2^24+2 exactly, while a
    # left-to-right sum or a tree that pairs lanes 16 apart gives 2^24.
    H = 256
    w = np.zeros((1, H), np.float32)
    w[0, 0] = 2.0 ** 24
    w[0, 16] = 1.0
    w[0, 24] = 1.0
    x = bf16_bits(np.ones((1, H)))
    assert oracle.router_logits(x, w)[0, 0] == np.float32(2.0 ** 24 + 2)
    # the bias is one fp32 add after the tree: 2^24+2 + 3 = 2^24+5 is a tie, rounded to even 2^24+4
    got = oracle.router_logits(x, w, np.float32([3.0]))[0, 0]
    assert got == np.float32(2.0 ** 24 + 4)


def _brute_topk(l, k):
    E = len(l)

    def before(a, b):
        return l[a] > l[b] or (l[a] == l[b] and a < b)

    sets = [S for S in itertools.combinations(range(E), k)
            if all(before(i, j) for i in S for j in range(E) if j not in S)]
    assert len(sets) == 1
    return sorted(sets[0], key=lambda i: (-l[i], i))


@pytest.mark.parametrize("score", [W.SCORE_SOFTMAX, W.SCORE_SIGMOID])
def test_topk_brute_force_with_ties(score):
    rng = np.random.default_rng(2)
    for E in range(3, 11):
        for k in range(1, min(3, E - 1) + 1):
            lg = rng.choice(np.float32([-1.0, 0.0, 0.5, 1.0, 2.0, -0.0]), size=(20, E)).astype(np.float32)
            ids, w = oracle.topk(lg, k, score)
            for t in range(lg.shape[0]):
                want = _brute_topk(list(lg[t]), k)
                assert list(ids[t]) == want
                sel = [float(lg[t, i]) for i in want]
                if score == W.SCORE_SOFTMAX:
                    z = [math.exp(v) for v in sel]
                else:
                    z = [1.0 / (1.0 + math.exp(-v)) for v in sel]
                np.testing.assert_allclose(w[t], np.array(z) / sum(z), rtol=1e-14)


def test_topk_equal_logits_pick_lowest_ids_with_equal_weights():
    ids, w = oracle.topk(np.zeros((3, 6), np.float32), 4, W.SCORE_SOFTMAX)
    assert (ids == np.arange(4)).all()
    assert np.allclose(w, 0.25, rtol=0, atol=1e-15)


# ------------------------------------------------------------------ dispatch
def test_dispatch_matches_stable_sort():
    rng = np.random.default_rng(3)
    for T, k, E in [(1, 1, 1), (17, 2, 8), (300, 8, 64), (1000, 8, 256)]:
        ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        ids[ids == 3] = 0 if E > 3 and k == 1 else ids[ids == 3]      # leave some experts empty
        counts, offsets, perm, inv = oracle.dispatch(ids, E)
        flat = ids.reshape(-1)
        assert counts.sum() == T * k
        assert (counts == np.bincount(flat, minlength=E)).all()
        assert (offsets == np.concatenate([[0], np.cumsum(counts)])).all()
        want = sorted(range(T * k), key=lambda a: flat[a])        # Python's sort is stable
        assert list(perm) == want
        assert (inv[perm] == np.arange(T * k)).all()


def test_schedule_tiles():
    # counts 0, 1, 129 (ragged: two tiles), 0, 384 (exactly three tiles)
    offsets = np.int32([0, 0, 1, 130, 130, 514])
    te, tr = oracle.schedule(offsets)
    assert list(te) == [1, 2, 2, 4, 4, 4]
    assert list(tr) == [0, 1, 129, 130, 258, 386]


# ------------------------------------------------------------------ quantisers
def test_fp8_row_quant_hand_example():
    x = np.zeros((2, 256), np.float32)
    x[0, :5] = [448.0, 224.0, -112.0, 0.0, 1.0]          # amax 448 -> s = 1 exactly
    codes, s = oracle.quant_rows(W.FMT_FP8_ROW, x)
    assert s[0] == 1.0 and s[1] == 0.0
    assert list(codes[0, :5]) == [0x7E, 0x76, 0xEE, 0x00, 0x38]
    assert (codes[1] == 0).all()


def test_fp8_block128_quant_hand_example():
    x = np.zeros((1, 256), np.float32)
    x[0, 0] = 448.0
    x[0, 128] = 224.0
    x[0, 129] = -56.0
    codes, s = oracle.quant_rows(W.FMT_FP8_BLOCK128, x)
    assert list(s[0]) == [1.0, 0.5]
    assert codes[0, 0] == 0x7E and codes[0, 128] == 0x7E and codes[0, 129] == 0xEE


def test_nvfp4_quant_hand_example():
    x = np.zeros((1, 32), np.float32)
    x[0, :4] = [6.0, 3.0, -1.5, 0.5]
    codes, sb = oracle.quant_rows(W.FMT_NVFP4, x, g=2.0 ** -8)
    assert sb[0, 0] == 0x78 and sb[0, 1] == 0x00     # 256 = 2^8 -> e=15, m=0
    assert list(codes[0, :2]) == [0x57, 0x1B] and (codes[0, 2:] == 0).all()
    assert oracle.nvfp4_global(np.float32([[-5376.0, 1.0]])) == 2.0


@pytest.mark.parametrize("fmt", [W.FMT_FP8_ROW, W.FMT_FP8_BLOCK128])
def test_fp8_quant_error_bound(fmt):
    rng = np.random.default_rng(4)
    x = (rng.normal(size=(8, 512)) * rng.uniform(0.01, 100, size=(8, 1))).astype(np.float32)
    codes, s = oracle.quant_rows(fmt, x)
    s_full = np.repeat(s.reshape(8, -1), 512 // s.reshape(8, -1).shape[1], axis=1)
    deq = torch_e4m3_value(codes) * s_full
    # half an e4m3 ulp: 2^-4 relative for normals, 2^-10 * s absolute in the subnormal range
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s_full * 2.0 ** -10) * (1 + 1e-6)
    assert (np.abs(deq - x) <= bound).all()
    # the element holding the block maximum gets the +-448 code: x/s = amax/fl(amax/448)
    nb = s.reshape(8, -1).shape[1]
    xb = np.abs(x).reshape(8, nb, -1)
    cb = codes.reshape(8, nb, -1)
    at_max = np.take_along_axis(cb, xb.argmax(axis=2)[..., None], axis=2)[..., 0]
    assert ((at_max & 0x7F) == 0x7E).all()


# ------------------------------------------------------------------ tile choice
def test_pick_down_tile_hand_example():
    # one token on one Mixtral-shaped expert: 1 m-tile, H/BN n-blocks, one wave
    P = dict(H=4096, I=14336, num_sms=148, alpha=240000, beta=2200, bw=60000, gamma=5000)
    c, costs = oracle.pick_down_tile(np.int32([1, 0]), **P)
    # BN=256: 112 K-blocks x (240000 + 256*2200) = 89958400 > load 61166933
    # BN=128: 112 x (240000 + 128*2200) = 58419200;  BN=64: 112 x 380800 = 42649600
    assert list(costs) == [5000 + 89958400, 5000 + 58419200, 5000 + 42649600]
    assert c == 2
    # no assignments: every cost is gamma, the widest tile wins the tie
    c, costs = oracle.pick_down_tile(np.zeros(8, np.int32), **P)
    assert c == 0 and list(costs) == [5000, 5000, 5000]


def test_pick_down_tile_load_term_and_waves():
    P = dict(H=2048, I=512, num_sms=4, alpha=0, beta=0, bw=1000, gamma=0)
    # beta = alpha = 0: only the load term counts; more active CTAs -> cheaper
    c, costs = oracle.pick_down_tile(np.int32([5]), **P)
    # m_tiles 1: tiles 8 / 16 / 32, all capped at 4 active CTAs -> equal -> widest
    load = 1 * 2048 * 512 * 1000000 // (4 * 1000)
    assert list(costs) == [load] * 3 and c == 0
    P.update(alpha=100, num_sms=1000)
    c, costs = oracle.pick_down_tile(np.int32([5]), **P)
    # one wave each, t_mma = 4 x 100 everywhere; load shrinks with more tiles
    loads = [1 * 2048 * 512 * 1000000 // (t * 1000) for t in (8, 16, 32)]
    assert list(costs) == [max(400, l) for l in loads] and c == 2


def test_pick_split_hand_examples():
    # Mixtral-shaped decode, one token on two experts: 2 m-tiles x 16 n-blocks =
    # 32 units; 32 x 4 = 128 <= 148 < 160 = 32 x 5, and s_max = min(8, 16/2, 112/4) = 8
    mix = dict(split_nb=16, split_kb=112, o_rows=2 + 7 * 2, num_sms=148)
    counts = np.int32([1, 0, 0, 1, 0, 0, 0, 0])
    assert oracle.pick_split(counts, **mix) == 4
    # one expert only: 16 units -> 16 x 8 = 128 <= 148, capped by 8
    assert oracle.pick_split(np.int32([2, 0, 0, 0, 0, 0, 0, 0]), **mix) == 8
    # the output buffer bounds the copies: o_rows / A = 16 / 4 = 4 ... = 16 / 5 = 3
    assert oracle.pick_split(np.int32([4, 0, 0, 0, 0, 0, 0, 0]), **mix) == 4
    assert oracle.pick_split(np.int32([5, 0, 0, 0, 0, 0, 0, 0]), **mix) == 3
    # at least four K-blocks per range: split_kb 8 -> s_max 2
    assert oracle.pick_split(counts, **dict(mix, split_kb=8)) == 2
    # units filling the SMs: 148 units -> every s costs a full unit round (840),
    # no split; 75 units -> rounds of 1/s for s = 2..8: 2, 2, 3, 3, 4, 4, 5, so
    # costs 840, 560, 630, 504, 560, 480, 525 -> 7; 74 -> 2 (one round of halves)
    many = dict(split_nb=1, split_kb=112, o_rows=10 ** 6, num_sms=148)
    assert oracle.pick_split(np.full(148, 1, np.int32), **many) == 1
    assert oracle.pick_split(np.full(75, 1, np.int32), **many) == 7
    assert oracle.pick_split(np.full(74, 1, np.int32), **many) == 2
    # 208 units (Mixtral-8x7B T = 512: 13 m-tiles x 16) with s_max 2: 2 rounds
    # (1680) against 3 rounds of halves (1260 <= 1344) -> 2; 128 units with
    # s_max 8: the best, s = 8 at 7 rounds of eighths (735), saves under a
    # fifth of one round (840) -> no split
    assert oracle.pick_split(np.full(208, 1, np.int32), **dict(many, o_rows=416)) == 2
    assert oracle.pick_split(np.full(128, 1, np.int32), **dict(many, o_rows=1024)) == 1
    # a 129-row expert is two m-tiles
    assert oracle.pick_split(np.int32([129]), **dict(many, num_sms=4)) == 2
    # no split for formats without one, nor for an empty batch
    assert oracle.pick_split(counts, **dict(mix, split_nb=0)) == 1
    assert oracle.pick_split(np.zeros(8, np.int32), **mix) == 1


# ------------------------------------------------------------------ gated activations
def test_gated_activations_closed_forms():
    # silu(1) = 1 / (1 + e^-1); Phi(1) = 0.8413447460685429 (normal CDF table value)
    assert oracle.glu(oracle.ACT_SWIGLU, 1.0, 2.0) == pytest.approx(2.0 / (1.0 + np.exp(-1.0)), rel=1e-15)
    assert oracle.glu(oracle.ACT_GEGLU, 1.0, 1.0) == pytest.approx(0.8413447460685429, rel=1e-15)
    assert oracle.glu(oracle.ACT_GEGLU, -1.0, 1.0) == pytest.approx(-(1.0 - 0.8413447460685429), rel=1e-14)
    # relu gate: exact
    assert oracle.glu(oracle.ACT_REGLU, -3.0, 5.0) == 0.0
    assert oracle.glu(oracle.ACT_REGLU, 3.0, 5.0) == 15.0
    # bounded: the gate is capped from above only, the up projection on both sides
    L = 10.0
    assert oracle.glu(oracle.ACT_SWIGLU_BOUNDED, 50.0, 50.0, limit=L) == \
        pytest.approx(10.0 / (1.0 + np.exp(-10.0)) * 10.0, rel=1e-15)
    assert oracle.glu(oracle.ACT_SWIGLU_BOUNDED, -50.0, -50.0, limit=L) == \
        pytest.approx(-50.0 / (1.0 + np.exp(50.0)) * -10.0, rel=1e-15)
    # OAI: g sigmoid(alpha g) (u + 1) with the same clamps
    assert oracle.glu(oracle.ACT_SWIGLU_OAI, 2.0, 3.0, alpha=1.702, limit=7.0) == \
        pytest.approx(2.0 / (1.0 + np.exp(-3.404)) * 4.0, rel=1e-15)
    assert oracle.glu(oracle.ACT_SWIGLU_OAI, 9.0, -9.0, alpha=1.702, limit=7.0) == \
        pytest.approx(7.0 / (1.0 + np.exp(-1.702 * 7.0)) * -6.0, rel=1e-15)
    # ReLU^2 ignores the gate: max(u, 0)^2
    assert oracle.glu(oracle.ACT_RELU2, 123.0, 3.0) == 9.0
    assert oracle.glu(oracle.ACT_RELU2, 1.0, -3.0) == 0.0
    # every gated variant is 0 at g = 0
    for act in range(5):
        assert oracle.glu(act, 0.0, 3.0, alpha=1.702, limit=7.0) == 0.0


def test_gated_activations_match_torch_library_routines():
    rng = np.random.default_rng(0)
    g, u = rng.normal(0, 3, 2000), rng.normal(0, 3, 2000)
    gt, ut = torch.from_numpy(g), torch.from_numpy(u)
    F = torch.nn.functional
    np.testing.assert_allclose(oracle.glu(oracle.ACT_SWIGLU, g, u), (F.silu(gt) * ut).numpy(), rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(oracle.glu(oracle.ACT_GEGLU, g, u), (F.gelu(gt) * ut).numpy(), rtol=1e-13, atol=1e-300)
    np.testing.assert_array_equal(oracle.glu(oracle.ACT_REGLU, g, u), (F.relu(gt) * ut).numpy())
    np.testing.assert_array_equal(oracle.glu(oracle.ACT_RELU2, g, u), (F.relu(ut) ** 2).numpy())
    ref = F.silu(torch.clamp(gt, max=2.0)) * torch.clamp(ut, -2.0, 2.0)
    np.testing.assert_allclose(oracle.glu(oracle.ACT_SWIGLU_BOUNDED, g, u, limit=2.0), ref.numpy(), rtol=1e-14, atol=1e-300)
    gc = torch.clamp(gt, max=2.0)
    ref = gc * torch.sigmoid(1.702 * gc) * (torch.clamp(ut, -2.0, 2.0) + 1.0)
    np.testing.assert_allclose(oracle.glu(oracle.ACT_SWIGLU_OAI, g, u, alpha=1.702, limit=2.0), ref.numpy(),
                               rtol=1e-13, atol=1e-300)


# ------------------------------------------------------------------ MX32 hidden rule
def test_mx32_quant_hand_example():
    x = np.zeros((4, 64), np.float32)
    x[0, 0] = 448.0            # 448 = 0.875 * 2^9 -> e = 0, code 127
    x[0, 32] = 449.0           # just above: e = 1, code 128, 449/2 = 224.5 -> e4m3 224
    x[1, 0] = 1.0              # 1 = 0.5 * 2^1 -> e = -8 (448 / 256 = 1.75 >= 1 > 0.875)
    x[1, 1] = -0.5
    codes, sc = oracle.quant_rows(oracle.FMT_MX32, x)
    assert list(sc[0]) == [127, 128] and list(sc[1]) == [119, 0]
    assert codes[0, 0] == 0x7E and codes[0, 32] == 0x76
    assert codes[1, 0] == 0x78 and codes[1, 1] == 0xF0      # 256 and -128
    assert (sc[2:] == 0).all() and (codes[2:] == 0).all()


def test_mx32_exponent_is_the_smallest_that_fits():
    rng = np.random.default_rng(11)
    x = (rng.normal(size=(16, 256)) * np.exp(rng.uniform(-20, 20, size=(16, 1)))).astype(np.float32)
    codes, sc = oracle.quant_rows(oracle.FMT_MX32, x)
    amax = np.abs(x).reshape(16, 8, 32).max(axis=2).astype(np.float64)
    scale = np.exp2(sc.astype(np.float64) - 127)
    assert (amax <= 448.0 * scale).all() and (amax > 224.0 * scale).all()
    deq = torch_e4m3_value(codes) * np.repeat(scale, 32, axis=1)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, np.repeat(scale, 32, axis=1) * 2.0 ** -10)
    assert (np.abs(deq - x) <= bound).all()


def test_gate_up_mode_rule_hand_cases():
    """The gate/up mode rule on histograms worked out by hand (148 SMs, nb
    256-wide n-blocks, kb K-blocks, per-unit costs kb a + b per mode)."""
    P = 3   # narrow tiles not allowed: single CTAs or pairs
    ps = [1000, 0, 1000, 0, 0, 0]      # equal per-unit cost: only the wave counts decide
    # 8 experts x 8 m-tiles (1024 rows each), nb = 112: single 64 x 112 = 7168
    # units -> 49 waves; pairs 32 x 112 = 3584 units -> ceil(3584 / 74) = 49 waves
    # -> equal cost, the lower mode (single CTAs)
    assert oracle.pick_gu_mode([1024] * 8, 112, 32, 148, ps, P) == 0
    # a pair unit cheaper than a single one (a_1 < a_0) breaks the tie for pairs
    assert oracle.pick_gu_mode([1024] * 8, 112, 32, 148, [1000, 0, 990, 0, 0, 0], P) == 1
    # one m-tile per expert: pairs are half empty -> as many pair units as single
    # ones on half the slots: 160 experts, nb = 4 -> single ceil(640/148) = 5,
    # pairs ceil(640/74) = 9 waves
    assert oracle.pick_gu_mode([100] * 160 + [0] * 96, 4, 16, 148, ps, P) == 0
    # odd counts: 3 m-tiles -> pairs (3 + 1) / 2 = 2 units per expert
    # single 150 x 8 = 1200 units -> 9 waves x 160; pairs 100 x 8 = 800 -> 11 waves
    assert oracle.pick_gu_mode([300] * 50, 8, 16, 148, [10, 0, 6, 0, 0, 0], P) == 1    # 11 x 96 = 1056 < 1440
    assert oracle.pick_gu_mode([300] * 50, 8, 16, 148, [10, 0, 9, 0, 0, 0], P) == 0    # 11 x 144 = 1584 > 1440
    # narrow tiles: 47 experts with one m-tile, nb = 4, kb = 16: wide 188 units ->
    # 2 waves x 16 a_0; narrow 376 units -> 3 waves x 16 a_2; pairs 188 units on
    # 74 -> 3 waves x 16 a_1
    q = [1000, 0, 990, 0, 600, 0]
    h47 = [10] * 47 + [0] * 209
    assert oracle.pick_gu_mode(h47, 4, 16, 148, q) == 2          # 3 x 9600 < 2 x 16000 < 3 x 15840
    assert oracle.pick_gu_mode(h47, 4, 16, 148, [1000, 0, 990, 0, 700, 0]) == 0   # 3 x 11200 > 32000
    # two experts with one m-tile, nb = 112, kb = 32: wide 224 units -> 2 waves,
    # narrow 448 -> 4 waves (3 x 148 = 444 < 448)
    assert oracle.pick_gu_mode([1, 1] + [0] * 6, 112, 32, 148, q) == 0   # 4 x 19200 > 2 x 32000
    # one wave either way (nb = 1, kb = 2): equal per-unit cost ties to wide,
    # a cheaper narrow unit wins
    assert oracle.pick_gu_mode([10] * 8, 1, 2, 148, [5, 0, 9, 0, 5, 0]) == 0
    assert oracle.pick_gu_mode([10] * 8, 1, 2, 148, [5, 0, 9, 0, 4, 0]) == 2
    # the allowed-mode mask: only one mode allowed -> that mode; none -> 0
    assert oracle.pick_gu_mode([1024] * 8, 112, 32, 148, q, 4) == 2
    assert oracle.pick_gu_mode([1, 1] + [0] * 6, 112, 32, 148, q, 2) == 1
    assert oracle.pick_gu_mode([1024] * 8, 112, 32, 148, q, 0) == 0
    # no n-blocks (not a gated FP8_ROW layer) or no rows: mode 0
    assert oracle.pick_gu_mode([1024] * 8, 0, 32, 148, [10, 0, 1, 0, 1, 0]) == 0
    assert oracle.pick_gu_mode([0] * 8, 112, 32, 148, [10, 0, 1, 0, 1, 0]) == 0