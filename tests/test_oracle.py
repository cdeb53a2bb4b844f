"""Pins for the CPU oracle (no GPU).

The oracle is only trusted because these tests tie it to things other than
itself: the E2M1 bit split and 32-element blocks the pages print, the pages'
memory figures, closed forms, invariants, and brute force written here
independently (Python loops over candidate values, math.fsum, torch's own
float32 -> bfloat16 rounding).  Each test says which mistake it would catch.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from moe_expert_gemm_mxfp4_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")
with open(os.path.join(GOLD, "e2m1_value_set.json")) as f:
    E2M1 = json.load(f)
GRID = [float(v) for v in E2M1["magnitudes"]]


# ----------------------------------------------------------------- independent helpers

def torch_bf16_bits(x_f32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns by torch's own round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_float(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def brute_scale_exp(amax: float, rule: int) -> int:
    """Search for the block exponent instead of computing it."""
    if amax == 0.0:
        return -127
    if rule == oracle.FLOOR:       # 4 * 2^s <= amax < 8 * 2^s
        s = next(s for s in range(-200, 200) if 4.0 * 2.0 ** s <= amax < 8.0 * 2.0 ** s)
    else:                          # smallest s with amax <= 6 * 2^s
        s = next(s for s in range(-200, 200) if amax <= 6.0 * 2.0 ** s)
    return max(-127, min(127, s))


def brute_code(v: float, s: int) -> int:
    """Nearest grid value by exhaustive distance, ties to the even code."""
    r = abs(v) / 2.0 ** s
    d = [abs(r - g) for g in GRID]
    best = min(d)
    cands = [i for i, x in enumerate(d) if x == best]
    idx = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
    return (8 if math.copysign(1.0, v) < 0 else 0) | idx


def brute_quantize(vals: np.ndarray, rule: int):
    """Per-block brute force; vals is a float64 1-D array of length 32*n."""
    nb = vals.size // 32
    codes, scales = [], []
    for b in range(nb):
        blk = vals[32 * b:32 * b + 32]
        if not np.all(np.isfinite(blk)):
            scales.append(255)
            codes.extend([0] * 32)
            continue
        s = brute_scale_exp(float(np.max(np.abs(blk))), rule)
        scales.append(s + 127)
        codes.extend(brute_code(float(v), s) for v in blk)
    packed = [codes[2 * j] | (codes[2 * j + 1] << 4) for j in range(len(codes) // 2)]
    return np.array(packed, dtype=np.uint8), np.array(scales, dtype=np.uint8)


def decode_value(code: int, S: int) -> float:
    if S == 255:
        return float("nan")
    v = GRID[code & 7] * 2.0 ** (S - 127)
    return -v if code & 8 else v


def decode_matrix(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    R, half = codes.shape
    out = np.empty((R, 2 * half))
    for r in range(R):
        for i in range(2 * half):
            byte = int(codes[r, i // 2])
            c = (byte >> 4) if i & 1 else (byte & 15)
            out[r, i] = decode_value(c, int(scales[r, i // 32]))
    return out


def bf16_round_ref(x: float) -> float:
    """Round to 8 significant bits, ties to even (normal range only)."""
    if x == 0.0:
        return x
    m, e = math.frexp(x)
    assert -125 < e < 127
    return math.ldexp(round(m * 256.0), e - 8)


# ----------------------------------------------------------------- E2M1 format

def test_e2m1_grid_matches_bit_split():
    """Pages: E2M1 = 1 sign, 2 exponent, 1 mantissa bit.  Catches a wrong bias,
    a swapped exponent/mantissa bit or a mis-placed sign bit."""
    assert [oracle.e2m1_magnitude(c) for c in range(8)] == GRID
    codes = np.array([[c | (c << 4) for c in range(16)]], dtype=np.uint8)   # 32 elements
    scales = np.array([[127]], dtype=np.uint8)
    vals = oracle.dequantize_f64(codes, scales)[0]
    for c in range(16):
        for half in (0, 1):
            v = vals[2 * c + half]
            assert abs(v) == GRID[c & 7]
            assert math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0)
    assert E2M1["block_size"] == 32 and E2M1["sign_bit"] == 3


def test_rne_ties_and_saturation_table():
    """Every tie point goes to the even code; values past 6 saturate."""
    cases = [(0.25, 0.0), (0.3, 0.5), (0.74, 0.5), (0.75, 1.0), (1.25, 1.0),
             (1.26, 1.5), (1.75, 2.0), (2.5, 2.0), (2.51, 3.0), (3.5, 4.0),
             (4.99, 4.0), (5.0, 4.0), (5.01, 6.0), (6.0, 6.0)]
    for s in (-3, 0, 5):
        blk = np.zeros(32, dtype=np.float32)
        blk[0] = 6.0 * 2.0 ** s           # fixes the block exponent at s
        for i, (r, _) in enumerate(cases):
            blk[1 + i] = r * 2.0 ** s
            blk[16 + i] = -r * 2.0 ** s
        codes, scales = oracle.quantize(blk[None, :], oracle.FLOOR)
        assert scales[0, 0] == s + 127
        deq = oracle.dequantize_f64(codes, scales)[0]
        for i, (_, q) in enumerate(cases):
            assert deq[1 + i] == q * 2.0 ** s
            assert deq[16 + i] == -q * 2.0 ** s
    for r in (6.5, 7.0, 7.96875):          # (6, 8) * 2^s saturates under the floor rule
        blk = np.zeros(32, dtype=np.float32)
        blk[0] = r
        codes, scales = oracle.quantize(blk[None, :], oracle.FLOOR)
        assert scales[0, 0] == 127 and (codes[0, 0] & 15) == 7


@pytest.mark.parametrize("rule", [oracle.FLOOR, oracle.CEIL])
def test_exhaustive_bf16_patterns_vs_bruteforce(rule):
    """All 65536 bf16 patterns, 32 consecutive patterns per block (so blocks span
    subnormals, normals, Inf and NaN).  Catches any error in the exponent,
    rounding, sign, saturation, NaN handling or nibble order."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(64, 1024)
    codes, scales = oracle.quantize(bits, rule, dtype="bf16")
    vals = bits_to_float(bits.reshape(-1))
    ref_c, ref_s = brute_quantize(vals, rule)
    assert np.array_equal(codes.reshape(-1), ref_c)
    assert np.array_equal(scales.reshape(-1), ref_s)


@pytest.mark.parametrize("rule", [oracle.FLOOR, oracle.CEIL])
def test_random_f32_vs_bruteforce(rule):
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(16, 256, generator=g) * torch.exp(torch.randn(16, 256, generator=g) * 4)).numpy()
    codes, scales = oracle.quantize(x, rule)
    ref_c, ref_s = brute_quantize(x.astype(np.float64).reshape(-1), rule)
    assert np.array_equal(codes.reshape(-1), ref_c)
    assert np.array_equal(scales.reshape(-1), ref_s)


def test_scale_closed_forms():
    """amax = 2^j * {1, 1.5, 1.99} -> byte j+125 (floor); ceil gives j+126 for 1.99;
    amax = 6 * 2^j -> byte j+127 under both rules."""
    for j in (-100, -10, 0, 7, 100):
        for m, fl, ce in ((1.0, 125, 125), (1.5, 125, 125), (1.99, 125, 126), (6.0, 127, 127)):
            blk = np.zeros((1, 32), dtype=np.float32)
            blk[0, 5] = m * 2.0 ** j
            assert oracle.quantize(blk, oracle.FLOOR)[1][0, 0] == j + fl
            assert oracle.quantize(blk, oracle.CEIL)[1][0, 0] == j + ce


def test_special_blocks():
    zero = np.zeros((1, 32), dtype=np.float32)
    c, s = oracle.quantize(zero)
    assert s[0, 0] == 0 and not c.any()
    negzero = np.full((1, 32), -0.0, dtype=np.float32)
    c, s = oracle.quantize(negzero)
    assert s[0, 0] == 0 and np.all(c == 0x88)
    for bad in (np.inf, -np.inf, np.nan):
        blk = np.ones((1, 32), dtype=np.float32)
        blk[0, 3] = bad
        c, s = oracle.quantize(blk)
        assert s[0, 0] == 0xFF and not c.any()
        assert np.all(np.isnan(oracle.dequantize_f64(c, s)))
    # bf16 subnormal amax: exponent clamps to -127; 127 * 2^-133 / 2^-127 = 1.98 -> 2
    bits = np.zeros((1, 32), dtype=np.uint16)
    bits[0, 0] = 0x007F
    c, s = oracle.quantize(bits, dtype="bf16")
    assert s[0, 0] == 0 and (c[0, 0] & 15) == 4
    # tiny negative rounds to -0 (code 8)
    blk = np.zeros((1, 32), dtype=np.float32)
    blk[0, 0], blk[0, 1] = 4.0, -0.01
    c, s = oracle.quantize(blk)
    assert (c[0, 0] >> 4) == 8


def test_dequantize_every_scale_and_code():
    """All 256 scale bytes x 16 codes against an independent decode, in fp64 and
    bf16 (the only rounding possible is overflow to Inf)."""
    codes = np.tile(np.array([c | (c << 4) for c in range(16)], dtype=np.uint8), (256, 1))
    scales = np.arange(256, dtype=np.uint8).reshape(256, 1)
    f = oracle.dequantize_f64(codes, scales)
    b = oracle.dequantize_bf16(codes, scales)
    for S in range(256):
        for i in range(32):
            ref = decode_value(i // 2, S)
            if math.isnan(ref):
                assert math.isnan(f[S, i]) and (b[S, i] & 0x7FFF) > 0x7F80
                continue
            assert f[S, i] == ref and math.copysign(1, f[S, i]) == math.copysign(1, ref)
            if abs(ref) >= 2.0 ** 128:
                assert b[S, i] == (0xFF80 if ref < 0 else 0x7F80)
            else:
                assert b[S, i] == (np.float32(ref).view(np.uint32) >> 16)


def test_bf16_rounding_vs_torch():
    """oracle.f64_to_bf16 on float32-representable inputs equals torch's own
    float32 -> bfloat16 rounding (covers ties, subnormals and overflow)."""
    g = torch.Generator().manual_seed(5)
    raw = torch.randint(0, 2 ** 32, (200000,), generator=g, dtype=torch.int64)
    f32 = raw.to(torch.int32).numpy().view(np.float32)
    f32 = f32[np.isfinite(f32)]
    special = np.array([2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135, 2.0 ** -149, 3.3895e38,
                        (2 - 2 ** -8) * 2.0 ** 127, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8,
                        -(1.0 + 2 ** -8)], dtype=np.float32)
    f32 = np.concatenate([f32, special])
    ours = oracle.f64_to_bf16(f32.astype(np.float64))
    ref = torch_bf16_bits(f32)
    assert np.array_equal(ours, ref)


# ----------------------------------------------------------------- invariants

def _data(seed=3, shape=(64, 512)):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * 3).numpy()


def test_roundtrip_invariants():
    x = _data()
    c, s = oracle.quantize(x, oracle.FLOOR)
    d = oracle.dequantize_bf16(c, s)
    c2, s2 = oracle.quantize(d, oracle.FLOOR, dtype="bf16")
    assert np.array_equal(c, c2) and np.array_equal(s, s2)          # quant(deq(quant)) == quant
    for rule in (oracle.FLOOR, oracle.CEIL):
        c, s = oracle.quantize(x, rule)
        d1 = oracle.dequantize_f64(c, s)
        c3, s3 = oracle.quantize(d1.astype(np.float32), rule)
        assert np.array_equal(oracle.dequantize_f64(c3, s3), d1)     # deq o quant idempotent
    # sign symmetry
    cn, sn = oracle.quantize(-x, oracle.FLOOR)
    cp, sp = oracle.quantize(x, oracle.FLOOR)
    assert np.array_equal(sn, sp) and np.array_equal(cn, cp ^ 0x88)
    # power-of-two scaling moves only the scale
    for j in (-5, 3):
        cj, sj = oracle.quantize((x * 2.0 ** j).astype(np.float32), oracle.FLOOR)
        assert np.array_equal(cj, cp) and np.array_equal(sj.astype(int), sp.astype(int) + j)


def test_on_grid_blocks_are_exact():
    g = torch.Generator().manual_seed(9)
    codes = torch.randint(0, 256, (8, 64), generator=g, dtype=torch.int64).numpy().astype(np.uint8)
    codes[:, ::16] |= 0x07     # every block holds a magnitude-6 element -> its scale is kept
    scales = torch.randint(100, 150, (8, 4), generator=g, dtype=torch.int64).numpy().astype(np.uint8)
    vals = oracle.dequantize_f64(codes, scales).astype(np.float32)
    c, s = oracle.quantize(vals, oracle.FLOOR)
    assert np.array_equal(s, scales)
    assert np.array_equal(oracle.dequantize_f64(c, s), vals.astype(np.float64))


def test_error_bound_floor_rule():
    x = _data(seed=4).astype(np.float64)
    c, s = oracle.quantize(x.astype(np.float32), oracle.FLOOR)
    d = oracle.dequantize_f64(c, s)
    scale = np.repeat(2.0 ** (s.astype(np.float64) - 127), 32, axis=1)
    r = np.abs(x) / scale
    gap = np.where(r < 2, 0.5, np.where(r < 4, 1.0, 2.0))
    err = np.abs(x - d) / scale
    unsat = r <= 6
    assert np.all(err[unsat] <= gap[unsat] / 2)
    assert np.all(err[~unsat] < 2.0)


def test_storage_ratio_matches_pages_memory_figures():
    """4 bits per code + one 8-bit scale per 32 codes = 4.25 bits per weight:
    0.265625 x bf16.  The pages' figures (~16 GB vs ~64 GB; ~80 GB vs > 300 GB;
    bf16 fallback ~4x the memory) follow from that ratio."""
    with open(os.path.join(GOLD, "memory_figures.json")) as f:
        mem = json.load(f)
    N, K = 5760, 2880
    c, s = oracle.quantize(np.zeros((N, K), dtype=np.float32))
    ratio = (c.nbytes + s.nbytes) / (N * K * 2)
    assert ratio == 0.265625
    assert abs(mem["gpt_oss_20b"]["bf16_gb"] * ratio - mem["gpt_oss_20b"]["mxfp4_gb"]) < 1.5
    assert abs(mem["gpt_oss_120b"]["bf16_gb_at_least"] * ratio - mem["gpt_oss_120b"]["mxfp4_gb"]) < 1.0
    assert abs(1 / ratio - mem["fallback_ratio"]) < 0.25
    # the 120b-shaped layer: 128 experts of [5760, 2880] + [2880, 2880] -> ~1.7 GB packed
    per_expert = (5760 * 2880 + 2880 * 2880) * 0.53125
    assert per_expert * 128 == 1_692_057_600


# ----------------------------------------------------------------- routing

def test_route_bruteforce():
    g = torch.Generator().manual_seed(21)
    T, E, k = 40, 12, 4
    logits = torch.randn(T, E, generator=g).numpy()
    logits[0, :] = 0.5            # all equal: ties go to the lowest ids
    logits[1, [3, 7, 9]] = 2.0    # a three-way tie at the top
    r = oracle.route(logits, k)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        assert list(r["ids"][t]) == order
        z = [math.exp(float(logits[t, e]) - float(logits[t, order[0]])) for e in order]
        tot = math.fsum(z)
        assert np.allclose(r["w"][t], [v / tot for v in z], rtol=1e-14, atol=0)
        assert abs(r["w"][t].sum() - 1.0) < 1e-12
    flat = r["ids"].reshape(-1)
    assert r["counts"].sum() == T * k
    assert np.array_equal(r["counts"], [int((flat == e).sum()) for e in range(E)])
    assert r["offsets"][0] == 0 and np.all(np.diff(r["offsets"]) == r["counts"])
    assert np.array_equal(np.sort(r["perm"]), np.arange(T * k))
    assert np.array_equal(r["inv"][r["perm"]], np.arange(T * k))
    for e in range(E):
        seg = r["perm"][r["offsets"][e]:r["offsets"][e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


def test_route_nan_logits_rank_below_every_number():
    # Reading: a NaN router logit ranks below every number, -inf included; NaNs
    # among themselves by expert id.  Brute force with that key.
    g = torch.Generator().manual_seed(22)
    T, E, k = 12, 9, 4
    logits = torch.randn(T, E, generator=g).numpy()
    logits[0, [1, 4]] = np.nan
    logits[1, :] = np.nan                      # all NaN: ids 0..k-1, NaN weights
    logits[2, [0, 2, 3, 5, 6, 7, 8]] = np.nan  # two numbers, then NaNs by id
    logits[3, [2, 6]] = -np.inf
    logits[3, [0, 1, 3, 4, 5]] = np.nan        # -inf ranks above NaN
    r = oracle.route(logits, k)

    def key(t, e):
        v = float(logits[t, e])
        return (1, 0.0, e) if math.isnan(v) else (0, -v, e)

    for t in range(T):
        order = sorted(range(E), key=lambda e: key(t, e))[:k]
        assert list(r["ids"][t]) == order, t
    assert list(r["ids"][2][:2]) == [1, 4] and np.isnan(r["w"][2]).all()
    assert sorted(r["ids"][3][:2]) == [7, 8] and list(r["ids"][3][2:]) == [2, 6]   # -inf above NaN
    assert np.isnan(r["w"][1]).all()
    assert np.all(np.isfinite(r["w"][4:]))


def test_moe_down_fed_with_moe_mlp_h_reproduces_moe_mlp():
    # the staged check's reference: moe_down(h of moe_mlp) is moe_mlp, bit for bit,
    # in both modes
    g = torch.Generator().manual_seed(23)
    T, H, I, E, k = 9, 64, 96, 5, 2
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    logits = torch.randn(T, E, generator=g).numpy()
    q13 = [oracle.quantize((torch.randn(2 * I, H, generator=g) * 0.1).numpy()) for _ in range(E)]
    q2 = [oracle.quantize((torch.randn(H, I, generator=g) * 0.1).numpy()) for _ in range(E)]
    w13c, w13s = np.stack([a for a, _ in q13]), np.stack([b for _, b in q13])
    w2c, w2s = np.stack([a for a, _ in q2]), np.stack([b for _, b in q2])
    for mode in ("w4a16", "w4a4"):
        out, h = oracle.moe_mlp(xb, logits, k, w13c, w13s, w2c, w2s, mode=mode, return_h=True)
        hb = oracle.f64_to_bf16(h)
        assert np.array_equal(oracle.moe_down(hb, logits, k, w2c, w2s, mode=mode), out)
        tok = np.array([1, 4, 8])
        assert np.array_equal(oracle.moe_down(hb[tok], logits, k, w2c, w2s, mode=mode, tokens=tok), out[tok])


def test_router_logits_bruteforce():
    g = torch.Generator().manual_seed(24)
    T, E, H = 5, 7, 96
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    w = (torch.randn(E, H, generator=g) * 0.1).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    got = oracle.router_logits(xb, wb)
    assert got.shape == (T, E)
    xf, wf = x.double().numpy(), w.double().numpy()
    for t in range(T):
        for e in range(E):
            assert got[t, e] == pytest.approx(math.fsum(float(xf[t, h]) * float(wf[e, h]) for h in range(H)),
                                              rel=1e-15, abs=1e-300)
    # a one-hot token picks a router column exactly; transposed operands would not
    onehot = np.zeros((1, H), np.uint16)
    onehot[0, 17] = 0x3F80                     # 1.0
    assert np.array_equal(oracle.router_logits(onehot, wb)[0], wf[:, 17])


def test_moe_mlp_dense_with_dequantized_weights_is_moe_mlp():
    # the bf16-weight layer's reference, fed the bf16 values of MXFP4 weights, is the
    # (pinned) MXFP4 layer bit for bit; a swapped gate/up or a missing weight would not be
    g = torch.Generator().manual_seed(25)
    T, H, I, E, k = 11, 64, 96, 4, 2
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    logits = torch.randn(T, E, generator=g).numpy()
    q13 = [oracle.quantize((torch.randn(2 * I, H, generator=g) * 0.1).numpy()) for _ in range(E)]
    q2 = [oracle.quantize((torch.randn(H, I, generator=g) * 0.1).numpy()) for _ in range(E)]
    w13c, w13s = np.stack([a for a, _ in q13]), np.stack([b for _, b in q13])
    w2c, w2s = np.stack([a for a, _ in q2]), np.stack([b for _, b in q2])
    ref = oracle.moe_mlp(xb, logits, k, w13c, w13s, w2c, w2s)
    w13b = oracle.dequantize_bf16(w13c, w13s)
    w2b = oracle.dequantize_bf16(w2c, w2s)
    assert np.array_equal(oracle.moe_mlp_dense(xb, logits, k, w13b, w2b), ref)
    swapped = np.concatenate([w13b[:, I:], w13b[:, :I]], axis=1)
    assert not np.allclose(oracle.moe_mlp_dense(xb, logits, k, swapped, w2b), ref)


# ----------------------------------------------------------------- GEMM

def test_gemm_bruteforce():
    g = torch.Generator().manual_seed(31)
    for M, N, K in ((1, 8, 32), (3, 64, 64), (8, 16, 96)):
        x = torch.randn(M, K, generator=g).to(torch.bfloat16)
        xb = x.view(torch.int16).numpy().view(np.uint16)
        w = (torch.randn(N, K, generator=g) * 0.05).numpy()
        c, s = oracle.quantize(w)
        wv = decode_matrix(c, s)
        xv = x.double().numpy()
        y = oracle.gemm_w4a16(xb, c, s)
        for m in range(M):
            for n in range(N):
                terms = [xv[m, kk] * wv[n, kk] for kk in range(K)]
                ref = math.fsum(terms)
                assert abs(y[m, n] - ref) <= 1e-13 * math.fsum(abs(t) for t in terms) + 1e-300


def test_gemm_closed_forms():
    g = torch.Generator().manual_seed(32)
    M, N, K = 4, 24, 128
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    for S in (120, 127, 131):
        c = np.full((N, K // 2), 0x22, dtype=np.uint8)     # every code = 1.0
        s = np.full((N, K // 32), S, dtype=np.uint8)
        y = oracle.gemm_w4a16(xb, c, s)
        rows = x.double().numpy().sum(axis=1) * 2.0 ** (S - 127)
        assert np.allclose(y, rows[:, None], rtol=1e-14, atol=1e-14)
    w = (torch.randn(N, K, generator=g) * 0.05).numpy()
    c, s = oracle.quantize(w)
    wv = decode_matrix(c, s)
    for kk in (0, 37, K - 1):
        onehot = np.zeros((1, K), dtype=np.uint16)
        onehot[0, kk] = 0x3F80                              # bf16 1.0
        assert np.array_equal(oracle.gemm_w4a16(onehot, c, s)[0], wv[:, kk])


def test_w4a4_equals_w4a16_on_grid_activations():
    g = torch.Generator().manual_seed(33)
    M, N, K = 5, 32, 128
    xc = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.int64).numpy().astype(np.uint8)
    xc[:, ::16] |= 0x07
    xs = torch.randint(120, 134, (M, K // 32), generator=g, dtype=torch.int64).numpy().astype(np.uint8)
    xb = oracle.dequantize_bf16(xc, xs)
    w = (torch.randn(N, K, generator=g) * 0.05).numpy()
    c, s = oracle.quantize(w)
    assert np.array_equal(oracle.gemm_w4a4(xb, c, s), oracle.gemm_w4a16(xb, c, s))
    # and off the grid they differ (the activation quantization is really applied)
    xr = torch.randn(M, K, generator=g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert not np.allclose(oracle.gemm_w4a4(xr, c, s), oracle.gemm_w4a16(xr, c, s))


# ----------------------------------------------------------------- MoE MLP

def _tiny_moe(seed, T=5, H=64, I=32, E=4, k=2, same_experts=False):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    logits = torch.randn(T, E, generator=g).numpy()
    w13 = [(torch.randn(2 * I, H, generator=g) * 0.2).numpy() for _ in range(E)]
    w2 = [(torch.randn(H, I, generator=g) * 0.2).numpy() for _ in range(E)]
    if same_experts:
        w13 = [w13[0]] * E
        w2 = [w2[0]] * E
    q13 = [oracle.quantize(w) for w in w13]
    q2 = [oracle.quantize(w) for w in w2]
    return dict(x=x, logits=logits, k=k, I=I,
                w13c=np.stack([q[0] for q in q13]), w13s=np.stack([q[1] for q in q13]),
                w2c=np.stack([q[0] for q in q2]), w2s=np.stack([q[1] for q in q2]))


def _run(m, mode="w4a16", **kw):
    return oracle.moe_mlp(m["x"], m["logits"], m["k"], m["w13c"], m["w13s"],
                          m["w2c"], m["w2s"], mode=mode, **kw)


def test_moe_bruteforce_loops():
    """Plain loops over tokens, slots, features: gate = rows [0, I), up = rows
    [I, 2I), h rounded to bf16, weighted sum of the k expert outputs."""
    m = _tiny_moe(41)
    out = _run(m)
    x = bits_to_float(m["x"])
    T, H = x.shape
    E, I, k = m["w13c"].shape[0], m["I"], m["k"]
    W13 = [decode_matrix(m["w13c"][e], m["w13s"][e]) for e in range(E)]
    W2 = [decode_matrix(m["w2c"][e], m["w2s"][e]) for e in range(E)]
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(m["logits"][t, e]), e))[:k]
        z = [math.exp(float(m["logits"][t, e]) - float(m["logits"][t, order[0]])) for e in order]
        ws = [v / math.fsum(z) for v in z]
        acc = [0.0] * H
        for j, e in enumerate(order):
            h = []
            for i in range(I):
                gte = math.fsum(x[t, c] * W13[e][i, c] for c in range(H))
                up = math.fsum(x[t, c] * W13[e][I + i, c] for c in range(H))
                h.append(bf16_round_ref(gte / (1.0 + math.exp(-gte)) * up))
            for n in range(H):
                acc[n] += ws[j] * math.fsum(h[i] * W2[e][n, i] for i in range(I))
        assert np.allclose(out[t], acc, rtol=1e-10, atol=1e-12)


def test_moe_identical_experts_independent_of_routing():
    m = _tiny_moe(42, same_experts=True)
    out = _run(m)
    x = m["x"]
    g = oracle.gemm_w4a16(x, m["w13c"][0], m["w13s"][0])
    I = m["I"]
    h = oracle.f64_to_bf16(oracle.silu(g[:, :I]) * g[:, I:])
    dense = oracle.gemm_w4a16(h, m["w2c"][0], m["w2s"][0])
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-14)
    m2 = dict(m, logits=m["logits"][:, ::-1].copy())
    assert np.allclose(_run(m2), dense, rtol=1e-12, atol=1e-14)


def test_moe_top1_is_the_selected_experts_dense_mlp():
    m = _tiny_moe(43, E=3, k=1)
    out = _run(m)
    ids = oracle.route(m["logits"], 1)["ids"][:, 0]
    I = m["I"]
    for t, e in enumerate(ids):
        g = oracle.gemm_w4a16(m["x"][t:t + 1], m["w13c"][e], m["w13s"][e])
        h = oracle.f64_to_bf16(oracle.silu(g[:, :I]) * g[:, I:])
        y = oracle.gemm_w4a16(h, m["w2c"][e], m["w2s"][e])
        assert np.allclose(out[t], y[0], rtol=1e-13, atol=1e-15)


def test_moe_token_subset_matches_full():
    m = _tiny_moe(44, T=9, E=5, k=3)
    full = _run(m)
    sub = _run(m, tokens=[7, 2, 4])
    assert np.array_equal(sub, full[[7, 2, 4]])
    full4 = _run(m, mode="w4a4")
    assert np.array_equal(_run(m, mode="w4a4", tokens=[1, 8]), full4[[1, 8]])


def test_moe_w4a4_quantizes_both_activations():
    """W4A4 with x already on the grid still differs from W4A16 (h is quantized),
    and equals a hand-assembled pipeline that quantizes x and h."""
    m = _tiny_moe(45, E=2, k=1)
    out4 = _run(m, mode="w4a4")
    ids = oracle.route(m["logits"], 1)["ids"][:, 0]
    I = m["I"]
    for t, e in enumerate(ids):
        xq = oracle.dequantize_bf16(*oracle.quantize(m["x"][t:t + 1], dtype="bf16"))
        g = oracle.gemm_w4a16(xq, m["w13c"][e], m["w13s"][e])
        h = oracle.f64_to_bf16(oracle.silu(g[:, :I]) * g[:, I:])
        hq = oracle.dequantize_bf16(*oracle.quantize(h, dtype="bf16"))
        y = oracle.gemm_w4a16(hq, m["w2c"][e], m["w2s"][e])
        assert np.allclose(out4[t], y[0], rtol=1e-13, atol=1e-15)
    assert not np.allclose(out4, _run(m))


# ----------------------------------------------------------------- inputs recipe

def test_quant_workload_recipe_statistics():
    x = inputs.quant_tensor(rows=256, cols=11520)
    v = x.float().view(256, -1, 32)
    zero_blocks = (v == 0).all(dim=2).float().mean().item()
    assert 0.003 < zero_blocks < 0.008
    big = (x.float().abs() > 8).float().mean().item()
    assert 0.005 < big < 0.015
