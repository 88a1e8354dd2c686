"""Pins of the CPU oracle against what the format and the mathematics fix.

None of these re-types the oracle's own algorithm: each pin uses another route
-- the format's bit-field definition, torch's float8_e4m3fn cast (a library
round-to-nearest-even), exact rational arithmetic, hand-derived worked
examples under tests/golden/, invariants (monotonicity, nearest-value, error
bounds) and closed forms (one-hot GEMMs, segment scaling) -- so that a dropped
term, a wrong sign or index, or a transposed operand in the oracle fails here.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def f32(x):
    return np.float32(x)


def all_bf16_nonneg_finite():
    bits = np.arange(0, 0x7F80, dtype=np.uint32)  # +0 .. largest finite
    return (bits << 16).view(np.float32)


# ---------------------------------------------------------------------------
# E2M1 element format
# ---------------------------------------------------------------------------

def e2m1_from_fields(code):
    """E2M1 value from its bit fields: sign | 2-bit exponent | 1-bit mantissa."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return s * (m / 2.0) * 2.0 ** (1 - 1)
    return s * (1.0 + m / 2.0) * 2.0 ** (e - 1)


def test_e2m1_values_golden(golden_dir):
    for line in read_golden(os.path.join(golden_dir, "e2m1_values.txt")):
        code, val = line.split()
        got = oracle.e2m1_value(int(code))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))
        assert got == e2m1_from_fields(int(code))


def test_e2m1_rne_golden(golden_dir):
    for line in read_golden(os.path.join(golden_dir, "e2m1_rne_points.txt")):
        t, code = line.split()
        assert int(oracle.e2m1_encode(np.array([float(t)], np.float32))[0]) == int(code), t


def test_e2m1_roundtrip_representable():
    vals = np.array([e2m1_from_fields(c) for c in range(16) if c != 8], np.float32)
    codes = oracle.e2m1_encode(vals)
    back = np.array([oracle.e2m1_value(int(c)) for c in codes])
    assert np.array_equal(back, vals.astype(np.float64))


def _nearest_dist(t):
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    return np.min(np.abs(np.minimum(np.abs(t.astype(np.float64)), 6.0)[:, None] - grid[None, :]), axis=1)


@pytest.mark.parametrize("d", [1.0, 0.5, 2.0 ** -7, 3.0, 1.0 / 3.0])
def test_e2m1_exhaustive_bf16_nearest_and_monotone(d):
    # every non-negative finite BF16 divided by d (an FP32 division, as in the
    # quantizer); the chosen value must be a nearest one, ties to an even code,
    # and the map must be monotone in t.
    with np.errstate(over="ignore"):
        t = (all_bf16_nonneg_finite() / np.float32(d)).astype(np.float32)
    codes = oracle.e2m1_encode(t)
    vals = np.array([oracle.e2m1_value(c) for c in range(8)])[codes & 7]
    err = np.abs(np.minimum(t.astype(np.float64), 6.0) - vals)
    best = _nearest_dist(t)
    assert np.all(err == best)
    tie = np.isclose(err, best) & (err > 0)
    # at exact midpoints both neighbours are at distance err: the even code wins
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    mids = (grid[1:] + grid[:-1]) / 2
    at_mid = np.isin(t.astype(np.float64), mids)
    assert np.all((codes[at_mid & tie] & 1) == 0)
    order = np.argsort(t, kind="stable")
    assert np.all(np.diff(vals[order]) >= 0)
    # negative inputs mirror positive ones with the sign bit set
    cn = oracle.e2m1_encode(-t)
    assert np.array_equal(cn, codes | 8)


def test_e2m1_saturates_and_keeps_sign_of_zero():
    t = np.array([6.0, 6.0001, 1e38, np.inf, -np.inf, -0.0, 0.0, -1e-30], np.float32)
    assert list(oracle.e2m1_encode(t)) == [7, 7, 7, 7, 15, 8, 0, 8]


# ---------------------------------------------------------------------------
# E4M3 scale format
# ---------------------------------------------------------------------------

def e4m3_from_fields(code):
    e = (code >> 3) & 15
    m = code & 7
    if e == 0:
        return m * 2.0 ** -9
    return (1 + m / 8.0) * 2.0 ** (e - 7)


def test_e4m3_values_fields_and_torch():
    codes = np.arange(0, 0x7F, dtype=np.uint8)
    lib = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    for c in codes:
        v = oracle.e4m3_value(int(c))
        assert v == e4m3_from_fields(int(c)) == float(lib[c])
    assert oracle.e4m3_value(0x7E) == 448.0
    assert math.isnan(oracle.e4m3_value(0x7F))


def test_e4m3_rne_golden(golden_dir):
    for line in read_golden(os.path.join(golden_dir, "e4m3_rne_points.txt")):
        v, code = line.split()
        assert int(oracle.e4m3_encode(np.array([float(v)], np.float32))[0]) == int(code, 16), v


def test_e4m3_encode_matches_torch_cast_exhaustive_bf16():
    s = all_bf16_nonneg_finite()
    s = s[s < 464.0]                 # torch's cast has no saturation above this
    ours = oracle.e4m3_encode(s)
    ref = torch.from_numpy(s.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_matches_torch_cast_random_fp32():
    rng = np.random.default_rng(123)
    s = np.concatenate([rng.uniform(0, 463.99, 400_000),
                        np.exp(rng.uniform(np.log(1e-6), np.log(460), 400_000))]).astype(np.float32)
    ours = oracle.e4m3_encode(s)
    ref = torch.from_numpy(s.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates_at_448():
    s = np.array([448.0, 463.9, 464.0, 500.0, 3e38, np.inf], np.float32)
    assert np.all(oracle.e4m3_encode(s) == 0x7E)


# ---------------------------------------------------------------------------
# FP64 -> BF16 single rounding
# ---------------------------------------------------------------------------

def test_bf16_round_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(200_000) * np.exp(rng.uniform(-30, 30, 200_000))).astype(np.float32)
    ours = oracle.bf16_from_double(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_round_single_step_ties_and_overflow():
    one = 1.0
    ulp = 2.0 ** -7
    cases = [
        (one + ulp / 2, 0x3F80),                 # tie -> even (1.0)
        (one + 3 * ulp / 2, 0x3F82),             # tie -> even (1 + 2ulp)
        (one + ulp / 2 + 2.0 ** -40, 0x3F81),    # just above the tie: up (a
                                                 # detour through FP32 would tie)
        (-(one + ulp / 2 + 2.0 ** -40), 0xBF81),
        (3.4e38, 0x7F80),                        # rounds past the largest finite
        (3.3895313892515355e38, 0x7F7F),
        (0.0, 0x0000), (-0.0, 0x8000),
        (2.0 ** -133, 0x0001),                   # smallest BF16 subnormal
        (2.0 ** -134, 0x0000),                   # tie with zero -> even (zero)
        (1.5 * 2.0 ** -133, 0x0002),             # tie between 1 and 2 -> 2
    ]
    for x, want in cases:
        assert int(oracle.bf16_from_double(np.array([x]))[0]) == want, x


# ---------------------------------------------------------------------------
# Step 1: global scale
# ---------------------------------------------------------------------------

def bf16_bits_of(arr):
    return torch.from_numpy(np.asarray(arr, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_global_scale_zero_tensor():
    g, amax = oracle.global_scale(np.zeros((3, 32), np.uint16))
    assert g == 1.0 and amax == 0.0


def test_global_scale_is_correctly_rounded_quotient():
    rng = np.random.default_rng(5)
    for trial in range(50):
        x = rng.standard_normal((7, 48)).astype(np.float32) * np.float32(10 ** rng.uniform(-20, 20))
        bits = bf16_bits_of(x)
        g, amax = oracle.global_scale(bits)
        vals = oracle.bf16_bits_to_f64(bits)
        assert amax == np.max(np.abs(vals))           # exact maximum
        q = Fraction(float(amax)) / 2688
        lo = np.nextafter(g, np.float32(0), dtype=np.float32)
        hi = np.nextafter(g, np.float32(np.inf), dtype=np.float32)
        dg = abs(Fraction(float(g)) - q)
        assert dg <= abs(Fraction(float(lo)) - q) and dg <= abs(Fraction(float(hi)) - q)


def test_global_scale_closed_forms():
    for amax, want in [(2688.0, 1.0), (1344.0, 0.5), (6.0 * 448.0 * 2 ** -20, 2 ** -20)]:
        x = np.zeros((2, 32), np.float32)
        x[1, 5] = -amax
        g, a = oracle.global_scale(bf16_bits_of(x))
        assert a == amax and g == np.float32(want)


# ---------------------------------------------------------------------------
# Steps 2-3: block scales and codes
# ---------------------------------------------------------------------------

def test_quantize_worked_blocks(golden_dir):
    for line in read_golden(os.path.join(golden_dir, "quantize_worked_blocks.txt")):
        name, g, vals, s8, codes = [p.strip() for p in line.split("|")]
        x = np.array([float(v) for v in vals.split()], np.float32)[None, :]
        bits = bf16_bits_of(x)
        assert np.array_equal(oracle.bf16_bits_to_f64(bits)[0], x[0].astype(np.float64)), name
        c, sf = oracle.quantize(bits, float(g))
        assert int(sf[0, 0]) == int(s8, 16), name
        assert [int(b) for b in c[0]] == [int(h, 16) for h in codes.split()], name


def test_absmax_block_gets_largest_scale():
    rng = np.random.default_rng(11)
    for _ in range(20):
        x = (rng.standard_t(3, (9, 64)) * 10 ** rng.uniform(-3, 3)).astype(np.float32)
        bits = bf16_bits_of(x)
        g, amax = oracle.global_scale(bits)
        _, sf = oracle.quantize(bits, g)
        vals = np.abs(oracle.bf16_bits_to_f64(bits))
        r, c = np.unravel_index(np.argmax(vals), vals.shape)
        assert sf[r, c // 16] == 0x7E


def test_block_scale_tracks_absmax_over_6():
    # dec(s8) * g is within the E4M3 half-spacing of (block absmax / 6)
    rng = np.random.default_rng(3)
    x = (rng.standard_t(3, (64, 256)) * np.exp(rng.uniform(-4, 4, (64, 1)))).astype(np.float32)
    bits = bf16_bits_of(x)
    g, _ = oracle.global_scale(bits)
    _, sf = oracle.quantize(bits, g)
    vals = np.abs(oracle.bf16_bits_to_f64(bits)).reshape(64, 16, 16)
    ab = vals.max(axis=2)
    target = ab / 6.0 / float(g)
    dec = np.vectorize(oracle.e4m3_value)(sf)
    normal = target >= 2.0 ** -6
    assert np.all(np.abs(dec[normal] - target[normal]) <= target[normal] * 2.0 ** -4 * (1 + 1e-6))
    assert np.all(np.abs(dec[~normal] - target[~normal]) <= 2.0 ** -10 * (1 + 1e-6))


# (block absmax, global scale as float32 bits): inputs near an E4M3 rounding
# midpoint where fl32(fl32(ab / 6) / g) and the one-division alternative
# fl32(ab / fl32(6 g)) round to different scale codes, in both directions
BLOCK_SCALE_ORDER_CASES = [
    (1.0078125, 0x3EA1E1E1), (1.0625, 0x3EAAAAAA), (1.0390625, 0x3EA6E6E6),
    (1.1640625, 0x3EBAFAFA), (1.1640625, 0x3E3AFAFA), (1.3828125, 0x3E5E1E1D),
    (1.328125, 0x3E1DAE61), (1.4375, 0x3E2AAAAB), (1.0546875, 0x3D555556),
    (1.109375, 0x3D606523),
]


def test_block_scale_is_two_float32_divisions():
    # the block scale takes the fixed sequence fl32(fl32(ab / 6) / g), then
    # E4M3 RNE: evaluated here with numpy's IEEE float32 division and torch's
    # float8_e4m3fn cast, on inputs where the order of the operations decides
    # the code (the alternative order must give another code, or the case
    # would prove nothing)
    for ab, gbits in BLOCK_SCALE_ORDER_CASES:
        g = np.array([gbits], np.uint32).view(np.float32)[0]
        spec = f32(f32(f32(ab) / f32(6.0)) / g)
        alt = f32(f32(ab) / f32(f32(6.0) * g))
        e4 = [int(torch.tensor([v]).to(torch.float8_e4m3fn).view(torch.uint8)[0]) for v in (spec, alt)]
        assert e4[0] != e4[1], (ab, hex(gbits))
        x = np.zeros((1, 16), np.float32)
        x[0, 0], x[0, 5] = ab, -ab / 2
        _, sf = oracle.quantize(bf16_bits_of(x), float(g))
        assert int(sf[0, 0]) == e4[0], (ab, hex(gbits))


def test_element_code_is_a_true_division_at_ties():
    # g = 1 and block absmax 11.25 give s8 = E4M3(1.875) = 0x3F and d = 1.875.
    # 2.34375, 4.6875 and 9.375 are exactly 1.25 d, 2.5 d and 5 d: E2M1 ties
    # that go to the even code (1.0, 2.0, 4.0).  1/1.875 is not a float32, so
    # a reciprocal multiply would land just above each tie and round up.
    x = np.zeros((1, 16), np.float32)
    x[0, :6] = [11.25, 2.34375, 4.6875, 9.375, -2.34375, -4.6875]
    codes, sf = oracle.quantize(bf16_bits_of(x), 1.0)
    assert int(sf[0, 0]) == 0x3F
    nib = [(int(b) >> (4 * h)) & 15 for b in codes[0] for h in (0, 1)]
    assert nib[:6] == [0x7, 0x2, 0x4, 0x6, 0xA, 0xC]
    assert nib[6:] == [0] * 10


def test_dequantization_error_bound():
    # |x - xhat| <= half the E2M1 spacing at |x/d| times d (plus the FP32
    # rounding of x/d), or the clip error when |x/d| > 6.
    rng = np.random.default_rng(9)
    x = (rng.standard_t(3, (32, 512)) * 0.7).astype(np.float32)
    x[:, 17] *= 200
    bits = bf16_bits_of(x)
    g, _ = oracle.global_scale(bits)
    codes, sf = oracle.quantize(bits, g)
    xh = oracle.dequantize_noglobal(codes, sf) * float(g)
    xv = oracle.bf16_bits_to_f64(bits)
    d = np.repeat(np.vectorize(oracle.e4m3_value)(sf), 16, axis=1) * float(g)
    d32 = d.astype(np.float32).astype(np.float64)
    t = np.abs(xv) / np.where(d32 > 0, d32, 1)
    half = np.where(t < 2, 0.25, np.where(t < 4, 0.5, 1.0))
    bound = np.where(t <= 6, half * d32, (t - 6) * d32) * (1 + 1e-6) + 1e-30
    ok = (d32 == 0) | (np.abs(xv - xh) <= bound + np.abs(d - d32) * 6)
    assert np.all(ok)


def test_nibble_order_low_first():
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0        # -> code 7 in the low nibble of byte 0
    x[0, 3] = -1.0       # -> code 0xA in the high nibble of byte 1
    codes, _ = oracle.quantize(bf16_bits_of(x), 1.0)
    assert codes[0, 0] == 0x07 and codes[0, 1] == 0xA0


# ---------------------------------------------------------------------------
# Scale-factor layout for the tensor cores
# ---------------------------------------------------------------------------

def test_sf_layout_hand_offsets():
    # atom = 128 rows x 4 scale columns = 512 B; inner (r%32)*16 + (r//32%4)*4 + c%4
    cases = [((0, 0), 0), ((1, 0), 16), ((31, 3), 31 * 16 + 3), ((32, 0), 4),
             ((33, 2), 16 + 4 + 2), ((127, 1), 31 * 16 + 12 + 1), ((0, 4), 512),
             ((128, 0), 512 * 5)]   # 20 scale columns -> 5 atoms per row block
    for (r, c), want in cases:
        assert oracle.sf_offset_tcgen05(r, c, 20) == want


def test_sf_layout_bijection_and_padding():
    rng = np.random.default_rng(1)
    rows, sfcols = 300, 10          # pads to 384 rows and 12 scale columns
    sf = rng.integers(1, 255, (rows, sfcols)).astype(np.uint8)
    out = oracle.sf_to_tcgen05(sf)
    assert out.size == 384 * 12
    offs = np.array([[oracle.sf_offset_tcgen05(r, c, 12) for c in range(12)] for r in range(384)])
    assert np.array_equal(np.sort(offs.ravel()), np.arange(384 * 12))
    assert np.array_equal(out[offs[:rows, :sfcols]], sf)
    pad = np.ones(384 * 12, bool)
    pad[offs[:rows, :sfcols].ravel()] = False
    assert np.all(out[pad] == 0)


# ---------------------------------------------------------------------------
# Step 4: the GEMM
# ---------------------------------------------------------------------------

def test_gemm_brute_force_exact_fractions():
    rng = np.random.default_rng(2)
    M, N, K = 3, 5, 32
    A = rng.integers(-6, 7, (M, K)) * 0.5
    W = rng.integers(-6, 7, (N, K)) * 0.25
    alpha = np.array([0.75, 1.0, 2.0 ** -9, 3.0, 1.5])
    y = oracle.gemm_f64(A, W, alpha)
    for m in range(M):
        for n in range(N):
            exact = Fraction(alpha[n]) * sum(Fraction(A[m, k]) * Fraction(W[n, k]) for k in range(K))
            assert y[m, n] == float(exact)


def test_gemm_matches_library_matmul_and_row_subset():
    rng = np.random.default_rng(4)
    A = rng.standard_normal((40, 96))
    W = rng.standard_normal((70, 96))
    alpha = rng.uniform(0.1, 2, 70)
    y = oracle.gemm_f64(A, W, alpha)
    assert np.allclose(y, (A @ W.T) * alpha[None, :], rtol=1e-12, atol=1e-12)
    rows = np.array([39, 0, 17])
    assert np.array_equal(oracle.gemm_f64(A, W, alpha, rows), y[rows])


def _quant(x32, g=None):
    bits = bf16_bits_of(x32)
    if g is None:
        g, _ = oracle.global_scale(bits)
    codes, sf = oracle.quantize(bits, g)
    return codes, sf, np.float32(g)


def test_one_hot_gemm_closed_form():
    # one nonzero per row: Y[m,n] = gA*gW*dec(sA)*dec(sW)*vA*vW
    M, N, K = 4, 3, 64
    xa = np.zeros((M, K), np.float32)
    xw = np.zeros((N, K), np.float32)
    ka = [0, 17, 33, 63]
    for m in range(M):
        xa[m, ka[m]] = [3.0, -1.5, 0.25, 40.0][m]
    for n in range(N):
        xw[n, ka] = [0.02, -0.5, 7.0][n]
    ca, sa, ga = _quant(xa)
    cw, sw, gw = _quant(xw)
    y64, _ = oracle.linear(ca, sa, ga, cw, sw, [(0, N, gw)])
    for m in range(M):
        k = ka[m]
        qa = ((ca[m, k // 2] >> (4 * (k % 2))) & 15)
        for n in range(N):
            qw = ((cw[n, k // 2] >> (4 * (k % 2))) & 15)
            want = (float(ga) * float(gw) * oracle.e4m3_value(sa[m, k // 16]) *
                    oracle.e4m3_value(sw[n, k // 16]) * oracle.e2m1_value(qa) * oracle.e2m1_value(qw))
            # same factors, another FP64 multiplication order: within 2 ulp
            assert abs(y64[m, n] - want) <= 4.5e-16 * abs(want)
    # the one-hot values are recovered to within the E2M1/E4M3 resolution
    assert abs(y64[0, 0] - 3.0 * 0.02) / (3.0 * 0.02) < 0.15


def test_fused_segments_equal_per_module_and_negative_control():
    rng = np.random.default_rng(8)
    K = 128
    x = rng.standard_t(3, (16, K)).astype(np.float32)
    mods = [(48, 0.02), (16, 0.2), (32, 0.002)]
    ws = [rng.standard_normal((n, K)).astype(np.float32) * s for n, s in mods]
    ca, sa, ga = _quant(x)
    qs = [_quant(w) for w in ws]
    cw = np.concatenate([q[0] for q in qs])
    sw = np.concatenate([q[1] for q in qs])
    segs, off = [], 0
    for (n, _), q in zip(mods, qs):
        segs.append((off, n, q[2]))
        off += n
    y_fused, yb_fused = oracle.linear(ca, sa, ga, cw, sw, segs)
    for (o, n, gw), q in zip(segs, qs):
        y_mod, yb_mod = oracle.linear(ca, sa, ga, q[0], q[1], [(0, n, gw)])
        assert np.array_equal(y_fused[:, o:o + n], y_mod)
        assert np.array_equal(yb_fused[:, o:o + n], yb_mod)
    # a single global scale for the fused GEMM mis-scales every other module by
    # its scale ratio -- the global-scale mismatch the pages repair
    y_one, _ = oracle.linear(ca, sa, ga, cw, sw, [(0, off, segs[0][2])])
    for (o, n, gw) in segs:
        ratio = float(segs[0][2]) / float(gw)
        nz = y_fused[:, o:o + n] != 0
        assert np.allclose(y_one[:, o:o + n][nz] / y_fused[:, o:o + n][nz], ratio, rtol=1e-12)
    assert float(segs[0][2]) / float(segs[2][2]) > 5      # really different scales


def test_quantized_gemm_close_to_bf16_gemm():
    # NVFP4 keeps a W4A4 GEMM within a few percent of the BF16 one on Gaussian
    # data (a property of 16-element block scaling, not a parity target)
    rng = np.random.default_rng(6)
    x = rng.standard_normal((32, 512)).astype(np.float32)
    w = (rng.standard_normal((48, 512)) * 0.02).astype(np.float32)
    ca, sa, ga = _quant(x)
    cw, sw, gw = _quant(w)
    y64, _ = oracle.linear(ca, sa, ga, cw, sw, [(0, 48, gw)])
    ref = oracle.bf16_bits_to_f64(bf16_bits_of(x)) @ oracle.bf16_bits_to_f64(bf16_bits_of(w)).T
    rel = np.linalg.norm(y64 - ref) / np.linalg.norm(ref)
    assert 0.01 < rel < 0.2


# ---------------------------------------------------------------------------
# MLP intermediate h = SiLU(gate) * up
# ---------------------------------------------------------------------------

def test_silu_mul_closed_forms():
    # SiLU(0) = 0; SiLU(v) - SiLU(-v) = v (odd part of v*sigmoid(v)); up = 1 and
    # up = -1 mirror; large |v| limits (SiLU -> v, SiLU -> 0)
    v = np.array([0.0, 0.5, 1.0, 2.0, 3.0, 8.0, 40.0, -40.0, 100.0], np.float32)
    gu = np.concatenate([np.concatenate([v, -v])[None, :],
                         np.ones((1, 2 * v.size), np.float32)], axis=1)
    # rows: [gate = (v, -v), up = 1]
    bits = bf16_bits_of(gu)
    h = oracle.bf16_bits_to_f64(oracle.silu_mul(bits))[0]
    n = v.size
    assert h[0] == 0.0
    for i in range(n):
        pos, neg = h[i], h[n + i]
        # difference is v up to the BF16 rounding of both terms
        assert abs((pos - neg) - v[i]) <= 2.0 ** -8 * (abs(pos) + abs(neg)) + 1e-30
    assert h[6] == 40.0 and h[n + 6] == 0.0 or abs(h[n + 6]) < 1e-15
    assert h[8] == 100.0
    up = np.concatenate([np.full(2 * n, 3.0, np.float32)])
    gu3 = np.concatenate([np.concatenate([v, -v]), -up])[None, :]
    h3 = oracle.bf16_bits_to_f64(oracle.silu_mul(bf16_bits_of(gu3)))[0]
    # up = -3: h = -3 SiLU(v), exact to one BF16 rounding of the FP64 product
    assert np.all(np.abs(h3 + 3 * oracle.bf16_bits_to_f64(oracle.silu_mul(bits))[0]) <=
                  2.0 ** -7 * np.abs(h3) + 1e-30)


def test_silu_mul_single_rounding_matches_exact_value():
    # for random inputs, h is the BF16 value nearest to g*sigmoid(g)*u (checked
    # through the neighbours of the returned BF16 value, in FP64)
    rng = np.random.default_rng(17)
    gu = (rng.standard_normal((16, 64)) * 3).astype(np.float32)
    bits = bf16_bits_of(gu)
    h = oracle.silu_mul(bits)
    vals = oracle.bf16_bits_to_f64(bits)
    g, u = vals[:, :32], vals[:, 32:]
    exact = g / (1 + np.exp(-g)) * u
    hv = oracle.bf16_bits_to_f64(h)
    up = oracle.bf16_bits_to_f64(h + 1)
    dn = oracle.bf16_bits_to_f64(h - 1)
    d0 = np.abs(hv - exact)
    assert np.all((d0 <= np.abs(up - exact)) | (h == 0x7F7F))
    assert np.all((d0 <= np.abs(dn - exact)) | ((h & 0x7FFF) == 0))


# --------------------------------------------------------------------------
# checkpoint-side scale harmonisation (chatpaper.ai abstract: the fused-module
# global-scale mismatch and its repair; reading: common scale = max module scale)
# --------------------------------------------------------------------------

def _harm_one(s8, gi, gc):
    sf = np.array([[s8], [0]], np.uint8)
    g_c, out = oracle.harmonize_scales(sf, [(0, 1, np.float32(gi)), (1, 1, np.float32(gc))])
    return g_c, int(out[0, 0])


def test_harmonize_golden(golden_dir):
    for line in read_golden(os.path.join(golden_dir, "harmonize_points.txt")):
        gi, gc, s8, expect = line.split()[:4]
        g_c, got = _harm_one(int(s8, 16), float(gi), float(gc))
        assert g_c == np.float32(max(float(gi), float(gc)))
        assert got == int(expect, 16), line


def test_harmonize_matches_torch_cast_exhaustive():
    # every scale byte x several ratios against an independent library path:
    # decode by the format's bit fields, one float32 multiply, torch's RNE cast
    codes = np.arange(0x7F, dtype=np.uint8)
    dec = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float()
    for gi, gc in [(0.3, 1.0), (1.0, 3.0), (0.01, 1.0), (0.77, 0.8), (1e-3, 0.2), (0.015, 0.02)]:
        ratio = np.float32(np.float32(gi) / np.float32(gc))
        prod = (dec * torch.tensor(ratio, dtype=torch.float32)).numpy()
        ref = torch.from_numpy(prod).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        sf = np.stack([codes, np.zeros_like(codes)])
        g_c, out = oracle.harmonize_scales(sf, [(0, 1, np.float32(gi)), (1, 1, np.float32(gc))])
        assert np.array_equal(out[0], ref), (gi, gc)
        assert np.all(out[1] == 0)


def test_harmonize_power_of_two_ratio_closed_form():
    # ratio 2^-k moves a normal scale k binades down: the code drops by 8k while
    # the exponent field stays >= 1, and the value is exactly E4M3(s8) * 2^-k
    for k in (1, 2, 3):
        for s8 in range(8 * (k + 1), 0x7F):
            _, got = _harm_one(s8, 2.0 ** -k, 1.0)
            assert got == s8 - 8 * k
            assert oracle.e4m3_value(got) == oracle.e4m3_value(s8) * 2.0 ** -k


def test_harmonize_max_module_unchanged_and_shape():
    rng = np.random.default_rng(7)
    sf = rng.integers(0, 0x7F, size=(40, 12), dtype=np.uint8)
    segs = [(0, 10, np.float32(0.02)), (10, 25, np.float32(0.2)), (35, 5, np.float32(0.002))]
    g_c, out = oracle.harmonize_scales(sf, segs)
    assert g_c == np.float32(0.2)
    assert np.array_equal(out[10:35], sf[10:35])            # the max-scale module
    assert np.all(out[:10] <= sf[:10]) and np.all(out[35:] <= sf[35:])   # ratio <= 1 never grows a scale
    # the other modules are the single-module formula row range by row range
    for off, n, g in segs:
        _, ref = oracle.harmonize_scales(np.concatenate([sf[off:off + n], np.zeros((1, 12), np.uint8)]),
                                         [(0, n, g), (n, 1, g_c)])
        assert np.array_equal(out[off:off + n], ref[:n])


# --------------------------------------------------------------------------
# FP8 E4M3 KV-cache quantization with a calibrated per-tensor scale
# (evolve.pub, Key claims under review, last bullet; reading beside the oracle)
# --------------------------------------------------------------------------

def _bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy() \
        .astype(np.uint16)


def test_kv_quantize_golden(golden_dir):
    for line in read_golden(os.path.join(golden_dir, "kv_e4m3_points.txt")):
        xv, sv, expect = line.split()[:3]
        got = oracle.kv_quantize(_bf16([[float(xv)]]), float(sv))[0, 0]
        assert got == int(expect, 16), line


def test_kv_code_is_a_true_division_at_ties():
    # s = 1.75: 2.734375, 3.171875 and 5.46875 are exactly 1.5625 s, 1.8125 s
    # and 3.125 s, E4M3 ties that go to the even code (1.5 = 0x3C,
    # 1.75 = 0x3E, 3.0 = 0x44); 1/1.75 is not a float32, so a reciprocal
    # multiply would land just above each tie and round up to the odd code
    got = oracle.kv_quantize(_bf16([[2.734375, 3.171875, 5.46875, -2.734375]]), 1.75)[0]
    assert [int(v) for v in got] == [0x3C, 0x3E, 0x44, 0xBC]


@pytest.mark.parametrize("s", [1.0, 0.37, 3.1e-3, 41.0])
def test_kv_quantize_matches_torch_cast_exhaustive_bf16(s):
    # every finite BF16 value: the quotient by one float32 division, then
    # torch's RNE float8_e4m3fn cast in range and +-448 beyond (satfinite)
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(vals)
    bits, vals = bits[keep], vals[keep]
    with np.errstate(over="ignore"):                 # quotients beyond float32 saturate too
        t = (vals / np.float32(s)).astype(np.float32)
    got = oracle.kv_quantize(bits.reshape(1, -1), s)[0]
    inr = np.abs(t) <= 448
    ref = torch.from_numpy(t[inr].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got[inr], ref)
    sat = np.where(np.signbit(t[~inr]), 0xFE, 0x7E).astype(np.uint8)
    assert np.array_equal(got[~inr], sat)


def test_kv_scale_maps_amax_to_448():
    rng = np.random.default_rng(3)
    for amax in [1.0, 448.0, 0.0123, 7.5e3, float(rng.uniform(0.1, 100))]:
        s = oracle.kv_scale(amax)
        assert s == np.float32(np.float32(amax) / np.float32(448.0))
        b = _bf16([[amax, -amax]])
        a_b = float(torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float()[0, 0])
        codes = oracle.kv_quantize(b, oracle.kv_scale(a_b))[0]
        assert codes[0] == 0x7E and codes[1] == 0xFE     # the calibration absmax is the largest code
    assert oracle.kv_scale(0.0) == np.float32(1.0)


# --------------------------------------------------------------------------
# Gated DeltaNet gate epilogue (evolve.pub, Key claims under review, second
# bullet: log-space softplus/exponential decay and sigmoid parameterizations)
# --------------------------------------------------------------------------

def test_gates_closed_forms():
    # sigmoid: exact values 1/2, 3/4, 1/4 at 0, +-ln 3
    y = np.array([[0.0, np.log(3.0), -np.log(3.0)]])
    assert list(oracle.gdn_gates(y, oracle.GATE_SIGMOID)[0]) == [0x3F00, 0x3F40, 0x3E80]
    # decay: softplus(ln(e - 1)) = 1, so g = -exp(A_log); softplus(0) = ln 2
    z = np.log(np.e - 1.0)
    a_log = np.array([0.0, np.log(np.float32(4.0)), 0.0], np.float32)
    g = oracle.gdn_gates(np.array([[z, z, 0.0]]), oracle.GATE_DECAY, a_log=a_log,
                         dt_bias=np.zeros(3, np.float32))[0]
    assert g[0] == 0xBF80 and g[1] == 0xC080                      # -1, -4
    assert g[2] == oracle.bf16_from_double(np.array([-np.log(2.0)]))[0]
    # dt_bias shifts the argument: y + b = 0 gives ln 2 whatever the split
    g2 = oracle.gdn_gates(np.array([[1.5]]), oracle.GATE_DECAY, a_log=np.zeros(1, np.float32),
                          dt_bias=np.array([-1.5], np.float32))[0, 0]
    assert g2 == g[2]


def test_gates_match_torch_float64():
    rng = np.random.default_rng(11)
    y = rng.uniform(-20, 20, size=(64, 48))
    a_log = rng.uniform(0.0, 2.8, size=48).astype(np.float32)
    dt_bias = rng.uniform(-7.0, -2.0, size=48).astype(np.float32)
    yt = torch.from_numpy(y)
    sig = torch.sigmoid(yt).numpy()
    assert np.array_equal(oracle.gdn_gates(y, oracle.GATE_SIGMOID), oracle.bf16_from_double(sig))
    z = yt + torch.from_numpy(dt_bias.astype(np.float64))
    dec = (-torch.exp(torch.from_numpy(a_log.astype(np.float64))) *
           torch.nn.functional.softplus(z, beta=1.0, threshold=50.0)).numpy()
    assert np.array_equal(oracle.gdn_gates(y, oracle.GATE_DECAY, a_log, dt_bias),
                          oracle.bf16_from_double(dec))


def test_gates_monotone_signs_and_tails():
    y = np.linspace(-60, 60, 4001).reshape(1, -1)
    s = oracle.bf16_bits_to_f64(oracle.gdn_gates(y, oracle.GATE_SIGMOID))[0]
    assert np.all(np.diff(s) >= 0) and s.min() >= 0 and s.max() <= 1
    n = y.shape[1]
    g = oracle.bf16_bits_to_f64(oracle.gdn_gates(y, oracle.GATE_DECAY, np.full(n, 0.5, np.float32),
                                                 np.zeros(n, np.float32)))[0]
    assert np.all(np.diff(g) <= 0) and g.max() <= 0
    # far tails: softplus(z) -> z for large z, -> e^z for very negative z
    big = oracle.gdn_gates(np.array([[300.0, -300.0]]), oracle.GATE_DECAY,
                           np.zeros(2, np.float32), np.zeros(2, np.float32))[0]
    assert big[0] == oracle.bf16_from_double(np.array([-300.0]))[0]
    assert big[1] == oracle.bf16_from_double(np.array([-np.exp(-300.0)]))[0]


def test_silu_mul_f64_agrees_with_bf16_input_form():
    # on BF16-representable inputs it is the (pinned) BF16-input SiLU * up
    rng = np.random.default_rng(21)
    gb = oracle.bf16_from_double(rng.normal(0, 4, size=(32, 40)))
    ub = oracle.bf16_from_double(rng.normal(0, 4, size=(32, 40)))
    h1 = oracle.silu_mul_f64(oracle.bf16_bits_to_f64(gb), oracle.bf16_bits_to_f64(ub))
    h2 = oracle.silu_mul(np.concatenate([gb, ub], axis=1))
    assert np.array_equal(h1, h2)


def test_silu_mul_f64_closed_forms():
    g = np.array([[0.0, 50.0, -50.0, np.log(3.0)]])
    u = np.array([[7.0, 2.0, 1.0, 4.0]])
    h = oracle.bf16_bits_to_f64(oracle.silu_mul_f64(g, u))[0]
    assert h[0] == 0.0                                        # SiLU(0) = 0
    assert h[1] == 100.0                                      # SiLU(50) = 50 to 2^-72
    assert h[2] == oracle.bf16_bits_to_f64(oracle.bf16_from_double(
        np.array([-50.0 / (1.0 + np.exp(50.0))])))[0]
    assert h[3] == oracle.bf16_bits_to_f64(oracle.bf16_from_double(np.array([np.log(3.0) * 0.75 * 4.0])))[0]
