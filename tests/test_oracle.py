"""Pins for the CPU oracle, checked against things other than the oracle itself.

The oracle (``oracle/w4_oracle.c``) is the yardstick of every GPU parity test,
so each of its steps is pinned here by a property, a closed form, a worked
value from the pages, an independent library routine (numpy's fp16
conversion, exact rational arithmetic), or brute force on tiny inputs.  A
plausible slip anywhere in it (a wrong sign of the zero point, the unrounded
scale used for the codes, a swapped nibble, a dropped AWQ factor, a transposed
operand, floor instead of round-half-even) fails at least one test below.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from weight_only_int4_w4_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
G = 128


def _groups(a, group=G):
    N, K = a.shape
    return a.reshape(N, K // group, group)


def _weights(N=64, K=512, std=0.02, outliers=0.001, tag="pin"):
    return synthetic.weight(K, N, std, outliers, ("oracle-pin", tag)).numpy()


# ---------------------------------------------------------------- fp16 rounding

def test_f16_conversion_matches_numpy():
    """The fp32 -> fp16 step agrees with numpy's independent RNE conversion,
    including ties, subnormals, overflow and the smallest normal."""
    rng = np.random.default_rng(1)
    vals = list((rng.standard_normal(4000) * np.exp(rng.uniform(-25, 12, 4000))).astype(np.float32))
    one = np.float32(1.0)
    vals += [one + np.float32(2.0 ** -11), one + np.float32(3 * 2.0 ** -11),  # ties to even
             np.float32(65504.0), np.float32(65520.0), np.float32(1e6),      # max, overflow tie, inf
             np.float32(2.0 ** -14), np.float32(2.0 ** -24), np.float32(2.0 ** -25),
             np.float32(3 * 2.0 ** -26), np.float32(0.0), np.float32(-0.0)]
    for v in vals:
        want = int(np.float32(v).astype(np.float16).view(np.uint16))
        assert oracle.f32_to_f16_bits(float(v)) == want, v
    for b in [0x0000, 0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0xC000]:
        assert oracle.f16_bits_to_f32(b) == float(np.uint16(b).view(np.float16))


# ---------------------------------------------------------------- quantize

def _check_grid_properties(W, codes, scales, zeros, awq_s=None):
    """Properties any correct affine per-group RTN must satisfy (fp64 checks)."""
    Wp = W.astype(np.float64)
    if awq_s is not None:
        Wp = Wp / awq_s.astype(np.float64)[None, :]
    wg = _groups(Wp)
    qg = _groups(codes).astype(np.float64)
    sc = scales.astype(np.float64)[:, :, None]
    z = zeros.astype(np.float64)[:, :, None]
    # zero points are integers in [0, 15]; codes too
    assert np.all(z == np.round(z)) and z.min() >= 0 and z.max() <= 15
    assert codes.max() <= 15
    # every code is the nearest grid point (q - z) * sc to w', among q in 0..15
    grid = (np.arange(16, dtype=np.float64)[None, None, None, :] - z[..., None]) * sc[..., None]
    dist_all = np.abs(wg[..., None] - grid)
    chosen = np.abs(wg - (qg - z) * sc)
    slack = 1e-6 * sc * (1.0 + np.abs(wg) / sc)
    assert np.all(chosen <= dist_all.min(axis=-1) + slack)
    # the scale is the fp16 value nearest to (max - min) / 15 (degenerate groups aside)
    rng_ = (wg.max(axis=-1) - wg.min(axis=-1)) / 15.0
    s = scales.astype(np.float64)
    ok = rng_ > 1e-4
    up = np.nextafter(scales, np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(scales, np.float16(-np.inf)).astype(np.float64)
    err = np.abs(s - rng_)
    assert np.all((err <= np.abs(up - rng_) * (1 + 1e-6) + 1e-12)[ok])
    assert np.all((err <= np.abs(dn - rng_) * (1 + 1e-6) + 1e-12)[ok])
    # the zero point is the integer nearest to -min / scale (clamped to [0, 15])
    t = -wg.min(axis=-1) / s
    zz = zeros.astype(np.float64)
    inside = (t >= 0) & (t <= 15)
    assert np.all((np.abs(zz - t) <= 0.5 + 1e-6)[inside])
    assert np.all(zz[t < -0.5] == 0) and np.all(zz[t > 15.5] == 15)
    # for groups that straddle zero, |w' - w^'| <= scale/2 except where the grid clamps
    straddle = (wg.min(axis=-1) <= 0) & (wg.max(axis=-1) >= 0)
    e = np.abs(wg - (qg - z) * sc)
    unclamped = (qg > 0) & (qg < 15)
    assert np.all((e <= sc / 2 * (1 + 1e-6))[straddle[..., None] & unclamped])


@pytest.mark.parametrize("outliers", [0.0, 0.001])
def test_rtn_grid_properties(outliers):
    W = _weights(outliers=outliers, tag=f"grid{outliers}")
    codes, scales, zeros = oracle.quantize(W)
    assert codes.shape == W.shape and scales.shape == (W.shape[0], W.shape[1] // G)
    _check_grid_properties(W, codes, scales, zeros)


def test_scale_uses_fp16_rounded_value():
    """Codes must be nearest on the grid of the STORED fp16 scale; a quantizer
    that used the unrounded fp32 scale for q fails the nearest-grid check on
    enough elements to be caught here."""
    W = _weights(N=256, K=1024, outliers=0.0, tag="fp16grid")
    codes, scales, zeros = oracle.quantize(W)
    _check_grid_properties(W, codes, scales, zeros)
    # and the fp16 rounding is real: many scales differ from their fp32 range/15
    r32 = (_groups(W).max(-1) - _groups(W).min(-1)).astype(np.float32) / np.float32(15)
    assert np.mean(r32 != scales.astype(np.float32)) > 0.5


def test_on_grid_weights_reconstruct_exactly():
    """Weights already on a grid (q - z) * sc, with codes 0 and 15 present in
    every group, come back with identical codes, zero point and scale."""
    rng = np.random.default_rng(7)
    N, Kg = 32, 4
    sc = rng.uniform(1e-3, 1e-1, (N, Kg)).astype(np.float16)
    z = rng.integers(0, 16, (N, Kg))
    q = rng.integers(0, 16, (N, Kg, G))
    q[:, :, 0] = 0
    q[:, :, 1] = 15
    W = ((q - z[..., None]).astype(np.float32) * sc.astype(np.float32)[..., None]).reshape(N, Kg * G)
    codes, scales, zeros = oracle.quantize(W)
    assert np.array_equal(codes.reshape(N, Kg, G), q.astype(np.uint8))
    assert np.array_equal(zeros.astype(np.int64), z)
    assert np.array_equal(scales.view(np.uint16), sc.view(np.uint16))
    What = oracle.dequant(codes, scales, zeros)
    assert np.array_equal(What, W)


def test_half_even_ties_worked_group():
    """A group spanning exactly 15 steps of c = 2^-6: scale = c, zero = rint(7.5)
    = 8 (ties to even), and the textbook half-even codes for +-0.5c, 1.5c, 2.5c."""
    c = 2.0 ** -6
    vals = np.zeros(G, np.float64)
    vals[0], vals[1] = -7.5 * c, 7.5 * c
    vals[2:8] = [0.5 * c, -0.5 * c, 1.5 * c, 2.5 * c, -2.5 * c, 3.0 * c]
    W = vals.astype(np.float32)[None, :]
    codes, scales, zeros = oracle.quantize(W)
    assert float(scales[0, 0]) == c
    assert float(zeros[0, 0]) == 8.0
    # rint(-7.5) = -8 -> 0 ; rint(7.5) = 8 -> 16 -> clamped to 15
    assert codes[0, 0] == 0 and codes[0, 1] == 15
    # rint(0.5)=0, rint(-0.5)=-0, rint(1.5)=2, rint(2.5)=2, rint(-2.5)=-2, rint(3)=3
    assert list(codes[0, 2:8]) == [8, 8, 10, 10, 6, 11]
    assert np.all(codes[0, 8:] == 8)


def test_degenerate_groups():
    """Constant groups: the fp16 scale is 0, taken as 1.0; integer constants and
    zero reconstruct exactly; a range below fp16's smallest subnormal too."""
    W = np.zeros((4, G), np.float32)
    W[0] = 3.0
    W[1] = 0.0
    W[2] = -2.0
    W[3] = 0.5
    W[3, 5] = 0.5 + 1e-9  # range/15 underflows fp16
    codes, scales, zeros = oracle.quantize(W)
    assert np.all(scales.astype(np.float32) == 1.0)
    assert list(zeros[:, 0].astype(int)) == [0, 0, 2, 0]
    # a zero point is an integer: zero is stored as +0 (bits 0x0000), never -0
    assert np.all(zeros.view(np.uint16)[[0, 1, 3], 0] == 0)
    What = oracle.dequant(codes, scales, zeros)
    assert np.array_equal(What[0], W[0]) and np.array_equal(What[1], W[1]) and np.array_equal(What[2], W[2])
    assert np.all(codes[3] == 0)  # rint(0.5) = 0 (ties to even), z = 0


def test_non_straddling_group_clamps():
    """A group entirely above zero: z clamps to 0 and codes beyond 15 clamp to
    15, so the scale/2 bound does not hold there (documented behaviour)."""
    W = np.linspace(1.0, 2.0, G, dtype=np.float32)[None, :]
    codes, scales, zeros = oracle.quantize(W)
    sc = float(scales[0, 0])
    assert float(zeros[0, 0]) == 0.0
    assert abs(sc - 1.0 / 15) <= 2.0 ** -15
    assert codes[0, -1] == 15 and codes[0, 0] == 15  # 1.0 / sc = 15 exactly after rounding
    What = oracle.dequant(codes, scales, zeros)
    assert abs(float(What[0, -1]) - 2.0) > 0.5


# ---------------------------------------------------------------- AWQ

def test_awq_unit_scale_is_plain_rtn():
    W = _weights(tag="awq1")
    plain = oracle.quantize(W)
    ones = oracle.quantize(W, awq_s=np.ones(W.shape[1], np.float32))
    for a, b in zip(plain, ones):
        assert np.array_equal(np.asarray(a).view(np.uint8), np.asarray(b).view(np.uint8))
    assert np.array_equal(oracle.dequant(*plain), oracle.dequant(*ones, awq_s=np.ones(W.shape[1], np.float32)))


@pytest.mark.parametrize("p", [2.0, 0.5])
def test_awq_power_of_two_scale_is_exact(p):
    """s = 2^j divides exactly, so codes and zeros equal plain RTN's, the scale
    is exactly RTN's / s, and W^ = quant(W/s) * s reproduces RTN's W^ bit for bit."""
    W = _weights(tag=f"awqpow{p}")
    s = np.full(W.shape[1], p, np.float32)
    c0, s0, z0 = oracle.quantize(W)
    c1, s1, z1 = oracle.quantize(W, awq_s=s)
    assert np.array_equal(c0, c1) and np.array_equal(z0, z1)
    assert np.array_equal(s1.astype(np.float64) * p, s0.astype(np.float64))
    assert np.array_equal(oracle.dequant(c1, s1, z1, awq_s=s), oracle.dequant(c0, s0, z0))


def test_awq_per_channel_identity():
    """W^ = quant(W / s) * s: the grid properties hold for W / s, and the
    reconstruction error of w is at most (scale / 2) * s_k where nothing clamps."""
    K = 512
    W = _weights(K=K, outliers=0.0, tag="awqchan")
    s = synthetic.awq_scale(K, ("oracle-pin", "awq")).numpy()
    assert s.dtype == np.float32 and s.min() > 0 and s.max() > 2.0 * np.median(s)
    codes, scales, zeros = oracle.quantize(W, awq_s=s)
    _check_grid_properties(W, codes, scales, zeros, awq_s=s)
    What = oracle.dequant(codes, scales, zeros, awq_s=s).astype(np.float64)
    sc = np.repeat(scales.astype(np.float64), G, axis=1)
    z = np.repeat(zeros.astype(np.float64), G, axis=1)
    exact = (codes - z) * sc * s.astype(np.float64)[None, :]
    assert np.all(np.abs(What - exact) <= 4 * 2.0 ** -24 * np.abs(exact) + 1e-30)
    unclamped = (codes > 0) & (codes < 15)
    bound = sc / 2 * s[None, :] * (1 + 1e-5)
    assert np.all((np.abs(W - What) <= bound)[unclamped])


# ---------------------------------------------------------------- packing and bytes

def test_pack_nibble_order_worked_bytes():
    codes = np.array([[1, 2, 15, 0, 7, 8, 0x1F, 0x13]], np.uint8)
    packed = oracle.pack(codes)
    assert list(packed[0]) == [0x21, 0x0F, 0x87, 0x3F]  # low nibble = even k; codes masked to 4 bits


def test_pack_round_trip():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, (17, 256)).astype(np.uint8)
    packed = oracle.pack(codes)
    assert packed.shape == (17, 128)
    assert np.array_equal(oracle.unpack(packed, 256), codes)


def test_byte_counts_match_pages():
    gold = json.load(open(os.path.join(GOLDEN, "page_byte_counts.json")))
    codes = np.zeros((96, 1024), np.uint8)
    packed = oracle.pack(codes)
    per_param = packed.nbytes / codes.size
    assert per_param == gold["bytes_per_param"]["INT4"] == 0.5
    seven = gold["model_7b_weight_gb"]
    assert seven["params"] * per_param / 1e9 == seven["INT4"]
    assert seven["params"] * 2 / 1e9 == seven["FP16/BF16"]
    # the 80-layer Llama-3-70B linear stack used by the whole-model workload
    params = synthetic.N_LAYERS_70B * sum(k * n for k, n in synthetic.SHAPES_70B.values())
    params += synthetic.LM_HEAD_70B[0] * synthetic.LM_HEAD_70B[1]
    codes_gb = params * per_param / 1e9
    seventy = gold["model_70b_weight_gb"]
    assert abs(codes_gb - seventy["INT4"]) / seventy["INT4"] < 0.01     # "about 35 GB"
    assert abs(params * 2 / 1e9 - seventy["FP16"]) / seventy["FP16"] < 0.01
    total_gb = params * (0.5 + 4.0 / G) / 1e9  # + fp16 scale and zero per group
    assert abs(codes_gb - 34.75) < 0.01 and abs(total_gb - 36.92) < 0.01
    a100 = gold["decode_weight_read_a100"]
    ms = a100["weights_gb"] / (a100["bandwidth_tb_s"] * 1000) * 1000
    assert a100["ms_per_token_min"] <= ms <= a100["ms_per_token_max"]


# ---------------------------------------------------------------- dequant + GEMM

def test_dequant_is_affine_of_stored_values():
    W = _weights(tag="deq")
    codes, scales, zeros = oracle.quantize(W)
    What = oracle.dequant(codes, scales, zeros).astype(np.float64)
    sc = np.repeat(scales.astype(np.float64), G, axis=1)
    z = np.repeat(zeros.astype(np.float64), G, axis=1)
    assert np.array_equal(What, (codes - z) * sc)  # (q - z) and its product with an fp16 are exact in fp32


@pytest.mark.parametrize("M,N,K", [(1, 1, 128), (3, 2, 128), (2, 4, 256), (4, 3, 256)])
def test_gemm_brute_force_exact_rationals(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    X = rng.standard_normal((M, K)).astype(np.float16).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Y, B, (codes, scales, zeros, What) = oracle.reference_linear(X, W)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(X[m, k])) * Fraction(float(What[n, k])) for k in range(K))
            absum = sum(abs(Fraction(float(X[m, k])) * Fraction(float(What[n, k]))) for k in range(K))
            assert abs(Fraction(Y[m, n]) - exact) <= Fraction(1, 10 ** 12) * absum
            assert abs(Fraction(B[m, n]) - absum) <= Fraction(1, 10 ** 12) * absum


def test_gemm_against_blas_dense():
    rng = np.random.default_rng(11)
    X = rng.standard_normal((5, 384)).astype(np.float32)
    What = rng.standard_normal((7, 384)).astype(np.float32)
    Y, B = oracle.gemm(X, What)
    ref = X.astype(np.float64) @ What.astype(np.float64).T
    assert np.all(np.abs(Y - ref) <= 1e-12 * B)
    assert np.allclose(B, np.abs(X.astype(np.float64)) @ np.abs(What.astype(np.float64)).T, rtol=1e-12)


def test_rows_are_independent():
    """Quantizing a subset of rows equals quantizing all rows then selecting
    them (what the sampled full-size parity tests rely on)."""
    W = _weights(N=300, K=256, tag="rows")
    rows = [0, 7, 128, 299]
    full = oracle.quantize(W)
    part = oracle.quantize(W[rows])
    for a, b in zip(full, part):
        assert np.array_equal(np.asarray(a)[rows].view(np.uint8), np.asarray(b).view(np.uint8))


def test_synthetic_row_blocks_are_consistent():
    full = synthetic.weight_rows(256, 300, 0.02, 0.001, "consistency")
    rows = [3, 130, 299]
    part = synthetic.weight_rows(256, 300, 0.02, 0.001, "consistency", rows=rows)
    assert np.array_equal(full[rows].numpy(), part.numpy())
    frac = (full.abs() > 0.1).float().mean().item()
    assert 0.0002 < frac < 0.003  # ~0.1% N(0,0.4) outliers, a few of them small


# ---------------------------------------------------------------- symmetric variant {-7..7}

@pytest.mark.parametrize("group", [32, 64, 128])
def test_symmetric_grid_properties(group):
    """Codes lie in {-7..7} + 8 with zero point 8. The scale is the nearest fp16
    to max|w|/7 (numpy's conversion). Every weight is within scale/2 of its
    reconstruction (checked in fp64)."""
    W = _weights(N=32, K=512, outliers=0.002, tag=("sym", group))
    codes, sc, zp = oracle.quantize_symmetric(W, group=group)
    assert codes.min() >= 1 and codes.max() <= 15
    assert np.all(zp.astype(np.float32) == 8.0)
    Wg = _groups(W.astype(np.float64), group)
    amax = np.abs(Wg).max(axis=2)
    expect = (amax.astype(np.float32) / np.float32(7.0)).astype(np.float16)
    assert np.array_equal(sc.view(np.uint16), expect.view(np.uint16))
    q = _groups(codes.astype(np.float64), group) - 8.0
    scale = sc.astype(np.float64)[:, :, None]
    assert np.all(np.abs(Wg - q * scale) <= scale / 2 + 1e-12)


def test_symmetric_on_grid_weights_reconstruct_exactly():
    """w = q * c with c an fp16 value and +-7 present in every group: the scale is
    c exactly and the codes are q + 8."""
    rng = np.random.default_rng(5)
    N, K = 8, 256
    q = rng.integers(-7, 8, size=(N, K))
    q[:, 0], q[:, 128] = 7, -7
    c = np.float16(0.0078125 * 1.25)
    W = (q * np.float32(c)).astype(np.float32)
    codes, sc, zp = oracle.quantize_symmetric(W)
    assert np.all(sc == c)
    assert np.array_equal(codes.astype(np.int64), q + 8)


def test_symmetric_sign_symmetry():
    """rint is symmetric and the set {-7..7} is too: quantizing -W negates every q."""
    W = _weights(N=16, K=384, tag="symneg")
    c1, s1, _ = oracle.quantize_symmetric(W)
    c2, s2, _ = oracle.quantize_symmetric(-W)
    assert np.array_equal(s1.view(np.uint16), s2.view(np.uint16))
    assert np.array_equal(16 - c1.astype(np.int64), c2.astype(np.int64))


def test_symmetric_half_even_ties_and_degenerate():
    """A worked group: with max|w| = 7 the scale is 1 and +-0.5, +-2.5 round to even
    (0, +-2). An all-zero group gets scale 1.0 and codes 8."""
    w = np.zeros((2, 128), np.float32)
    w[0, :6] = [7.0, -7.0, 0.5, -0.5, 2.5, -2.5]
    codes, sc, zp = oracle.quantize_symmetric(w)
    assert sc[0, 0] == 1.0 and sc[1, 0] == 1.0
    assert list(codes[0, :6].astype(int) - 8) == [7, -7, 0, 0, 2, -2]
    assert np.all(codes[1] == 8)


def test_symmetric_awq_unit_scale_and_dequant_matches_q_times_scale():
    """s = 1 changes nothing. The shared dequantization ((code - 8) * scale)
    gives q * scale exactly."""
    W = _weights(N=8, K=256, tag="symawq")
    c0, s0, z0 = oracle.quantize_symmetric(W)
    c1, s1, z1 = oracle.quantize_symmetric(W, np.ones(256, np.float32))
    assert np.array_equal(c0, c1) and np.array_equal(s0.view(np.uint16), s1.view(np.uint16))
    What = oracle.dequant(c0, s0, z0)
    q = c0.astype(np.float32) - 8.0
    expect = (q.reshape(8, 2, 128) * s0.astype(np.float32)[:, :, None]).reshape(8, 256)
    assert np.array_equal(What, expect)


# ---------------------------------------------------------------- dense + sparse outlier split

def _outlier_weights(N=64, K=512, tag="outl"):
    return synthetic.weight(K, N, 0.02, 0.002, ("oracle-pin", tag)).numpy()


def test_outlier_mask_is_top_count_by_magnitude():
    """The sparse entries are exactly the `count` largest |w| (distinct magnitudes),
    checked against numpy's independent partition."""
    W = _outlier_weights()
    count = 40
    codes, sc, zp, row_ptr, col, val = oracle.outlier_split(W, count)
    assert row_ptr[-1] == count and len(col) == count
    flat = np.abs(W).ravel()
    top = np.argpartition(flat, -count)[-count:]
    rows = np.repeat(np.arange(W.shape[0]), np.diff(row_ptr))
    assert set(top.tolist()) == set((rows * W.shape[1] + col).tolist())
    assert np.all(np.diff(row_ptr) >= 0)
    for n in range(W.shape[0]):  # increasing k within a row
        assert np.all(np.diff(col[row_ptr[n]:row_ptr[n + 1]]) > 0)


def test_outlier_dense_part_is_zero_at_outliers_and_values_are_fp16():
    W = _outlier_weights(tag="outl2")
    codes, sc, zp, row_ptr, col, val = oracle.outlier_split(W, 50)
    rows = np.repeat(np.arange(W.shape[0]), np.diff(row_ptr))
    dense = oracle.dequant(codes, sc, zp)
    assert np.all(dense[rows, col] == 0.0)
    assert np.array_equal(val, W[rows, col].astype(np.float16))
    What = oracle.outlier_dequant(codes, sc, zp, row_ptr, col, val)
    assert np.array_equal(What[rows, col], W[rows, col].astype(np.float16).astype(np.float32))
    mask = np.zeros(W.shape, bool)
    mask[rows, col] = True
    # elsewhere: plain RTN of the matrix with the outliers set to 0
    c2, s2, z2 = oracle.quantize(np.where(mask, 0, W).astype(np.float32))
    assert np.array_equal(What[~mask], oracle.dequant(c2, s2, z2)[~mask])


def test_outlier_split_reduces_weight_error_on_outlier_heavy_weights():
    """Groups with a large outlier get a coarse RTN grid; splitting the outliers off
    lowers the reconstruction error (seeded data, 0.2% N(0,0.4) outliers)."""
    W = _outlier_weights(N=128, K=1024, tag="outl3")
    count = int(np.ceil(0.002 * W.size))
    codes, sc, zp, row_ptr, col, val = oracle.outlier_split(W, count)
    err_split = np.abs(W - oracle.outlier_dequant(codes, sc, zp, row_ptr, col, val)).sum()
    c, s, z = oracle.quantize(W)
    err_rtn = np.abs(W - oracle.dequant(c, s, z)).sum()
    assert err_split < 0.8 * err_rtn


def test_outlier_ties_at_threshold_are_all_kept():
    W = np.full((2, 128), 0.01, np.float32)
    W[0, 3] = W[1, 7] = W[1, 9] = 0.5  # three tied largest magnitudes, count = 2
    codes, sc, zp, row_ptr, col, val = oracle.outlier_split(W, 2)
    assert list(row_ptr) == [0, 1, 3] and list(col) == [3, 7, 9]


# ---------------------------------------------------------------- GPTQ column sweep

def _gptq_numpy(W, X, group=G, damp_frac=0.01):
    """Independent route: numpy/LAPACK inverse and Cholesky for U, the same sweep rule."""
    W = W.astype(np.float64)
    H = 2.0 * (X.astype(np.float64).T @ X.astype(np.float64))
    H[np.diag_indices_from(H)] += damp_frac * np.trace(H) / H.shape[0]
    U = np.linalg.cholesky(np.linalg.inv(H)).T  # upper factor: H^-1 = U^T U
    N, K = W.shape
    codes = np.zeros((N, K), np.uint8)
    for n in range(N):
        w = W[n].copy()
        for j in range(K):
            if j % group == 0:
                c, s, z = oracle.quantize(w[j:j + group].astype(np.float32)[None, :], group=group)
                sc, zp = np.float32(s[0, 0]), np.float32(z[0, 0])
            q = min(max(np.rint(np.float32(w[j]) / sc) + zp, 0), 15)
            codes[n, j] = q
            err = (w[j] - np.float64((np.float32(q) - zp) * sc)) / U[j, j]
            w[j + 1:] -= err * U[j, j + 1:]
    return codes


def test_gptq_matches_independent_linear_algebra_route():
    """The oracle's own Cholesky/inverse loops against numpy's LAPACK route: same codes."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((12, 64)) * 0.02).astype(np.float32)
    X = rng.standard_normal((48, 64)).astype(np.float32)
    X += 0.7 * X[:, [3]]  # correlated channels, a non-trivial Hessian
    c, s, z = oracle.gptq(W, X, group=32)
    assert np.array_equal(c, _gptq_numpy(W, X, group=32))


def test_gptq_with_diagonal_hessian_is_plain_rtn():
    """X = 2 I (orthogonal channels): H is diagonal, no error is fed forward, so the
    sweep reduces to round-to-nearest with the same per-group rule."""
    K = 256
    W = _weights(N=16, K=K, tag="gptq-diag")
    X = (2.0 * np.eye(K)).astype(np.float32)
    c, s, z = oracle.gptq(W, X)
    c2, s2, z2 = oracle.quantize(W)
    assert np.array_equal(c, c2)
    assert np.array_equal(s.view(np.uint16), s2.view(np.uint16))
    assert np.array_equal(z.view(np.uint16), z2.view(np.uint16))


def test_gptq_lowers_the_layer_output_error():
    """The objective ||X W^T - X W^^T||^2 is lower than plain RTN's on correlated data."""
    rng = np.random.default_rng(3)
    W = _weights(N=32, K=256, tag="gptq-obj")
    X = rng.standard_normal((128, 256)).astype(np.float32)
    X += 0.5 * X[:, [0]]
    def err(c, s, z):
        return float(np.sum((X @ W.T - X @ oracle.dequant(c, s, z).T) ** 2))
    assert err(*oracle.gptq(W, X)) < 0.5 * err(*oracle.quantize(W))


# ---------------------------------------------------------------- AWQ exponent search
# The search (aiwing.uk ch. 22, section 22.3: s from calibration activation
# magnitudes, W^ = quant(W / s) * s, a layer judged by ||X W^T - X W^^T||^2) is
# pinned step by step against numpy routes that share nothing with the C loops:
# the channel magnitude m_k, the exponent s = m^a, each exponent's output error
# (quantization by the pinned quantizer, the products by BLAS), the argmin with
# the first index on ties, and a constructed layer whose best exponent is known
# by hand.

def _search_numpy(W, X, alphas, group=G):
    """Independent route: numpy magnitudes and powers, BLAS products in fp64."""
    X64 = X.astype(np.float64)
    m = np.abs(X64).mean(axis=0)  # one magnitude per input channel k
    Yref = X64 @ W.astype(np.float64).T
    errs, ss = [], []
    for a in alphas:
        s = np.where(m > 0, np.power(m, a), 1.0).astype(np.float32)
        c, sc, zp = oracle.quantize(W, awq_s=s, group=group)
        # W^ = (q - z) * scale * s, fp32 left to right, from the stored values
        What = ((c.astype(np.float32) - np.repeat(zp.astype(np.float32), group, axis=1))
                * np.repeat(sc.astype(np.float32), group, axis=1)) * s[None, :]
        d = Yref - X64 @ What.astype(np.float64).T
        errs.append(float(np.sum(d * d)))
        ss.append(s)
    return np.array(errs), ss, m


def test_awq_search_magnitude_is_channel_mean_of_abs():
    """With a = 1, s is m_k = mean over the calibration ROWS of |x_k| (fp64,
    rounded to fp32).  Dyadic inputs make every sum exact, so the comparison
    is bit for bit; a non-square X tells rows from channels apart."""
    rng = np.random.default_rng(21)
    Mc, K = 24, 256
    X = (rng.integers(-64, 65, (Mc, K)) / 8.0).astype(np.float32)
    X[:, 7] = 0.0  # a silent channel: m = 0, s must be 1
    W = _weights(N=8, K=K, tag="awq-m")
    _, s, best = oracle.awq_search(W, X, [1.0])
    m = np.abs(X.astype(np.float64)).mean(axis=0)
    want = np.where(m > 0, m, 1.0).astype(np.float32)
    assert best == 0
    assert np.array_equal(s, want)
    assert s[7] == 1.0


@pytest.mark.parametrize("a", [0.5, -0.3, 0.0, 1.0])
def test_awq_search_scale_is_power_of_magnitude(a):
    """s = m^a for the exponent returned, against numpy's power (1 fp32 ulp)."""
    rng = np.random.default_rng(22)
    X = rng.standard_normal((40, 128)).astype(np.float32) * np.exp(rng.uniform(-3, 3, 128)).astype(np.float32)
    W = _weights(N=4, K=128, tag="awq-pow")
    _, s, best = oracle.awq_search(W, X, [a])
    m = np.abs(X.astype(np.float64)).mean(axis=0)
    want = np.power(m, a).astype(np.float32)
    assert best == 0
    assert np.all(np.abs(s - want) <= np.spacing(np.abs(want)))
    if a == 0.0:
        assert np.all(s == 1.0)


@pytest.mark.parametrize("group", [128, 64])
def test_awq_search_errors_match_blas_route(group):
    """Every exponent's error ||X W^T - X W^^T||_F^2 equals the numpy/BLAS route
    (quantizer pinned above, products in fp64 by BLAS) to 1e-9 relative, and the
    returned index is the argmin of those errors."""
    rng = np.random.default_rng(23)
    Mc, K, N = 48, 256, 24
    X = rng.standard_normal((Mc, K)).astype(np.float32)
    X[:, rng.choice(K, 3, replace=False)] *= 10.0  # heavy channels
    W = _weights(N=N, K=K, outliers=0.0, tag=("awq-blas", group))
    alphas = [-1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0]
    errs, s, best = oracle.awq_search(W, X, alphas, group=group)
    e_np, s_np, _ = _search_numpy(W, X, alphas, group=group)
    assert np.allclose(errs, e_np, rtol=1e-9, atol=0.0), (errs, e_np)
    assert best == int(np.argmin(e_np))
    assert np.array_equal(s, s_np[best])
    assert len(set(errs.tolist())) == len(alphas)  # the exponents really differ


def test_awq_search_first_index_on_ties():
    """Equal errors keep the first exponent: repeated exponents give bit-equal
    errors, and channels of equal magnitude make every exponent's s the same."""
    rng = np.random.default_rng(24)
    X = rng.standard_normal((16, 128)).astype(np.float32)
    X[:, 0] *= 10.0
    W = _weights(N=6, K=128, tag="awq-tie")
    errs, _, best = oracle.awq_search(W, X, [0.5, 0.0, 0.5, -0.5])
    assert errs[0] == errs[2]
    assert best == (0 if errs[0] <= min(errs[1], errs[3]) else int(np.argmin(errs)))
    # |x| = 1 everywhere: m = 1, s = 1 for every exponent -> all errors equal -> index 0
    Xs = np.where(rng.standard_normal((16, 128)) > 0, 1.0, -1.0).astype(np.float32)
    errs, s, best = oracle.awq_search(W, Xs, [0.7, -0.2, 0.0])
    assert errs[0] == errs[1] == errs[2]
    assert best == 0 and np.all(s == 1.0)


def test_awq_search_constructed_layer_prefers_positive_exponent():
    """A layer built so that only a = 0.5 quantizes exactly.  Channels 0..3 are
    heavy (|x| = 4, so m = 4 and s = 4^a), the rest have |x| = 1 (s = 1).  The
    weights are W = g * s(0.5) with g on a power-of-two grid (scale 2^-6, zero 8,
    codes 0 and 15 present, heavy values inside the range).  At a = 0.5, W / s = g
    exactly, so W^ = W and the error is exactly 0; at a = 0 the heavy weights
    leave the range, at a = 1 they fall halfway between grid points, at a < 0
    they grow further: every other exponent has a positive error."""
    K, N, Mc = 128, 3, 8
    sc = 2.0 ** -6
    rng = np.random.default_rng(25)
    q = rng.integers(1, 15, (N, K))
    q[:, 4] = 0
    q[:, 5] = 15  # min and max codes present in every row: scale = sc, zero = 8
    q[:, 0:4] = [13, 3, 11, 9]  # heavy channels: (q - 8) = 5, -5, 3, 1 (odd: halving leaves the grid)
    g = (q - 8) * sc
    s_true = np.ones(K)
    s_true[0:4] = 2.0  # 4 ** 0.5
    W = (g * s_true[None, :]).astype(np.float32)
    signs = np.where(rng.standard_normal((Mc, K)) > 0, 1.0, -1.0)
    X = (signs * np.where(np.arange(K) < 4, 4.0, 1.0)[None, :]).astype(np.float32)
    alphas = [-1.0, -0.5, 0.0, 0.5, 1.0]
    errs, s, best = oracle.awq_search(W, X, alphas)
    assert alphas[best] == 0.5
    assert errs[best] == 0.0
    assert all(e > 0.0 for i, e in enumerate(errs) if i != best)
    assert np.array_equal(s, s_true.astype(np.float32))
    # the same ordering from the independent route
    e_np, _, _ = _search_numpy(W, X, alphas)
    assert int(np.argmin(e_np)) == best and e_np[best] == 0.0
