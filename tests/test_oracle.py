"""Pins for the CPU oracle against things other than itself.

Each test names what fixes the expected value: a number printed on the pages
(tests/golden/worked_example.txt), a closed form, exact rational brute force,
an independent library routine (scipy's normal CDF, torch's bf16 cast,
torch.autograd), or an invariant the method must satisfy.  CPU only.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import ndtr

import oracle
from oracle import nf4 as O


# ---------------------------------------------------------------------------
# NF4 table
# ---------------------------------------------------------------------------

def test_nf4_table_structure():
    """'That is NF4': 16 values, one exactly 0, spanning [-1, 1]."""
    q = oracle.nf4_table()
    assert q.dtype == np.float32 and q.shape == (16,)
    assert np.all(np.diff(q) > 0)
    assert q[0] == -1.0 and q[15] == 1.0
    assert q[7] == 0.0 and np.count_nonzero(q == 0) == 1
    assert np.sum(q < 0) == 7 and np.sum(q > 0) == 8


def test_nf4_table_is_normal_quantiles():
    """The positive levels sit at evenly spaced probabilities of N(0,1), from
    1/2 up to 1 - delta; the negative ones likewise with one level fewer.
    Checked with scipy's forward CDF (ndtr), not the inverse used to build it."""
    q = oracle.nf4_table().astype(np.float64)
    delta = 0.5 * (1 / 30 + 1 / 32)
    zmax = None
    # un-normalise with the top quantile: Phi(zmax) = 1 - delta
    lo, hi = 0.0, 10.0
    for _ in range(200):
        mid = (lo + hi) / 2
        lo, hi = (mid, hi) if ndtr(mid) < 1 - delta else (lo, mid)
    zmax = lo
    pos = ndtr(q[8:] * zmax)                 # 8 positive levels, ascending
    neg = ndtr(-q[:7] * zmax)                # 7 negative levels, descending mass
    # fp32 rounding of q moves Phi by at most ~ pdf * zmax * 2^-24 * |q|
    assert np.allclose(np.diff(np.concatenate([[0.5], pos])), (1 - delta - 0.5) / 8, atol=2e-7)
    assert np.allclose(np.diff(np.concatenate([[0.5], neg[::-1]])), (1 - delta - 0.5) / 7, atol=2e-7)


def test_nf4_finer_near_zero():
    """'The steps are noticeably finer near zero ... coarser out in the tails'."""
    q = oracle.nf4_table().astype(np.float64)
    gaps_pos = np.diff(q[7:])
    gaps_neg = np.diff(q[:8])[::-1]
    assert np.all(np.diff(gaps_pos) > 0)
    assert np.all(np.diff(gaps_neg) > 0)
    assert gaps_pos[0] < 2 / 15 and gaps_neg[0] < 2 / 15


def test_nf4_beats_uniform_on_gaussian_weights():
    """'Same four bits ... buys back a large part of the accuracy that even
    spacing threw away' (That is NF4); NF4 beats uniform INT4 (quiz page)."""
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((256, 1024)) * 0.02).astype(np.float32)
    errs = {}
    for name, table in (("nf4", oracle.nf4_table()), ("uniform", oracle.uniform_table())):
        codes, a = oracle.quantize(W, table)
        Wd = oracle.dequantize(oracle.pack(codes), a, W.shape, table)
        errs[name] = float(np.sqrt(np.mean((Wd - W) ** 2)))
    assert errs["nf4"] < 0.95 * errs["uniform"]


# ---------------------------------------------------------------------------
# Nearest code: thresholds vs exact rational brute force
# ---------------------------------------------------------------------------

def _brute_code(x: float, table) -> int:
    """argmin over codes of |x - q_code| in exact rationals; ties -> the
    higher value, then the lower code (+0 before -0)."""
    fx = Fraction(float(x))
    best, bi = None, -1
    for i, qi in enumerate(table):
        fq = Fraction(float(qi))
        key = (abs(fx - fq), -fq, i)
        if best is None or key < best:
            best, bi = key, i
    return bi


_TABLES = {"nf4": oracle.nf4_table, "uniform": oracle.uniform_table, "fp4": oracle.fp4_table}


@pytest.mark.parametrize("table_name", ["nf4", "uniform", "fp4"])
def test_threshold_code_equals_brute_force(table_name):
    table = _TABLES[table_name]()
    xs = []
    q = np.unique(table.astype(np.float64))
    for j in range(q.size - 1):
        m = np.float32((q[j] + q[j + 1]) / 2)
        v = m
        for _ in range(5):
            v = np.nextafter(v, np.float32(-2))
        for _ in range(11):
            xs.append(v)
            v = np.nextafter(v, np.float32(2))
    rng = np.random.default_rng(3)
    xs += list(rng.uniform(-1, 1, 2000).astype(np.float32))
    xs += [np.float32(v) for v in (-1.0, 1.0, 0.0, -0.0)] + list(table)
    xs = np.array(xs, dtype=np.float32)
    got = oracle.nearest_code(xs, table)
    want = np.array([_brute_code(x, table) for x in xs])
    assert np.array_equal(got, want)


def test_fp4_table_from_the_float_layout():
    """The FP4 reading: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 under codes
    0..7 (the E2M1 values listed, not derived from the bit fields), the sign
    in bit 3, divided by 6; 15 distinct values ascending with +0 stored as
    code 0."""
    t = oracle.fp4_table()
    listed = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        want = np.float32(listed[c & 7] / 6.0)
        assert t[c] == (-want if c & 8 else want)
    assert np.signbit(t[8]) and not np.signbit(t[0])
    vals, codes = oracle.distinct_values(t)
    assert vals.size == 15 and np.all(np.diff(vals) > 0)
    assert vals[0] == -1 and vals[-1] == 1 and codes[7] == 0
    assert oracle.thresholds(t).size == 14
    # the ends are exact: the absmax element dequantises to +/- the scale
    W = np.array([[0.3, -0.02, 0.0, -0.7] + [0.01] * 60], dtype=np.float32)
    c, a = oracle.quantize(W, t)
    deq = oracle.dequantize(oracle.pack(c), a, W.shape, table=t)
    assert deq[0, 3] == oracle.round_bf16(np.float32(-0.7)) and deq[0, 2] == 0.0


@pytest.mark.parametrize("table_name", ["nf4", "fp4"])
def test_quantize_tiny_blocks_brute_force(table_name):
    """Whole quantise path on tiny random blocks vs rational brute force."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((4, 128)) * 0.02).astype(np.float32)
    W[1, :64] = 0.0                                       # zero block: every code is +0's
    table = _TABLES[table_name]()
    codes, a = oracle.quantize(W, table)
    blk = W.reshape(-1, 64)
    assert np.array_equal(a, np.abs(blk).max(axis=1))
    for b in range(blk.shape[0]):
        for i in range(64):
            x = np.float32(0) if a[b] == 0 else np.float32(blk[b, i]) / np.float32(a[b])   # RN32 division
            assert codes[64 * b + i] == _brute_code(x, table)


# ---------------------------------------------------------------------------
# The pages' worked example, uniform table
# ---------------------------------------------------------------------------

def _example_block(values, scale=0.08):
    blk = np.zeros(64, dtype=np.float32)
    blk[0] = np.float32(scale)
    blk[1:1 + len(values)] = np.array(values, dtype=np.float32)
    return blk.reshape(1, 64)


def test_worked_example_uniform_table(golden):
    g = golden
    u = oracle.uniform_table()
    assert u[1] - u[0] == pytest.approx(g["uniform_step"], abs=5e-4)
    assert u[1] == pytest.approx(g["uniform_row_1"], abs=5e-4)
    assert u[2] == pytest.approx(g["uniform_row_2"], abs=5e-4)

    W = _example_block([g["example_w"], g["small_w"], 0.0])
    codes, a = oracle.quantize(W, u)
    assert a[0] == np.float32(g["example_scale"])
    x = oracle.normalise(W, a)[0]
    assert x[1] == pytest.approx(g["example_x"], abs=5e-4)
    assert x[2] == pytest.approx(g["small_x"], abs=5e-5)
    # step 3: nearest rows
    assert u[codes[1]] == pytest.approx(g["example_row"], abs=5e-4)
    assert u[codes[1] - 1] == pytest.approx(g["example_lower_row"], abs=5e-4)
    assert (u[codes[2] - 1], u[codes[2]]) == pytest.approx(g["small_rows"], abs=5e-5)
    # step 4 and the two failures: read back = row * scale (fp32, before bf16)
    back = (u[codes] * a[0]).astype(np.float32)
    assert back[1] == pytest.approx(g["example_back"], abs=5e-5)
    assert abs(back[1] - g["example_w"]) == pytest.approx(g["example_loss"], abs=5e-5)
    assert back[2] == pytest.approx(g["small_back"], abs=5e-5)
    assert abs(back[2] - g["small_w"]) / g["small_w"] == pytest.approx(g["small_rel_err"], abs=5e-3)
    # zero lands exactly between the two middle rows and goes up
    assert codes[3] == 8
    assert back[3] == pytest.approx(g["zero_back"], abs=5e-5)


# ---------------------------------------------------------------------------
# Quantise invariants
# ---------------------------------------------------------------------------

def test_zero_block_and_signed_zero():
    W = np.zeros((1, 128), dtype=np.float32)
    W[0, 64] = -0.0
    W[0, 65] = 0.5
    codes, a = oracle.quantize(W)
    assert a[0] == 0 and a[1] == 0.5
    assert np.all(codes[:64] == 7)        # all-zero block -> the exact-zero row
    assert codes[64] == 7                 # -0.0 -> zero row
    assert codes[65] == 15                # +absmax -> +1 row
    Wd = oracle.dequantize(oracle.pack(codes), a, W.shape)
    assert np.all(Wd[0, :64] == 0) and not np.signbit(Wd[0, 64])


def test_absmax_element_maps_to_table_ends():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32)
    codes, a = oracle.quantize(W)
    blk = W.reshape(-1, 64)
    c = codes.reshape(-1, 64)
    for b in range(blk.shape[0]):
        i = int(np.argmax(np.abs(blk[b])))
        assert c[b, i] == (15 if blk[b, i] > 0 else 0)


def test_permutation_and_power_of_two_scaling():
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((2, 64)) * 0.02).astype(np.float32)
    codes, a = oracle.quantize(W)
    perm = rng.permutation(64)
    codes_p, a_p = oracle.quantize(W[:, perm])
    assert np.array_equal(codes_p.reshape(2, 64), codes.reshape(2, 64)[:, perm])
    assert np.array_equal(a_p, a)
    codes_s, a_s = oracle.quantize(W * np.float32(2.0 ** -5))
    assert np.array_equal(codes_s, codes)
    assert np.array_equal(a_s, a * np.float32(2.0 ** -5))


def test_outlier_damage_stays_in_its_block():
    """'Keeping groups small keeps an outlier's damage inside its own group.'"""
    rng = np.random.default_rng(13)
    W = (rng.standard_normal((4, 256)) * 0.02).astype(np.float32)
    W2 = W.copy()
    W2[1, 70] = 3.0                       # block index (256 + 70) // 64 = 5
    c1, a1 = oracle.quantize(W)
    c2, a2 = oracle.quantize(W2)
    diff_blocks = np.unique(np.nonzero(c1 != c2)[0] // 64)
    assert list(diff_blocks) == [5]
    assert list(np.nonzero(a1 != a2)[0]) == [5]
    # the outlier block's ordinary weights collapse onto the middle rows
    assert np.all(np.isin(np.delete(c2.reshape(-1, 64)[5], 6), [6, 7, 8]))


def test_nonfinite_rejected():
    W = np.zeros((1, 64), dtype=np.float32)
    W[0, 3] = np.nan
    with pytest.raises(ValueError):
        oracle.quantize(W)
    W[0, 3] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(W)


def test_pack_nibble_order_and_roundtrip():
    codes = np.array([1, 2, 3, 4, 15, 0], dtype=np.uint8)
    p = oracle.pack(codes)
    assert list(p) == [0x12, 0x34, 0xF0]
    rng = np.random.default_rng(1)
    c = rng.integers(0, 16, 1000).astype(np.uint8)
    assert np.array_equal(oracle.unpack(oracle.pack(c)), c)
    assert oracle.pack(c).size == 500


# ---------------------------------------------------------------------------
# bf16 rounding vs torch
# ---------------------------------------------------------------------------

def test_round_bf16_matches_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * 0.02,
        rng.standard_normal(1000).astype(np.float32) * 1e-38,
        # exact ties: low 16 bits == 0x8000, both parities of the kept part
        (np.arange(1000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0], dtype=np.float32),
    ])
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = oracle.round_bf16(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


# ---------------------------------------------------------------------------
# Double quantisation
# ---------------------------------------------------------------------------

def test_dq_mean_exact():
    """mu against an exact rational mean (tiny) and an fp64 running sum (large)."""
    rng = np.random.default_rng(4)
    a = np.abs(rng.standard_normal(1000).astype(np.float32)) * np.float32(0.05)
    exact = sum(Fraction(float(v)) for v in a) / len(a)
    mu = oracle.dq_mean(a)
    # RN32 of RN64(sum)/n: within half an fp32 ulp of the exact mean plus 2^-52 relative
    assert abs(Fraction(float(mu)) - exact) <= Fraction(float(np.spacing(mu))) / 2 + exact * Fraction(1, 2 ** 51)
    big = np.abs(rng.standard_normal(200000).astype(np.float32))
    s = 0.0
    for v in big.astype(np.float64):
        s += v
    assert oracle.dq_mean(big) == np.float32(s / big.size)


def test_double_quantize_properties():
    rng = np.random.default_rng(6)
    a = np.abs(rng.standard_normal(1000).astype(np.float32)) * np.float32(0.05)   # 3 full groups + 1 partial
    q, s, mu = oracle.double_quantize(a)
    assert q.dtype == np.int8 and s.shape == (4,)
    d = (a - mu).astype(np.float32)
    for g in range(4):
        dg = d[g * 256:(g + 1) * 256]
        assert s[g] == np.abs(dg).max()
        qg = q[g * 256:(g + 1) * 256]
        assert np.abs(qg).max() == 127
        assert qg[int(np.argmax(np.abs(dg)))] == (127 if dg[np.argmax(np.abs(dg))] > 0 else -127)
    ah = oracle.dq_absmax(q, s, mu)
    sg = np.repeat(s, 256)[:a.size]
    bound = sg / 254 + 4 * np.spacing(np.maximum(np.abs(a), np.abs(ah)))
    assert np.all(np.abs(ah.astype(np.float64) - a) <= bound)


def test_double_quantize_constant_group():
    a = np.full(300, 0.25, dtype=np.float32)
    q, s, mu = oracle.double_quantize(a)
    assert mu == np.float32(0.25)
    assert np.all(s == 0) and np.all(q == 0)
    assert np.all(oracle.dq_absmax(q, s, mu) == np.float32(0.25))


# ---------------------------------------------------------------------------
# The rounding sequence of double quantisation, restated in exact rationals
# ---------------------------------------------------------------------------

def _round_binary(x: Fraction, p: int, emin: int) -> Fraction:
    """Round a rational to the nearest binary float with p significand bits
    and minimum normal exponent emin (subnormals below), ties to even.
    Written from the IEEE 754 definition, independent of NumPy."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    m = abs(x)
    e = m.numerator.bit_length() - m.denominator.bit_length()
    if Fraction(2) ** e > m:
        e -= 1                                   # now 2^e <= m < 2^(e+1)
    e = max(e, emin)
    quantum = Fraction(2) ** (e - p + 1)         # spacing of the grid at m
    k, rem = divmod(m, quantum)                  # m = k * quantum + rem
    half = quantum / 2
    if rem > half or (rem == half and k % 2 == 1):
        k += 1
    return sign * k * quantum


def _rn32(x: Fraction) -> Fraction:
    return _round_binary(x, 24, -126)


def _rn64(x: Fraction) -> Fraction:
    return _round_binary(x, 53, -1022)


def _round_half_even_int(x: Fraction) -> int:
    k = math.floor(x)
    rem = x - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2 == 1):
        k += 1
    return k


def _dq_exact(a: np.ndarray, group: int = 256):
    """Double quantisation restated step by step in rationals: the mean
    RN32(RN64(exact sum)/n) with the fp64 division correctly rounded, then per
    group d = RN32(a - mu), s_g = max|d|, t = RN32(d / s_g), u = RN32(t * 127),
    c = round-half-even(u) (page "QLoRA Explained", section "Shrink the scale
    factors too"; the int8 scale-and-round reading of the same page)."""
    fa = [Fraction(float(v)) for v in a]
    total = _rn64(sum(fa, Fraction(0)))
    mu = _rn32(_rn64(total / len(fa)))
    d = [_rn32(v - mu) for v in fa]
    codes, scales = [], []
    for g0 in range(0, len(d), group):
        dg = d[g0:g0 + group]
        sg = max(abs(v) for v in dg)
        scales.append(sg)
        for v in dg:
            if sg == 0:
                codes.append(0)
                continue
            t = _rn32(v / sg)
            u = _rn32(t * 127)
            codes.append(max(-127, min(127, _round_half_even_int(u))))
    return codes, scales, mu


def _tie_offsets(sg: float, count: int):
    """Offsets e (exact fp32, |e| < sg) for which RN32(RN32(e / sg) * 127) is
    exactly k + 1/2: the integer step then meets a tie."""
    out = []
    fsg = Fraction(sg)
    for k in range(126, -1, -1):
        target = Fraction(2 * k + 1, 2 * 127) * fsg
        e0 = np.float32(float(target))
        for step in range(-24, 25):
            e = np.float32(e0)
            for _ in range(abs(step)):
                e = np.nextafter(e, np.float32(np.inf if step > 0 else -np.inf))
            t = _rn32(Fraction(float(e)) / fsg)
            if _rn32(t * 127) == Fraction(2 * k + 1, 2):
                out.append(float(e))
                break
        if len(out) >= count:
            break
    return out


def test_double_quantize_rounding_sequence_exact_rationals():
    """Every code, scale and the mean of oracle.double_quantize equal the
    rational restatement of the reading c = rint(RN32(RN32(d / s_g) * 127)),
    rounding each step to fp32 by hand.  The inputs include constructed
    near-ties of the integer step (u = k + 1/2 exactly), where swapping the
    order to RN32(d * 127) / s_g or rounding half away from zero changes
    the code."""
    rng = np.random.default_rng(31)
    # (1) random Gaussian-like absmax values: 2 full groups + a partial one
    a1 = (np.abs(rng.standard_normal(600)) * 0.02 + 0.01).astype(np.float32)
    # (2) exact ties: a = 1 +/- e in symmetric pairs, so the mean is exactly 1,
    # d = +/-e exactly, and s_g = 0.5 (the group holds 1.5 and 0.5)
    ties = _tie_offsets(0.5, 100)
    assert len(ties) >= 40
    a2 = [1.5, 0.5]
    for e in ties:
        a2 += [1.0 + e, 1.0 - e]
    a2 = np.array(a2[:256], dtype=np.float32)
    assert np.all((a2.astype(np.float64) - 1.0) == np.array([Fraction(float(v)) - 1 for v in a2], dtype=np.float64))
    for a in (a1, a2):
        q, s, mu = oracle.double_quantize(a)
        codes, scales, mu_x = _dq_exact(a)
        assert Fraction(float(mu)) == mu_x
        assert [Fraction(float(v)) for v in s] == scales
        assert q.astype(int).tolist() == codes
    # the ties decide: rounding half away from zero changes those codes
    q2, _, mu2 = oracle.double_quantize(a2)
    assert mu2 == np.float32(1.0)
    away = 0
    for v, c in zip(a2, q2.astype(int)):
        u = _rn32(_rn32((Fraction(float(v)) - 1) / Fraction(0.5)) * 127)
        if u - math.floor(u) == Fraction(1, 2):
            away += int(math.copysign(math.floor(abs(u)) + 1, float(u))) != c
    assert away >= 20
    # (3) the order of the two fp32 steps matters: with s_g not a power of
    # two, offsets near a tie give other codes under RN32(RN32(d * 127) / s_g)
    sg = float(np.float32(round(0.37 * 2 ** 23) / 2 ** 23))
    fsg = Fraction(sg)
    a3, n_swap = [1.0 + sg, 1.0 - sg], 0
    for k in range(1, 127):
        e0 = round(float(Fraction(2 * k + 1, 254) * fsg) * 2 ** 23)
        for j in range(e0 - 200, e0 + 201):
            d = Fraction(j, 2 ** 23)
            ours = _round_half_even_int(_rn32(_rn32(d / fsg) * 127))
            other = _round_half_even_int(_rn32(_rn32(d * 127) / fsg))
            if ours != other:
                a3 += [1.0 + float(d), 1.0 - float(d)]
                n_swap += 1
                break
    assert n_swap >= 5
    a3 = np.array(a3[:256], dtype=np.float32)
    q3, s3, mu3 = oracle.double_quantize(a3)
    codes, scales, mu_x = _dq_exact(a3)
    assert mu3 == np.float32(1.0) and s3[0] == np.float32(sg)
    assert q3.astype(int).tolist() == codes


def test_storage_closed_forms(golden):
    g = golden
    n = 4096 * 4096
    assert oracle.stored_bits_per_param(n, double_quant=False) - 4 == g["fp32_scale_bits"]
    assert (oracle.stored_bits_per_param(n, double_quant=False) - 4) / 4 == g["fp32_scale_surcharge"]
    bits = oracle.stored_bits_per_param(n)
    assert bits == 4 + 8 / 64 + 32 / 16384 + 32 / n
    assert 8 / 64 == g["dq_scale_bits"]
    assert 32 / 16384 == pytest.approx(g["dq_group_bits"], abs=5e-4)
    assert bits == pytest.approx(g["total_bits"], abs=0.005)
    assert g["total_bits"] / 8 == g["bytes_per_param"]
    saving = oracle.stored_bits_per_param(n, double_quant=False) - bits + 32 / n
    assert saving == 0.373046875
    assert saving == pytest.approx(g["dq_saving_bits"], abs=0.005)
    assert saving < g["dq_saving_bits_upper"]
    assert g["model_7b_params"] * g["bytes_per_param"] / 1e9 == pytest.approx(g["model_7b_nf4_gb"], abs=0.05)
    assert g["model_7b_params"] * 2 / 1e9 == pytest.approx(g["model_7b_bf16_gb"], abs=0.05)
    # N x b / 8
    assert g["model_13b_params"] * 16 / 8 / 1e9 == g["model_13b_fp16_gb"]
    assert g["model_13b_params"] * 4 / 8 / 1e9 == g["model_13b_4bit_gb"]
    # rank-16 adapter on a 4096 x 4096 projection: r*(d+k) = 2rd
    r, d = 16, 4096
    assert r * (d + d) == 2 * r * d == 131072
    assert r * (d + d) == pytest.approx(g["lora_rank16_4096_params"], rel=0.01)
    assert d * d == pytest.approx(g["base_4096_params"], rel=0.01)


# ---------------------------------------------------------------------------
# Dequantise
# ---------------------------------------------------------------------------

def test_dequantize_invariants():
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32)
    codes, a = oracle.quantize(W)
    q, s, mu = oracle.double_quantize(a)
    ah = oracle.dq_absmax(q, s, mu)
    for aa in (a, ah):
        Wd = oracle.dequantize(oracle.pack(codes), aa, W.shape)
        blk = Wd.reshape(-1, 64)
        wb = W.reshape(-1, 64)
        for b in range(blk.shape[0]):
            assert len(np.unique(blk[b])) <= 16
            i = int(np.argmax(np.abs(wb[b])))
            want = oracle.round_bf16(np.array([aa[b]], np.float32))[0]
            assert blk[b, i] == (want if wb[b, i] > 0 else -want)
        # values are bf16-representable
        assert np.array_equal(oracle.round_bf16(Wd), Wd)
        # re-quantising the dequantised weights reproduces the codes (soft
        # invariant; holds on this seed)
        c2, _ = oracle.quantize(Wd)
        assert np.mean(c2 == codes) > 0.999


def test_dequantize_matches_table_times_scale_closed_form():
    """Each element equals RNbf16(q[code] * a^): check with torch's bf16 cast."""
    rng = np.random.default_rng(10)
    W = (rng.standard_normal((4, 128)) * 0.02).astype(np.float32)
    codes, a = oracle.quantize(W)
    Wd = oracle.dequantize(oracle.pack(codes), a, W.shape)
    q = oracle.nf4_table()
    ref = torch.from_numpy((q[codes] * np.repeat(a, 64)).astype(np.float32)).to(torch.bfloat16).float()
    assert np.array_equal(Wd.reshape(-1), ref.numpy())


# ---------------------------------------------------------------------------
# Linear layer vs torch.autograd (fp64)
# ---------------------------------------------------------------------------

def test_linear_fwd_bwd_vs_autograd():
    torch.manual_seed(0)
    M, N, K, r, alpha = 5, 7, 64, 4, 8.0
    X = torch.randn(M, K, dtype=torch.float64, requires_grad=True)
    W = torch.randn(N, K, dtype=torch.float64)
    A = torch.randn(r, K, dtype=torch.float64, requires_grad=True)
    B = torch.randn(N, r, dtype=torch.float64, requires_grad=True)
    dY = torch.randn(M, N, dtype=torch.float64)
    # W' = W + s B A (LoRA page), applied as a Linear: Y = X W'^T
    Y = torch.nn.functional.linear(X, W + (alpha / r) * (B @ A))
    Y.backward(dY)
    Yo, T = oracle.linear_fwd(X.detach().numpy(), W.numpy(), A.detach().numpy(),
                              B.detach().numpy(), alpha, r)
    dX, dA, dB = oracle.linear_bwd(X.detach().numpy(), dY.numpy(), W.numpy(),
                                   A.detach().numpy(), B.detach().numpy(), alpha, r)
    assert np.allclose(Yo, Y.detach().numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dX, X.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dA, A.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dB, B.grad.numpy(), rtol=1e-12, atol=1e-12)
    dA2, dB2 = oracle.linear_bwd_adapters(X.detach().numpy(), dY.numpy(), A.detach().numpy(),
                                          B.detach().numpy(), alpha, r)
    assert np.allclose(dA2, A.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dB2, B.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_linear_special_cases():
    rng = np.random.default_rng(12)
    M, N, K, r = 6, 8, 64, 4
    X = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    A = rng.standard_normal((r, K))
    Y, _ = oracle.linear_fwd(X, W, A, np.zeros((N, r)), 8.0, r)
    assert np.allclose(Y, torch.from_numpy(X) @ torch.from_numpy(W).T, rtol=1e-13)
    # one-hot token rows with A = 0 read out columns of W exactly
    E = np.eye(K)[:M]
    Y, _ = oracle.linear_fwd(E, W, np.zeros((r, K)), rng.standard_normal((N, r)), 8.0, r)
    assert np.array_equal(Y, W[:, :M].T)
    # finite difference on one A entry
    B = rng.standard_normal((N, r))
    dY = rng.standard_normal((M, N))
    _, dA, _ = oracle.linear_bwd(X, dY, W, A, B, 8.0, r)
    eps = 1e-6
    A2 = A.copy()
    A2[1, 3] += eps
    Y1, _ = oracle.linear_fwd(X, W, A, B, 8.0, r)
    Y2, _ = oracle.linear_fwd(X, W, A2, B, 8.0, r)
    fd = np.sum(dY * (Y2 - Y1)) / eps
    assert fd == pytest.approx(dA[1, 3], rel=1e-5)


def test_bf16_in_fp64_products_are_exact():
    """The oracle's fp64 matmul of bf16 inputs: each product is exact (8+8
    significant bits), so for K <= 2^20 the fp64 sum error is tiny relative to
    the 1e-2 bar.  Check one dot product against exact rationals."""
    rng = np.random.default_rng(14)
    x = oracle.round_bf16(rng.standard_normal(4096).astype(np.float32)).astype(np.float64)
    w = oracle.round_bf16((rng.standard_normal(4096) * 0.02).astype(np.float32)).astype(np.float64)
    exact = sum(Fraction(a) * Fraction(b) for a, b in zip(x, w))
    got = float(np.dot(x, w))
    assert abs(Fraction(got) - exact) <= Fraction(1, 2 ** 40) * max(1, abs(exact))
    assert math.isfinite(got)


# ---------------------------------------------------------------------------
# Merge (base dequantised, then the adapter product added)
# ---------------------------------------------------------------------------

def test_round_bf16_f64_matches_torch_on_exact_fp32_values_and_ties():
    """One-step fp64 -> bf16 rounding: equals torch's fp32 -> bf16 cast where
    the fp64 value is an fp32 value, and breaks exact halves to even."""
    rng = np.random.default_rng(41)
    x = (rng.standard_normal(20000) * 0.05).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(oracle.round_bf16_f64(x.astype(np.float64)), want)
    one = 1.0 + 2.0 ** -8                               # halfway between 1 and 1 + 2^-7
    assert oracle.round_bf16_f64(np.array([one]))[0] == 1.0
    assert oracle.round_bf16_f64(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    assert oracle.round_bf16_f64(np.array([one + 2.0 ** -40]))[0] == 1.0 + 2.0 ** -7


def test_merge_special_cases_and_orientation():
    """B = 0 returns the dequantised weight; a rank-1 case worked by hand
    fixes the orientation W[n, k] += s B[n] A[k]; the merged weight is within
    half a bf16 ulp of the exact sum."""
    rng = np.random.default_rng(42)
    W = oracle.round_bf16((rng.standard_normal((6, 64)) * 0.02).astype(np.float32)).astype(np.float64)
    A = rng.standard_normal((8, 64)) * 0.02
    assert np.array_equal(oracle.merge(W, A, np.zeros((6, 8)), 16.0, 8), W)
    A1 = np.zeros((1, 64)); A1[0, 5] = 0.5
    B1 = np.zeros((6, 1)); B1[3, 0] = 0.25
    M1 = oracle.merge(np.zeros((6, 64)), A1, B1, 4.0, 1)
    assert M1[3, 5] == 4.0 * 0.25 * 0.5 and np.count_nonzero(M1) == 1
    B = rng.standard_normal((6, 8)) * 0.02
    Mg = oracle.merge(W, A, B, 16.0, 8)
    exact = W + 2.0 * (B @ A)
    ulp = np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64) * 2.0 ** 16
    assert np.all(np.abs(Mg - exact) <= ulp / 2)


def test_merged_weight_reproduces_the_layer():
    """X W_merged^T equals the layer's forward X W'^T + s (X A^T) B^T (pinned
    against autograd above) up to the bf16 rounding of the merged weight."""
    rng = np.random.default_rng(43)
    N, K, M, r, alpha = 48, 128, 10, 16, 32.0
    W = oracle.round_bf16((rng.standard_normal((N, K)) * 0.02).astype(np.float32)).astype(np.float64)
    A = rng.standard_normal((r, K)) * 0.02
    B = rng.standard_normal((N, r)) * 0.02
    X = rng.standard_normal((M, K))
    Y, _ = oracle.linear_fwd(X, W, A, B, alpha, r)
    Ym = X @ oracle.merge(W, A, B, alpha, r).T
    bound = np.abs(X) @ (np.abs(W + (alpha / r) * B @ A).T * 2.0 ** -8)
    assert np.all(np.abs(Ym - Y) <= bound + 1e-15)
    # and the adapter term is far above that bound (the check has teeth)
    assert np.max(np.abs(X @ oracle.merge(W, A, B, alpha, r).T - (X @ W.T))) > 10 * np.max(bound)


# ---------------------------------------------------------------------------
# LoRA dropout (counter-based mask)
# ---------------------------------------------------------------------------

def test_philox4x64_matches_numpy():
    """oracle.dropout.philox4x64_10 equals NumPy's Philox bit generator (the
    same published generator; NumPy increments its counter before each block,
    so its state c - 1 yields block c)."""
    from oracle import dropout as D
    rng = np.random.default_rng(5)
    for _ in range(20):
        key = [int(v) for v in rng.integers(0, 2 ** 63, 2)]
        ctr = [int(v) for v in rng.integers(1, 2 ** 63, 4)]
        bg = np.random.Philox(key=key, counter=[ctr[0] - 1, ctr[1], ctr[2], ctr[3]])
        want = [int(v) for v in bg.random_raw(4)]
        assert list(D.philox4x64_10(ctr, key)) == want
    bg = np.random.Philox(key=[0, 0])
    st = bg.state                                        # the counter's carry into word 1
    st["state"]["counter"] = np.array([2 ** 64 - 1, 0, 0, 0], dtype=np.uint64)
    st["buffer_pos"] = 4
    bg.state = st
    assert list(D.philox4x64_10((0, 1, 0, 0), (0, 0))) == [int(v) for v in bg.random_raw(4)]


def test_dropout_mask_rate_and_p_zero():
    from oracle import dropout as D
    m = D.keep_mask(64, 256, 0.05, seed=12345)
    n = m.size
    assert abs(m.mean() - 0.95) < 4 * np.sqrt(0.05 * 0.95 / n)
    assert not np.array_equal(m, D.keep_mask(64, 256, 0.05, seed=12346))
    assert D.keep_mask(8, 64, 0.0, seed=1).all()
    # p = 0: the layer is the plain layer
    rng = np.random.default_rng(6)
    X = oracle.round_bf16(rng.standard_normal((8, 64)).astype(np.float32))
    W = rng.standard_normal((16, 64)) * 0.02
    A = rng.standard_normal((8, 64)) * 0.02
    B = rng.standard_normal((16, 8)) * 0.02
    Y0, T0 = oracle.linear_fwd(X, W, A, B, 16.0, 8)
    Y1, T1 = D.linear_fwd_dropout(X, W, A, B, 16.0, 8, np.ones((8, 64), bool), 0.0)
    assert np.array_equal(Y0, Y1) and np.array_equal(T0, T1)


def test_dropout_layer_vs_autograd():
    """With p = 1/2 the kept inputs scale by exactly 2 (no rounding), so the
    fp64 autograd of Y = X W^T + s ((D * 2 X) A^T) B^T pins the forward and
    all three gradients of the dropout layer."""
    from oracle import dropout as D
    rng = np.random.default_rng(7)
    M, K, N, r, alpha, p = 12, 64, 24, 8, 16.0, 0.5
    X = oracle.round_bf16(rng.standard_normal((M, K)).astype(np.float32)).astype(np.float64)
    W = rng.standard_normal((N, K)) * 0.02
    A = rng.standard_normal((r, K)) * 0.02
    B = rng.standard_normal((N, r)) * 0.02
    dY = rng.standard_normal((M, N))
    mask = D.keep_mask(M, K, p, seed=99)
    assert D.keep_scale(p) == 2.0 and 0 < mask.mean() < 1
    Xt = torch.tensor(X, requires_grad=True)
    At = torch.tensor(A, requires_grad=True)
    Bt = torch.tensor(B, requires_grad=True)
    Dm = torch.tensor(mask.astype(np.float64))
    Y = Xt @ torch.tensor(W).T + (alpha / r) * (((Dm * 2.0 * Xt) @ At.T) @ Bt.T)
    Y.backward(torch.tensor(dY))
    Yo, _ = D.linear_fwd_dropout(X, W, A, B, alpha, r, mask, p)
    dX, dA, dB = D.linear_bwd_dropout(X, dY, W, A, B, alpha, r, mask, p)
    np.testing.assert_allclose(Yo, Y.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dX, Xt.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dA, At.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dB, Bt.grad.numpy(), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# 8-bit float double quantisation
# ---------------------------------------------------------------------------

def test_e4m3_encode_matches_torch():
    """The oracle's E4M3 rounding equals torch's float8_e4m3fn cast (round to
    nearest, ties to even) on random values, every representable value and
    every midpoint between neighbours (|x| <= 448, where the cast does not
    saturate)."""
    v = oracle.e4m3_values()
    mids = (v[:-1] + v[1:]) / 2
    rng = np.random.default_rng(12)
    x = np.concatenate([v, mids, -v, -mids, rng.uniform(-300, 300, 5000),
                        rng.standard_normal(5000) * 1e-2]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x)
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.e4m3_decode(got), torch.from_numpy(got).view(torch.float8_e4m3fn).double().numpy())
    assert oracle.e4m3_values()[-1] == 448.0 and oracle.e4m3_values().size == 127


def test_double_quantize_fp8_properties():
    """fp8 variant: the group max maps to code 256 (0x78 = 2^8, t = +/-1
    exactly), and the recovered scales are within E4M3's half-ulp relative
    error of d plus rounding."""
    rng = np.random.default_rng(16)
    a = (np.abs(rng.standard_normal(1000)) * 0.05).astype(np.float32)
    q, s, mu = oracle.double_quantize(a, fmt="fp8")
    d = (a - mu).astype(np.float32)
    for g in range(4):
        dg = d[g * 256:(g + 1) * 256]
        i = int(np.argmax(np.abs(dg)))
        assert (q[g * 256 + i].view(np.uint8) & 0x7F) == 0x78
    ah = oracle.dq_absmax(q, s, mu, fmt="fp8")
    sg = np.repeat(s, 256)[:a.size].astype(np.float64)
    bound = np.abs(d).astype(np.float64) * 2.0 ** -4 + sg * 2.0 ** -17 + 4 * np.spacing(np.abs(a))
    assert np.all(np.abs(ah.astype(np.float64) - a) <= bound)
    q8, _, _ = oracle.double_quantize(a)
    assert not np.array_equal(q, q8)
