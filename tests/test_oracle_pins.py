"""Pins for the CPU oracle (runs without a GPU).

Each test checks one oracle function against something other than the
oracle itself: hand-derived golden cases, exact rational arithmetic with
Python's ``fractions``, closed-form statistics, numpy library routines or
brute-force enumeration.  A plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong rounding direction) fails
at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from sparse_linear_layers_bitlinear_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16_bits(values):
    return synth.bits(torch.tensor(values, dtype=torch.float32).to(torch.bfloat16))


def _bf16_float(bits_u16):
    """Exact float value of bf16 bit patterns (via the fp32 pattern)."""
    return (np.asarray(bits_u16, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Independent exact rounding helpers (rational arithmetic, no shared code).
# ---------------------------------------------------------------------------
def _rne(q: Fraction) -> int:
    return round(q)  # Fraction.__round__ rounds half to even


def _fraction_to_f32(q: Fraction) -> np.float32:
    """Nearest-even fp32 of a non-negative rational, via exact arithmetic."""
    assert q >= 0
    if q == 0:
        return np.float32(0.0)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    lsb = max(e - 23, -149)
    n = _rne(q / Fraction(2) ** lsb)
    return np.float32(math.ldexp(n, lsb))


def _fraction_to_bf16_value(q: Fraction) -> float:
    sign = -1.0 if q < 0 else 1.0
    q = abs(q)
    if q == 0:
        return 0.0
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    lsb = max(e - 7, -133)
    n = _rne(q / Fraction(2) ** lsb)
    v = math.ldexp(n, lsb)
    if v >= 2.0 ** 128:
        return sign * math.inf
    return sign * v


def _exact_mean_f32(w_bits) -> np.float32:
    vals = _bf16_float(w_bits).ravel()
    s = sum((Fraction(abs(float(v))) for v in vals), Fraction(0))
    return _fraction_to_f32(s / len(vals))


# ---------------------------------------------------------------------------
# A1: absmean scale
# ---------------------------------------------------------------------------
def test_gamma_golden_cases():
    for case in _golden("gamma_cases.json")["cases"]:
        w = _bf16_bits(case["w"])
        gamma = oracle.absmean_gamma(w)
        assert gamma == np.float32(case["gamma"]), case
        assert oracle.clamped_scale(gamma) == np.float32(case["g"]), case


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_gamma_equals_exact_rational_mean(seed):
    rng = np.random.default_rng(seed)
    n = 3001 + 997 * seed
    # Mix of scales, including subnormal bf16 magnitudes and large exponents,
    # so that the exact sum spans far more than 53 bits.
    bits = rng.integers(0, 0x7F80, size=n, dtype=np.uint32).astype(np.uint16)
    bits |= (rng.integers(0, 2, size=n, dtype=np.uint32) << 15).astype(np.uint16)
    if seed % 2:
        bits[: n // 3] &= 0x807F  # subnormal and zero magnitudes
    assert oracle.absmean_gamma(bits) == _exact_mean_f32(bits)


@pytest.mark.parametrize("seed", [5, 6])
def test_gamma_gaussian_weights_exact(seed):
    w = synth.master_weights(64, 96, seed)
    assert oracle.absmean_gamma(w) == _exact_mean_f32(synth.bits(w))


def test_gamma_constant_magnitude():
    for c in [1.0, 0.015625, 3.0e38, 2.0 ** -133, 2.0 ** -126, 0.3]:
        vals = np.full(777, c, dtype=np.float32)
        vals[::3] *= -1
        w = _bf16_bits(vals)
        c_bf16 = float(_bf16_float(w[:1])[0])
        c_bf16 = abs(c_bf16)
        assert float(oracle.absmean_gamma(w)) == float(np.float32(c_bf16))


def test_gamma_underflow_to_fp32_subnormal_and_zero():
    w = np.zeros(1 << 16, dtype=np.uint16)
    w[7] = 0x0001  # 2^-133, the smallest bf16 subnormal
    # exact mean 2^-149 is the smallest fp32 subnormal
    assert oracle.absmean_gamma(w) == np.float32(2.0 ** -149)
    w2 = np.zeros(1 << 17, dtype=np.uint16)
    w2[3] = 0x0001  # mean 2^-150: a tie between 0 and 2^-149, even gives 0
    assert oracle.absmean_gamma(w2) == np.float32(0.0)
    w3 = np.zeros(1 << 17, dtype=np.uint16)
    w3[3] = 0x0001
    w3[4] = 0x0001  # 2^-149 exactly
    assert oracle.absmean_gamma(w3) == np.float32(2.0 ** -149)
    assert oracle.clamped_scale(np.float32(0.0)) == np.float32(1e-5)


def test_gamma_nonfinite_is_nan():
    w = _bf16_bits([1.0, float("inf"), 2.0])
    assert np.isnan(oracle.absmean_gamma(w))
    w = _bf16_bits([1.0, float("nan")])
    assert np.isnan(oracle.absmean_gamma(w))


def test_gamma_gaussian_statistic():
    # E|w| = sigma * sqrt(2/pi) for w ~ N(0, sigma^2); standard error of the
    # mean is sigma * sqrt(1 - 2/pi) / sqrt(n).
    w = synth.master_weights(1024, 1024, seed=11)
    n = w.numel()
    expect = 0.02 * math.sqrt(2 / math.pi)
    se = 0.02 * math.sqrt(1 - 2 / math.pi) / math.sqrt(n)
    assert abs(float(oracle.absmean_gamma(w)) - expect) < 6 * se + 1e-5 * expect


# ---------------------------------------------------------------------------
# A2: N:M mask
# ---------------------------------------------------------------------------
def test_mask_golden_cases():
    for case in _golden("mask_cases.json")["cases"]:
        w = _bf16_bits(case["w"]).reshape(1, -1)
        mask = oracle.nm_mask(w, case["n"], case["m"])
        assert int(mask[0, 0]) == case["mask"], case


def _brute_force_mask(mags, n):
    """The kept set is the unique size-n subset whose every member beats every
    non-member under (magnitude descending, index ascending)."""
    m = len(mags)
    winners = []
    for subset in itertools.combinations(range(m), n):
        s = set(subset)
        ok = all(
            (mags[i] > mags[j]) or (mags[i] == mags[j] and i < j)
            for i in s
            for j in range(m)
            if j not in s
        )
        if ok:
            winners.append(subset)
    assert len(winners) == 1
    return sum(1 << i for i in winners[0])


@pytest.mark.parametrize("n,m", [(1, 2), (2, 4), (1, 4), (3, 4), (6, 8), (4, 8), (3, 8), (2, 8), (5, 8)])
def test_mask_brute_force(n, m):
    rng = np.random.default_rng(100 * n + m)
    rows, groups = 9, 13
    # Draw from a small set of values so that ties (and +-0) are frequent.
    pool = np.array([0.0, -0.0, 0.5, -0.5, 0.25, 1.0, -1.0, 0.125, 2.0], dtype=np.float32)
    vals = pool[rng.integers(0, len(pool), size=rows * groups * m)].reshape(rows, groups * m)
    w = _bf16_bits(vals)
    mask = oracle.nm_mask(w, n, m)
    mags = np.abs(_bf16_float(w))
    for r in range(rows):
        for g in range(groups):
            want = _brute_force_mask(list(mags[r, g * m:(g + 1) * m]), n)
            assert int(mask[r, g]) == want


@pytest.mark.parametrize("n,m", [(2, 4), (6, 8), (4, 8), (8, 8)])
def test_mask_invariants_gaussian(n, m):
    w = synth.master_weights(40, 64, seed=3)
    wb = synth.bits(w)
    mask = oracle.nm_mask(wb, n, m)
    mags = np.abs(_bf16_float(wb))
    for r in range(wb.shape[0]):
        for g in range(wb.shape[1] // m):
            bits = int(mask[r, g])
            kept = [j for j in range(m) if bits >> j & 1]
            dropped = [j for j in range(m) if not bits >> j & 1]
            assert len(kept) == n
            grp = mags[r, g * m:(g + 1) * m]
            for i in kept:
                for j in dropped:
                    assert grp[i] > grp[j] or (grp[i] == grp[j] and i < j)


def test_mask_from_codes_golden_cases():
    for case in _golden("mask_from_codes_cases.json")["cases"]:
        q = np.array(case["q"], dtype=np.int8).reshape(1, -1)
        mask = oracle.nm_mask_from_codes(q, case["n"], case["m"])
        assert int(mask[0, 0]) == case["mask"], case


@pytest.mark.parametrize("n,m", [(1, 2), (2, 4), (3, 4), (6, 8), (4, 8), (3, 8)])
def test_mask_from_codes_brute_force(n, m):
    rng = np.random.default_rng(300 + 10 * n + m)
    q = rng.choice(np.array([-1, 0, 1], dtype=np.int8), size=(7, 11 * m))
    mask = oracle.nm_mask_from_codes(q, n, m)
    for r in range(q.shape[0]):
        for g in range(q.shape[1] // m):
            want = _brute_force_mask([abs(int(v)) for v in q[r, g * m:(g + 1) * m]], n)
            assert int(mask[r, g]) == want


def test_mask_from_codes_differs_from_master_mask():
    """The two masks coincide where the codes separate the magnitudes and
    differ where a kept master magnitude quantises to 0 next to a nonzero one
    that the master mask dropped; on Gaussian masters both must occur."""
    w = synth.master_weights(64, 256, seed=8)
    p_master = oracle.prepare(w, 2, 4)
    p_codes = oracle.prepare(w, 2, 4, mask_from_codes=True)
    assert np.array_equal(p_master["q"], p_codes["q"])
    same = p_master["mask"] == p_codes["mask"]
    assert same.any() and (~same).any()
    # every code the master mask keeps nonzero is at least matched in count
    nz_kept = lambda p: int(np.count_nonzero(p["weff"]))
    assert nz_kept(p_codes) >= nz_kept(p_master)


# ---------------------------------------------------------------------------
# A3: ternary codes, quant-then-mask, packing
# ---------------------------------------------------------------------------
def test_ternary_golden_cases():
    gold = _golden("ternary_cases.json")
    w = _bf16_bits([c["w"] for c in gold["cases"]])
    q = oracle.ternary(w, np.float32(gold["g"]))
    assert list(q) == [c["q"] for c in gold["cases"]]


@pytest.mark.parametrize("seed", [0, 1])
def test_ternary_equals_rational_round_clip(seed):
    w = synth.master_weights(32, 80, seed)
    wb = synth.bits(w)
    g = oracle.clamped_scale(oracle.absmean_gamma(wb))
    q = oracle.ternary(wb, g)
    gq = Fraction(float(g))
    vals = _bf16_float(wb).ravel()
    for v, code in zip(vals, q.ravel()):
        r = Fraction(float(v)) / gq
        r = max(Fraction(-1), min(Fraction(1), r))
        assert _rne(r) == int(code)
    # exact boundary |w| = g/2 maps to 0, just above maps to sign(w)
    g2 = np.float32(0.03125)
    wb2 = _bf16_bits([0.015625, -0.015625, 0.0157470703125, -0.0157470703125])
    assert list(oracle.ternary(wb2, g2)) == [0, 0, 1, -1]


def test_ternary_zero_fraction_closed_form():
    # P(|w| <= g/2) for w ~ N(0, s^2) with g = s*sqrt(2/pi) is 2*Phi(sqrt(2/pi)/2) - 1.
    w = synth.master_weights(1024, 1024, seed=21)
    wb = synth.bits(w)
    g = oracle.clamped_scale(oracle.absmean_gamma(wb))
    q = oracle.ternary(wb, g)
    z = math.sqrt(2 / math.pi) / 2
    p = math.erf(z / math.sqrt(2))  # = 2*Phi(z) - 1
    frac = float(np.mean(q == 0))
    se = math.sqrt(p * (1 - p) / q.size)
    assert abs(frac - p) < 6 * se + 2e-3, (frac, p)
    assert abs(p - 0.3101) < 1e-3


def test_quant_then_mask_and_dense_limit():
    w = synth.master_weights(24, 64, seed=7)
    for n, m in [(2, 4), (6, 8), (4, 8)]:
        p = oracle.prepare(w, n, m)
        q, mask, weff = p["q"], p["mask"], p["weff"]
        expand = np.repeat(mask, m, axis=1)
        pos = np.tile(np.arange(m), mask.shape[1])
        kept = (expand >> pos) & 1
        assert np.array_equal(weff, q * kept)
        assert set(np.unique(weff)).issubset({-1, 0, 1})
        # at most n non-zeros per group of m
        nz = (weff != 0).reshape(weff.shape[0], -1, m).sum(-1)
        assert nz.max() <= n
    # N = M is plain ternary BitLinear: the mask keeps every weight
    p = oracle.prepare(w, 4, 4)
    assert np.array_equal(p["weff"], p["q"])


def test_pack24_round_trip():
    w = synth.master_weights(16, 64, seed=9)
    p = oracle.prepare(w, 2, 4)
    vals, meta = oracle.pack24(p["weff"], p["mask"])
    rebuilt = np.zeros_like(p["weff"])
    for r in range(16):
        for g in range(16):
            byte = int(meta[r, g // 2])
            nib = (byte >> (4 * (g % 2))) & 0xF
            i0, i1 = nib & 3, nib >> 2
            assert i0 < i1
            assert int(p["mask"][r, g]) == (1 << i0) | (1 << i1)
            rebuilt[r, 4 * g + i0] = vals[r, 2 * g]
            rebuilt[r, 4 * g + i1] = vals[r, 2 * g + 1]
    assert np.array_equal(rebuilt, p["weff"])


def test_pack_nm_golden_cases():
    """Hand-worked bytes of the compressed-index pack (mask byte per block of
    8, kept 2-bit codes in index order, least significant bit first)."""
    for case in _golden("pack_nm_cases.json")["cases"]:
        n, m, k = case["n"], case["m"], 64
        weff = np.zeros((1, k), dtype=np.int8)
        mask = np.full((1, k // m), case["rest_group_mask"], dtype=np.uint8)
        for b, blk in enumerate(case["blocks"]):
            weff[0, 8 * b:8 * b + 8] = blk["weff"]
            mask[0, b * (8 // m):(b + 1) * (8 // m)] = blk["group_masks"]
        masks8, codes = oracle.pack_nm(weff, mask, n, m)
        assert list(masks8[0]) == case["masks8"], case["why"]
        assert list(codes[0]) == case["codes"], case["why"]


def _unpack_nm(masks8, codes, n, m, k):
    """Decode the compressed-index pack back to dense codes, block by block."""
    n_out = masks8.shape[0]
    out = np.zeros((n_out, k), dtype=np.int8)
    value = {0: 0, 1: 1, 3: -1}
    for r in range(n_out):
        stream = int.from_bytes(codes[r].tobytes(), "little")
        pos = 0
        for b in range(k // 8):
            mb = int(masks8[r, b])
            for j in range(8):
                if mb >> j & 1:
                    c = (stream >> pos) & 3
                    assert c != 2, "code 10 is never written"
                    out[r, 8 * b + j] = value[c]
                    pos += 2
        assert pos == 2 * (8 * n // m) * (k // 8)
    return out


@pytest.mark.parametrize("n,m", [(6, 8), (4, 8), (3, 8), (1, 8), (7, 8), (8, 8), (1, 4), (3, 4), (1, 2), (2, 4)])
def test_pack_nm_round_trip_and_invariants(n, m):
    """The pack decodes back to W_eff exactly; every block keeps 8n/m
    positions, each group of m exactly n, and they are the mask's."""
    k = 128
    w = synth.master_weights(12, k, seed=40 + 8 * n + m)
    p = oracle.prepare(w, n, m)
    masks8, codes = oracle.pack_nm(p["weff"], p["mask"], n, m)
    assert masks8.shape == (12, k // 8) and codes.shape == (12, k * n // (4 * m))
    bits = np.unpackbits(masks8[..., None], axis=-1, bitorder="little").reshape(12, k)
    assert (bits.reshape(12, -1, m).sum(-1) == n).all()
    dense_mask = np.unpackbits(p["mask"][..., None], axis=-1, bitorder="little")[..., :m].reshape(12, k)
    assert np.array_equal(bits, dense_mask)
    assert np.array_equal(_unpack_nm(masks8, codes, n, m, k), p["weff"])
    # the pack is no larger than 1 + 2n/m bits per weight (2.5 at 6:8)
    assert masks8.nbytes + codes.nbytes == 12 * k * (1 + 2 * n / m) / 8


def test_pack24_code6_golden_cases():
    """Hand-worked bytes of the 6-bit 2:4 group code."""
    for case in _golden("pack24_code6_cases.json")["cases"]:
        weff = np.array([case["weff"]], dtype=np.int8)
        mask = np.array([case["group_masks"]], dtype=np.uint8)
        assert list(oracle.pack24_code6(weff, mask)[0]) == case["bytes"], case["why"]


_PAIRS = [(a, b) for a in range(4) for b in range(a + 1, 4)]


def _unpack_code6(packed, k):
    """Decode the 6-bit group code by division: (weff [n_out, k], group masks)."""
    n_out = packed.shape[0]
    weff = np.zeros((n_out, k), dtype=np.int8)
    masks = np.zeros((n_out, k // 4), dtype=np.uint8)
    value = {0: 0, 1: 1, 2: -1}
    for r in range(n_out):
        stream = int.from_bytes(packed[r].tobytes(), "little")
        for gi in range(k // 4):
            state = (stream >> (6 * gi)) & 63
            assert state < 54
            p, rest = divmod(state, 9)
            d0, d1 = divmod(rest, 3)
            i0, i1 = _PAIRS[p]
            weff[r, 4 * gi + i0], weff[r, 4 * gi + i1] = value[d0], value[d1]
            masks[r, gi] = (1 << i0) | (1 << i1)
    return weff, masks


def test_pack24_code6_is_a_bijection_onto_54_states():
    """Every (kept pair, code, code) of a group gets its own state below 54,
    and the all-zero group under the pair (0, 1) is state 0 (so zero bytes
    decode to zero weights)."""
    combos = [(pair, c0, c1) for pair in _PAIRS for c0 in (-1, 0, 1) for c1 in (-1, 0, 1)]
    k = 4 * 56  # 54 groups, padded to a multiple of 16 with zero groups under (0, 1)
    weff = np.zeros((1, k), dtype=np.int8)
    mask = np.full((1, k // 4), 3, dtype=np.uint8)
    for gi, ((i0, i1), c0, c1) in enumerate(combos):
        weff[0, 4 * gi + i0], weff[0, 4 * gi + i1] = c0, c1
        mask[0, gi] = (1 << i0) | (1 << i1)
    packed = oracle.pack24_code6(weff, mask)
    stream = int.from_bytes(packed[0].tobytes(), "little")
    states = [(stream >> (6 * gi)) & 63 for gi in range(k // 4)]
    assert sorted(states[:54]) == list(range(54))
    assert states[54:] == [0, 0]
    assert states[combos.index(((0, 1), 0, 0))] == 0
    back, masks = _unpack_code6(packed, k)
    assert np.array_equal(back, weff) and np.array_equal(masks, mask)


@pytest.mark.parametrize("seed", [0, 1])
def test_pack24_code6_round_trip(seed):
    """On prepared 2:4 weights the code decodes back to W_eff and the mask,
    at 1.5 bits a weight."""
    k = 256
    w = synth.master_weights(10, k, seed=70 + seed)
    p = oracle.prepare(w, 2, 4)
    packed = oracle.pack24_code6(p["weff"], p["mask"])
    assert packed.shape == (10, 3 * k // 16)
    back, masks = _unpack_code6(packed, k)
    assert np.array_equal(back, p["weff"])
    assert np.array_equal(masks, p["mask"])


# ---------------------------------------------------------------------------
# A4: activation quantisation
# ---------------------------------------------------------------------------
def test_act_quant_golden_cases():
    for case in _golden("act_quant_cases.json")["cases"]:
        x = _bf16_bits(case["x"]).reshape(1, -1)
        xq, ap = oracle.act_quant(x)
        assert list(xq[0]) == case["xq"], case
        assert ap[0] == np.float32(case["a_prime"]), case


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_act_quant_equals_rational_rne(seed):
    x = synth.activations(6, 200, seed)
    xb = synth.bits(x)
    xq, ap = oracle.act_quant(xb)
    vals = _bf16_float(xb)
    for r in range(vals.shape[0]):
        a = max(abs(float(v)) for v in vals[r])
        assert ap[r] == np.float32(max(a, np.float32(1e-5)))
        A = Fraction(a)
        for v, code in zip(vals[r], xq[r]):
            n = _rne(127 * abs(Fraction(float(v))) / A)
            n = min(n, 127)
            want = -n if v < 0 else n
            assert int(code) == want
        assert np.max(np.abs(xq[r])) == 127  # the argmax element maps to +-127


# ---------------------------------------------------------------------------
# A5 / A6: integer product and dequant
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("t,n_out,k", [(1, 8, 16), (5, 12, 64), (17, 33, 96)])
def test_gemm_acc_equals_numpy_int64(t, n_out, k):
    rng = np.random.default_rng(t + n_out + k)
    xq = rng.integers(-127, 128, size=(t, k), dtype=np.int64).astype(np.int8)
    weff = rng.integers(-1, 2, size=(n_out, k), dtype=np.int64).astype(np.int8)
    acc = oracle.gemm_acc(xq, weff)
    ref = xq.astype(np.int64) @ weff.astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), ref)
    assert oracle.acc_at(xq, weff, t - 1, n_out - 1) == int(ref[-1, -1])


def test_gemm_acc_extreme_range():
    # |acc| = 127 * k at the extremes: no int32 overflow for realistic k
    k = 8192
    xq = np.full((2, k), 127, dtype=np.int8)
    xq[1] = -127
    weff = np.ones((3, k), dtype=np.int8)
    weff[1] = -1
    weff[2] = 0
    acc = oracle.gemm_acc(xq, weff)
    assert acc.tolist() == [[127 * k, -127 * k, 0], [-127 * k, 127 * k, 0]]


def test_dequant_within_three_roundings_of_exact():
    rng = np.random.default_rng(4)
    acc = rng.integers(-400000, 400000, size=(7, 11), dtype=np.int64).astype(np.int32)
    ap = rng.uniform(0.5, 6.0, size=7).astype(np.float32)
    g = np.float32(0.0159)
    y = oracle.dequant(acc, ap, g)
    u = 2.0 ** -24
    for i in range(7):
        for j in range(11):
            exact = Fraction(int(acc[i, j])) * Fraction(float(g)) * Fraction(float(ap[i])) / 127
            err = abs(Fraction(float(y[i, j])) - exact)
            assert err <= Fraction(4 * u) * abs(exact)
    # g * a' = 127 makes the scale exactly 1
    y1 = oracle.dequant(np.array([[254, -3, 0]], dtype=np.int32), np.array([127.0], np.float32), 1.0)
    assert y1.tolist() == [[254.0, -3.0, 0.0]]


def test_forward_end_to_end_small():
    w = synth.master_weights(8, 32, seed=1)
    x = synth.activations(3, 32, seed=2)
    out = oracle.forward(w, x, 2, 4)
    ref = out["xq"].astype(np.int64) @ out["weff"].astype(np.int64).T
    assert np.array_equal(out["acc"], ref)
    scale = (np.float32(out["g"]) * out["a_prime"]) / np.float32(127)
    assert np.allclose(out["y"], ref * scale[:, None], rtol=1e-6, atol=0)


# ---------------------------------------------------------------------------
# A7 / A8: STE gradients
# ---------------------------------------------------------------------------
def test_grad_x_equals_numpy_matmul():
    w = synth.master_weights(24, 48, seed=3)
    dy = synth.upstream_grad(5, 24, seed=4)
    p = oracle.prepare(w, 2, 4)
    dx = oracle.grad_x(dy, p["weff"], p["g"])
    ref = float(p["g"]) * (_bf16_float(synth.bits(dy)) @ p["weff"].astype(np.float64))
    assert np.allclose(dx, ref, rtol=1e-12, atol=1e-12)
    assert math.isclose(oracle.grad_x_at(dy, p["weff"], p["g"], 4, 47), ref[4, 47], rel_tol=1e-12, abs_tol=1e-12)
    # the gradient ignores pruned weights: changing a pruned code changes nothing
    assert dx.shape == (5, 48)


def test_grad_w_equals_numpy_matmul_and_is_dense():
    dy = synth.upstream_grad(9, 20, seed=5)
    x = synth.activations(9, 36, seed=6)
    dw = oracle.grad_w(dy, x)
    ref = _bf16_float(synth.bits(dy)).T @ _bf16_float(synth.bits(x))
    assert np.allclose(dw, ref, rtol=1e-12, atol=1e-12)
    assert math.isclose(oracle.grad_w_at(dy, x, 19, 35), ref[19, 35], rel_tol=1e-12, abs_tol=1e-12)
    # dense gradient flow: every master weight gets a gradient, including pruned ones
    assert np.count_nonzero(dw) == dw.size


def test_grad_w_masked_blocks_exactly_the_pruned_positions():
    dy = synth.upstream_grad(9, 16, seed=15)
    x = synth.activations(9, 40, seed=16)
    w = synth.master_weights(16, 40, seed=17)
    for n, m in [(2, 4), (6, 8), (1, 2), (8, 8)]:
        mask = oracle.nm_mask(synth.bits(w), n, m)
        dw = oracle.grad_w_masked(dy, x, mask, m)
        dense = _bf16_float(synth.bits(dy)).T @ _bf16_float(synth.bits(x))
        keep = np.repeat(mask[:, :, None], m, axis=2) >> np.arange(m, dtype=np.uint8) & 1
        keep = keep.reshape(16, 40).astype(bool)
        assert np.allclose(dw[keep], dense[keep], rtol=1e-12, atol=1e-12)
        assert (dw[~keep] == 0).all()
        assert keep.sum() == 16 * 40 * n // m
        if n == m:
            assert np.array_equal(dw, oracle.grad_w(dy, x))


def test_round_bf16_matches_rational_rounding():
    rng = np.random.default_rng(8)
    vals = np.concatenate([
        rng.normal(size=500) * 10.0 ** rng.integers(-40, 38, size=500),
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -134, 3 * 2.0 ** -135,
                  2.0 ** -140, 3.4e38, 3.3961e38, 0.0, -0.0]),
    ])
    out = oracle.round_bf16(vals)
    got = _bf16_float(out)
    for v, gv, b in zip(vals, got, out):
        want = _fraction_to_bf16_value(Fraction(float(v)))
        if math.isinf(want):
            assert (int(b) & 0x7FFF) == 0x7F80
        else:
            assert gv == want, (v, gv, want)
    # ties go to even
    assert got[500] == 1.0 and got[501] == 1.0 + 2.0 ** -6 and got[502] == -1.0


# ---------------------------------------------------------------------------
# Thread count: every oracle sum is exact or runs in a fixed order per output,
# so one thread and all threads give identical bits.
# ---------------------------------------------------------------------------
def test_results_do_not_depend_on_thread_count():
    w = synth.master_weights(40, 96, seed=21)
    x = synth.activations(7, 96, seed=22)
    dy = synth.upstream_grad(7, 40, seed=23)

    def run():
        out = oracle.forward(w, x, 2, 4)
        dx = oracle.grad_x(dy, out["weff"], out["g"])
        dw = oracle.grad_w(dy, x)
        return out, dx, dw

    cores = oracle.threads()
    many = run()
    oracle.set_threads(1)
    try:
        assert oracle.threads() == 1 or cores == 1
        one = run()
    finally:
        oracle.set_threads(cores)
    assert oracle.threads() == cores
    for key in ("g", "mask", "weff", "xq", "a_prime", "acc", "y"):
        assert np.array_equal(np.asarray(many[0][key]), np.asarray(one[0][key])), key
    assert np.array_equal(many[1], one[1]) and np.array_equal(many[2], one[2])


# ---------------------------------------------------------------------------
# Detach-form STE operand for dW (SBL_DW_QUANT_X): xhat = RN_bf16(xq a' / 127)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [31, 32])
def test_dequant_act_equals_exact_rational_rounding(seed):
    x = synth.activations(6, 200, seed=seed)
    xb = synth.bits(x).copy()
    xb[0, :3] = [0x0000, 0x8000, 0x3F80]        # zeros and 1.0
    xb[1, :] = 0                                 # all-zero row: a' = 1e-5
    xb[2, 5] = 0x7F7F                            # near the bf16 maximum
    xq, ap = oracle.act_quant(xb)
    got = oracle.dequant_act(xq, ap)
    for r in range(xq.shape[0]):
        for c in range(xq.shape[1]):
            want = _fraction_to_bf16_value(Fraction(int(xq[r, c])) * Fraction(float(ap[r])) / 127)
            gv = float(_bf16_float(got[r, c:c + 1])[0])
            assert gv == want, (r, c, int(xq[r, c]), float(ap[r]), gv, want)
            if xq[r, c] == 0:
                assert got[r, c] == 0  # +0, whatever the sign of x


def test_dequant_act_invariants():
    x = synth.activations(16, 256, seed=33)
    xb = synth.bits(x)
    xq, ap = oracle.act_quant(xb)
    xhat = _bf16_float(oracle.dequant_act(xq, ap)).reshape(xq.shape)
    xf = _bf16_float(xb).reshape(xq.shape)
    for r in range(xq.shape[0]):
        j = int(np.argmax(np.abs(xf[r])))
        # the row's absmax element has code +-127 and comes back exactly
        assert abs(int(xq[r, j])) == 127 and xhat[r, j] == xf[r, j]
        # quantisation error: half a step a'/127, plus the bf16 rounding of xhat
        err = np.abs(xhat[r] - xf[r])
        bound = float(ap[r]) / 254.0 * (1 + 1e-6) + np.abs(xhat[r]) * 2.0 ** -8
        assert np.all(err <= bound)
        assert np.all(np.sign(xhat[r]) * np.sign(xf[r]) >= 0)


def test_grad_w_quant_x_uses_the_dequantised_operand():
    dy = synth.upstream_grad(9, 24, seed=34)
    x = synth.activations(9, 64, seed=35)
    dw_q = oracle.grad_w_quant_x(dy, x)
    xq, ap = oracle.act_quant(x)
    xhat = _bf16_float(oracle.dequant_act(xq, ap)).reshape(xq.shape)
    ref = _bf16_float(synth.bits(dy)).reshape(9, 24).T @ xhat
    assert np.allclose(dw_q, ref, rtol=1e-12, atol=1e-12)
    # and it is not the raw-X gradient
    assert not np.allclose(dw_q, oracle.grad_w(dy, x), rtol=1e-4, atol=0)


# ---------------------------------------------------------------------------
# Property checks over random small cases (hypothesis): the packs decode back
# to W_eff whatever the pattern, shape and codes, and the mask keeps the
# largest magnitudes.
# ---------------------------------------------------------------------------
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

_NM = [(1, 2), (2, 2), (1, 4), (2, 4), (3, 4), (4, 4), (1, 8), (2, 8), (3, 8), (4, 8), (5, 8), (6, 8), (7, 8), (8, 8)]


@st.composite
def _masked_codes(draw):
    n, m = draw(st.sampled_from(_NM))
    rows = draw(st.integers(1, 4))
    k = 64 * draw(st.integers(1, 2))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    mask = np.zeros((rows, k // m), dtype=np.uint8)
    for r in range(rows):
        for g in range(k // m):
            for j in rng.choice(m, size=n, replace=False):
                mask[r, g] |= 1 << int(j)
    codes = rng.integers(-1, 2, size=(rows, k)).astype(np.int8)
    keep = np.unpackbits(mask[..., None], axis=-1, bitorder="little")[..., :m].reshape(rows, k).astype(bool)
    return n, m, np.where(keep, codes, 0).astype(np.int8), mask


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(_masked_codes())
def test_pack_nm_round_trip_on_random_masks(case):
    n, m, weff, mask = case
    masks8, codes = oracle.pack_nm(weff, mask, n, m)
    assert np.array_equal(_unpack_nm(masks8, codes, n, m, weff.shape[1]), weff)


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(_masked_codes().filter(lambda c: (c[0], c[1]) == (2, 4)))
def test_pack24_code6_round_trip_on_random_masks(case):
    _, _, weff, mask = case
    back, masks = _unpack_code6(oracle.pack24_code6(weff, mask), weff.shape[1])
    assert np.array_equal(back, weff) and np.array_equal(masks, mask)


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.sampled_from(_NM), st.integers(0, 2**31 - 1))
def test_mask_keeps_the_largest_magnitudes(nm, seed):
    """Every kept magnitude is at least every dropped one in its group, and a
    drop of an equal magnitude only happens to a higher index (ties to the
    lowest index)."""
    n, m = nm
    rng = np.random.default_rng(seed)
    k = 64
    # few distinct magnitudes, so that ties are common
    w = (rng.integers(-3, 4, size=(2, k)) * 0.25).astype(np.float32)
    wb = synth.bits(torch.from_numpy(w).to(torch.bfloat16))
    mask = oracle.nm_mask(wb, n, m)
    mags = np.abs(w)
    for r in range(2):
        for g in range(k // m):
            bits = [(int(mask[r, g]) >> j) & 1 for j in range(m)]
            assert sum(bits) == n
            for a in range(m):
                for b in range(m):
                    if bits[a] and not bits[b]:
                        ma, mb = mags[r, g * m + a], mags[r, g * m + b]
                        assert ma > mb or (ma == mb and a < b)
