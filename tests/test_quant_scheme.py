"""The division-free activation-quantiser scheme of the CUDA kernels, checked
against the oracle on the CPU (no GPU needed).

The kernels compute a code as the low byte of RN_fp32(x * c + 1.5 * 2^23)
with c = RU_fp32(127 / a'), one fused multiply-add per element, for every row
whose a' is a bf16 value in [1e-5, 2^120).  The oracle rounds the IEEE
quotient fl32(127 |x|) / a' to nearest even.  This test restates the kernel's
scheme in float64 (the product of a bf16 value and an fp32 value is exact
there, and so is its sum with 1.5 * 2^23, so one cast to float32 is the FMA's
single rounding) and compares it with the oracle on every bf16 |x| <= a' in
the twelve binades at and below a', for all bf16 a' of several binades.
The same scheme with c rounded to nearest must disagree (at the ties
|x| = a' / 2), which shows the comparison can fail.
"""
import numpy as np
import pytest
import torch

import oracle

MAGIC = 12582912.0  # 1.5 * 2^23: the sum's ulp is 1


def _bf16_binades(lo, hi):
    e = np.arange(lo, hi)[:, None]
    return ((1.0 + np.arange(128)[None, :] / 128.0) * 2.0 ** e).ravel()


def _reciprocal_127(ap, round_up):
    c = np.float32(127.0 / ap)
    if round_up and float(c) * ap < 127.0:  # the product of the two is exact in float64
        c = np.nextafter(c, np.float32(np.inf))
    return float(c)


def _scheme_codes(xs, ap, round_up):
    s = (xs * _reciprocal_127(ap, round_up) + MAGIC).astype(np.float32)
    return (s.astype(np.float64) - MAGIC).astype(np.int64)


def _rows(exp):
    """Rows for every bf16 a' of binade `exp`: a', then every bf16 |x| < a'
    of the twelve binades up to a''s, with alternating signs."""
    aps = _bf16_binades(exp, exp + 1)
    xs_all = _bf16_binades(exp - 11, exp + 1)
    k = 12 * 128 * 2 + 64
    rows = np.zeros((aps.size, k), dtype=np.float64)
    for r, ap in enumerate(aps):
        xs = xs_all[xs_all < ap]
        rows[r, 0] = ap
        rows[r, 1:1 + xs.size] = xs
        rows[r, 1 + xs.size:1 + 2 * xs.size] = -xs
    return aps, rows


@pytest.mark.parametrize("exp", [-16, -1, 0, 7, 64, 119])
def test_fma_with_rounded_up_reciprocal_matches_oracle(exp):
    aps, rows = _rows(exp)
    x = torch.from_numpy(rows.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(x.double().numpy(), rows)  # every value is a bf16 value
    xq_ref, ap_ref = oracle.act_quant(x)
    assert np.array_equal(ap_ref.astype(np.float64), aps)
    ties = 0
    for r, ap in enumerate(aps):
        got = _scheme_codes(rows[r], ap, round_up=True)
        assert np.array_equal(got, xq_ref[r].astype(np.int64)), (exp, ap)
        ties += int((np.abs(rows[r]) == ap / 2).sum())
    assert ties >= 2 * 127  # the |x| = a'/2 ties are in the grid


def test_round_to_nearest_reciprocal_fails_on_ties():
    aps, rows = _rows(0)
    x = torch.from_numpy(rows.astype(np.float32)).to(torch.bfloat16)
    xq_ref, _ = oracle.act_quant(x)
    wrong = 0
    for r, ap in enumerate(aps):
        got = _scheme_codes(rows[r], ap, round_up=False)
        bad = got != xq_ref[r].astype(np.int64)
        wrong += int(bad.sum())
        # every disagreement is a tie |x| = a'/2 rounded to 63 instead of 64
        assert (np.abs(rows[r][bad]) == ap / 2).all() and (np.abs(got[bad]) == 63).all()
    assert wrong > 0
