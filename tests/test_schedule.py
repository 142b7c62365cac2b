"""The learning-rate schedule (Table 10: cosine with linear warmup) and its conversion to
the integer multiply-shifts the SGD kernels take (host logic, no GPU)."""
import math

import pytest

from integer_only_nn_02_b200 import schedule as S


def test_cosine_warmup_shape():
    base, total, warm = 0.1, 1000, 50
    lrs = [S.cosine_warmup(t, total, base, warm) for t in range(total + 1)]
    assert lrs[0] == pytest.approx(base / warm)
    assert lrs[warm - 1] == pytest.approx(base)  # warmup ends at the base rate
    assert all(a < b for a, b in zip(lrs[:warm - 1], lrs[1:warm]))  # rises linearly
    assert all(a >= b for a, b in zip(lrs[warm:], lrs[warm + 1:]))  # then only falls
    assert lrs[warm + (total - warm) // 2] == pytest.approx(base / 2, rel=1e-2)  # half way: half
    assert lrs[total] == pytest.approx(0.0, abs=1e-12)
    assert S.cosine_warmup(10, 100, 0.05) == pytest.approx(0.05 * 0.5 * (1 + math.cos(math.pi * 0.1)))


@pytest.mark.parametrize("x", [0.1, 0.05, 0.001, 1e-4, 0.8984375, 0.0625, 1.0, 3.7, 1e-9])
def test_mul_shift_nearest(x):
    mul, shift = S.mul_shift(x, bits=8)
    assert 0 <= mul < 256 and 0 <= shift <= 62
    if mul == 0:
        assert x < 2.0 ** -62
        return
    got = mul * 2.0 ** -shift
    # the best 8-bit multiplier at this shift: within half a unit of the last place
    assert abs(got - x) <= 0.5 * 2.0 ** -shift + 1e-18
    assert mul >= 128 or shift == 0  # all 8 bits used unless the shift bottoms out


def test_paper_constants():
    assert S.MOMENTUM_0_9 == S.mul_shift(0.9, bits=8)
    m, s = S.WEIGHT_DECAY_1E_4
    assert abs(m * 2.0 ** -s - 1e-4) / 1e-4 < 0.002
    assert S.mul_shift(0.0) == (0, 0)
    with pytest.raises(ValueError):
        S.mul_shift(-1.0)
    with pytest.raises(ValueError):
        S.mul_shift(300.0, bits=8)  # needs a negative shift


def test_lr_mul_shift_follows_schedule():
    for t in (0, 10, 499, 900):
        m, s = S.lr_mul_shift(t, 1000, 0.1, 5)
        assert m * 2.0 ** -s == pytest.approx(S.cosine_warmup(t, 1000, 0.1, 5), rel=2 ** -7)
