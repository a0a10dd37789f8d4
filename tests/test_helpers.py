"""CPU checks of the parity helpers themselves: each accepts the oracle's own results and rejects
a planted mistake (planted on the CPU, in oracle output)."""
import numpy as np
import pytest

import oracle as O
from _util import check_fp4_near, check_topk


def _rows(n, d, seed=7):
    return np.random.default_rng(seed).standard_normal((n, d))


def test_fp4_near_accepts_the_oracle_quantisation():
    x = _rows(64, 128)
    codes, scales = O.quant_fp4(x.astype(np.float32))
    assert check_fp4_near(codes, scales, x) == 0


def test_fp4_near_rejects_a_wrong_code_away_from_a_boundary():
    x = _rows(64, 128)
    codes, scales = O.quant_fp4(x.astype(np.float32))
    v = O.dequant_fp4(codes, scales)
    s = np.ldexp(1.0, scales.astype(np.int64) - 127).repeat(32, axis=1)
    # an element far from every rounding midpoint: |x/s - code value| small
    r, j = np.argwhere(np.abs(x / s - v / s) < 0.05)[0]
    bad = codes.copy()
    bad[r, j // 2] ^= np.uint8(0x1 << (4 * (j % 2)))  # flip the low mantissa/exponent bit of that nibble
    with pytest.raises(AssertionError):
        check_fp4_near(bad, scales, x)


def test_fp4_near_rejects_a_wrong_scale():
    x = _rows(64, 128)
    codes, scales = O.quant_fp4(x.astype(np.float32))
    bad = scales.copy()
    bad[3, 1] += 1
    with pytest.raises(AssertionError):
        check_fp4_near(codes, bad, x)


def test_fp4_near_allows_either_neighbour_on_a_midpoint():
    # 0.25 * 2^e lies halfway between codes 0 and 0.5 * 2^e; round-half-even gives 0, the
    # other neighbour is accepted within the tolerance band
    x = np.zeros((1, 32))
    x[0, 0] = 6.0      # fixes the block scale at 2^0
    x[0, 1] = 0.25
    codes, scales = O.quant_fp4(x.astype(np.float32))
    alt = codes.copy()
    alt[0, 0] = (alt[0, 0] & 0x0F) | 0x10   # element 1 -> 0.5
    assert check_fp4_near(alt, scales, x, max_frac=1.0) == 1


def test_topk_check_rejects_a_wrong_member():
    rng = np.random.default_rng(3)
    S = rng.standard_normal((1, 500))
    idx = np.argsort(-S[0])[:16][None].astype(np.int32)
    assert check_topk(idx, idx, S, [500], 16) == 1
    bad = idx.copy()
    bad[0, 3] = np.argsort(-S[0])[100]
    with pytest.raises(AssertionError):
        check_topk(bad, idx, S, [500], 16)
