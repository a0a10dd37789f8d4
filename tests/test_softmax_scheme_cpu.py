"""The online-softmax scheme the tensor-core attention kernels use, modelled in numpy and checked
against the exact softmax with the sink on the CPU.

The scheme (prefill kernels, both key layouts): keys arrive in tiles of 128; per head a running
max m moves only when a tile raises it by more than 8 (log2 units), the earlier accumulators are
then rescaled by 2^(m_old - m_new); P = bf16(2^(s - m)) feeds the P V product (bf16 V, fp32
accumulation); the denominator sums the fp32 values of 2^(s - m) and adds the sink 2^(sink - m).
The keys-on-M kernel takes each tile's maximum from bf16 copies of the scores plus a margin of
|max| / 128 (a bf16 copy is within 2^-8 of its score), so 2^(s - m) stays below 2^8 after the
margin.  Outputs are compared row by row (max |o - r| / max |r| < 2e-2, the parity tolerance) and
the log-sum-exp to 2e-3.  Special cases: a dominant key, equal scores, wide score ranges, fully
masked tiles, a sink that outweighs every key."""
import zlib

import numpy as np
import pytest

from _util import row_rel_err

LOG2E = 1.4426950408889634


def bf16(x):
    """Round fp32 values to bf16 (round to nearest even), returned as fp32."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    return np.where(np.isfinite(x), out, np.asarray(x, np.float32))


def scheme(s, v, sink, bf16_max):
    """s [H, n] natural-log scores (-inf = masked), v [n, c] values, sink [H]."""
    H, n = s.shape
    s2 = (s * LOG2E).astype(np.float32)
    m = np.full(H, -np.inf, np.float32)
    l = np.zeros(H, np.float32)
    O = np.zeros((H, v.shape[1]), np.float32)
    vb = bf16(v)
    for t0 in range(0, n, 128):
        st = s2[:, t0:t0 + 128]
        if bf16_max:
            mt = bf16(st).max(1)
            with np.errstate(invalid="ignore"):
                mt = np.where(np.isfinite(mt), mt + np.abs(mt) / 128, mt)
        else:
            mt = st.max(1)
        m_new = np.maximum(m, mt)
        move = np.isfinite(m_new) & (~np.isfinite(m) | (m_new > m + 8))
        resc = np.where(move, np.where(np.isfinite(m), np.exp2(m - m_new), 0.0), 1.0).astype(np.float32)
        m = np.where(move, m_new, m)
        with np.errstate(invalid="ignore"):
            p = np.where(np.isfinite(m)[:, None], np.exp2(st - m[:, None]), 0.0).astype(np.float32)
        l = l * resc + p.sum(1, dtype=np.float32)
        O = O * resc[:, None] + bf16(p) @ vb[t0:t0 + 128]
    den = l + np.exp2(sink * LOG2E - m)
    o = O / den[:, None]
    lse = np.where(np.isfinite(m), (m + np.log2(den)) / LOG2E, sink)
    return o, lse


def exact(s, v, sink):
    s = s.astype(np.float64)
    mx = np.maximum(np.max(np.where(np.isfinite(s), s, -np.inf), 1), sink)
    e = np.exp(s - mx[:, None])
    den = e.sum(1) + np.exp(sink - mx)
    return (e @ bf16(v).astype(np.float64)) / den[:, None], mx + np.log(den)


def _case(kind, rng):
    H, n, c = 64, 384, 64
    s = rng.standard_normal((H, n)).astype(np.float32)
    v = rng.standard_normal((n, c)).astype(np.float32)
    sink = rng.standard_normal(H).astype(np.float32)
    if kind == "wide":          # scores spread over a wide range, rising across the tiles
        s = s * 6 + np.linspace(-40, 40, n, dtype=np.float32)[None, :]
    elif kind == "dominant":    # one key far above the rest, in the last tile
        s[:, -5] += 60
    elif kind == "equal":
        s[:] = 1.25
    elif kind == "masked":      # the first tile fully masked, a few masked keys elsewhere
        s[:, :128] = -np.inf
        s[:, 200:210] = -np.inf
    elif kind == "sink":        # the sink outweighs every key
        sink[:] = 30.0
    elif kind == "falling":     # the largest scores come first (no rescale after tile 0)
        s = s + np.linspace(20, -20, n, dtype=np.float32)[None, :]
    return s, v, sink


@pytest.mark.parametrize("bf16_max", [False, True])
@pytest.mark.parametrize("kind", ["normal", "wide", "dominant", "equal", "masked", "sink", "falling"])
def test_online_softmax_scheme_matches_exact(kind, bf16_max):
    rng = np.random.default_rng(zlib.crc32(kind.encode()))
    s, v, sink = _case(kind, rng)
    o, lse = scheme(s, v, sink, bf16_max)
    o_ref, lse_ref = exact(s, v, sink)
    assert row_rel_err(o, o_ref).max() < 2e-2
    np.testing.assert_allclose(lse, lse_ref, atol=2e-3, rtol=0)


def test_model_flags_a_scheme_without_the_rescale():
    """The check has teeth: dropping the rescale of the earlier accumulators (a plausible slip)
    breaks the rising-scores case."""
    rng = np.random.default_rng(5)
    s, v, sink = _case("wide", rng)
    H, n = s.shape
    s2 = (s * LOG2E).astype(np.float32)
    m = np.full(H, -np.inf, np.float32)
    l = np.zeros(H, np.float32)
    O = np.zeros((H, v.shape[1]), np.float32)
    for t0 in range(0, n, 128):
        st = s2[:, t0:t0 + 128]
        m = np.maximum(m, st.max(1))       # max moves but nothing is rescaled
        p = np.exp2(st - m[:, None])
        l = l + p.sum(1)
        O = O + p @ v[t0:t0 + 128]
    o = O / (l + np.exp2(sink * LOG2E - m))[:, None]
    o_ref, _ = exact(s, v, sink)
    assert row_rel_err(o, o_ref).max() > 2e-2
