"""csa_prep_rows -- RMSNorm of entries, rotary embedding of the last dims, Hadamard rotation and the
cache quantisers -- against the fp64 oracle of the same steps ([notes] Sec. 2.3 Compressor and
Indexer listings).  The kernel computes in fp32 (angles in fp64), so dense outputs are compared at
fp32 / bf16 accuracy, and quantised outputs may differ from the oracle's quantisation only where a
value lies within the fp32 error of a rounding boundary."""
import numpy as np
import pytest
import torch

import oracle as O
from _util import check_fp4_near, dev, host, row_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(gpu):
    import compressed_sparse_kv_csa_b200 as C
    return C


def _ref(x, g, eps, rd, pos, base, had):
    y = np.asarray(x, np.float64)
    if g is not None:
        y = O.rmsnorm(y, g, eps)
    if rd:
        y = O.rope(y, pos, rd, base)
    if had:
        y = O.hadamard(y)
    return y


@pytest.mark.parametrize("d,n,norm,rd,had,dtype", [
    (512, 1000, True, 64, False, "bf16"),   # KV entries: RMSNorm + RoPE on the last 64
    (128, 777, True, 64, True, "bf16"),     # index keys: RMSNorm + RoPE + Hadamard
    (128, 4096, False, 64, True, "f32"),    # index queries: RoPE + Hadamard
    (256, 33, False, 0, True, "f32"),       # Hadamard alone
    (64, 5, True, 0, False, "f32"),         # RMSNorm alone
    (32, 9, False, 32, False, "f32"),       # RoPE over the whole row
])
def test_prep_rows_dense(C, d, n, norm, rd, had, dtype):
    g = np.random.default_rng(d + n)
    x = g.standard_normal((n, d)).astype(np.float32)
    if dtype == "bf16":
        x = O.bf16_value(O.bf16_bits(x)).astype(np.float32)
    gain = (1.0 + 0.3 * g.standard_normal(d)).astype(np.float32) if norm else None
    pos = g.integers(0, 1 << 20, size=n).astype(np.int64)
    pos[0] = 0
    eps = 1e-6
    ref = _ref(x, gain, eps, rd, pos, 10000.0, had)
    out = torch.empty((n, d), dtype=torch.float32, device="cuda")
    C.csa_prep_rows(dev(x, dtype), g=None if gain is None else dev(gain), eps=eps, rd=rd,
                    pos=torch.from_numpy(pos).cuda(), hadamard=had, out=out)
    torch.cuda.synchronize()
    assert row_rel_err(host(out), ref).max() < 2e-6
    ob = torch.empty((n, d), dtype=torch.bfloat16, device="cuda")
    C.csa_prep_rows(dev(x, dtype), g=None if gain is None else dev(gain), eps=eps, rd=rd,
                    pos=torch.from_numpy(pos).cuda(), hadamard=had, out=ob)
    assert row_rel_err(host(ob), ref).max() <= 2.0 ** -8


def test_prep_rows_into_the_caches(C):
    """KV entries -> FP8/BF16 rows and index keys -> FP4 rows, quantise-on-write, against the
    oracle's quantisation of its own fp64 result (codes may differ only at a rounding boundary)."""
    g = np.random.default_rng(77)
    n = 600
    x = O.bf16_value(O.bf16_bits(g.standard_normal((n, 512)).astype(np.float32))).astype(np.float32)
    gain = (1.0 + 0.3 * g.standard_normal(512)).astype(np.float32)
    pos = g.integers(0, 1 << 20, size=n).astype(np.int64)
    ref = _ref(x, gain, 1e-6, 64, pos, 10000.0, False)
    kv = C.KvRows.empty(n, 512, 64, "cuda")
    C.csa_prep_rows(dev(x, "bf16"), g=dev(gain), eps=1e-6, rd=64, pos=torch.from_numpy(pos).cuda(), out_kv=kv)
    torch.cuda.synchronize()
    f8, rb, sc = kv.fp8.cpu().numpy(), kv.rope.view(torch.int16).cpu().numpy().view(np.uint16), kv.scale.cpu().numpy()
    f8r, rbr, scr = O.quant_kv(ref.astype(np.float32))
    np.testing.assert_allclose(sc, scr, rtol=2e-6)
    vg, vr = O.dequant_kv(f8, rb, sc), O.dequant_kv(f8r, rbr, scr)
    tol = 2e-6 * np.abs(ref).max(1, keepdims=True)
    bad = (vg != vr) & (np.abs(vg - ref) > np.abs(vr - ref) + 2 * tol)
    assert not bad.any(), np.argwhere(bad)[:4]
    assert (f8 != f8r).mean() < 1e-3 and (rb != rbr).mean() < 1e-3   # codes differ only at boundaries
    # index keys: RMSNorm + RoPE + Hadamard -> FP4
    xi = O.bf16_value(O.bf16_bits(g.standard_normal((n, 128)).astype(np.float32))).astype(np.float32)
    gi = np.ones(128, np.float32)
    refi = _ref(xi, gi, 1e-6, 64, pos, 10000.0, True)
    f4 = C.Fp4Rows.empty(n, 128, "cuda")
    C.csa_prep_rows(dev(xi, "bf16"), g=dev(gi), eps=1e-6, rd=64, pos=torch.from_numpy(pos).cuda(), hadamard=True,
                    out_fp4=f4)
    torch.cuda.synchronize()
    check_fp4_near(f4.codes.cpu().numpy(), f4.scales.cpu().numpy(), refi, atol=1e-5)
    assert C.csa_device_error() == 0


def test_prep_rows_argument_checks(C):
    x = torch.zeros((4, 96), device="cuda")
    out = torch.empty_like(x)
    with pytest.raises(C.CsaError) as e:
        C.csa_prep_rows(x, out=out)
    assert e.value.status == C.CSA_ERR_UNSUPPORTED
    x = torch.zeros((4, 128), device="cuda")
    with pytest.raises(C.CsaError) as e:
        C.csa_prep_rows(x, rd=64, out=torch.empty_like(x))  # rotary embedding without positions
    assert e.value.status == C.CSA_ERR_INVALID_ARG
    with pytest.raises(C.CsaError) as e:
        C.csa_prep_rows(x, rd=63, pos=torch.zeros(4, dtype=torch.int64, device="cuda"), out=torch.empty_like(x))
    assert e.value.status == C.CSA_ERR_INVALID_ARG
