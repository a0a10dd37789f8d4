"""Mutation check of the oracle's pins: plant one plausible mistake in a copy of the oracle and
require that at least one pin of ``test_oracle_pins`` fails on it.

Each mutant is a textual edit of ``oracle/csa_oracle.c`` or ``oracle/__init__.py``, applied to a
copy in a temporary folder that is compiled by the copy's own ``build()`` (same gcc flags); the
real oracle is never touched.  Only mutants that change what the method computes are listed
(no rewrites that are equal in exact arithmetic), and none reads outside its buffers.
CPU only.
"""
import importlib.util
import inspect
import os

import numpy as np
import pytest

import oracle as O
import test_oracle_pins as PINS

ORACLE_DIR = os.path.dirname(os.path.abspath(O.__file__))
C_SRC = open(os.path.join(ORACLE_DIR, "csa_oracle.c")).read()
PY_SRC = open(os.path.join(ORACLE_DIR, "__init__.py")).read()

# (name, old text, new text): each old text occurs exactly once in the C source.
C_MUTANTS = [
    # CSA compression (V4 paper notes Sec. 2.3, Eq. 11-12)
    ("csa_drop_bias_a", "logit[cnt] = Za[p * c + d] + B[(int64_t)j * c + d];", "logit[cnt] = Za[p * c + d];"),
    ("csa_prev_block_uses_bias_a", "Zb[p * c + d] + B[(int64_t)(m + j) * c + d]", "Zb[p * c + d] + B[(int64_t)j * c + d]"),
    ("csa_prev_values_from_ca", "val[cnt] = Cb[p * c + d];", "val[cnt] = Ca[p * c + d];"),
    ("csa_prev_logits_from_za", "logit[cnt] = Zb[p * c + d]", "logit[cnt] = Za[p * c + d]"),
    ("csa_overlap_starts_at_entry2", "if (i > 0) {", "if (i > 1) {"),
    ("csa_overlap_reads_current_block", "int64_t p = (i - 1) * m + j;", "int64_t p = i * m + j;"),
    ("csa_unweighted_sum", "num += e * val[u];", "num += val[u];"),
    ("csa_bias_b_rows_reversed", "B[(int64_t)(m + j) * c + d]", "B[(int64_t)(2 * m - 1 - j) * c + d]"),
    # HCA compression (Sec. 2.4, Eq. 22-23)
    ("hca_drop_bias", "double e = exp(Z[p * c + d] + B[(int64_t)j * c + d] - mx);", "double e = exp(Z[p * c + d] - mx);"),
    ("hca_pools_logits", "num += e * C[p * c + d];", "num += e * Z[p * c + d];"),
    ("hca_bias_rows_reversed", "double e = exp(Z[p * c + d] + B[(int64_t)j * c + d] - mx);",
     "double e = exp(Z[p * c + d] + B[(int64_t)(m - 1 - j) * c + d] - mx);"),
    ("hca_weights_not_normalised", "out[i * c + d] = num / den;\n        }\n    }\n}", "out[i * c + d] = num;\n        }\n    }\n}"),
    # indexer (Eq. 16)
    ("indexer_no_relu", "acc += w[r * H + h] * (dot > 0.0 ? dot : 0.0);", "acc += w[r * H + h] * dot;"),
    ("indexer_relu_after_weight", "acc += w[r * H + h] * (dot > 0.0 ? dot : 0.0);",
     "acc += (w[r * H + h] * dot > 0.0 ? w[r * H + h] * dot : 0.0);"),
    ("indexer_weight_of_head0", "acc += w[r * H + h] *", "acc += w[r * H] *"),
    ("indexer_query_of_head0", "dot += qr[(int64_t)h * d + e] * ks[e];", "dot += qr[e] * ks[e];"),
    ("indexer_ignores_kbase", "K + (kbase[r] + s) * (int64_t)d", "K + s * (int64_t)d"),
    # top-k
    ("topk_ties_to_higher_index", "return (x->idx < y->idx) ? -1 : (x->idx > y->idx);",
     "return (x->idx > y->idx) ? -1 : (x->idx < y->idx);"),
    ("topk_ascending", "if (x->score > y->score) return -1;\n    if (x->score < y->score) return 1;",
     "if (x->score > y->score) return 1;\n    if (x->score < y->score) return -1;"),
    ("topk_pads_with_zero", "(int32_t)p[j].idx : -1;", "(int32_t)p[j].idx : 0;"),
    # attention (Sec. 2.3-2.4; Q&A essay Question 1 mechanism 3)
    ("attn_no_sink", "double den = exp(sink[h] - mx);", "double den = 0.0;"),
    ("attn_sink_counted_twice", "double den = exp(sink[h] - mx);", "double den = 2.0 * exp(sink[h] - mx);"),
    ("attn_no_scale", "z[j] = scale * dot;", "z[j] = dot;"),
    ("attn_lse_drops_max", "lse[r * H + h] = mx + log(den);", "lse[r * H + h] = log(den);"),
    ("attn_not_normalised", "for (int e = 0; e < c; e++) oh[e] /= den;", ""),
    # bf16
    ("bf16_truncates", "u += 0x7fffu + lsb;", "u += 0u;"),
    ("bf16_ties_away", "u += 0x7fffu + lsb;", "u += 0x8000u;"),
    # FP8 E4M3 (OCP OFP8)
    ("e4m3_saturates_to_nan", "return (uint8_t)(sign | 0x7e);", "return (uint8_t)(sign | 0x7f);"),
    ("e4m3_subnormal_step", "float j = orc_rne(ldexpf(a, 9));", "float j = orc_rne(ldexpf(a, 10));"),
    ("e4m3_encode_bias", "code = (uint8_t)(((e + 7) << 3)", "code = (uint8_t)(((e + 8) << 3)"),
    ("e4m3_truncates", "float q = orc_rne(ldexpf(a, 3 - e));", "float q = floorf(ldexpf(a, 3 - e));"),
    ("e4m3_decode_bias", "ldexp(1.0 + f / 8.0, e - 7)", "ldexp(1.0 + f / 8.0, e - 8)"),
    ("e4m3_decode_subnormal", "ldexp((double)f, -9)", "ldexp((double)f, -10)"),
    # FP4 E2M1 + E8M0 (OCP MX)
    ("e2m1_truncates_mid", "code = (int)orc_rne(a) + 2;", "code = (int)a + 2;"),
    ("e2m1_table", "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}", "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0}"),
    ("e2m1_negative_zero", "if (code == 0) return 0;", ""),
    ("fp4_scale_boundary", "(amax <= ldexpf(1.5f, e0))", "(amax < ldexpf(1.5f, e0))"),
    ("fp4_scale_one_low", "? e0 - 2 : e0 - 1;", "? e0 - 3 : e0 - 2;"),
    ("fp4_nibble_order", "(uint8_t)(lo | (hi << 4))", "(uint8_t)(hi | (lo << 4))"),
    ("fp4_amax_signed", "amax = fmaxf(amax, fabsf(xb[j]));", "amax = fmaxf(amax, xb[j]);"),
    ("fp4_dequant_bias", "int e = (int)scales[r * (d / 32) + j / 32] - 127;", "int e = (int)scales[r * (d / 32) + j / 32] - 128;"),
    # mixed-precision KV rows
    ("kv_scale_240", "float s = amax / 448.0f;", "float s = amax / 240.0f;"),
    ("kv_amax_includes_rope", "for (int j = 0; j < cn; j++) amax = fmaxf(amax, fabsf(xr[j]));",
     "for (int j = 0; j < c; j++) amax = fmaxf(amax, fabsf(xr[j]));"),
    ("kv_rope_from_first_dims", "orc_bf16_bits(xr[cn + j])", "orc_bf16_bits(xr[j])"),
    ("kv_dequant_divides", "* (double)scale[r];", "/ (double)scale[r];"),
    # stacked-decode glue
    ("glue_drop_sqrt_c", "1.0 / sqrt(ss / c) / sqrt((double)c)", "1.0 / sqrt(ss / c)"),
    ("glue_transposed_p", "P[(int64_t)i * c + j]", "P[(int64_t)j * c + i]"),
    ("glue_index_query_norm_by_c", "1.0 / sqrt(ss / d) : 0.0", "1.0 / sqrt(ss / c) : 0.0"),
    # layer fidelity (Sec. 2.3 Compressor and Indexer listings)
    ("rmsnorm_drops_eps", "const double f = 1.0 / sqrt(ss / d + eps);", "const double f = 1.0 / sqrt(ss / d);"),
    ("rmsnorm_sum_not_mean", "const double f = 1.0 / sqrt(ss / d + eps);", "const double f = 1.0 / sqrt(ss + eps);"),
    ("rmsnorm_drops_gain", "out[r * d + j] = x[r * d + j] * f * g[j];", "out[r * d + j] = x[r * d + j] * f;"),
    ("rope_clockwise", "yr[d - rd + 2 * i] = x0 * cos(a) - x1 * sin(a);", "yr[d - rd + 2 * i] = x0 * cos(a) + x1 * sin(a);"),
    ("rope_exponent_sign", "pow(base, -2.0 * i / rd)", "pow(base, 2.0 * i / rd)"),
    ("rope_exponent_not_halved", "pow(base, -2.0 * i / rd)", "pow(base, -1.0 * i / rd)"),
    ("rope_first_dims", "const double x0 = xr[d - rd + 2 * i], x1 = xr[d - rd + 2 * i + 1];",
     "const double x0 = xr[2 * i], x1 = xr[2 * i + 1];"),
    ("hadamard_not_normalised", "out[r * d + i] = acc * s;", "out[r * d + i] = acc;"),
    ("hadamard_wrong_sign_rule", "(__builtin_popcount((unsigned)(i & j)) & 1)", "(__builtin_popcount((unsigned)(i | j)) & 1)"),
]

# (name, old text, new text) on the Python half: key lists and visibility.
PY_MUTANTS = [
    ("n_vis_off_by_one", "return (np.asarray(t, dtype=np.int64) + 1) // m", "return np.asarray(t, dtype=np.int64) // m"),
    ("window_one_too_wide", "w = np.arange(max(0, t - W + 1), t + 1, dtype=np.int64)",
     "w = np.arange(max(0, t - W), t + 1, dtype=np.int64)"),
    ("window_excludes_own_token", "w = np.arange(max(0, t - W + 1), t + 1, dtype=np.int64)",
     "w = np.arange(max(0, t - W + 1), t, dtype=np.int64)"),
    ("hca_prefill_ignores_causality", "cmp_ = np.arange(min(int(n_vis(t, m)), n_comp), dtype=np.int64)",
     "cmp_ = np.arange(n_comp, dtype=np.int64)"),
    ("csa_prefill_keeps_padding", "cmp_ = r[r >= 0]", "cmp_ = r"),
    ("prefill_compressed_keys_not_offset", "np.concatenate([w, c + T])", "np.concatenate([w, c])"),
    ("prefill_compressed_keys_off_by_one", "np.concatenate([w, c + T])", "np.concatenate([w, c + T - 1])"),
    ("decode_window_ignores_length", "w = b * W + np.arange(int(win_len[b]), dtype=np.int64)",
     "w = b * W + np.arange(W, dtype=np.int64)"),
    ("decode_ignores_sequence_offset", "Nw + int(comp_off[b]) + s", "Nw + s"),
    ("decode_hca_visibility", "s = np.arange(int(n_vis(int(pos[b]), m)), dtype=np.int64)",
     "s = np.arange(int(pos[b]) // m, dtype=np.int64)"),
    ("decode_csa_keeps_padding", "            s = r[r >= 0]\n", "            s = r\n"),
    ("append_emits_one_token_late", "        if (t + 1) % m:\n            return None", "        if t % m or t == 0:\n            return None"),
    ("append_overlap_skips_previous_block", "            first = max(0, (e - 1) * m)", "            first = e * m"),
    ("append_ring_too_short", "        self.L = 2 * m if overlap else m", "        self.L = m"),
    ("bf16_vector_ties_away", "r = ((u + 0x7FFF + lsb) >> 16)", "r = ((u + 0x8000) >> 16)"),
]


def _mutate(src, old, new):
    assert src.count(old) == 1, f"mutation site must be unique: {old!r}"
    return src.replace(old, new)


def _oracle_copy(tmp_path, c_src, py_src):
    """A separate oracle module built from the given sources in ``tmp_path``."""
    (tmp_path / "csa_oracle.c").write_text(c_src)
    (tmp_path / "__init__.py").write_text(py_src)
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{tmp_path.name}",
                                                  str(tmp_path / "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.lib()  # compile now so a build error is reported as such
    return mod


def _pin_cases():
    """Every pin of test_oracle_pins, parametrisations expanded, in file order."""
    cases = []
    for name, fn in vars(PINS).items():
        if not (name.startswith("test_") and callable(fn)):
            continue
        params = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if params:
            (argname, values), = [m.args for m in params]
            names = [a.strip() for a in argname.split(",")]
            for v in values:
                kw = dict(zip(names, v)) if len(names) > 1 else {argname: v}
                cases.append((f"{name}[{v}]", fn, kw))
        else:
            cases.append((name, fn, {}))
        needed = set(inspect.signature(fn).parameters)
        assert needed <= set(cases[-1][2]), f"{name} needs fixtures {needed}"
    return cases


def _first_failing_pin(mod, monkeypatch):
    monkeypatch.setattr(PINS, "O", mod)
    monkeypatch.setattr(PINS, "RNG", np.random.default_rng(1234))
    for name, fn, kw in _pin_cases():
        try:
            fn(**kw)
        except Exception:  # an assertion or a numerical error: the pin rejects this oracle
            return name
    return None


def test_mutant_harness_accepts_the_oracle(tmp_path, monkeypatch):
    """The unmodified sources, built and run through the same harness, pass every pin."""
    mod = _oracle_copy(tmp_path, C_SRC, PY_SRC)
    assert _first_failing_pin(mod, monkeypatch) is None


@pytest.mark.parametrize("name,old,new", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_mutant_c_is_caught(name, old, new, tmp_path, monkeypatch):
    mod = _oracle_copy(tmp_path, _mutate(C_SRC, old, new), PY_SRC)
    assert _first_failing_pin(mod, monkeypatch) is not None, f"no pin catches mutant {name}"


@pytest.mark.parametrize("name,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_mutant_py_is_caught(name, old, new, tmp_path, monkeypatch):
    mod = _oracle_copy(tmp_path, C_SRC, _mutate(PY_SRC, old, new))
    assert _first_failing_pin(mod, monkeypatch) is not None, f"no pin catches mutant {name}"

