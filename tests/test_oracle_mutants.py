"""Plant plausible mistakes in copies of the oracle and check that the pins catch each one.

The mistakes are planted in temporary copies of the oracle's C source, on the
CPU; the committed oracle is never changed.
"""
import os
import shutil

import pytest

import oracle
import oracle_pins
from oracle import build as obuild

MUTANTS = {
    "phase_sign": ("const double phi = qarg[h * F + f] - karg[f];",
                   "const double phi = qarg[h * F + f] + karg[f];"),
    "unrotate_sign": ("double pi = -xr * sn + xi * c;", "double pi = xr * sn + xi * c;"),
    "distance_sign": ("const double delta = (double)((int64_t)t + offsets[j]) - p;",
                      "const double delta = p - (double)((int64_t)t + offsets[j]);"),
    "weight_R_not_1mR": ("norm += (1.0 - (double)R[h * F + f])", "norm += ((double)R[h * F + f])"),
    "pairing_adjacent": ("*im = f + d / 2;", "*im = f + 1;"),
    "omega_over_F": ("omega[f] = pow(base, -2.0 * (double)f / (double)d);",
                     "omega[f] = pow(base, -2.0 * (double)f / (double)(d / 2));"),
    "sum_not_mean": ("trig /= (double)n_off;", "trig /= 1.0;"),
    "max_over_delta": ("trig += series;", "trig = (j == 0 || series > trig) ? series : trig;"),
    "sample_std": ("sqrt(m2 / (double)N)", "sqrt(m2 / (double)(N > 1 ? N - 1 : 1))"),
    "ties_to_higher_slot": ("return (a->i > b->i) - (a->i < b->i);", "return (a->i < b->i) - (a->i > b->i);"),
    "drop_norm_term": ("s_out[(size_t)h * N + i] = trig + norm;", "s_out[(size_t)h * N + i] = trig;"),
    "qmag_not_kmag": ("series += qmag[h * F + f] * kmag[f] *", "series += qmag[h * F + f] *"),
    "flat_head_not_zero": ("const int flat = !(hi > lo);", "const int flat = 0;"),
    "no_resort": ("qsort(kept_out, (size_t)M, sizeof(int32_t), idx_cmp);", ""),
    "max_mode_takes_min": ("if (j == 0 || series > best) best = series;", "if (j == 0 || series < best) best = series;"),
    "max_mode_keeps_mean": ("if (combine == TRI_ORACLE_MAX_OVER_DELTA) trig = best;", ""),
    "calib_R_inverted": ("mm > 0.0 ? sqrt(mr * mr + mi * mi) / mm : 0.0;", "mm > 0.0 ? mm / sqrt(mr * mr + mi * mi) : 0.0;"),
    "calib_squared_modulus": ("sm += sqrt(re * re + im * im);", "sm += re * re + im * im;"),
    "calib_sum_not_mean": ("const double mr = sr / (double)T, mi = si / (double)T, mm = sm / (double)T;",
                           "const double mr = sr, mi = si, mm = sm;"),
    "calib_sample_mean_T_minus_1": ("const double mr = sr / (double)T, mi = si / (double)T, mm = sm / (double)T;",
                                    "const double mr = sr / (double)(T - 1), mi = si / (double)(T - 1), mm = sm / (double)(T - 1);"),
    "calib_centre_modulus_first": ("                    sr += re;\n                    si += im;",
                                   "                    sr += fabs(re);\n                    si += fabs(im);"),
    "attn_scale_by_d": ("const double scale = 1.0 / sqrt((double)d);", "const double scale = 1.0 / (double)d;"),
    "attn_no_normalisation": ("out[(size_t)h * d + i] = acc / denom;", "out[(size_t)h * d + i] = acc;"),
    "attn_values_from_keys": ("acc += logit[j] * bf16_value(V[(size_t)j * d + i]);",
                              "acc += logit[j] * bf16_value(K[(size_t)j * d + i]);"),
    "attn_first_head_only": ("dot += bf16_value(q[(size_t)h * d + i]) * bf16_value(K[(size_t)j * d + i]);",
                             "dot += bf16_value(q[i]) * bf16_value(K[(size_t)j * d + i]);"),
    "attn_minus_logit": ("logit[j] = exp(logit[j] - top);", "logit[j] = exp(top - logit[j]);"),
    "batch_qnorm_offset_drops_group": ("q_norm + (size_t)u * G * F", "q_norm + (size_t)u * F"),
    "batch_keys_offset_by_length": ("K + (size_t)u * stride * d", "K + (size_t)u * N * d"),
    "batch_kept_offset_by_count": ("tri_oracle_select(N, B, zm, kept_out + (size_t)u * B)",
                                   "tri_oracle_select(N, B, zm, kept_out + (size_t)u * (N < B ? N : B))"),
    "select_f32_truncates": ("for (int i = 0; i < N; ++i) z[i] = (double)zmax[i];",
                             "for (int i = 0; i < N; ++i) z[i] = floor((double)zmax[i]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    msrc = tmp_path / "tri_oracle_mutant.c"
    msrc.write_text(src.replace(old, new))
    mlib = tmp_path / "libtri_oracle_mutant.so"
    obuild.build(force=True, src=str(msrc), lib=str(mlib))
    L = oracle.lib(str(mlib))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(L)
        except (AssertionError, ValueError, ZeroDivisionError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
