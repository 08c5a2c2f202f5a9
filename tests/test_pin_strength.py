"""Strength of the oracle's pins: plant one plausible mistake at a time in a scratch copy
of the oracle (a flipped sign, a dropped term, a transposed operand, an off-by-one index, a
wrong tie rule, a swapped nibble or slot order) and check that the CPU pin suite
(tests/test_oracle_*.py) fails on every one of them. The unmutated copy must pass in the
same harness, so a broken harness cannot pass the check by failing everything.

Each mutant is (name, text in the oracle's source, replacement, which occurrence): MUTANTS
for csa_oracle.cpp, PY_MUTANTS for the Python layer. All of them change the oracle's
arithmetic or layout; none of them touches the tests.
"""

import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

import pytest

from tests import mutation

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = [
    ("bf16_dec_subnormal",
     "-126 - 7",
     "-126 - 8", 0),
    ("round_ties_away",
     "std::nearbyint(r)",
     "std::round(r)", 0),
    ("e4m3_dec_bias",
     "e - 7);\n"
     "  return s ? -v : v;",
     "e - 8);\n"
     "  return s ? -v : v;", 0),
    ("e4m3_enc_sat",
     "if (v > 448.0) v = 448.0;",
     "if (v > 480.0) v = 480.0;", 0),
    ("e4m3_enc_sub",
     "std::ldexp(v, 9)",
     "std::ldexp(v, 10)", 0),
    ("e2m1_dec_sub",
     "(e == 0) ? 0.5 * m",
     "(e == 0) ? 1.0 * m", 0),
    ("e2m1_enc_tie025",
     "if (a <= 0.25) c = 0;",
     "if (a < 0.25) c = 0;", 0),
    ("e2m1_enc_tie25",
     "else if (a <= 2.5) c = 4;",
     "else if (a < 2.5) c = 4;", 0),
    ("e2m1_enc_tie5",
     "else if (a <= 5.0) c = 6;",
     "else if (a < 5.0) c = 6;", 0),
    ("e2m1_enc_tie075",
     "else if (a < 0.75) c = 1;",
     "else if (a <= 0.75) c = 1;", 0),
    ("mx_exp_minus3",
     "ex - 1 - 2",
     "ex - 1 - 3", 0),
    ("mx_exp_ceil",
     "ex - 1 - 2",
     "ex - 2", 0),
    ("e8m0_bias",
     "(int)e - 127",
     "(int)e - 128", 0),
    ("sf_off_swap",
     "16 * (r % 32) + 4 * (r / 32) + s",
     "16 * (r / 32) + 4 * (r % 32) + s", 0),
    ("sf_off_s_rev",
     "16 * (r % 32) + 4 * (r / 32) + s",
     "16 * (r % 32) + 4 * (r / 32) + 3 - s", 0),
    ("cmp_own_bias_rev",
     "(double)za[o] + (double)bias[r]",
     "(double)za[o] + (double)bias[m - 1 - r]", 0),
    ("cmp_prev_bias",
     "(double)zb[o] + (double)bias[m + r]);\n"
     "            } else if",
     "(double)zb[o] + (double)bias[r]);\n"
     "            } else if", 0),
    ("cmp_prev_uses_a",
     "xs.push_back(or_bf16_decode(b[o]));",
     "xs.push_back(or_bf16_decode(a[o]));", 0),
    ("cmp_prev_uses_za",
     "zs.push_back((double)zb[o] + (double)bias[m + r]);",
     "zs.push_back((double)za[o] + (double)bias[m + r]);", 0),
    ("cmp_no_den",
     "e[d] = num / den;",
     "e[d] = num;", 0),
    ("cmp_state_bias",
     "(double)prev_zb[o] + (double)bias[m + r]",
     "(double)prev_zb[o] + (double)bias[r]", 0),
    ("cmp_state_idx",
     "const size_t o = ((size_t)bb * m + r) * kD + d;",
     "const size_t o = ((size_t)bb * m + (m - 1 - r)) * kD + d;", 0),
    ("rms_no_mean",
     "1.0 / std::sqrt(ss / kD + eps)",
     "1.0 / std::sqrt(ss + eps)", 0),
    ("rms_no_eps",
     "1.0 / std::sqrt(ss / kD + eps)",
     "1.0 / std::sqrt(ss / kD)", 0),
    ("rms_no_w",
     "y[d] = e[d] * inv * (norm_w ? (double)norm_w[d] : 1.0);",
     "y[d] = e[d] * inv;", 0),
    ("rope_pos_end",
     "(double)(pos0 + (int64_t)m * i)",
     "(double)(pos0 + (int64_t)m * i + m - 1)", 0),
    ("rope_sign",
     "y[kNope + 2 * j] = x0 * c - x1 * s;\n"
     "        y[kNope + 2 * j + 1] = x0 * s + x1 * c;",
     "y[kNope + 2 * j] = x0 * c + x1 * s;\n"
     "        y[kNope + 2 * j + 1] = -x0 * s + x1 * c;", 0),
    ("rope_theta",
     "std::pow(rope_base, -(double)j / (kRope / 2))",
     "std::pow(rope_base, -(double)j / kRope)", 0),
    ("rope_halfsplit",
     "const double x0 = y[kNope + 2 * j], x1 = y[kNope + 2 * j + 1];\n"
     "        y[kNope + 2 * j] = x0 * c - x1 * s;\n"
     "        y[kNope + 2 * j + 1] = x0 * s + x1 * c;",
     "const double x0 = y[kNope + j], x1 = y[kNope + j + 32];\n"
     "        y[kNope + j] = x0 * c - x1 * s;\n"
     "        y[kNope + j + 32] = x0 * s + x1 * c;", 0),
    ("q_scale_240",
     "(float)(amax / 448.0)",
     "(float)(amax / 240.0)", 0),
    ("q_amax_all",
     "for (int d = 0; d < kNope; ++d) amax = std::max(amax, std::fabs(y[d]));",
     "for (int d = 0; d < kD; ++d) amax = std::max(amax, std::fabs(y[d]));", 0),
    ("q_bf16_part_skip",
     "const uint16_t h = or_bf16_encode(y[d]);",
     "const uint16_t h = or_bf16_encode(e[d]);", 0),
    ("ik_own_bias_rev",
     "(double)za[o] + (double)bias[r]",
     "(double)za[o] + (double)bias[m - 1 - r]", 1),
    ("ik_prev_uses_a",
     "xs.push_back(or_bf16_decode(b[o]));",
     "xs.push_back(or_bf16_decode(a[o]));", 1),
    ("ik_nib_swap",
     "for (int j = 0; j < kDI / 2; ++j) krow[j] = (uint8_t)(nib[2 * j] | (nib[2 * j + 1] << 4));",
     "for (int j = 0; j < kDI / 2; ++j) krow[j] = (uint8_t)(nib[2 * j + 1] | (nib[2 * j] << 4));", 0),
    ("ik_sf_row_i",
     "sfb[or_key_sf_offset(row, s)] = code;",
     "sfb[or_key_sf_offset(i, s)] = code;", 0),
    ("ik_no_den",
     "y[d] = num / den;",
     "y[d] = num;", 0),
    ("iq_nib_swap",
     "row[j] = (uint8_t)(nib[2 * j] | (nib[2 * j + 1] << 4));",
     "row[j] = (uint8_t)(nib[2 * j + 1] | (nib[2 * j] << 4));", 0),
    ("iq_sf_rev",
     "q_sf + ((size_t)t * H_I + h) * 4 + sb);",
     "q_sf + ((size_t)t * H_I + h) * 4 + 3 - sb);", 0),
    ("iq_W_transposed",
     "const uint16_t* w = W + (size_t)o * r;\n"
     "      for (int j = 0; j < r; ++j) acc += or_bf16_decode(w[j])",
     "const uint16_t* w = W + (size_t)o;\n"
     "      for (int j = 0; j < r; ++j) acc += or_bf16_decode(w[(size_t)j * O])", 0),
    ("op_no_round",
     "md[(size_t)g * d_g + o] = or_bf16_decode(or_bf16_encode(acc));",
     "md[(size_t)g * d_g + o] = acc;", 0),
    ("op_group_off",
     "acc += or_bf16_decode(w[j]) * x[(size_t)g * K1 + j];",
     "acc += or_bf16_decode(w[j]) * x[(size_t)j];", 0),
    ("ix_no_relu",
     "std::max(0.0, dot)",
     "dot", 0),
    ("ix_no_w",
     "s += (double)w[(size_t)bb * H_I + h] * std::max(0.0, dot);",
     "s += std::max(0.0, dot);", 0),
    ("ix_w_batch",
     "s += (double)w[(size_t)bb * H_I + h] *",
     "s += (double)w[(size_t)h] *", 0),
    ("ix_qnib_swap",
     "const uint8_t nib = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);",
     "const uint8_t nib = (d % 2 == 0) ? (byte >> 4) : (byte & 0xF);", 0),
    ("ix_knib_swap",
     "(d % 2 == 0) ? (kr[d / 2] & 0xF) : (kr[d / 2] >> 4)",
     "(d % 2 == 0) ? (kr[d / 2] >> 4) : (kr[d / 2] & 0xF)", 0),
    ("ix_qsf_idx",
     "q_sf[((size_t)bb * H_I + h) * 4 + d / 32]",
     "q_sf[((size_t)bb * H_I + h) * 4 + d % 4]", 0),
    ("ix_ksf_plain",
     "ks[or_key_sf_offset(j, d / 32)]",
     "ks[j * 4 + d / 32]", 0),
    ("ix_ksf_nobatch",
     "const uint8_t* ks = k_sf + (size_t)bb * Nmax * 4;",
     "const uint8_t* ks = k_sf;", 0),
    ("ix_nan_off1",
     "if (j >= n_entries[bb]) {",
     "if (j > n_entries[bb]) {", 0),
    ("tk_tie_desc",
     "return x < y;\n"
     "  });",
     "return x > y;\n"
     "  });", 0),
    ("tk_no_index_order",
     "std::sort(order.begin(), order.begin() + keep);",
     "", 0),
    ("tk_keep_off1",
     "const int64_t keep = std::min<int64_t>(k, n);",
     "const int64_t keep = std::min<int64_t>(k - 1, n);", 0),
    ("tk_bf16_noround",
     "r[(size_t)j] = or_bf16_decode(or_bf16_encode(scores[j]));",
     "r[(size_t)j] = scores[j];", 0),
    ("at_win_129",
     "for (int64_t p = std::max<int64_t>(0, t - (kWin - 1)); p <= t; ++p) {\n"
     "        const uint16_t* sr",
     "for (int64_t p = std::max<int64_t>(0, t - kWin); p <= t; ++p) {\n"
     "        const uint16_t* sr", 0),
    ("at_win_excl",
     "p <= t; ++p) {\n"
     "        const uint16_t* sr",
     "p < t; ++p) {\n"
     "        const uint16_t* sr", 0),
    ("at_sink_dropped",
     "double Z = std::exp(sig - lmax);",
     "double Z = 0.0;", 0),
    ("at_sink_tau",
     "const double sig = (double)sink[h];",
     "const double sig = tau * (double)sink[h];", 0),
    ("at_no_tau",
     "l[r] = tau * dot;",
     "l[r] = dot;", 0),
    ("at_derot_sign",
     "o[kNope + 2 * j] = x0 * c + x1 * s;\n"
     "            o[kNope + 2 * j + 1] = -x0 * s + x1 * c;",
     "o[kNope + 2 * j] = x0 * c - x1 * s;\n"
     "            o[kNope + 2 * j + 1] = x0 * s + x1 * c;", 0),
    ("at_derot_pos",
     "const double c = std::cos((double)t * theta), s = std::sin((double)t * theta);\n"
     "            const double x0 = o[",
     "const double c = std::cos((double)(t + 1) * theta), s = std::sin((double)(t + 1) * theta);\n"
     "            const double x0 = o[", 0),
    ("at_lse_nomax",
     "lse[(size_t)bb * H + h] = lmax + std::log(Z);",
     "lse[(size_t)bb * H + h] = std::log(Z);", 0),
    ("at_hca_off1",
     "for (int32_t j = 0; j < n_entries[bb]; ++j) {",
     "for (int32_t j = 0; j + 1 < n_entries[bb]; ++j) {", 0),
    ("dq_no_scale",
     "v[d] = or_e4m3_decode(row[d]) * (double)scale;",
     "v[d] = or_e4m3_decode(row[d]);", 0),
    ("dq_rope_stride",
     "std::memcpy(&h, row + kNope + 2 * (d - kNope), 2);",
     "std::memcpy(&h, row + kNope + (d - kNope), 2);", 0),
    ("at_ring_slot",
     "swa + ((size_t)bb * kWin + (size_t)(p % kWin)) * kD",
     "swa + ((size_t)bb * kWin + (size_t)((p + 1) % kWin)) * kD", 0),
    ("at_q_head",
     "const uint16_t* qh = q + ((size_t)bb * H + h) * kD;",
     "const uint16_t* qh = q + ((size_t)bb * H) * kD;", 0),
    ("pf_n_off1",
     "const int32_t n = (int32_t)((strict_eligibility ? t : t + 1) / m);",
     "const int32_t n = (int32_t)(t / m);", 0),
    ("pf_strict_ignored",
     "const int32_t n = (int32_t)((strict_eligibility ? t : t + 1) / m);",
     "const int32_t n = (int32_t)((t + 1) / m);", 0),
    ("pf_strict_off1",
     "const int32_t n = (int32_t)((strict_eligibility ? t : t + 1) / m);",
     "const int32_t n = (int32_t)((strict_eligibility ? t - 1 : t + 1) / m);", 0),
    ("sw_pos",
     "const double c = std::cos((double)t * theta), s = std::sin((double)t * theta);\n"
     "    const double x0 = y[",
     "const double c = std::cos((double)(t + 1) * theta), s = std::sin((double)(t + 1) * theta);\n"
     "    const double x0 = y[", 0),
    ("sw_no_mean",
     "const double inv = 1.0 / std::sqrt(ss / kD + eps);\n"
     "  for (int d = 0; d < kD; ++d) y[d] = y[d]",
     "const double inv = 1.0 / std::sqrt(ss + eps);\n"
     "  for (int d = 0; d < kD; ++d) y[d] = y[d]", 0),
    ("pf_prefix_off1",
     "if (p < P)\n"
     "          std::memcpy",
     "if (p < P - 1)\n"
     "          std::memcpy", 0),
    ("pf_row_q",
     "q + (size_t)r * H * kD, &tq",
     "q + (size_t)i * H * kD, &tq", 0),
    ("pf_qsf_row",
     "q_sf + (size_t)r * H_I * 4, w + (size_t)r * H_I",
     "q_sf + (size_t)r * H_I * 4, w", 0),
    ("sw_no_w",
     "for (int d = 0; d < kD; ++d) y[d] = y[d] * inv * (norm_w ? (double)norm_w[d] : 1.0);",
     "for (int d = 0; d < kD; ++d) y[d] = y[d] * inv;", 0),
    ("ik_prev_bias",
     "(double)zb[o] + (double)bias[m + r]);\n"
     "            } else if",
     "(double)zb[o] + (double)bias[r]);\n"
     "            } else if", 1),
    ("ik_state_idx",
     "const size_t o = ((size_t)bb * m + r) * kDI + d;",
     "const size_t o = ((size_t)bb * m + (m - 1 - r)) * kDI + d;", 0),
    ("at_sink_inf_branch",
     "if (sig == kInf) {",
     "if (false) {", 0),
    ("bf16_enc_sub",
     "std::ldexp(v, 133)",
     "std::ldexp(v, 134)", 0),
    ("e4m3_dec_sub",
     "v = std::ldexp((double)m, -9);",
     "v = std::ldexp((double)m, -10);", 0),
    ("sf_off_group",
     "g * 512 + 16 * (r % 32)",
     "g * 256 + 16 * (r % 32)", 0),
]


# Mistakes planted in the oracle's Python layer (oracle/__init__.py): the paged-cache view
# and scatter, whose arithmetic is written there rather than in the C++ file.
PY_MUTANTS = [
    ("pv_table_ignored",
     "out[b, lp * per_page:(lp + 1) * per_page] = pool[page]",
     "out[b, lp * per_page:(lp + 1) * per_page] = pool[lp % pool.shape[0]]", 0),
    ("pv_negative_page_read",
     "if 0 <= page < pool.shape[0]:",
     "if page < pool.shape[0]:", 0),
    ("pv_group_offset",
     "out[b, lp * per_page:(lp + 1) * per_page] = pool[page]",
     "out[b, lp * (page_entries // 128):(lp + 1) * (page_entries // 128)] = pool[page]", 0),
    ("ps_wrong_sequence",
     "pool[page, :hi - lo] = view[b, lo:hi]",
     "pool[page, :hi - lo] = view[(b + 1) % B, lo:hi]", 0),
    ("ps_table_transposed",
     "page = int(table[b, lp])",
     "page = int(table[lp % B, b % pages_max])", 1),
    ("ps_slot_shift",
     "pool[page, :hi - lo] = view[b, lo:hi]",
     "pool[page, :hi - lo] = np.roll(view[b, lo:hi], 1, axis=0)", 0),
]


def _prepare(base, name, text, py_text):
    """Copy the pins and the oracle under base/name with the given oracle sources (C++ and
    the Python layer) and build it; returns (name, directory, build ok, compiler message)."""
    d = os.path.join(base, name)
    shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(d, "synth"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(d, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__", "c", "test_[!o]*"))
    os.makedirs(os.path.join(d, "oracle"))
    with open(os.path.join(d, "oracle", "__init__.py"), "w") as f:
        f.write(py_text)
    shutil.copy(os.path.join(ROOT, "pytest.ini"), d)
    cpp = os.path.join(d, "oracle", "csa_oracle.cpp")
    with open(cpp, "w") as f:
        f.write(text)
    so = os.path.join(d, "oracle", "liboracle.so")
    b = subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", "-o", so,
                        cpp], capture_output=True, text=True)
    return name, d, b.returncode == 0, b.stderr[-300:]


@pytest.mark.slow
def test_every_planted_mistake_fails_a_pin(tmp_path):
    if not shutil.which("g++"):
        pytest.skip("no g++")
    with open(os.path.join(ROOT, "oracle", "csa_oracle.cpp")) as f:
        src = f.read()
    with open(os.path.join(ROOT, "oracle", "__init__.py")) as f:
        py = f.read()
    jobs = ([("unmutated", src, py)] +
            [(n, mutation.apply(src, o, r, w), py) for n, o, r, w in MUTANTS] +
            [(n, src, mutation.apply(py, o, r, w)) for n, o, r, w in PY_MUTANTS])
    workers = max(1, min(8, os.cpu_count() or 2))
    with ThreadPoolExecutor(workers) as ex:
        built = list(ex.map(lambda j: _prepare(str(tmp_path), *j), jobs))
    unbuilt = [(n, msg) for n, _, ok, msg in built if not ok]
    assert not unbuilt, f"copies that do not compile: {unbuilt}"
    names, dirs = [b[0] for b in built], [b[1] for b in built]
    status = mutation.run(dirs, ["test_oracle_"], str(tmp_path), workers)
    mutation.verdict(names, dirs, status, "oracle")
