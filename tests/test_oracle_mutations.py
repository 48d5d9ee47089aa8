"""The pins have teeth: plant one plausible mistake at a time in a copy of the
oracle source, build it on the CPU, and check that at least one pin fails."""
import os
import shutil
import subprocess

import pytest

import oracle
from tests import test_oracle_composed_pins as cpins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "mta_oracle.c")

# (name, original text, mutated text)
MUTATIONS = [
    ("mix matrix transposed", "wg[ho * c_h + hi]", "wg[hi * c_h + ho]"),
    ("key offset sign flipped", "int c = j - jp;", "int c = j + jp;"),
    ("query taps reversed", "theta[ip * c_k + (jp - jlo)]",
     "theta[(c_q - 1 - ip) * c_k + (jp - jlo)]"),
    ("no Mask_0 before the conv", "const int last = a->exact ? r + s->c_q - 1 : r;",
     "const int last = T - 1;"),
    ("Mask_-inf replaced by zero", "rows, a->exact, -INFINITY, C);", "rows, a->exact, 0.0, C);"),
    ("unbiased variance", "    var /= d;\n    double inv", "    var /= (d - 1);\n    double inv"),
    ("eps outside the square root", "1.0 / sqrt(var + s->gn_eps)",
     "1.0 / (sqrt(var) + s->gn_eps)"),
    ("scale 1/d instead of 1/sqrt(d)", "1.0 / sqrt((double)d)", "1.0 / (double)d"),
    ("value of the input head", "const double *vj = row_of(a->v, s, b, h, j);",
     "const double *vj = row_of(a->v, s, b, (h / s->c_h) * s->c_h + (s->c_h - 1 - h % s->c_h), j);"),
    ("even-c_k window mirrored", "const int jlo = -(c_k / 2);",
     "const int jlo = -((c_k - 1) / 2);"),
    ("depth scale dropped", ": a->depth_scale;", ": 1.0;"),
    ("gate sign flipped", "exp(-a->gate[h])", "exp(a->gate[h])"),
    ("gate applied before the affine bias", "out_row[chn] = scale * y;",
     "out_row[chn] = scale * (y - a->gn_bias[chn]) + a->gn_bias[chn];"),
    # compositions of "Putting Everything Together"
    ("post-softmax conv keeps future keys", "rows, 0, 0.0,", "rows, 0, 1.0,"),
    ("second head mix skipped", "a->w_head_post ? a->w_head_post + (size_t)g * c_h * c_h : NULL",
     "NULL"),
    ("post-softmax conv fed unmixed rows", "u.A1 + (size_t)hh * T,", "u.P + (size_t)hh * T,"),
    ("fresh first-stage rows fed unmixed rows", "memcpy(slot, u->A1 + (size_t)hh * T,",
     "memcpy(slot, u->P + (size_t)hh * T,"),
    ("fresh first-stage rows from the wrong logits",
     "masked0_logit_row(s, a, b, g * c_h + hh, r - ip2, slot);",
     "masked0_logit_row(s, a, b, g * c_h + hh, i - ip2, slot);"),
    ("no Mask_-inf without a key-query conv", "C[j] = (j <= r) ? rows[0][j] : -INFINITY;",
     "C[j] = rows[0][j];"),
    ("post-softmax conv reads the current row only",
     "point_rows(s, u.ring1, i, u.zero, u.rows1);",
     "point_rows(s, u.ring1, i, u.zero, u.rows1);\n"
     "            for (int z = 0; z < s->c_h * s->c_q; ++z) u.rows1[z] = u.rows1[z - z % s->c_q];"),
    # pre-softmax head mix and the exact indicator of Eq. (4)
    ("logit mix transposed", "acc += wrow[hi] *", "acc += wg[(size_t)hi * c_h + ho] *"),
    ("logit mix fills future keys with zero",
     "if (j > r) { out[(size_t)ho * T + j] = -INFINITY; continue; }",
     "if (j > r) { out[(size_t)ho * T + j] = 0.0; continue; }"),
    ("logit mix skipped", "    if (a->w_head_pre) {", "    if (0) {"),
    ("exact indicator tested against the shifted query", "if (exact && c > i) continue;",
     "if (exact && c > i - ip) continue;"),
    ("exact rows without the keys past the query", "const int last = a->exact ? r + s->c_q - 1 : r;",
     "const int last = a->exact ? r + s->c_q - 2 : r;"),
    # the 3-D convolution over (query, key, head)
    ("3-D conv reads the output head's own logits", "rows0 + (size_t)hi * c_q, a->exact",
     "rows0 + (size_t)hh * c_q, a->exact"),
    ("3-D kernel indexed [in][out]", "a->w_kq_3d + ((size_t)h * c_h + hi)",
     "a->w_kq_3d + (((size_t)g * c_h + hi) * c_h + hh)"),
]

PIN_CHECKS = [
    lambda: [pins.test_oracle_matches_library_composition(s) for s in pins.SHAPES],
    pins.test_identity_kernels_give_causal_softmax_attention,
    lambda: [pins.test_single_tap_kernel_closed_form(a, b) for a, b in ((6, 11), (3, 4))],
    pins.test_receptive_field_matches_golden,
    pins.test_zero_kernel_gives_prefix_mean,
    pins.test_diff_transformer_special_case,
    pins.test_causality_future_tokens_do_not_leak,
    pins.test_row_sums_pre_and_post_mix,
    pins.test_groupnorm_statistics_and_depth_scale,
    pins.test_sigmoid_gate_scales_each_head_after_the_affine,
    lambda: [cpins.test_composition_matches_library_brute_force(s, n)
             for s in cpins.SHAPES[:2] for n in ("repeat", "post_kq_only", "plain_attention")],
    lambda: cpins.test_post_conv_single_tap_closed_form(3, 5),
    cpins.test_plain_composition_is_causal_attention,
    lambda: [cpins.test_composed_rows_and_forward_agree(n) for n in ("repeat", "both_post")],
    lambda: [cpins.test_pre_softmax_compositions_match_brute_force(cpins.SHAPES[1], n)
             for n in ("both_pre", "exact_everything")],
    lambda: cpins.test_exact_indicator_single_tap_closed_form(3, 5),
    cpins.test_logit_mix_is_softmax_of_mixed_logits,
    lambda: cpins.test_pre_softmax_rows_and_forward_agree("exact_everything"),
    lambda: [cpins.test_conv3d_matches_brute_force(cpins.SHAPES[1], e) for e in (False, True)],
    cpins.test_conv3d_single_cross_head_tap,
]


def _build_mutant(tmp_path, before, after):
    text = open(SRC).read()
    assert text.count(before) == 1, before
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(before, after))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(src),
                    "-lm"], check=True)
    return str(lib)


@pytest.mark.parametrize("name,before,after", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_some_pin_catches(tmp_path, name, before, after):
    lib = _build_mutant(tmp_path, before, after)
    caught = []
    with oracle.use_library(lib):
        for check in PIN_CHECKS:
            try:
                check()
            except AssertionError:
                caught.append(check)
    assert caught, "no pin caught the planted mistake: " + name


def test_unmutated_source_passes_every_pin(tmp_path):
    lib = tmp_path / "libsame.so"
    shutil.copy(SRC, tmp_path / "same.c")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(lib),
                    str(tmp_path / "same.c"), "-lm"], check=True)
    with oracle.use_library(str(lib)):
        for check in PIN_CHECKS:
            check()
