"""Planted mistakes in the oracle must each break at least one pin (CPU only).

Every mutant is a copy of the oracle's C source with one plausible slip (a
dropped term, a wrong sign, a transposed operand, a wrong index), compiled to
a temporary library.  The pins of ``test_oracle_pins`` are then run against
it; a mutant that passes all of them would mean the pins cannot tell that
slip from the real oracle.
"""
import os
import tempfile

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdpa_oracle.c")

MUTANTS = {
    "silu_sign": ("pi[k] = si[k] / (1.0 + exp(-si[k]));", "pi[k] = si[k] / (1.0 + exp(si[k]));"),
    "softmax_no_max": ("pi[k] = exp(si[k] - mx) / sum;", "pi[k] = exp(si[k]) / sum;"),
    "lse_no_max": ("lse_rows[i] = mx + log(sum);", "lse_rows[i] = log(sum);"),
    "logit_no_scale": ("S[(size_t)i * m + k] = scale * acc + (b1b ? (double)b1b[k] : 0.0);",
                       "S[(size_t)i * m + k] = acc + (b1b ? (double)b1b[k] : 0.0);"),
    "logit_k_transposed": ("acc += (double)qi[d] * (double)kk[d];",
                           "acc += (double)qi[d] * (double)kb[(size_t)d * m + k];"),
    "pv_v_transposed": ("acc += P[(size_t)i * m + kk] * (double)vb[(size_t)kk * dh + d];",
                        "acc += P[(size_t)i * m + kk] * (double)vb[(size_t)d * m + kk];"),
    "q_head_offset": ("const float* qb = q + ((size_t)t0 * h + j) * dh;\n    const float* kb = k + ((size_t)b * h + j) * (size_t)m * dh;\n    const float* vb = v + ((size_t)b * h + j) * (size_t)m * dh;\n    const float* b1b = b1 ? b1 + ((size_t)b * h + j) * (size_t)m : NULL;\n    const float* b2b",
                      "const float* qb = q + ((size_t)t0 * h) * dh;\n    const float* kb = k + ((size_t)b * h + j) * (size_t)m * dh;\n    const float* vb = v + ((size_t)b * h + j) * (size_t)m * dh;\n    const float* b1b = b1 ? b1 + ((size_t)b * h + j) * (size_t)m : NULL;\n    const float* b2b"),
    # the biased variant
    "b1_ignored": ("S[(size_t)i * m + k] = scale * acc + (b1b ? (double)b1b[k] : 0.0);",
                   "S[(size_t)i * m + k] = scale * acc;"),
    "b1_per_token": ("S[(size_t)i * m + k] = scale * acc + (b1b ? (double)b1b[k] : 0.0);",
                     "S[(size_t)i * m + k] = scale * acc + (b1b ? (double)b1b[i % m] : 0.0);"),
    "b1_unscaled_twice": ("S[(size_t)i * m + k] = scale * acc + (b1b ? (double)b1b[k] : 0.0);",
                          "S[(size_t)i * m + k] = scale * (acc + (b1b ? (double)b1b[k] : 0.0));"),
    "b2_dropped": ("oi[d] = acc + (b2b ? (double)b2b[d] : 0.0);", "oi[d] = acc;"),
    "b2_wrong_head": ("const float* b2b = b2 ? b2 + ((size_t)b * h + j) * (size_t)dh : NULL;",
                      "const float* b2b = b2 ? b2 + ((size_t)b * h) * (size_t)dh : NULL;"),
    "db1_sums_p": ("for (int i = 0; i < n; ++i) acc += dP[(size_t)i * m + kk];\n        db1b[kk] = acc;",
                   "for (int i = 0; i < n; ++i) acc += P[(size_t)i * m + kk];\n        db1b[kk] = acc;"),
    "db1_scaled": ("db1b[kk] = acc;", "db1b[kk] = scale * acc;"),
    "db2_row_stride": ("for (int i = 0; i < n; ++i) acc += (double)gb[(size_t)i * h * dh + d];",
                       "for (int i = 0; i < n; ++i) acc += (double)gb[(size_t)i * dh + d];"),
    "silu_grad_term": ("dpi[kk] = dpi[kk] * sg * (1.0 + si[kk] * (1.0 - sg));",
                       "dpi[kk] = dpi[kk] * sg * (1.0 + si[kk] * sg);"),
    "softmax_grad_sign": ("dpi[kk] = pi[kk] * (dpi[kk] - D);", "dpi[kk] = pi[kk] * (dpi[kk] + D);"),
    "dq_no_scale": ("dqi[d] = scale * acc;", "dqi[d] = acc;"),
    "dk_row_stride": ("acc += dP[(size_t)i * m + kk] * (double)qb[(size_t)i * h * dh + d];",
                      "acc += dP[(size_t)i * m + kk] * (double)qb[(size_t)i * dh + d];"),
    "dv_uses_logits": ("for (int i = 0; i < n; ++i) acc += P[(size_t)i * m + kk] * (double)gb[(size_t)i * h * dh + d];",
                       "for (int i = 0; i < n; ++i) acc += S[(size_t)i * m + kk] * (double)gb[(size_t)i * h * dh + d];"),
    "relu_negative_half": ("pi[k] = si[k] > 0.0 ? si[k] : 0.0;", "pi[k] = si[k] > 0.0 ? si[k] : 0.01 * si[k];"),
    "relu_grad_always": ("dpi[kk] = si[kk] > 0.0 ? dpi[kk] : 0.0;", "dpi[kk] = dpi[kk];"),
    "gelu_cdf_scale": ("return 0.5 * (1.0 + erf(x * 0.70710678118654752440));",
                       "return 0.5 * (1.0 + erf(x));"),
    "gelu_grad_no_pdf": ("dpi[kk] = dpi[kk] * (normal_cdf(si[kk]) + si[kk] * normal_pdf(si[kk]));",
                         "dpi[kk] = dpi[kk] * normal_cdf(si[kk]);"),
    "dp_uses_q": ("acc += (double)gb[(size_t)i * h * dh + d] * (double)vb[(size_t)kk * dh + d];",
                  "acc += (double)gb[(size_t)i * h * dh + d] * (double)kb[(size_t)kk * dh + d];"),
}

PIN_CALLS = (
    [(pins.test_hand_derived_golden, (phi,)) for phi in pins.PHIS]
    + [(pins.test_identity_equals_other_association, ())]
    + [(pins.test_matches_library_routines, (phi,)) for phi in pins.PHIS]
    + [(pins.test_softmax_matches_sdpa_and_lse, ()), (pins.test_softmax_special_cases, ()),
       (pins.test_silu_closed_forms, ()), (pins.test_identity_backward_closed_forms, ()),
       (pins.test_softmax_backward_invariants, ())]
    + [(pins.test_backward_matches_torch_autograd, (phi,)) for phi in pins.PHIS]
    + [(pins.test_relu_gelu_closed_forms, ())]
    + [(pins.test_matches_library_routines, (phi,)) for phi in ("relu", "gelu")]
    + [(pins.test_backward_matches_torch_autograd, (phi,)) for phi in ("relu", "gelu")]
    + [(pins.test_bias_hand_derived_golden, (phi,)) for phi in pins.PHIS]
    + [(pins.test_key_bias_is_an_extra_head_dim_column, (phi,)) for phi in ("silu", "softmax")]
    + [(pins.test_output_bias_shifts_o_and_its_gradient_is_the_token_sum, ("silu",))]
    + [(pins.test_softmax_key_bias_shift_invariance, ())]
    + [(pins.test_biased_operator_matches_torch_autograd, (phi,)) for phi in ("silu", "softmax")]
)


def _failing_pins(lib):
    saved = oracle._lib
    oracle._lib = lib
    failed = []
    try:
        for fn, args in PIN_CALLS:
            try:
                fn(*args)
            except AssertionError:
                failed.append(fn.__name__ + str(args))
    finally:
        oracle._lib = saved
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    with tempfile.TemporaryDirectory() as d:
        msrc = os.path.join(d, "mutant.c")
        with open(msrc, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.load(oracle.build(force=True, src=msrc, out=os.path.join(d, "libmutant.so")))
        failed = _failing_pins(lib)
    assert failed, f"mutant {name} passed every pin"


def test_unmutated_oracle_passes_every_pin():
    assert _failing_pins(oracle.load()) == []
