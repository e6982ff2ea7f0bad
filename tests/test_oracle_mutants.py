"""Every plausible slip in the oracle's arithmetic fails at least one pin.

The oracle is test infrastructure, and its pins are meant to fail on any
plausible mistake in it: a dropped term, a wrong sign, shift or index, a
transposed operand, truncation where the method floors.  This test plants
one such mistake at a time in a copy of the oracle's C source (on the CPU),
builds the copy, and runs the pins of test_oracle_pins.py and
test_oracle_next.py against it in a separate process, which stops at the
first failing pin.  A copy that passes
every pin is a slip the pins miss, and fails this test.

Deliberately absent: removing the quantiser's clip to [-m, m].  The clamp to
the narrow range +-(2^(k-1) - 1) that follows already gives every input
beyond m the same code, so that change alters no result.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ivit_oracle.c")
WORK = os.path.join(ROOT, "_build", "oracle_mutants")

# (what the slip is, text in the oracle's source, the same text with the slip)
MUTANTS = [
    # integer helpers
    ("floor division truncates", "if ((a % b) != 0 && a < 0)\n        q -= 1;", "if (0)\n        q -= 1;"),
    ("saturation low end one too high", "int64_t lo = -((int64_t)1 << (bits - 1));",
     "int64_t lo = -((int64_t)1 << (bits - 1)) + 1;"),
    ("bit length one too long", "int n = 0;\n    while (v > 0)", "int n = 1;\n    while (v > 0)"),
    # quantiser, dyadic numbers, I_0
    ("quantiser step 2m / 2^k", "double S = 2.0 * m / (double)((1 << k) - 1);", "double S = 2.0 * m / (double)(1 << k);"),
    ("quantiser range to 2^(k-1)", "double lim = (double)((1 << (k - 1)) - 1);", "double lim = (double)(1 << (k - 1));"),
    ("dyadic multiplier below 2^30", "if (v < 2147483648.0) {", "if (v < 1073741824.0) {"),
    ("dyadic multiplier truncated", "double v = round(ldexp(s, cc));", "double v = floor(ldexp(s, cc));"),
    ("dyadic pair takes the larger shift", "int32_t cc = cc1 < cc2 ? cc1 : cc2;", "int32_t cc = cc1 > cc2 ? cc1 : cc2;"),
    ("I_0 floors", "double v = round(1.0 / S);", "double v = floor(1.0 / S);"),
    # linear layers and residual additions
    ("bias dropped", "acc += bias[j];", "acc += 0;"),
    ("reduction misses the last k", "for (int32_t k = 0; k < K; ++k)\n                acc +=",
     "for (int32_t k = 0; k < K - 1; ++k)\n                acc +="),
    ("weight read transposed", "(int64_t)W[(int64_t)j * K + k]", "(int64_t)W[(int64_t)k * N + j]"),
    ("output width ignored", "linear_requant_one(acc, b[j], c[j], out_bits)", "linear_requant_one(acc, b[j], c[j], 8)"),
    ("residual multipliers swapped", "(int64_t)b_skip * s + (int64_t)b_branch * o",
     "(int64_t)b_branch * s + (int64_t)b_skip * o"),
    ("residual shifted by the channel shift", "c_res), 8);", "c[j]), 8);"),
    ("round-half-up adds 2^c", "((int64_t)1 << (c - 1))", "((int64_t)1 << c)"),
    # Shiftmax
    ("log2 e term added", "- shr_floor(I_delta, 4);", "+ shr_floor(I_delta, 4);"),
    ("remainder sign flipped", "I0 + shr_floor(-r, 1)", "I0 + shr_floor(r, 1)"),
    ("large-q shortcut returns I_0", "return 0;                 /* t < 2^62", "return I0;                 /* t < 2^62"),
    ("IntDiv shift M - k_out", "return shr_floor(Dv * e, M - (k_out - 1));", "return shr_floor(Dv * e, M - k_out);"),
    ("IntDiv divides by sum + 1", "floor_div((int64_t)1 << M, sum);", "floor_div((int64_t)1 << M, sum + 1);"),
    ("row minimum for the maximum", "if (L[j] > mx) mx = L[j];", "if (L[j] < mx) mx = L[j];"),
    ("row sum skips the first key", "for (int j = 0; j < n; ++j)\n        sum +=", "for (int j = 1; j < n; ++j)\n        sum +="),
    # attention
    ("logit multiplier dropped", "L[j] = (int32_t)orc_requant(s, b_s, c_s, k_s);",
     "L[j] = (int32_t)orc_requant(s, 1, c_s, k_s);"),
    ("logits shifted by the output shift", "L[j] = (int32_t)orc_requant(s, b_s, c_s, k_s);",
     "L[j] = (int32_t)orc_requant(s, b_s, c_o, k_s);"),
    ("logits saturate at 8 bits", "orc_requant(s, b_s, c_s, k_s)", "orc_requant(s, b_s, c_s, 8)"),
    ("output multiplier dropped", "out[d] = (int8_t)orc_requant(acc, b_o, c_o, 8);",
     "out[d] = (int8_t)orc_requant(acc, 1, c_o, 8);"),
    ("V read from the K columns", "2 * D + h * 64 + d]", "D + h * 64 + d]"),
    ("query ignores the head offset", "(int64_t)i * ld + h * 64;", "(int64_t)i * ld;"),
    # ShiftGELU
    ("1.702 with x >> 2 for x >> 3", "shr_floor(x, 1) + shr_floor(x, 3)", "shr_floor(x, 1) + shr_floor(x, 2)"),
    ("1.702 without x >> 4", "shr_floor(x, 3) + shr_floor(x, 4);", "shr_floor(x, 3);"),
    ("I_max the smaller exponent", "I_p > 0 ? I_p : 0", "I_p < 0 ? I_p : 0"),
    ("second exponent of the wrong sign", "orc_shift_exp(-I_max, I0)", "orc_shift_exp(I_max - I_p, I0)"),
    ("sigmoid over e1 alone", "return orc_int_div(e1, e1 + e2, M, k_out);", "return orc_int_div(e1, e1 + e1, M, k_out);"),
    ("product with I_p instead of x", "orc_requant(x * sigma, b_g, c_g, 8)", "orc_requant(I_p * sigma, b_g, c_g, 8)"),
    # I-LayerNorm
    ("nine Newton steps", "it < 10", "it < 9"),
    ("mean truncates", "int64_t mu = floor_div(sx, cols);", "int64_t mu = sx / cols;"),
    ("variance over n - 1", "floor_div(sd2, cols);", "floor_div(sd2, cols > 1 ? cols - 1 : 1);"),
    ("no lower bound on sigma", "if (sigma < 1)\n            sigma = 1;", "if (sigma < 0)\n            sigma = 1;"),
    ("factor 2^(M-1) / sigma", "int64_t f = floor_div((int64_t)1 << M_ln, sigma);",
     "int64_t f = floor_div((int64_t)1 << (M_ln - 1), sigma);"),
    ("normalisation shift one too far", "shr_floor(d * f, M_ln - F)", "shr_floor(d * f, M_ln - F + 1)"),
    ("gamma dropped", "nv * gamma[i] + beta[i]", "nv + beta[i]"),
    ("beta subtracted", "nv * gamma[i] + beta[i]", "nv * gamma[i] - beta[i]"),
    # block composition
    ("first residual skips from LN1", "x, p->res1_b_skip", "ln, p->res1_b_skip"),
    ("second residual skips from the block input", "xh, p->res2_b_skip", "x, p->res2_b_skip"),
    ("LN2 reads the attention context", "orc_layernorm(xh, T, D, p->ln2_gamma", "orc_layernorm(ctx, T, D, p->ln2_gamma"),
    ("LN2 with LN1's gamma", "p->ln2_gamma, p->ln2_beta", "p->ln1_gamma, p->ln2_beta"),
    ("attention output with the logit dyadic", "p->attn_out_b, p->attn_out_c, ctx);", "p->logit_b, p->logit_c, ctx);"),
    # patch embedding and head
    ("patch flattened channel-last", "(ch * P + ky) * P + kx] = img[src]", "(ky * P + kx) * C + ch] = img[src]"),
    ("patches in column-major order", "z[(int64_t)(py * gx + px) * K", "z[(int64_t)(px * gy + py) * K"),
    ("position and token multipliers swapped", "(int64_t)b_u * u + (int64_t)b_v * v", "(int64_t)b_v * u + (int64_t)b_u * v"),
    ("position rows off by one", "const int64_t v = pos[(int64_t)t * D + j];",
     "const int64_t v = pos[(int64_t)(t == 0 ? 0 : t - 1) * D + j];"),
    ("head reads the last token", "x[(int64_t)bi * Ntok * D + j]", "x[((int64_t)bi * Ntok + Ntok - 1) * D + j]"),
    ("head LayerNorm shift off by one", "orc_layernorm(t, B, D, gamma, beta, F, M_ln, ln_b, ln_c, n);",
     "orc_layernorm(t, B, D, gamma, beta, F, M_ln, ln_b, ln_c + 1, n);"),
    # ShiftGELU with a row maximum
    ("row-max ShiftGELU takes the row minimum", "if (I_p > I_max)\n                I_max = I_p;",
     "if (I_p < I_max)\n                I_max = I_p;"),
    ("row maximum without the floor at 0", "int64_t I_max = 0;\n        for (int32_t i = 0; i < cols; ++i) {\n            int64_t v",
     "int64_t I_max = -300;\n        for (int32_t i = 0; i < cols; ++i) {\n            int64_t v"),
    ("second exponential at 0", "int64_t e2 = orc_shift_exp(-I_max, I0);\n        for",
     "int64_t e2 = orc_shift_exp(0, I0);\n        for"),
    ("0 / 0 read as one half", "int64_t sigma = orc_int_div(e1, sum > 0 ? sum : 1, M, k_out);",
     "int64_t sigma = sum > 0 ? orc_int_div(e1, sum, M, k_out) : ((int64_t)1 << (k_out - 2));"),
    # Log-Int-Softmax
    ("log2 rounded at 2 instead of sqrt 2", "((int64_t)1 << (2 * fl + 1))", "((int64_t)1 << (2 * fl + 2))"),
    ("zero probability coded 0", "if (P16 <= 0)\n        return 15;", "if (P16 <= 0)\n        return 0;"),
    ("LIS probability to 15 bits", "sum, M, 16));", "sum, M, 15));"),
    ("BitShift one place short", "((int64_t)1 << (15 - K[j]))", "((int64_t)1 << (14 - K[j]))"),
    ("LIS reads V from the K columns", "base[(int64_t)j * ld + 2 * D + h * 64 + d] * ((int64_t)1",
     "base[(int64_t)j * ld + D + h * 64 + d] * ((int64_t)1"),
    # I-LayerNorm with power-of-two factors
    ("PTF mean without the factors", "sx += (int64_t)xr[i] * ((int64_t)1 << alpha[i]);", "sx += (int64_t)xr[i];"),
    ("PTF variance without the factors",
     "int64_t d = (int64_t)xr[i] * ((int64_t)1 << alpha[i]) - mu;\n            sd2",
     "int64_t d = (int64_t)xr[i] - mu;\n            sd2"),
    ("PTF normalises the unshifted input",
     "int64_t d = (int64_t)xr[i] * ((int64_t)1 << alpha[i]) - mu;\n            int64_t nv",
     "int64_t d = (int64_t)xr[i] - mu;\n            int64_t nv"),
]

# Runs the pins against one build, stopping at the first failure: exit 1 if
# a pin fails, 0 if all pass (a crash exits otherwise, which also counts).
RUNNER = r"""
import inspect, sys
sys.path[:0] = [sys.argv[2], sys.argv[3]]
import oracle
oracle.use_library(sys.argv[1])
import test_oracle_pins, test_oracle_next
for pins in (test_oracle_pins, test_oracle_next):
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if name.startswith("test_") and not inspect.signature(fn).parameters:
            try:
                fn()
            except Exception:
                sys.exit(1)
sys.exit(0)
"""


def run_pins(so):
    r = subprocess.run([sys.executable, "-c", RUNNER, so, ROOT, os.path.join(ROOT, "tests")],
                       capture_output=True, text=True, timeout=600)
    return r.returncode


@pytest.mark.slow
def test_every_planted_slip_fails_a_pin():
    src = open(SRC).read()
    for name, old, new in MUTANTS:
        assert src.count(old) >= 1, f"{name}: the text to alter is no longer in the oracle"
    shutil.rmtree(WORK, ignore_errors=True)
    os.makedirs(WORK)
    import oracle
    builds = []
    for i, (name, old, new) in enumerate(MUTANTS):
        c_path = os.path.join(WORK, f"m{i}.c")
        with open(c_path, "w") as f:
            f.write(src.replace(old, new, 1))
        builds.append((name, oracle.compile_source(c_path, os.path.join(WORK, f"m{i}.so"))))
    # the unaltered source passes every pin, so a failure below is the slip's
    clean = oracle.compile_source(SRC, os.path.join(WORK, "clean.so"))
    assert run_pins(clean) == 0
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        codes = list(ex.map(lambda b: run_pins(b[1]), builds))
    missed = [name for (name, _), code in zip(builds, codes) if code == 0]
    shutil.rmtree(WORK, ignore_errors=True)
    assert not missed, f"slips no pin catches: {missed}"
