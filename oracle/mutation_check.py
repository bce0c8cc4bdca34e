"""Planted-mistake check of the oracle's pins -- TEST INFRASTRUCTURE ONLY.

    python -m oracle.mutation_check [-k SUBSTRING]

Each entry below plants one plausible mistake (a dropped term, a wrong sign,
bound, index or rounding) in a COPY of mixq_oracle.c, builds that copy into a
temporary shared library, and runs tests/test_oracle_pins.py against it (the
oracle package loads the library named by MIXQ_ORACLE_LIB).  A pin suite that
does its job fails on every planted mistake that changes an output.  The
committed oracle source and library are never touched.

One entry is expected to survive: clamping codes at -128 instead of -127 is
unobservable, because every quantized element satisfies |x| <= a, so
|x * 127/a| never rounds past 127.

Exit status 0 when every other mistake is caught and the expected survivor
survives; 1 otherwise.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys
import tempfile

from . import CFLAGS, _SRC

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, text in mixq_oracle.c, replacement); the first occurrence is replaced
MUTATIONS = [
    # 8-bit weights and the shared symmetric code
    ("weight range without abs", "      float m = fabsf(v);\n      if (m > a) a = m;",
     "      float m = v;\n      if (m > a) a = m;"),
    ("scale a/128", "static float quant_scale(float a) { return a / 127.0f; }",
     "static float quant_scale(float a) { return a / 128.0f; }"),
    ("code truncated, not rounded",
     "  float v = x * inv;\n  return (int8_t)clamp_i32(rint_even(v), -127, 127);",
     "  float v = x * inv;\n  return (int8_t)clamp_i32((int32_t)v, -127, 127);"),
    ("W_out columns reversed",
     "W_out[(size_t)n * K_out_pad + j] = j < K_out ? w[idx[j]] : (uint16_t)0;",
     "W_out[(size_t)n * K_out_pad + j] = j < K_out ? w[idx[K_out - 1 - j]] : (uint16_t)0;"),
    # activations
    ("threshold >=", "int mixed = K_out > 0 && amax > T;", "int mixed = K_out > 0 && amax >= T;"),
    ("mixed from the idx amax only", "float amax = aI > aN ? aI : aN;", "float amax = aI;"),
    ("mixed token keeps the full amax", "float a = mixed ? aN : amax;", "float a = amax;"),
    ("outlier channels not zeroed",
     "Xq[(size_t)m * K + k] = (mixed && mask[k]) ? (int8_t)0 : quant_code(h2f(x[k]), inv);",
     "Xq[(size_t)m * K + k] = quant_code(h2f(x[k]), inv);"),
    ("X_out filled for unmixed tokens",
     "X_out[(size_t)m * K_out_pad + j] = (mixed && j < K_out) ? x[idx[j]] : (uint16_t)0;",
     "X_out[(size_t)m * K_out_pad + j] = (j < K_out) ? x[idx[j]] : (uint16_t)0;"),
    ("detection >=", "if (mag > T) hit[k] = 1;", "if (mag >= T) hit[k] = 1;"),
    ("flags[1] counts idx channels too", "if (!mask[k]) ++outside;", "++outside;"),
    ("bitmap bit order reversed", "bitmap[k / 32] |= 1u << (k % 32);",
     "bitmap[k / 32] |= 1u << (31 - k % 32);"),
    # the layer
    ("layer drops the outlier product",
     "      y[at] = (double)s * (double)s_x[m] * (double)s_w[n] + o;\n",
     "      y[at] = (double)s * (double)s_x[m] * (double)s_w[n];\n"),
    ("layer weight scale by token index",
     "      y[at] = (double)s * (double)s_x[m] * (double)s_w[n] + o;\n",
     "      y[at] = (double)s * (double)s_x[m] * (double)s_w[m % N] + o;\n"),
    ("INT32 product with the next weight row",
     "(int64_t)Wq[(size_t)n * K + k];\n      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;\n"
     "      acc[(size_t)(m - m0) * N + n] = (int32_t)s;",
     "(int64_t)Wq[(size_t)((n + 1) % N) * K + k];\n      if (s > INT32_MAX || s < INT32_MIN) "
     "overflow = 1;\n      acc[(size_t)(m - m0) * N + n] = (int32_t)s;"),
    # 4-bit progressive level 2
    ("s2 floor instead of ceil", "int scale = (span + 14) / 15;", "int scale = span / 15;"),
    ("z2 sign", "int zero = clamp_i32(rint_even(-(float)lo / (float)scale), 0, 15);",
     "int zero = clamp_i32(rint_even((float)lo / (float)scale), 0, 15);"),
    ("q upper bound ignores int8", "      if (qhi > 15) qhi = 15;\n",
     "      qhi = 15;\n"),
    ("effective weight sign", "w8eff[at] = (int8_t)((code - zero) * scale);",
     "w8eff[at] = (int8_t)((zero - code) * scale);"),
    # 4-bit reading B
    ("B: zero added in the layer", "(int64_t)((int)q[(size_t)n * K + k] - z)",
     "(int64_t)((int)q[(size_t)n * K + k] + z)"),
    ("B: zero from lo/s", "zero = clamp_i32(rint_even(-lo / s), 0, 15);",
     "zero = clamp_i32(rint_even(lo / s), 0, 15);"),
    ("B: range / 16", "range / 15.0f", "range / 16.0f"),
    ("B: range not widened to 0",
     "      float lo = 0.0f, hi = 0.0f;\n      for (int i = 0; i < ORC_GROUP; ++i) {\n"
     "        float v = h2f(w[i]);",
     "      float lo = h2f(w[0]), hi = 0.0f;\n      for (int i = 0; i < ORC_GROUP; ++i) {\n"
     "        float v = h2f(w[i]);"),
    ("B: zero of the next group", "const int z = z_g[(size_t)n * ng + g];",
     "const int z = z_g[(size_t)n * ng + (g + 1) % ng];"),
    ("B: scale of the mirrored group",
     "acc += (double)h2f(s_g[(size_t)n * ng + g]) * (double)p;",
     "acc += (double)h2f(s_g[(size_t)n * ng + (ng - 1 - g)]) * (double)p;"),
    ("B: layer drops the outlier product",
     "y[(size_t)(m - m0) * N + n] = (double)s_x[m] * acc + o;",
     "y[(size_t)(m - m0) * N + n] = (double)s_x[m] * acc;"),
    ("B: codes clamped to 14", "clamp_i32(rint_even(h2f(w[i]) / s) + zero, 0, 15)",
     "clamp_i32(rint_even(h2f(w[i]) / s) + zero, 0, 14)"),
    ("B: code truncated", "clamp_i32(rint_even(h2f(w[i]) / s) + zero, 0, 15)",
     "clamp_i32((int32_t)(h2f(w[i]) / s) + zero, 0, 15)"),
    ("B: scale not rounded to fp16", "float s = h2f(s_bits);", "float s = range / 15.0f;"),
    # RMS normalisation
    ("RMSNorm without eps", "double den = sqrt(ss / (double)K + eps);",
     "double den = sqrt(ss / (double)K);"),
    ("RMSNorm sum, not mean", "double den = sqrt(ss / (double)K + eps);",
     "double den = sqrt(ss + eps);"),
    ("RMSNorm gain dropped",
     "double v = den > 0.0 ? (double)h2f(x[k]) / den * (double)h2f(g[k]) : 0.0;",
     "double v = den > 0.0 ? (double)h2f(x[k]) / den : 0.0;"),
    # expected survivor (see the module docstring)
    ("codes clamped at -128", "return (int8_t)clamp_i32(rint_even(v), -127, 127);",
     "return (int8_t)clamp_i32(rint_even(v), -128, 127);"),
]
EXPECTED_SURVIVORS = {"codes clamped at -128"}


def run(select: str | None = None) -> int:
    with open(_SRC) as f:
        original = f.read()
    bad = 0
    with tempfile.TemporaryDirectory() as tmp:
        for i, (name, find, repl) in enumerate(MUTATIONS):
            if select and select not in name:
                continue
            if find not in original:
                print(f"{name:40s} NOT APPLICABLE (text not found)")
                bad += 1
                continue
            src = os.path.join(tmp, f"m{i}.c")
            lib = os.path.join(tmp, f"m{i}.so")
            with open(src, "w") as f:
                f.write(original.replace(find, repl, 1))
            subprocess.run(["gcc", *CFLAGS, "-w", "-o", lib, src, "-lm"], check=True)
            env = dict(os.environ, MIXQ_ORACLE_LIB=lib)
            r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                                os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                               cwd=ROOT, env=env, capture_output=True, text=True)
            caught = r.returncode != 0
            expected = name not in EXPECTED_SURVIVORS
            verdict = "caught" if caught else "survived"
            ok = caught == expected
            bad += 0 if ok else 1
            print(f"{name:40s} {verdict}{'' if ok else '  <-- UNEXPECTED'}")
    return 1 if bad else 0


if __name__ == "__main__":
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("-k", default=None, help="run only mutations whose name contains this")
    sys.exit(run(ap.parse_args().k))
