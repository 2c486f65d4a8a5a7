"""Plant plausible mistakes in a copy of the oracle source (on the CPU) and check
that at least one pin catches each of them."""
import pytest

import oracle
from oracle_pins import PINS

# (name, text to find, replacement, expected count of occurrences replaced)
MUTANTS = [
    ("residual dropped (explicit fwd)",
     "double acc = x[((size_t)b * T + t) * D + c];\n                for (int k = 0; k < W; ++k) {\n"
     "                    if (t - k < 0) break;\n                    acc += wt[k]",
     "double acc = 0.0;\n                for (int k = 0; k < W; ++k) {\n"
     "                    if (t - k < 0) break;\n                    acc += wt[k]"),
    ("tap order reversed (lowrank fwd)",
     "acc += wt[g * W + k] * x[(bt - k) * D + c];",
     "acc += wt[g * W + (W - 1 - k)] * x[(bt - k) * D + c];"),
    ("tying map c mod (D/G)", "const int g = c / G;", "const int g = c % (D / G);"),
    ("U column order tap-major (lowrank weights)",
     "s += z[bt * R + r] * U[(size_t)r * N + j];\n            w[bt * N + j] = s;",
     "s += z[bt * R + r] * U[(size_t)r * N + (j % W) * (N / W) + j / W];\n            w[bt * N + j] = s;"),
    ("dx sign flipped (lowrank bwd)",
     "dx[(bt - k) * D + c] += wt[g * W + k] * gy;",
     "dx[(bt - k) * D + c] -= wt[g * W + k] * gy;"),
    ("dU misses the z factor",
     "dU[(size_t)r * N + j] += zr * dwt[j];", "dU[(size_t)r * N + j] += dwt[j];"),
    ("dz uses U transposed index",
     "s += dwt[j] * U[(size_t)r * N + j];", "s += dwt[j] * U[(size_t)((j + r) % R) * N + j];"),
    ("sequences leak into each other (explicit fwd)",
     "if (t - k < 0) break;\n                    acc += wt[k]",
     "if ((long)b * T + t - k < 0) break;\n                    acc += wt[k]"),
    ("static dx misses the residual",
     "memcpy(dx, dy, sizeof(double) * (size_t)B * T * D);\n    memset(dws",
     "memset(dx, 0, sizeof(double) * (size_t)B * T * D);\n    memset(dws"),
    ("static dws shifted by one tap",
     "dws[(size_t)c * W + k] += gy * x[(bt - k) * D + c];",
     "dws[(size_t)c * W + k] += gy * x[(bt - (k > 0 ? k - 1 : 0)) * D + c];"),
    ("decode window read newest first",
     "acc += wt[g * W + k] * state[(size_t)(W - 1 - k) * D + c];",
     "acc += wt[g * W + k] * state[(size_t)(k - 1) * D + c];"),
    ("decode window not shifted",
     "state_out[(size_t)i * D + c] = state[(size_t)(i + 1) * D + c];",
     "state_out[(size_t)i * D + c] = state[(size_t)i * D + c];"),
    ("decode drops the residual",
     "double acc = x_t[c];\n        acc += wt[g * W + 0] * x_t[c];",
     "double acc = 0.0;\n        acc += wt[g * W + 0] * x_t[c];"),
    ("rope rotates the other way",
     "row[c0 + 2 * i] = a * co - e * si;\n                    row[c0 + 2 * i + 1] = a * si + e * co;",
     "row[c0 + 2 * i] = a * co + e * si;\n                    row[c0 + 2 * i + 1] = -a * si + e * co;"),
    ("rope pairs channel i with i + dh/2",
     "const double a = row[c0 + 2 * i], e = row[c0 + 2 * i + 1];\n                    row[c0 + 2 * i] = a * co - e * si;\n                    row[c0 + 2 * i + 1] = a * si + e * co;",
     "const double a = row[c0 + i], e = row[c0 + np + i];\n                    row[c0 + i] = a * co - e * si;\n                    row[c0 + np + i] = a * si + e * co;"),
    ("rope transpose ignored",
     "const double si = transpose ? -cs[((size_t)t * np + i) * 2 + 1]",
     "const double si = transpose ? cs[((size_t)t * np + i) * 2 + 1]"),
    ("explicit dw misses the group sum (last channel wins)",
     "dw[(bt * NG + g) * W + k] += gy * x[(bt - k) * D + c];",
     "dw[(bt * NG + g) * W + k] = gy * x[(bt - k) * D + c];"),
]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(mutant, tmp_path):
    name, find, repl = mutant
    src = oracle.source()
    assert find in src, "mutation site not found: %s" % name
    variant = oracle.from_source(src.replace(find, repl), str(tmp_path))
    failed = []
    for pin in PINS:
        try:
            pin(variant)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "no pin caught the planted mistake: %s" % name
