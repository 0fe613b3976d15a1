"""Plant plausible mistakes in copies of the oracle's C source (on the CPU) and check that
each one trips at least one pin of tests/oracle_pins.py.  A mutant that passes every pin
would mean the pins cannot tell that mistake from the truth."""
import subprocess
import sys
from pathlib import Path

import pytest

import oracle as oracle_pkg

ROOT = Path(__file__).resolve().parents[1]

# (id, text in e2d2_oracle.c, replacement)
MUTANTS = [
    ("enc-excludes-own-block", "(uint8_t)(block_of(j, S) <= block_of(i, S))",
     "(uint8_t)(block_of(j, S) < block_of(i, S))"),
    ("dec-enc-includes-own-block", "mask[i * W + j] = (uint8_t)(block_of(j, S) < block_of(i, S));",
     "mask[i * W + j] = (uint8_t)(block_of(j, S) <= block_of(i, S));"),
    ("dec-own-becomes-causal-blocks", "mask[i * W + L + j] = (uint8_t)(block_of(j, S) == block_of(i, S));",
     "mask[i * W + L + j] = (uint8_t)(block_of(j, S) <= block_of(i, S));"),
    ("dec-own-is-causal-within-block", "mask[i * W + L + j] = (uint8_t)(block_of(j, S) == block_of(i, S));",
     "mask[i * W + L + j] = (uint8_t)(block_of(j, S) == block_of(i, S) && j <= i);"),
    ("sample-drops-last-prefix-key", "mask[(size_t)i * (P + S) + j] = 1;",
     "mask[(size_t)i * (P + S) + j] = (uint8_t)(j != P - 1);"),
    ("block-of-off-by-one", "static int block_of(int pos, int S) { return pos / S; }",
     "static int block_of(int pos, int S) { return (pos + 1) / S; }"),
    ("dropped-scale", "s[j] = scale * acc;", "s[j] = acc;"),
    ("wrong-default-scale", "1.0 / sqrt((double)d)", "1.0 / (double)d"),
    ("sign-of-exponent", "double p = exp(s[j] - m);", "double p = exp(m - s[j]);"),
    ("missing-normalisation", "for (int c = 0; c < d; ++c) o[c] /= l;", ""),
    ("lse-drops-max", "lse[i] = m + log(l);", "lse[i] = log(l);"),
    ("lse-log2", "lse[i] = m + log(l);", "lse[i] = m + log2(l);"),
    ("gqa-modulo-mapping", "const int g = h / G;\n            double* kd = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));",
     "const int g = h % Hkv;\n            double* kd = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));"),
    ("dec-swapped-key-sources", "rows_to_double(k_enc + ko, L, d, kd);\n            rows_to_double(k_dec + ko, L, d, kd + (size_t)L * d);",
     "rows_to_double(k_dec + ko, L, d, kd);\n            rows_to_double(k_enc + ko, L, d, kd + (size_t)L * d);"),
    ("dec-values-from-keys", "rows_to_double(v_dec + ko, L, d, vd + (size_t)L * d);",
     "rows_to_double(k_dec + ko, L, d, vd + (size_t)L * d);"),
    ("sample-cache-stride-P", "const size_t co = ((size_t)b * Hkv + g) * (size_t)capacity * d;",
     "const size_t co = ((size_t)b * Hkv + g) * (size_t)(P + S) * d;"),
    ("transposed-q-index", "acc += (double)q[(size_t)i * d + c] * keys[(size_t)j * d + c];",
     "acc += (double)q[(size_t)c * d + (i % d)] * keys[(size_t)j * d + c];"),
    ("append-off-by-one", "capacity + P + r) * d;", "capacity + P + r + 1) * d;"),
    ("append-swaps-k-and-v", "memcpy(v_cache + dst, v_new + src, sizeof(uint16_t) * d);",
     "memcpy(v_cache + dst, k_new + src, sizeof(uint16_t) * d);"),
    # BD3LM's 2L-token attention
    ("bd3lm-noised-sees-own-clean-block", "if (noised_row) a = noised_col ? (bj == bi) : (bj < bi);",
     "if (noised_row) a = noised_col ? (bj == bi) : (bj <= bi);"),
    ("bd3lm-clean-sees-noised", "else a = noised_col ? 0 : (bj <= bi);", "else a = noised_col ? (bj < bi) : (bj <= bi);"),
    ("bd3lm-clean-rows-read-noised-keys", "rows_to_double(k + ((size_t)b * Hkv + g) * W * d, (int)W, d, kd);",
     "rows_to_double(k + ((size_t)b * Hkv + g) * W * d, (int)W / 2, d, kd);\n            rows_to_double(k + ((size_t)b * Hkv + g) * W * d, (int)W / 2, d, kd + (size_t)L * d);"),
    # backward of the train calls
    ("bwd-drops-row-term", "const double ds = exp(s[j] - lse) * (dp[j] - dsum);",
     "const double ds = exp(s[j] - lse) * dp[j];"),
    ("bwd-dk-wrong-sign", "dk[(size_t)j * d + c] += scale * ds * (double)qi[c];",
     "dk[(size_t)j * d + c] -= scale * ds * (double)qi[c];"),
    ("bwd-dq-missing-scale", "dqi[c] += scale * ds * keys[(size_t)j * d + c];",
     "dqi[c] += ds * keys[(size_t)j * d + c];"),
    ("bwd-dv-without-p", "dv[(size_t)j * d + c] += p * (double)gi[c];",
     "dv[(size_t)j * d + c] += (double)gi[c];"),
    ("bwd-dec-swaps-sources", "memcpy(dk_enc + ko, dkd, sizeof(double) * (size_t)L * d);",
     "memcpy(dk_enc + ko, dkd + (size_t)L * d, sizeof(double) * (size_t)L * d);"),
    # ragged prefixes
    ("ragged-first-entry-prefix", "const int Pb = P[b];", "const int Pb = P[0];"),
    ("ragged-block-read-from-cache", "rows_to_double(k_blk + bo, S, d, kd + (size_t)Pb * d);",
     "rows_to_double(k_cache + co + (size_t)Pb * d, S, d, kd + (size_t)Pb * d);"),
]

_RUNNER = r"""
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
from oracle import Oracle
import oracle_pins
orc = Oracle({lib!r})
failed = []
for pin in oracle_pins.ALL_PINS:
    try:
        pin(orc)
    except Exception as exc:
        failed.append(pin.__name__)
print("FAILED_PINS", ",".join(failed))
sys.exit(0 if failed else 3)
"""


@pytest.mark.parametrize("mid,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, mid, old, new):
    src = oracle_pkg.SOURCE.read_text()
    assert src.count(old) >= 1, f"mutation site for {mid} not found"
    mutated = src.replace(old, new, 1)
    c_path = tmp_path / "mutant.c"
    c_path.write_text(mutated)
    lib = tmp_path / "libmutant.so"
    oracle_pkg.build(c_path, lib)
    code = _RUNNER.format(root=str(ROOT), tests=str(ROOT / "tests"), lib=str(lib))
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    # exit 0: some pin failed (caught); a crash (signal / nonzero other than 3) also counts as
    # caught; exit 3 means every pin passed on the mutant.
    assert res.returncode != 3, f"mutant {mid} survived every pin:\n{res.stdout}\n{res.stderr}"
