"""Each plausible mistake planted in a copy of the oracle fails some pin.

The copies are compiled on the CPU into a temporary directory; the real
oracle source is never modified.  A mutant that no pin catches would mean a
part of the oracle is not pinned.
"""
import os
import shutil
import subprocess
import sys

import pytest

import oracle
import oracle_pins

SRC = os.path.dirname(os.path.abspath(oracle.__file__))

# (name, exact text in gdn_oracle.c, replacement)
MUTANTS = [
    ("delta_sign", "delta[c] = beta * (bf16_bits_to_real(v_row[c]) - kv[c]);",
     "delta[c] = beta * (bf16_bits_to_real(v_row[c]) + kv[c]);"),
    ("beta_on_v_only", "delta[c] = beta * (bf16_bits_to_real(v_row[c]) - kv[c]);",
     "delta[c] = beta * bf16_bits_to_real(v_row[c]) - kv[c];"),
    ("S_k_not_transposed", "acc += S[(size_t)r * V + c] * k_hat[r];",
     "acc += S[(size_t)c * V + r] * k_hat[r];"),
    ("output_uses_k", "acc += S[(size_t)r * V + c] * q_hat[r];",
     "acc += S[(size_t)r * V + c] * k_hat[r];"),
    ("gqa_modulo", "const int32_t h = hv / G;", "const int32_t h = hv % H;"),
    ("scale_missing", "q_hat[r] = bf16_bits_to_real(q_row[r]) * q_norm * (real)scale;",
     "q_hat[r] = bf16_bits_to_real(q_row[r]) * q_norm;"),
    ("scale_on_k_too", "k_hat[r] = bf16_bits_to_real(k_row[r]) * k_norm;",
     "k_hat[r] = bf16_bits_to_real(k_row[r]) * k_norm * (real)scale;"),
    ("decay_dropped", "S[e] *= decay;", "S[e] *= 1;"),
    ("g_sign", "g = -exp((real)A_log[hv]) * softplus(x);",
     "g = exp((real)A_log[hv]) * softplus(x);"),
    ("A_log_not_exponentiated", "g = -exp((real)A_log[hv]) * softplus(x);",
     "g = -(real)A_log[hv] * softplus(x);"),
    ("given_g_sign", "g = (real)g_in[(size_t)tok * HV + hv];", "g = -(real)g_in[(size_t)tok * HV + hv];"),
    ("given_beta_ignored", "beta = (real)beta_in[(size_t)tok * HV + hv];", "beta = 1;"),
    ("given_g_indexed_by_head_only", "g = (real)g_in[(size_t)tok * HV + hv];", "g = (real)g_in[hv];"),
    ("gating_beta_complement", "beta_out[(size_t)tok * HV + hv] = sigmoid(", "beta_out[(size_t)tok * HV + hv] = 1 - sigmoid("),
    ("gating_g_unscaled", "g_out[(size_t)tok * HV + hv] = -exp((real)A_log[hv]) * softplus(x);",
     "g_out[(size_t)tok * HV + hv] = -softplus(x);"),
    ("fp32_inputs_truncated", "    return (real)x;", "    return (real)(int)x;"),
    ("dt_bias_dropped", "+ (real)dt_bias[hv];", ";"),
    ("softplus_is_identity", "return log1p(exp(x));", "return log(exp(x));"),
    ("sigmoid_sign", "return (real)1 / ((real)1 + exp(-x));", "return (real)1 / ((real)1 + exp(x));"),
    ("norm_without_sqrt", "(real)1 / sqrt(sum_kk + eps)", "(real)1 / (sum_kk + eps)"),
    ("a_index_transposed", "a[(size_t)tok * HV + hv]", "a[(size_t)hv * T_tot + tok]"),
    ("inter_per_sequence_index", "real *dst = inter + ((size_t)tok * HV + hv) * head_elems;",
     "real *dst = inter + ((size_t)(tok - bos) * HV + hv) * head_elems;"),
    ("padded_rows_not_zero", "out[((size_t)tok * HV + hv) * V + c] = 0;",
     "out[((size_t)tok * HV + hv) * V + c] = 1;"),
    ("no_writeback", "if (final_write) {", "if (0) {"),
    ("writeback_ignores_flag", "if (final_write) {", "if (1) {"),
    ("slot_bound_off_by_one", "slot >= num_slots", "slot > num_slots"),
]


def _build_mutant(tmpdir, name, old, new):
    d = os.path.join(tmpdir, name)
    os.makedirs(d)
    for f in ("gdn_oracle.c", "gdn_oracle_f32.c", "gdn_oracle_fin.c", "gdn_oracle.h"):
        shutil.copy(os.path.join(SRC, f), d)
    path = os.path.join(d, "gdn_oracle.c")
    text = open(path).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    open(path, "w").write(text.replace(old, new))
    lib = os.path.join(d, "libmutant.so")
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-w",
                    "-o", lib, os.path.join(d, "gdn_oracle.c"), os.path.join(d, "gdn_oracle_f32.c"),
                    os.path.join(d, "gdn_oracle_fin.c"), "-lm"],
                   check=True)
    return lib


# Runs every pin on one library in a child process; exit status 0 means every
# pin passed.  A mutant that reads out of bounds may crash the child, which
# counts as caught.
_RUNNER = """
import sys
sys.path[:0] = [{tests!r}, {root!r}]
import oracle_pins
failed = []
for pin in oracle_pins.ALL_PINS:
    try:
        pin(library={lib!r})
    except Exception as exc:
        failed.append(pin.__name__)
print("caught by:", failed)
sys.exit(1 if failed else 0)
"""


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path, oracle_lib):
    lib = _build_mutant(str(tmp_path), name, old, new)
    tests = os.path.dirname(os.path.abspath(__file__))
    code = _RUNNER.format(tests=tests, root=os.path.dirname(tests), lib=lib)
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert res.returncode != 0, f"mutant {name} passes every pin: {res.stdout}"


def test_unmutated_copy_passes_every_pin(tmp_path, oracle_lib):
    """The same build recipe without a mutation passes, so a caught mutant is
    caught for its mutation and not for the way it was built."""
    lib = _build_mutant(str(tmp_path), "identity", "#include", "#include")
    tests = os.path.dirname(os.path.abspath(__file__))
    code = _RUNNER.format(tests=tests, root=os.path.dirname(tests), lib=lib)
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
