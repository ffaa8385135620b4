"""Mutation check for the oracle's pins.

Each case compiles a copy of the oracle with one plausible mistake planted in
its source (a dropped scale, a wrong block index, a transposed operand, double
rounding, an off-by-one in the masked bound, ...) and runs the whole pin suite
against it in a child process.  The pins are only worth something if every
mutant fails at least one of them.  The mistakes are planted in the oracle, on
the CPU; nothing here touches a GPU.
"""
import json
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dg_oracle.c")

# (name, exact text in dg_oracle.c, replacement)
MUTANTS = [
    ("drop_sfa", "* (double)sfa_row[k / ORACLE_BLOCK_K]", "* 1.0"),
    ("drop_sfb", "* (double)sfb_nblock_row[k / ORACLE_BLOCK_K]", "* 1.0"),
    ("sfb_block_by_k_only", "sfb + (n / ORACLE_BLOCK_N) * KB", "sfb"),
    ("sfa_kblock_off_by_one", "sfa_row[k / ORACLE_BLOCK_K]", "sfa_row[(k + 1) / ORACLE_BLOCK_K % (K / ORACLE_BLOCK_K)]"),
    ("transposed_b_index", "const uint8_t *b_row = b + n * K;", "const uint8_t *b_row = b + (n % 2) * K;"),
    ("skip_last_k", "for (int64_t k = 0; k < K; ++k)", "for (int64_t k = 0; k < K - 1; ++k)"),
    ("float_accumulator", "double s = 0.0;\n    for", "float s = 0.0f;\n    for"),
    ("e4m3_bias_8", "ldexp(1.0 + mant / 8.0, expo - 7)", "ldexp(1.0 + mant / 8.0, expo - 8)"),
    ("e4m3_mantissa_16", "ldexp(1.0 + mant / 8.0, expo - 7)", "ldexp(1.0 + mant / 16.0, expo - 7)"),
    ("e4m3_subnormal_scale", "ldexp((double)mant, -9)", "ldexp((double)mant, -10)"),
    ("e4m3_sign_dropped", "return sign ? -mag : mag;", "return mag;"),
    ("bf16_double_rounding", "double ax = fabs(x);", "double ax = (double)(float)fabs(x);"),
    ("bf16_ties_away", "double r = nearbyint(n);", "double r = round(n);"),
    ("bf16_truncate", "double r = nearbyint(n);", "double r = trunc(n);"),
    ("bf16_subnormal_quantum", "(E < -126) ? -133 : E - 7", "(E < -126) ? -134 : E - 7"),
    ("masked_bound_inclusive", "if (m >= valid)", "if (m > valid)"),
    ("masked_mask_ignored", "if (m >= valid)", "if (m >= max_m)"),
    ("masked_mask_of_group0", "masked_m[g] < 0 ? 0 : (masked_m[g] > max_m ? max_m : masked_m[g])",
     "masked_m[0] < 0 ? 0 : (masked_m[0] > max_m ? max_m : masked_m[0])"),
    ("contiguous_pad_as_expert0", "if (e < 0)\n            continue;", "if (e < 0)\n            e = 0;"),
    ("contiguous_wrong_sfb_group", "sfb + e * NB * KB", "sfb"),
    ("masked_wrong_b_group", "b + g * N * K, sfb + g * NB * KB", "b, sfb + g * NB * KB"),
    ("bf16_operand_bias_126", "ldexp(1.0 + mant / 128.0, expo - 127)", "ldexp(1.0 + mant / 128.0, expo - 126)"),
    ("bf16_operand_mantissa_64", "ldexp(1.0 + mant / 128.0, expo - 127)", "ldexp(1.0 + mant / 64.0, expo - 127)"),
    ("bf16_operand_subnormal", "ldexp((double)mant, -133)", "ldexp((double)mant, -134)"),
    ("bf16_operand_sign_dropped", "int sign = (bits >> 15) & 1;", "int sign = 0;"),
    ("bf16_operand_nan_as_inf", "mag = mant ? NAN : INFINITY;", "mag = INFINITY;"),
    ("bf16_gemm_transposed_b", "const uint16_t *b_row = b + n * K;", "const uint16_t *b_row = b + (n % 2) * K;"),
    ("bf16_gemm_skip_first_k", "s += tab[a_row[k]] * tab[b_row[k]];", "s += k ? tab[a_row[k]] * tab[b_row[k]] : 0.0;"),
    ("bf16_gemm_float_acc", "double s = 0.0;\n        for", "float s = 0.0f;\n        for"),
    ("bf16_gemm_a_row_for_b", "s += tab[a_row[k]] * tab[b_row[k]];", "s += tab[a_row[k]] * tab[a_row[k]];"),
    ("bf16_contiguous_wrong_group", "bf16_gemm_row(tab, a + r * K, b + e * N * K,", "bf16_gemm_row(tab, a + r * K, b,"),
    ("bf16_masked_wrong_group", "bf16_gemm_row(tab, a + r * K, b + g * N * K,", "bf16_gemm_row(tab, a + r * K, b,"),
    ("kgrouped_local_scale_block", "sfa[m * KB + k / ORACLE_BLOCK_K]", "sfa[m * KB + (k - k_off[g]) / ORACLE_BLOCK_K]"),
    ("kgrouped_group_shifted", "for (int64_t k = k_off[g]; k < k_off[g + 1]; ++k)",
     "for (int64_t k = k_off[g] / 2; k < k_off[g + 1]; ++k)"),
    ("kgrouped_addend_dropped", "acc[o] = (c ? (double)c[o] : 0.0) + s;", "acc[o] = s;"),
    ("kgrouped_sfb_one_n_block", "(double)sfb[(n / ORACLE_BLOCK_N) * KB + k / ORACLE_BLOCK_K]",
     "(double)sfb[k / ORACLE_BLOCK_K]"),
    ("kgrouped_b_row_of_a", "tab[b[k * N + n]]", "tab[b[k * N + (n % M)]]"),
]

_CHILD = r"""
import json, sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle, oracle_pins
o = oracle.Oracle(oracle.load({lib!r}))
print(json.dumps(oracle_pins.run_all(o)))
"""


def _compile(src_text: str, out_dir: str, tag: str) -> str:
    csrc = os.path.join(out_dir, f"{tag}.c")
    with open(csrc, "w") as f:
        f.write(src_text)
    lib = os.path.join(out_dir, f"lib{tag}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", csrc, "-o", lib, "-lm"],
                   check=True)
    return lib


def _run_pins(lib: str):
    """Run the pin suite in a child process; None if the child crashed."""
    code = _CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), lib=lib)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                       env={**os.environ, "OMP_NUM_THREADS": "1"})
    if r.returncode != 0:
        return None
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_every_mutant_is_caught(tmp_path):
    src = open(SRC).read()
    for name, old, new in MUTANTS:
        assert src.count(old) >= 1, f"mutation site for {name} not found"

    def one(case):
        name, old, new = case
        lib = _compile(src.replace(old, new), str(tmp_path), name)
        return name, _run_pins(lib)

    workers = max(2, min(8, os.cpu_count() or 2))
    with ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(one, MUTANTS + [("unmutated", "", "")]))
    escaped = [name for name, failed in results if name != "unmutated" and failed == []]
    assert not escaped, f"mutants that passed every pin: {escaped}"
    clean = dict(results)["unmutated"]
    assert clean == [], f"the unmutated copy failed pins: {clean}"
