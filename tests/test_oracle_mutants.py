"""Sensitivity of the oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of oracle.c (a wrong head
index, an off-by-one in the causal count, a dropped scale or normaliser, a
flipped sign, a reversed or misindexed operand, a min taken for the max),
compiles it, and runs the fast oracle pins against that copy in a fresh
process.  The pins must fail for every mutant: a pin set that a plausible bug
passes would not be pinning anything.
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "head_mapping_modulo": ("const int hk = h / G;", "const int hk = h % Hkv;"),
    "causal_off_by_one": ("int64_t n = Lk - Lq + qi + 1;", "int64_t n = Lk - Lq + qi;"),
    "scale_dropped": ("s[j] = scale * acc;", "s[j] = acc;"),
    "lse_sign": ("*lse_row = m + log(l);", "*lse_row = m - log(l);"),
    "normaliser_dropped": ("out_row[d] /= l;", "out_row[d] /= 1.0;"),
    "v_reversed": ("const uint16_t *vrow = v + ((k_tok0 + j) * Hkv + hk)",
                   "const uint16_t *vrow = v + ((k_tok0 + n - 1 - j) * Hkv + hk)"),
    "k_transposed": ("bf16_bits_to_double(qrow[d]) * bf16_bits_to_double(krow[d]);",
                     "bf16_bits_to_double(qrow[d]) * bf16_bits_to_double(krow[D - 1 - d]);"),
    "min_for_max": ("if (s[j] > m)\n            m = s[j];", "if (s[j] < m)\n            m = s[j];"),
    "merge_weight_dropped": ("L += l[s] * w;", "L += w;"),
    "query_token_fixed": ("const int64_t tok = cu_q[b] + qi;", "const int64_t tok = cu_q[b];"),
    "query_head_is_kv_head": ("const uint16_t *qrow = q + (q_tok * Hq + h)",
                              "const uint16_t *qrow = q + (q_tok * Hq + hk)"),
    "key_offset_dropped": ("const uint16_t *krow = k + ((k_tok0 + j) * Hkv + hk)",
                           "const uint16_t *krow = k + ((j) * Hkv + hk)"),
}


def _run_mutant(name, workdir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    if src.count(old) != 1:
        return name, None, f"mutation site for {name} not found exactly once"
    mutated = os.path.join(workdir, f"oracle_{name}.c")
    with open(mutated, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(workdir, f"liboracle_{name}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", lib,
                    mutated, "-lm"], check=True)
    env = dict(os.environ, VGQA_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py"), "-k", "not exhaustive"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    workdir = str(tmp_path_factory.mktemp("mutants"))
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda n: _run_mutant(n, workdir), sorted(MUTANTS)))
    return {name: (rc, out) for name, rc, out in results}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, mutant_results):
    rc, out = mutant_results[name]
    assert rc is not None, out
    assert rc != 0, f"mutant {name} passed every pin:\n{out}"
    assert "failed" in out, out
