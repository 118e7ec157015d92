"""Plant plausible mistakes in a copy of the oracle's C source and check that
every one of them fails at least one pin.  The real oracle is never modified:
each mutant is a temporary copy compiled with gcc on the CPU.
"""
import os
import re
import subprocess
import sys

import pytest

import oracle

# (name, pattern, replacement) -- each a mistake someone could plausibly make.
MUTANTS = [
    ("scale_dropped", r"s\[j\] = scale \* dot;", "s[j] = dot;"),
    ("gqa_modulo", r"g = h / G;", "g = h % Hkv;"),
    ("causal_off_by_one", r"return \(last \+ 1 < Lkv\) \? last \+ 1 : Lkv;",
     "return (last < Lkv) ? last : Lkv;"),
    ("causal_top_left", r"int64_t last = i \+ \(Lkv - Lq\);", "int64_t last = i;"),
    ("lse_missing_max", r"\*lse = m \+ log\(l\);", "*lse = log(l);"),
    ("lse_log2", r"\*lse = m \+ log\(l\);", "*lse = (m + log(l)) / log(2.0);"),
    ("no_normalisation", r"double p = exp\(s\[j\] - m\) / l;", "double p = exp(s[j] - m);"),
    ("keys_read_from_v", r"const uint16_t \*kj = k_base \+ k_off\[j\];",
     "const uint16_t *kj = v_base + v_off[j];"),
    ("ragged_kv_base_from_q", r"int64_t t = \(int64_t\)cu_kv\[b\] \+ j;",
     "int64_t t = (int64_t)cu_q[b] + j;"),
    ("paged_slot_swapped", r"int64_t slot = t % page_size;", "int64_t slot = t / page_size % page_size;"),
    ("paged_table_row", r"page_table\[\(int64_t\)b \* pt_stride \+ t / page_size\]",
     "page_table[(int64_t)b + t / page_size * pt_stride]"),
    ("merge_weight_sign", r"double w = exp\(lse_part\[\(int64_t\)s \* R \+ r\] - L\);",
     "double w = exp(L - lse_part[(int64_t)s * R + r]);"),
    ("merge_lse_no_max", r"double L = M \+ log\(sum\);", "double L = log(sum);"),
    ("empty_row_lse_zero", r"\*lse = -INFINITY;\n        return;", "*lse = 0.0;\n        return;"),
    ("dense_batch_stride_k", r"ko\[j\] = \(int64_t\)b \* ks\[0\] \+ j \* ks\[1\]",
     "ko[j] = j * ks[1]"),
]


_RUNNER = r"""
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle
from oracle_pin_battery import ALL_PINS
orc = oracle.Oracle({so!r})
failed = []
for pin in ALL_PINS:
    try:
        pin(orc)
    except Exception as e:
        failed.append(pin.__name__)
print("FAILED_PINS", ",".join(failed))
"""


def _run_pins(so_path):
    """Run the pin battery on a mutant in a child process; a crash (a mutant
    that reads out of bounds) counts as caught."""
    here = os.path.dirname(os.path.abspath(__file__))
    code = _RUNNER.format(root=os.path.dirname(here), tests=here, so=so_path)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                       timeout=600)
    if r.returncode != 0:
        return [f"crashed rc={r.returncode}"]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("FAILED_PINS")][-1]
    names = line.split(" ", 1)[1].strip() if " " in line else ""
    return [n for n in names.split(",") if n]


@pytest.mark.parametrize("name,pat,rep", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, pat, rep):
    src = open(oracle.SOURCE).read()
    mutated, n = re.subn(pat, rep, src)
    assert n >= 1, f"mutation {name} did not apply"
    c_path = os.path.join(tmp_path, f"m_{name}.c")
    so_path = os.path.join(tmp_path, f"m_{name}.so")
    open(c_path, "w").write(mutated)
    oracle.compile_source(c_path, so_path)
    failed = _run_pins(so_path)
    assert failed, f"mutant {name} passed every pin"
