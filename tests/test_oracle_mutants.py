"""Planted mistakes in the oracle must fail its pins.

Each case copies moe_oracle.cpp to a temporary directory, plants one plausible
mistake (a flipped comparison, a dropped term, a wrong sign or index, a broken
order), compiles it with the oracle's own flags and runs every pin against it.
A mutant that passes every pin would mean the pins cannot see that mistake.
CPU only; nothing here touches the CUDA path.
"""
import os
import subprocess
import sys

import pytest

import oracle
import oracle_pins

_RUNNER = """
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle, oracle_pins
orc = oracle.Oracle({lib!r})
caught = []
for pin in oracle_pins.ALL_PINS:
    try:
        pin(orc)
    except Exception:
        caught.append(pin.__name__)
print("CAUGHT", ",".join(caught))
"""

MUTANTS = [
    ("tie-break picks the highest index",
     "if (best < 0 || x[e] > x[best]) best = e;", "if (best < 0 || x[e] >= x[best]) best = e;"),
    ("renormalise flag ignored",
     "denom = S;", "denom = Z;"),
    ("softmax denominator over the selected experts only",
     "for (int32_t e = 0; e < E; ++e) Z += std::exp(x[e] - m);",
     "for (int32_t j = 0; j < k; ++j) Z += std::exp(x[sel[j]] - m);"),
    ("sign error in the exponent",
     "double wj = std::exp(x[sel[j]] - m) / denom;", "double wj = std::exp(m - x[sel[j]]) / denom;"),
    ("weight taken from the wrong expert",
     "double wj = std::exp(x[sel[j]] - m) / denom;", "double wj = std::exp(x[j] - m) / denom;"),
    ("max not subtracted",
     "if (x[e] > m) m = x[e];", "if (x[e] > m) m = m;"),
    ("unstable order inside an expert",
     "if (le >= 0) rows_of[le].push_back(s);", "if (le >= 0) rows_of[le].insert(rows_of[le].begin(), s);"),
    ("padding adds a block to full blocks",
     "int64_t padded = ((n + block_size - 1) / block_size) * block_size;",
     "int64_t padded = ((n + block_size) / block_size) * block_size;"),
    ("remote slots counted on expert 0",
     "if (le >= 0) rows_of[le].push_back(s);", "rows_of[le < 0 ? 0 : le].push_back(s);"),
    ("expert_ids one block too long",
     "b < offsets[e + 1] / block_size; ++b", "b <= offsets[e + 1] / block_size && b < NB; ++b"),
    ("gather copies the wrong token",
     "hidden + (s / k) * H", "hidden + (s % k) * H"),
    ("combine accumulates in descending j",
     "for (int32_t j = 0; j < k; ++j) {\n                int64_t r = inv_perm[t * k + j];",
     "for (int32_t j = k - 1; j >= 0; --j) {\n                int64_t r = inv_perm[t * k + j];"),
    ("combine rounds the product before adding",
     "acc = std::fma(topk_weights[t * k + j], y, acc);",
     "{ volatile float prod = topk_weights[t * k + j] * y; acc = prod + acc; }"),
    ("bf16 output truncated instead of rounded",
     "u += 0x7fffu + lsb;", "u += 0u * lsb;"),
    ("combine ignores the remote marker",
     "if (r < 0) continue;", "if (r < 0) r = 0;"),
    ("sigmoid with the sign of the exponent flipped",
     "score[j] = 1.0 / (1.0 + std::exp(-x[sel[j]]));", "score[j] = 1.0 / (1.0 + std::exp(x[sel[j]]));"),
    ("sigmoid renormalise flag ignored",
     "const double wj = renormalize ? (S > 0.0 ? score[j] / S : 1.0 / k) : score[j];",
     "const double wj = score[j];"),
    ("sigmoid weight taken from the wrong expert",
     "score[j] = 1.0 / (1.0 + std::exp(-x[sel[j]]));", "score[j] = 1.0 / (1.0 + std::exp(-x[j]));"),
    ("reduce adds the ranks in descending order",
     "for (int32_t r = 0; r < n; ++r) acc = acc + bf16_to_float(partials[r * m + i]);",
     "for (int32_t r = n - 1; r >= 0; --r) acc = acc + bf16_to_float(partials[r * m + i]);"),
    ("reduce accumulates in bf16",
     "for (int32_t r = 0; r < n; ++r) acc = acc + bf16_to_float(partials[r * m + i]);",
     "for (int32_t r = 0; r < n; ++r) acc = bf16_to_float(float_to_bf16_rne(acc + bf16_to_float(partials[r * m + i])));"),
    ("reduce drops the last rank",
     "for (int32_t r = 0; r < n; ++r) acc = acc + bf16_to_float(partials[r * m + i]);",
     "for (int32_t r = 0; r + 1 < n; ++r) acc = acc + bf16_to_float(partials[r * m + i]);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_fails_a_pin(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"mutation site not unique/absent: {old!r}"
    mutated = tmp_path / "moe_oracle_mutant.cpp"
    mutated.write_text(src.replace(old, new))
    lib = oracle.compile_oracle(str(mutated), str(tmp_path / "libmutant.so"))
    tests_dir = os.path.dirname(os.path.abspath(__file__))
    code = _RUNNER.format(root=os.path.dirname(tests_dir), tests=tests_dir, lib=lib)
    # a child process: a mutant that writes out of bounds may crash, which also fails the pins
    proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    if proc.returncode == 0:
        line = [ln for ln in proc.stdout.splitlines() if ln.startswith("CAUGHT")][-1]
        caught = [c for c in line[len("CAUGHT "):].split(",") if c]
        assert caught, f"planted mistake '{name}' passed every pin"
