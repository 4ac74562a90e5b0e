"""The oracle's pins must catch plausible mistakes (no GPU).

Each case plants one mistake in a copy of oracle/gqa_oracle.cpp on the CPU,
compiles it, and runs the pin suites against the mutant through the
ORACLE_LIB override; the suites must fail.  This shows the pins tie every
step of the oracle to something outside it.
"""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gqa_oracle.cpp")

MUTANTS = {
    "strided_group_map": ("    return h / R;", "    return h % p.H_KV;"),
    "dropped_scale": ("    return p.scale * ks * acc;", "    return ks * acc;"),
    "exponent_sign": ("    for (int64_t t = 0; t < L; ++t) {\n        s[t] = std::exp(s[t] - m);",
                      "    for (int64_t t = 0; t < L; ++t) {\n        s[t] = std::exp(m - s[t]);"),
    "prefill_exponent_sign": ("            s[t] = std::exp(s[t] - m);", "            s[t] = std::exp(m - s[t]);"),
    "drops_last_token": ("    int64_t L = p.seq_lens[b];\n    std::vector<double> s(",
                         "    int64_t L = p.seq_lens[b] > 1 ? p.seq_lens[b] - 1 : p.seq_lens[b];\n    std::vector<double> s("),
    "values_from_keys": ("            out[i] += w[t] * vs * load_elem(p.v, p.kv_dtype, kv_index(p, b, t, g, i));",
                         "            out[i] += w[t] * vs * load_elem(p.k, p.kv_dtype, kv_index(p, b, t, g, i));"),
    "batch_stride": ("    return ((static_cast<int64_t>(b) * p.S_max + t) * p.H_KV + g) * p.D + i;",
                     "    return ((static_cast<int64_t>(b) * (p.S_max > 1 ? p.S_max - 1 : 1) + t) * p.H_KV + g) * p.D + i;"),
    "query_stride": ("    return (static_cast<int64_t>(b) * p.H_Q + h) * p.D + i;",
                     "    return (static_cast<int64_t>(h) * p.B + b) * p.D + i;"),
    "unnormalised_weights": ("    for (int64_t t = 0; t < L; ++t) s[t] /= sum;", "    (void)sum;"),
    "lossy_bf16": ("        uint32_t wide = static_cast<uint32_t>(bits) << 16;",
                   "        uint32_t wide = static_cast<uint32_t>(bits & 0xFFFEu) << 16;"),
    "lse_merge_shift": ("        double wj = std::exp(lse[j] - M) / total;", "        double wj = std::exp(lse[j]) / total;"),
    "partial_lse": ("    double l = m + std::log(sum);", "    double l = std::log(sum);"),
    "cache_bytes_factor": ("    return 2.0 * static_cast<double>(layers)", "    return 1.0 * static_cast<double>(layers)"),
    "rope_frequency": ("                const double theta = std::pow(base, -2.0 * i / D);",
                       "                const double theta = std::pow(base, -1.0 * i / D);"),
    "rope_rotation_sign": ("                out[row + i1] = x0 * sn + x1 * c;", "                out[row + i1] = -x0 * sn + x1 * c;"),
    "e4m3_bias": ("        mag = std::ldexp(1.0 + m / 8.0, e - 7);", "        mag = std::ldexp(1.0 + m / 8.0, e - 8);"),
    "e4m3_subnormal": ("        mag = std::ldexp(static_cast<double>(m), -9);", "        mag = std::ldexp(static_cast<double>(m), -10);"),
    "value_scale_dropped": ("    const double vs = p.v_scale ? p.v_scale[g] : 1.0;", "    const double vs = 1.0;"),
    "prefill_ignores_prefix": ("        const int64_t pos = seq_lens[b] - n_b + (i - cu_q[b]);",
                               "        const int64_t pos = i - cu_q[b];"),
    "prefill_sees_next_key": ("        const int64_t pos = seq_lens[b] - n_b + (i - cu_q[b]);",
                              "        const int64_t pos = seq_lens[b] - n_b + (i - cu_q[b]) + 1;"),
    "prefill_span_lookup": ("        while (cu_q[b + 1] <= i) ++b;", "        while (cu_q[b + 1] < i) ++b;"),
    "prefill_query_layout": ("load_elem(q, q_dtype, (i * H_Q + h) * D + e)",
                             "load_elem(q, q_dtype, (h * cu_q[B] + i) * D + e)"),
    "rope_pairing": ("                const int i1 = pairing == 0 ? 2 * i + 1 : i + half;",
                     "                const int i1 = pairing == 0 ? 2 * i + 1 : i + half - 1;"),
}

PIN_SUITES = ["tests/test_oracle_pins.py", "tests/test_oracle_rope_pins.py", "tests/test_oracle_fp8_pins.py",
              "tests/test_oracle_prefill_pins.py"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutant_src = tmp_path / "mutant.cpp"
    mutant_src.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-O1", "-std=c++17", "-shared", "-fPIC", "-pthread", str(mutant_src), "-o", str(lib)],
                   check=True)
    env = dict(os.environ, ORACLE_LIB=str(lib))
    proc = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_SUITES],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert proc.returncode != 0, f"pins did not catch mutant {name}:\n{proc.stdout[-2000:]}"
    assert "failed" in proc.stdout or "error" in proc.stdout.lower()
