"""Plant mistakes in copies of oracle.c and check that the pins catch every one.

Each mutant is a plausible slip (a dropped term, a wrong sign, index or
operand).  All mutants keep every memory access inside its buffer, so running
them on the CPU is safe.
"""
import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = [
    ("exponent sign", "exp(x[t] - mu)", "exp(mu - x[t])"),
    ("no max subtraction", "exp(x[t] - mu)", "exp(x[t])"),
    ("min instead of max", "if (x[t] > mu)", "if (x[t] < mu)"),
    ("no normalisation", "out[d] /= z;", "out[d] /= 1.0;"),
    ("normalise by count", "z += w;", "z += 1.0;"),
    ("scale dropped", "x[t] = scale * dot;", "x[t] = dot;"),
    ("head grouping j mod Hkv", "const int h = j / group;", "const int h = j % num_kv_heads;"),
    ("q row of the kv head", "q + ((int64_t)s * num_q_heads + j) * head_dim",
     "q + ((int64_t)s * num_q_heads + j / (num_q_heads / num_kv_heads)) * head_dim"),
    ("values read from K", "pool_value(V, vrow + d, h)", "pool_value(K, vrow + d, h)"),
    ("block table ignored", "table[t / block_size]", "(t / block_size)"),
    ("offset off by one", "pool_row(p, t % block_size", "pool_row(p, (t + 1) % block_size"),
    ("last token dropped from PV", "for (int t = 0; t < context_len; ++t) {\n        double w",
     "for (int t = 0; t + 1 < context_len; ++t) {\n        double w"),
    ("pool layout transposed", "((p * block_size + off) * num_kv_heads + h)", "((p * num_kv_heads + h) * block_size + off)"),
    ("append ignores head", "int64_t src = (i * num_kv_heads + h) * (int64_t)head_dim;",
     "int64_t src = (i * num_kv_heads) * (int64_t)head_dim;"),
    ("append crosses k and v", "k_cache[dst + d] = k[src + d];", "k_cache[dst + d] = v[src + d];"),
    ("append offset 0", "int off = (int)(slot % block_size);", "int off = 0;"),
    ("e4m3 exponent bias", "ldexp((double)(8 + m), e - 10)", "ldexp((double)(8 + m), e - 9)"),
    ("e4m3 subnormal step", "ldexp((double)m, -9)", "ldexp((double)m, -8)"),
    ("e4m3 encode truncates", "double m = nearbyint((a / ldexp(1.0, E) - 1.0) * 8.0);",
     "double m = floor((a / ldexp(1.0, E) - 1.0) * 8.0);"),
    ("e4m3 no saturation", "if (a >= 448.0)", "if (a >= 480.0)"),
    ("fp8 scale of head 0", "* (double)P->scale[h];", "* (double)P->scale[0];"),
    ("fp8 append uses the K scale for V", "/ v_scale[h];", "/ k_scale[h];"),
    ("prefill sees one token too few", "int p = context_lens[s] - n + i;", "int p = context_lens[s] - n + i - 1;"),
    ("prefill sees the whole context", "int p = context_lens[s] - n + i;", "int p = context_lens[s] - 1;"),
    ("prefill reads the chunk's first query", "q + (row * num_q_heads + j) * (int64_t)head_dim",
     "q + ((int64_t)query_start[s] * num_q_heads + j) * (int64_t)head_dim"),
    ("prefill output rows transposed", "mine = decode_one(out + (row * num_q_heads + j) * head_dim, x,",
     "mine = decode_one(out + ((int64_t)j * num_tokens + row) * head_dim, x,"),
    ("prefill chunk rows reversed", "int64_t row = (int64_t)query_start[s] + i;",
     "int64_t row = (int64_t)query_start[s + 1] - 1 - i;"),
    ("prefill reads sequence 0's table", "p + 1, s, j, num_q_heads", "p + 1, 0, j, num_q_heads"),
]


@pytest.mark.parametrize("label,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(label, old, new, tmp_path):
    src = oracle.source()
    assert old in src, f"mutation site for '{label}' not found"
    lib = oracle.build_variant(src.replace(old, new), str(tmp_path))
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib=lib)
        except (AssertionError, oracle.OracleError) as e:
            caught.append(pin.__name__)
            break
    assert caught, f"no pin caught the mutant '{label}'"
