"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a private copy of ``oracle/oracle.c``
(a dropped term, a wrong sign, index or operand, an off-by-one), builds it,
and runs the pin suite ``test_oracle.py`` against that copy in a child
process.  The pins are only worth something if every such mutant fails them.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, text in oracle.c, replacement, expected number of occurrences)
MUTANTS = [
    ("offsets_start", "cu[0] = 0;\n    for (int b = 0; b < batch; ++b) cu[b + 1]",
     "cu[0] = lengths[0];\n    for (int b = 0; b < batch; ++b) cu[b + 1]", 1),
    ("offsets_bound", "lengths[b] > pad_len) ok = 0", "lengths[b] > pad_len + 1) ok = 0", 1),
    ("remove_stride", "src[((int64_t)b * pad_len + s) * row_bytes + k]",
     "src[((int64_t)b * len + s) * row_bytes + k]", 1),
    ("rebuild_pads_kept", "? src[((int64_t)cu[b] + s) * row_bytes + k] : 0;",
     "? src[((int64_t)cu[b] + s) * row_bytes + k] : dst[((int64_t)b * pad_len + s) * row_bytes + k];", 1),
    ("trebuild_block_order", "int64_t i = ((int64_t)cu[b] + s) * row + ((int64_t)c * n_heads + h) * head_bytes;",
     "int64_t i = ((int64_t)cu[b] + s) * row + ((int64_t)h * parts + c) * head_bytes;", 1),
    ("trebuild_head_seq_swapped", "int64_t o = ((((int64_t)c * batch + b) * n_heads + h) * pad_len + s) * head_bytes;",
     "int64_t o = ((((int64_t)c * batch + b) * pad_len + s) * n_heads + h) * head_bytes;", 1),
    ("trebuild_pads_kept", "dst[o + k] = s < len ? src[i + k] : 0;", "if (s < len) dst[o + k] = src[i + k];", 1),
    ("tremove_batch_part_swapped", "int64_t i = ((((int64_t)c * batch + b) * n_heads + h) * pad_len + s) * head_bytes;",
     "int64_t i = ((((int64_t)b * parts + c) * n_heads + h) * pad_len + s) * head_bytes;", 1),
    ("decode_f16_bias", "ldexp((double)(1024 + m), e - 25)", "ldexp((double)(1024 + m), e - 24)", 1),
    ("ln_unbiased_var", "var /= hidden;", "var /= (hidden - 1);", 1),
    ("ln_no_eps", "1.0 / sqrt(var + eps)", "1.0 / sqrt(var)", 1),
    ("ln_gamma_beta_swapped", "* inv * elem(g, wdtype, k) + elem(beta, wdtype, k)",
     "* inv * elem(beta, wdtype, k) + elem(g, wdtype, k)", 1),
    ("linear_transposed", "elem(W, wdtype, (int64_t)n * in_dim + k)",
     "elem(W, wdtype, (int64_t)k * out_dim + n)", 1),
    ("linear_no_bias", "y[t * out_dim + n] = acc + bn;", "y[t * out_dim + n] = acc;", 1),
    ("gelu_constant", "(v + 0.044715 * v * v * v)", "(v + 0.04715 * v * v * v)", 1),
    ("attn_strict_mask", "t <= s; ++t)", "t < s; ++t)", 3),
    ("attn_no_scale", "p[t] = dot * scale;", "p[t] = dot;", 1),
    ("attn_softmax_sign", "exp(p[t] - m)", "exp(m - p[t])", 1),
    ("attn_keys_are_queries", "qkv + t * ld + hidden + (int64_t)j * d", "qkv + t * ld + (int64_t)j * d", 1),
    ("attn_v_head0", "2 * (int64_t)hidden + (int64_t)j * d + e]", "2 * (int64_t)hidden + e]", 1),
    ("layer_no_attn_residual", "x1[i] += x[i];", "x1[i] += 0.0 * x[i];", 1),
    ("layer_wrong_ffn_residual", "y[i] += x1[i];", "y[i] += x[i];", 1),
    ("layer_pads_not_zeroed", "yb[i] = 0.0;", "yb[i] = yb[i];", 1),
]


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new, count):
    src = open(SRC).read()
    assert src.count(old) == count, f"mutation site for {name} not found as expected"
    mutant_c = tmp_path / "oracle_mutant.c"
    mutant_c.write_text(src.replace(old, new))
    mutant_so = tmp_path / "liboracle_mutant.so"
    sys.path.insert(0, ROOT)
    import oracle
    oracle.compile_to(str(mutant_c), str(mutant_so))
    env = dict(os.environ, ORACLE_LIB_OVERRIDE=str(mutant_so), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
