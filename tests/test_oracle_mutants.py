"""The oracle's pins have teeth: each plausible mistake below, planted in a
copy of the oracle's C source (never in the oracle itself), makes at least one
of the pin tests for that part fail.  Each mutant is compiled with the
oracle's own flags into a temporary library, and the pin tests run against it
in a separate process (the oracle module pointed at the mutant)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "nvfp4_oracle.c")

CODEC = ["test_oracle_codec.py"]
FORMATS = ["test_oracle_formats.py"]
GEMM = ["test_oracle_gemm.py"]

# (mistake, text in the oracle, planted text, pin files that must catch it)
MUTANTS = [
    ("tensor scale constant", "*s_t_out = amax / 2688.0f;", "*s_t_out = amax / 2680.0f;",
     CODEC),
    ("E2M1 ties to odd",
     "double d = fabs(x - orc_e2m1_value(c));\n    if (d < bd || (d == bd && (c & 1) == 0))",
     "double d = fabs(x - orc_e2m1_value(c));\n    if (d < bd || (d == bd && (c & 1) == 1))",
     FORMATS),
    ("E4M3 ties to odd",
     "double d = fabs(x - orc_e4m3_value(c));\n    if (d < bd || (d == bd && (c & 1) == 0))",
     "double d = fabs(x - orc_e4m3_value(c));\n    if (d < bd || (d == bd && (c & 1) == 1))",
     FORMATS),
    ("E2M1 sign dropped", "return best | (signbit(y) ? 0x8 : 0);", "return best;", FORMATS),
    ("nibbles swapped", "(uint8_t)(q0 | (q1 << 4))", "(uint8_t)(q1 | (q0 << 4))", CODEC),
    ("block scale onto 8", "float six_st = 6.0f * s_t;", "float six_st = 8.0f * s_t;", CODEC),
    ("block scale evaluation order", "float six_st = 6.0f * s_t;\n  float r = amax_b / six_st;",
     "float six_st = 6.0f;\n  float r = amax_b / s_t / six_st;", CODEC),
    ("element code without s_t", "float d = s_b * s_t;\n  float y = x / d;",
     "float y = x / s_b;", CODEC),
    ("element code evaluation order", "float d = s_b * s_t;\n  float y = x / d;",
     "float d = s_b;\n  float y = x / d / s_t;", CODEC),
    ("bf16 ties away from zero",
     "return (uint16_t)((((t >> 16) & 1u) == 0) ? (t >> 16) : (u >> 16));",
     "return (uint16_t)(u >> 16);", FORMATS),
    ("dequant rounds s_b * s_t first", "float vs = v * s_b;\n  float f = vs * s_t;",
     "float bs = s_b * s_t;\n  float f = v * bs;", CODEC),
    ("scale layout rows and quadrants swapped", "(row % 32) * 16 + ((row / 32) % 4) * 4",
     "(row % 32) * 4 + ((row / 32) % 4) * 16", FORMATS),
    ("GEMM drops W's tensor scale",
     "w[k] = orc_e2m1_value(q) * orc_e4m3_value(w_sf[n * (K / 16) + k / 16]) * (double)w_st;",
     "w[k] = orc_e2m1_value(q) * orc_e4m3_value(w_sf[n * (K / 16) + k / 16]);", GEMM),
    ("GEMM reads W's nibbles swapped",
     "int q = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);\n        w[k]",
     "int q = (k % 2 == 1) ? (byte & 0xF) : (byte >> 4);\n        w[k]", GEMM),
    ("GEMM magnitude sum signed", "mag += fabs(p);", "mag += p;", GEMM),
    ("Four Over Six keeps 4 on a tie",
     "block_sq_error(xs, s4, s_t) < block_sq_error(xs, s6, s_t) ? s4 : s6",
     "block_sq_error(xs, s4, s_t) <= block_sq_error(xs, s6, s_t) ? s4 : s6",
     ["test_oracle_four_over_six.py"]),
    ("Four Over Six onto 3", "int s4 = block_scale_onto(amax_b, s_t, 4.0f);",
     "int s4 = block_scale_onto(amax_b, s_t, 3.0f);", ["test_oracle_four_over_six.py"]),
    ("KV chunk ignores the token stride", "kv + t * token_stride", "kv + t * row_elems", CODEC),
    ("GELU coefficient", "0.044715 * (v * v * v)", "0.0447 * (v * v * v)",
     ["test_oracle_gelu.py"]),
    ("GELU sign", "out[i] = 0.5 * v * (1.0 + tanh(inner));",
     "out[i] = 0.5 * v * (1.0 - tanh(inner));", ["test_oracle_gelu.py"]),
    ("attention scale dropped", "logit[j] = scale * dot;", "logit[j] = dot;",
     ["test_oracle_attention.py"]),
    ("attention reads head 0's keys",
     "const uint16_t* kj = k + (j * heads + h) * (int64_t)head_dim;",
     "const uint16_t* kj = k + (j * heads) * (int64_t)head_dim;", ["test_oracle_attention.py"]),
    ("attention magnitude sum signed", "e[d] += p * fabs(x);", "e[d] += p * x;",
     ["test_oracle_attention.py"]),
    ("tensor amax ignores the sign", "else amax = fmaxf(amax, fabsf(v));",
     "else amax = fmaxf(amax, v);", CODEC),
    ("E4M3 saturates to the NaN byte", "if (x >= 448.0) return 0x7E | (signbit(r) ? 0x80 : 0);",
     "if (x >= 448.0) return 0x7F | (signbit(r) ? 0x80 : 0);", FORMATS),
    ("exact dequant uses the next block's scale",
     "out[i * cols + j] = orc_e2m1_value(q) * orc_e4m3_value(sf[i * nkb + j / 16]) * (double)s_t;",
     "out[i * cols + j] = orc_e2m1_value(q) * orc_e4m3_value(sf[i * nkb + (j / 16 + 1) % nkb]) "
     "* (double)s_t;", GEMM),
    ("window rebuild takes the list position's tensor scale",
     "pool_sf + s * frame_sf, pool_st[s], rows,", "pool_sf + s * frame_sf, pool_st[i], rows,",
     CODEC),
]

# the same for the oracle's Python functions: (mistake, function, text, planted text, pins)
PY_MUTANTS = [
    ("sink window one frame short", "sink_window_frames", "in_window = f >= f1 - window",
     "in_window = f > f1 - window", ["test_oracle_sink_plan.py"]),
    ("shot sinks never re-bound", "sink_window_frames", "if new_shot or f0 == 0:",
     "if f0 == 0:", ["test_oracle_sink_plan.py"]),
    ("shot sinks one frame too many", "sink_window_frames",
     "in_shot = shot <= f < shot + shot_sinks", "in_shot = shot <= f <= shot + shot_sinks",
     ["test_oracle_sink_plan.py"]),
]


@pytest.mark.parametrize("mistake,old,new,files", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_planted_mistake(tmp_path, mistake, old, new, files):
    sys.path.insert(0, ROOT)
    import oracle
    src = open(SRC).read()
    assert src.count(old) == 1, f"{mistake}: the text to mutate must occur exactly once"
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(src.replace(old, new))
    mutant_so = str(tmp_path / "libmutant.so")
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", mutant_so, str(mutant_c), "-lm"], check=True)
    paths = [os.path.join(ROOT, "tests", f) for f in files]
    code = (f"import sys; sys.path.insert(0, {ROOT!r}); import oracle; "
            f"oracle._LIB = {mutant_so!r}; oracle.build = lambda force=False: oracle._LIB; "
            f"import pytest; sys.exit(pytest.main(['-q', '-x', '-p', 'no:cacheprovider', "
            f"'-m', 'not gpu', *{paths!r}]))")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 1 and " failed" in r.stdout, (
        f"{mistake}: the pins did not catch it (exit {r.returncode})\n{r.stdout[-1500:]}")


@pytest.mark.parametrize("mistake,func,old,new,files", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_pins_reject_planted_mistake_python(mistake, func, old, new, files):
    sys.path.insert(0, ROOT)
    import inspect

    import oracle
    assert inspect.getsource(getattr(oracle, func)).count(old) == 1, mistake
    paths = [os.path.join(ROOT, "tests", f) for f in files]
    code = (f"import sys, inspect; sys.path.insert(0, {ROOT!r}); import oracle; "
            f"src = inspect.getsource(oracle.{func}).replace({old!r}, {new!r}); "
            f"exec(src, oracle.__dict__); "
            f"import pytest; sys.exit(pytest.main(['-q', '-x', '-p', 'no:cacheprovider', "
            f"'-m', 'not gpu', *{paths!r}]))")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 1 and " failed" in r.stdout, (
        f"{mistake}: the pins did not catch it (exit {r.returncode})\n{r.stdout[-1500:]}")
