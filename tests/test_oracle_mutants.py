"""Sensitivity of the oracle's pins: each plausible mistake below is planted in
a copy of the C oracle (never in the repository's own file), and the pin
suite (tests/test_oracle_pins.py, run against that copy in a subprocess) must
fail for every one of them.  A mistake no pin catches would be a part of the
oracle whose correctness rests on nothing but itself.

The mistakes are the kinds a restatement of the format and the method could
plausibly contain: a wrong table entry, bias or subnormal exponent; a tie
rule to the odd code or toward zero; a lost sign of zero; a reciprocal where
the method divides; a different rounding order; swapped nibbles; a transposed
or mis-strided scale layout; a dropped term of the dot product; gate and up
exchanged; a gate with a parameter missing or a sign flipped."""
import os
import re
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "nvfp4_oracle.c")
PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")

# (name, text in the oracle, replacement, which occurrence (0 = first))
MUTANTS = [
    # formats
    ("e2m1 largest value 5", "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}",
     "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0}", 0),
    ("e2m1 ties to odd", "(dist == best_d && (c & 1) == 0 && (best & 1) == 1)",
     "(dist == best_d && (c & 1) == 1 && (best & 1) == 0)", 0),
    ("e2m1 ties toward zero", "(dist < best_d || (dist == best_d && (c & 1) == 0 && (best & 1) == 1))",
     "(dist < best_d)", 0),
    ("e2m1 zero loses its sign", "return signbit(t) ? (best | 8) : best;",
     "return (signbit(t) && best) ? (best | 8) : best;", 0),
    ("e2m1 no saturation of inf", "if (a > 6.0) a = 6.0;", "", 0),
    ("e4m3 bias 8", "ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)", 0),
    ("e4m3 subnormal step 2^-10", "ldexp((double)m, -9)", "ldexp((double)m, -10)", 0),
    ("e4m3 ties to odd", "(dist == best_d && (c & 1) == 0 && (best & 1) == 1)",
     "(dist == best_d && (c & 1) == 1 && (best & 1) == 0)", 1),
    ("bf16 ties away from zero", "nearbyint(ldexp(a, -ulp_exp))", "round(ldexp(a, -ulp_exp))", 0),
    ("bf16 no subnormals", "if (ulp_exp < -133) ulp_exp = -133;", "if (ulp_exp < -126) ulp_exp = -126;", 0),
    # global scale
    ("global scale without the 6", "float g = amax / 2688.0f;", "float g = amax / 448.0f;", 0),
    ("global scale by reciprocal", "float g = amax / 2688.0f;", "float g = amax * (1.0f / 2688.0f);", 0),
    ("zero tensor scale 0", "if (amax == 0.0f) return 1.0f;", "if (amax == 0.0f) return 0.0f;", 0),
    # block scales and codes
    ("block scale in one division", "float sf = ab / 6.0f;\n            sf = sf / g;",
     "float sf = ab / (6.0f * g);", 0),
    ("block absmax over 8 elements", "for (int i = 0; i < 16; ++i) {\n                float v",
     "for (int i = 0; i < 8; ++i) {\n                float v", 0),
    ("element scale before rounding", "float d = (float)oracle_e4m3_value(s8) * g;", "float d = sf * g;", 0),
    ("element by reciprocal", "float t0 = bf16_to_float(blk[i]) / d;",
     "float t0 = bf16_to_float(blk[i]) * (1.0f / d);", 0),
    ("zero block divided anyway", "if (d != 0.0f) {", "if (1) {", 0),
    ("nibbles swapped", "(uint8_t)(c0 | (c1 << 4))", "(uint8_t)(c1 | (c0 << 4))", 0),
    # scale layout
    ("sf atom rows transposed", "(r % 32) * 16 + ((r / 32) % 4) * 4", "(r % 32) * 4 + ((r / 32) % 4) * 128", 0),
    ("sf atoms mis-strided", "(r / 128) * (sfcols_padded / 4) + (c / 4)", "(r / 128) * sfcols_padded + (c / 4)", 0),
    # dequantization and GEMM
    ("dequant nibbles swapped", "(k % 2 == 0) ? (byte & 15) : (byte >> 4)",
     "(k % 2 == 0) ? (byte >> 4) : (byte & 15)", 0),
    ("dequant scale per 32", "sf_linear[r * (cols / 16) + k / 16]", "sf_linear[r * (cols / 16) + k / 32]", 0),
    ("gemm operand reversed along k", "acc += a[k] * w[k];", "acc += a[k] * w[K - 1 - k];", 0),
    ("gemm last k dropped", "for (int64_t k = 0; k < K; ++k) acc += a[k] * w[k];",
     "for (int64_t k = 0; k + 1 < K; ++k) acc += a[k] * w[k];", 0),
    # MLP intermediate
    ("silu of the wrong sign", "double s = g / (1.0 + exp(-g));", "double s = g / (1.0 + exp(g));", 0),
    ("gate and up exchanged", "double g = (double)bf16_to_float(gu[r * ld + c]);\n"
     "            double u = (double)bf16_to_float(gu[r * ld + f + c]);",
     "double u = (double)bf16_to_float(gu[r * ld + c]);\n"
     "            double g = (double)bf16_to_float(gu[r * ld + f + c]);", 0),
    ("fused silu without up", "h[r * f + c] = oracle_bf16_from_double(g / (1.0 + exp(-g)) * u);",
     "h[r * f + c] = oracle_bf16_from_double(g / (1.0 + exp(-g)));", 0),
    # harmonisation
    ("common scale the smallest", "if (seg_g[i] > gc) gc = seg_g[i];", "if (seg_g[i] < gc) gc = seg_g[i];", 0),
    ("ratio inverted", "const float ratio = seg_g[i] / gc;", "const float ratio = gc / seg_g[i];", 0),
    # KV cache
    ("kv scale from 240", "return amax > 0.0f ? amax / 448.0f : 1.0f;",
     "return amax > 0.0f ? amax / 240.0f : 1.0f;", 0),
    ("kv zero loses its sign", "if (signbit(t)) code |= 0x80;", "if (t < 0.0f) code |= 0x80;", 0),
    ("kv by reciprocal", "const float t = bf16_to_float(x[r * ld + c]) / s;",
     "const float t = bf16_to_float(x[r * ld + c]) * (1.0f / s);", 0),
    # gates
    ("decay without exp(A_log)", "o = -exp((double)a_log[c]) * sp;", "o = -(double)a_log[c] * sp;", 0),
    ("decay without dt_bias", "const double z = v + (double)dt_bias[c];", "const double z = v;", 0),
    ("softplus missing z", "z > 0.0 ? z + log1p(exp(-z)) : log1p(exp(z))",
     "z > 0.0 ? log1p(exp(-z)) : log1p(exp(z))", 0),
    ("sigmoid of -y", "o = 1.0 / (1.0 + exp(-v));", "o = 1.0 / (1.0 + exp(v));", 0),
]


# the same for the oracle's Python wrapper (argument marshalling and the
# per-column alpha); every one stays inside the buffers it touches
PY_MUTANTS = [
    ("alpha without the weight scale", "alpha[int(off):int(off) + int(size)] = float(np.float32(g_a)) * float(np.float32(gw))",
     "alpha[int(off):int(off) + int(size)] = float(np.float32(g_a))"),
    ("alpha with the weight scale squared", "alpha[int(off):int(off) + int(size)] = float(np.float32(g_a)) * float(np.float32(gw))",
     "alpha[int(off):int(off) + int(size)] = float(np.float32(gw)) * float(np.float32(gw))"),
    ("harmonisation rows from the offsets", "seg_rows = np.array([int(s[1]) for s in segments], np.int64)",
     "seg_rows = np.array([int(s[0]) for s in segments], np.int64)"),
    ("SiLU row stride f", "_L().oracle_silu_mul(_ptr(gu), rows, f, two_f, _ptr(h))",
     "_L().oracle_silu_mul(_ptr(gu), rows, f, f, _ptr(h))"),
    ("gate parameters swapped", "_ptr(y), rows, ncols, ncols, _ptr(al), _ptr(db), int(kind)",
     "_ptr(y), rows, ncols, ncols, _ptr(db), _ptr(al), int(kind)"),
    ("quantizer row stride halved", "_L().oracle_quantize(_ptr(x), rows, cols, cols, ctypes.c_float(float(g)),",
     "_L().oracle_quantize(_ptr(x), rows, cols, cols // 2, ctypes.c_float(float(g)),"),
]


def _apply(src: str, old: str, new: str, nth: int) -> str:
    """src with the nth occurrence of `old` in code (comments skipped, so a
    mistake is never planted where the compiler ignores it) replaced."""
    spans = [m.span() for m in re.finditer(r"/\*.*?\*/|//[^\n]*", src, flags=re.S)]
    in_comment = lambda i: any(a <= i < b for a, b in spans)
    hits = [m.start() for m in re.finditer(re.escape(old), src) if not in_comment(m.start())]
    if len(hits) <= nth:
        return ""
    pos = hits[nth]
    return src[:pos] + new + src[pos + len(old):]


def _tree(base: str, c_source: str, py_source: str) -> str:
    """A minimal copy in which `import oracle` and the pins resolve to the
    planted oracle: oracle/ (wrapper + C source), tests/ (conftest, pins,
    golden files)."""
    os.makedirs(os.path.join(base, "oracle"))
    with open(os.path.join(base, "oracle", "__init__.py"), "w") as f:
        f.write(py_source)
    with open(os.path.join(base, "oracle", "nvfp4_oracle.c"), "w") as f:
        f.write(c_source)
    os.makedirs(os.path.join(base, "tests"))
    for name in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(base, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(base, "tests", "golden"))
    return base


def _run_pins(base: str) -> subprocess.CompletedProcess:
    env = dict(os.environ, OMP_NUM_THREADS="1", PYTHONDONTWRITEBYTECODE="1")
    return subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
         os.path.join(base, "tests", "test_oracle_pins.py")],
        cwd=base, env=env, capture_output=True, text=True, timeout=600)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc for the C oracle")
def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = open(SRC).read()
    py = open(PY_SRC).read()
    planted = []
    for i, (name, old, new, nth) in enumerate(MUTANTS):
        mutated = _apply(src, old, new, nth)
        assert mutated, f"mutant '{name}' no longer applies to the oracle source"
        planted.append((name, _tree(str(tmp_path / f"m{i:02d}"), mutated, py)))
    for i, (name, old, new) in enumerate(PY_MUTANTS):
        assert py.count(old) == 1, f"mutant '{name}' no longer applies to the oracle wrapper"
        planted.append((name, _tree(str(tmp_path / f"p{i:02d}"), src, py.replace(old, new))))
    control = _tree(str(tmp_path / "control"), src, py)

    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as pool:
        ctrl = pool.submit(_run_pins, control)
        results = [(name, pool.submit(_run_pins, base)) for name, base in planted]
        c = ctrl.result()
        outcome = [(name, fut.result()) for name, fut in results]
    # the copy itself is sound: unplanted, every pin passes there
    assert c.returncode == 0, c.stdout[-2000:] + c.stderr[-2000:]
    survivors = [name for name, r in outcome if r.returncode == 0]
    assert not survivors, f"no pin fails for: {survivors}"
    for name, r in outcome:
        # a failing pin, not a crash of the harness (exit 1 = tests failed)
        assert r.returncode == 1, f"{name}: exit {r.returncode}\n{r.stdout[-1500:]}{r.stderr[-1500:]}"
