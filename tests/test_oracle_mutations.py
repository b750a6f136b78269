"""The oracle's pins catch plausible mistakes: each test copies nvfp4_oracle.c,
plants one mistake in the copy (a wrong sign, operand, index or pairing), builds
it with the oracle's own compiler flags into a temporary library, and checks that
at least one pin fails on it, while the unchanged copy passes every pin.  The
oracle package itself is never modified.

Covered: the keys' rotary embedding ahead of the quantize (reading R24, the fused
RoPE of the anzhuoshouzhuan.com LongLive 2.0 article, section "NVFP4 量化"), with
the pins of test_oracle_rope.py restated against a library handle; and the rest of
the oracle (the format and scaling rules R3-R10 of "LongLive-2.0：用 NVFP4 并行底座做
长视频生成", section "NVFP4 量化格式", the GEMM and its epilogue, R19, R20, R22),
each mutant run against every other oracle pin file in a child process; and the
numpy attention and chunk-set functions (section 二's sink + window set), each
mutant compiled from the function's source and patched in for the test."""
import ctypes
import inspect
import os
import shutil
import subprocess
import sys
import textwrap

import numpy as np
import pytest

import oracle

from . import test_oracle_attention as _ta
from .test_oracle_rope import U, _f32, _nonzero_chunk, _quarter_turned_bits, _turn

SRC = os.path.join(os.path.dirname(oracle.__file__), "nvfp4_oracle.c")


def _build(tmp_path, replacements):
    src = open(SRC).read()
    for old, new in replacements:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    c = tmp_path / "mut.c"
    so = tmp_path / "libmut.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
                           "-shared", "-fvisibility=hidden", str(c), "-o", str(so), "-lm"])
    L = ctypes.CDLL(str(so))
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    L.orc_rope.argtypes = [vp, i64, i64, i64, vp, vp, vp]
    L.orc_kv_append_rope.argtypes = [vp, i64, i64, i64, vp, vp, ctypes.c_int, vp, vp, vp, vp, ctypes.c_int]
    L.orc_kv_append_rope.restype = ctypes.c_int
    return L


def _p(a):
    return None if a is None else a.ctypes.data


def _rope(L, x, cs, sn):
    T, H, d = x.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    cs = np.ascontiguousarray(cs, dtype=np.float32)
    sn = np.ascontiguousarray(sn, dtype=np.float32)
    y = np.zeros((T, H, d), np.float32)
    L.orc_rope(_p(x), T, H, d, _p(cs), _p(sn), _p(y))
    return y


def _append(L, x, cs, sn, smooth):
    T, H, d = x.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    cs = np.ascontiguousarray(cs, dtype=np.float32)
    sn = np.ascontiguousarray(sn, dtype=np.float32)
    codes = np.zeros((T * H, d // 2), np.uint8)
    scales = np.zeros((T * H, d // 16), np.uint8)
    a = np.zeros(1, np.float32)
    mean = np.zeros(H * d, np.float32) if smooth else None
    assert L.orc_kv_append_rope(_p(x), T, H, d, _p(cs), _p(sn), 0, _p(codes), _p(scales), _p(a), _p(mean), 0) == 0
    return codes, scales, np.float32(a[0]), mean


def _failed_pins(L):
    """Names of the R24 pins that the library fails."""
    failed = []
    # complex product within three roundings (random angles)
    T, H, d = 24, 3, 32
    x = _nonzero_chunk(T, H, d, seed=1)
    g = np.random.default_rng(2)
    ang = g.uniform(-np.pi, np.pi, size=(T, d // 2))
    cs, sn = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    y = _rope(L, x, cs, sn).astype(np.float64)
    xf = _f32(x).astype(np.float64).reshape(T, H, d // 2, 2)
    z = (xf[..., 0] + 1j * xf[..., 1]) * (cs.astype(np.float64) + 1j * sn.astype(np.float64))[:, None, :]
    ref = np.stack([z.real, z.imag], axis=-1).reshape(T, H, d)
    bound = np.repeat(2.02 * U * (np.abs(xf[..., 0]) + np.abs(xf[..., 1])), 2, axis=-1).reshape(T, H, d)
    if not np.all(np.abs(y - ref) <= bound):
        failed.append("complex product")
    # the exact quarter turn
    T, H, d = 8, 2, 16
    x = _nonzero_chunk(T, H, d, seed=3)
    xf = _f32(x)
    q = _rope(L, x, *_turn(T, d, 0.0, 1.0))
    if not (np.array_equal(q[..., 0::2], -xf[..., 1::2]) and np.array_equal(q[..., 1::2], xf[..., 0::2])):
        failed.append("quarter turn")
    # one pair of one token, in every head
    T, H, d = 9, 4, 16
    x = _nonzero_chunk(T, H, d, seed=4)
    cs, sn = _turn(T, d, 1.0, 0.0)
    cs[5, 3], sn[5, 3] = 0.0, 1.0
    y = _rope(L, x, cs, sn)
    changed = np.argwhere(y != _f32(x))
    if {(int(t), int(j)) for t, _, j in changed} != {(5, 6), (5, 7)} or len(changed) != 2 * H:
        failed.append("one pair")
    # the appends against the pinned plain and smoothed appends of the turned keys
    T, H, d = 70, 2, 16
    x = _nonzero_chunk(T, H, d, seed=6)
    got = _append(L, x, *_turn(T, d, 0.0, 1.0), smooth=False)
    ref = oracle.kv_append(_quarter_turned_bits(x))
    if not (np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1]) and got[2] == ref[2]):
        failed.append("append")
    got = _append(L, x, *_turn(T, d, 0.0, 1.0), smooth=True)
    ref = oracle.kv_append_smooth(_quarter_turned_bits(x))
    if not all(np.array_equal(a, b) for a, b in zip(got, ref)):
        failed.append("smoothed append")
    return failed


MUTATIONS = {
    "difference turned into a sum": [("y[base + 2 * p] = a - b;", "y[base + 2 * p] = a + b;")],
    "operands of the second output swapped": [
        ("const float a = x0 * c, b = x1 * s, e = x0 * s, f = x1 * c;",
         "const float a = x0 * c, b = x1 * s, e = x1 * s, f = x0 * c;")],
    "sine of the neighbouring pair": [
        ("const float c = cs[t * (d / 2) + p], s = sn[t * (d / 2) + p];",
         "const float c = cs[t * (d / 2) + p], s = sn[t * (d / 2) + (p ^ 1)];")],
    "table row by head instead of token": [
        ("const float c = cs[t * (d / 2) + p], s = sn[t * (d / 2) + p];",
         "const float c = cs[h * (d / 2) + p], s = sn[h * (d / 2) + p];")],
    "rotate-half pairing (p, p + d/2)": [
        ("const float x0 = orc_bf16_to_f32(x[base + 2 * p]);\n"
         "                const float x1 = orc_bf16_to_f32(x[base + 2 * p + 1]);",
         "const float x0 = orc_bf16_to_f32(x[base + p]);\n"
         "                const float x1 = orc_bf16_to_f32(x[base + p + d / 2]);")],
    "means of the unturned keys": [("if (!mean_given) orc_channel_mean_f32(y, T, C, mean);",
                                    "if (!mean_given) orc_channel_mean(x, T, C, mean);")],
}


@pytest.fixture(scope="module")
def gcc():
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")


def test_unchanged_copy_passes_every_pin(gcc, tmp_path):
    assert _failed_pins(_build(tmp_path, [])) == []


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_fails_a_pin(gcc, tmp_path, name):
    failed = _failed_pins(_build(tmp_path, MUTATIONS[name]))
    assert failed, f"no pin caught: {name}"


# ---------------------------------------------------------------------------
# The whole pin suite against planted mistakes in the rest of the oracle: each
# mutant runs every other test_oracle_*.py file in a child process (the oracle
# package builds the modified copy there) and at least one pin must fail.
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = sorted(os.path.join(ROOT, "tests", f) for f in os.listdir(os.path.join(ROOT, "tests"))
                   if f.startswith("test_oracle_") and f.endswith(".py") and f != "test_oracle_mutations.py")

ORACLE_MUTATIONS = {
    "R3/R6 ties away from even": [("return (i % 2 == 0) ? i : i + 1;", "return i + 1;")],
    "R7 sign from a comparison, not the sign bit": [
        ("return mag | (signbit(y) ? 8u : 0u);", "return mag | ((y < 0.0f) ? 8u : 0u);")],
    "R3 block scale without the 6": [("    float d = target * a32;\n", "    float d = a32;\n")],
    "R4 zero scale not flushed": [("if (s != 0.0f) { /* R4 */", "if (1) { /* R4 */")],
    "R5 division instead of the reciprocal": [("float y = xb[i] * inv;", "float y = xb[i] / denom;")],
    "R9 swizzle row and group offsets swapped": [
        ("(rr % 32) * 16 + (rr / 32) * 4 + cc", "(rr % 32) * 4 + (rr / 32) * 16 + cc")],
    "GEMM sum drops the last k": [("for (int64_t k = 0; k < K; k++) acc += ad[k] * br[k];",
                                   "for (int64_t k = 0; k + 1 < K; k++) acc += ad[k] * br[k];")],
    "GEMM without the tensor scales": [("double v = alpha * acc;", "double v = acc;")],
    "modulate without the 1 +": [("v = v * (1.0 + sc) + sh;", "v = v * sc + sh;")],
    "R10 one rounding instead of two": [
        ("            float v = qs * alpha;\n            out[r * cols + c] = orc_f32_to_bf16(v);",
         "            out[r * cols + c] = orc_f64_to_bf16((double)qs * (double)alpha);")],
    "R19 eps outside the root": [("stats[2 * r + 1] = (float)(1.0 / sqrt(var + (double)eps));",
                                  "stats[2 * r + 1] = (float)(1.0 / (sqrt(var) + (double)eps));")],
    "R19 one 16-element block in 32 left out of the row sum": [
        ("for (int64_t c = 0; c < cols; c++) s1 += (double)orc_bf16_to_f32(x[r * ld + c]);",
         "for (int64_t c = 0; c < cols; c++) if ((c / 16) % 32 != 31) s1 += (double)orc_bf16_to_f32(x[r * ld + c]);")],
    "R19 squares taken about 0 instead of the mean": [
        ("const double d = (double)orc_bf16_to_f32(x[r * ld + c]) - mu;",
         "const double d = (double)orc_bf16_to_f32(x[r * ld + c]);")],
    "R20 first 32 tokens dropped": [
        ("for (int64_t t = 0; t < T; t++) s += (double)orc_bf16_to_f32(x[t * C + c]);",
         "for (int64_t t = 32; t < T; t++) s += (double)orc_bf16_to_f32(x[t * C + c]);")],
    "R20 one token in 32 left out of the sum": [
        ("for (int64_t t = 0; t < T; t++) s += (double)orc_bf16_to_f32(x[t * C + c]);",
         "for (int64_t t = 0; t < T; t++) if (t % 32 != 31) s += (double)orc_bf16_to_f32(x[t * C + c]);")],
    "R22 signs inverted": [("v[i] = sign[i] < 0 ? -v[i] : v[i];", "v[i] = sign[i] > 0 ? -v[i] : v[i];")],
    "R22 normalised by 1/2": [("for (int i = 0; i < 16; i++) v[i] = v[i] * 0.25f;",
                               "for (int i = 0; i < 16; i++) v[i] = v[i] * 0.5f;")],
    "R1 tensor scale amax / 448": [
        ("        a32 = amax / 2688.0f; /* R1 */\n        *alpha = a32;\n    } else {\n        a32 = *alpha;\n"
         "    }\n    const int64_t nb = cols / 16;",
         "        a32 = amax / 448.0f; /* R1 */\n        *alpha = a32;\n    } else {\n        a32 = *alpha;\n"
         "    }\n    const int64_t nb = cols / 16;")],
    "R8 nibbles swapped": [("(uint8_t)(q[2 * i] | (q[2 * i + 1] << 4)); /* R8 */",
                            "(uint8_t)((q[2 * i] << 4) | q[2 * i + 1]); /* R8 */")],
    "R11 GELU cube dropped to a square": [("0.044715 * y * y * y", "0.044715 * y * y")],
    "R18 a tie takes the target-4 candidate": [
        ("block_sq_error(xb, sc4, q4, a32) < block_sq_error(xb, sc, q, a32)",
         "block_sq_error(xb, sc4, q4, a32) <= block_sq_error(xb, sc, q, a32)")],
    "R19 sample variance (n - 1)": [("const double var = s2 / (double)cols;",
                                     "const double var = s2 / (double)(cols - 1);")],
    "R21 transposed operand not transposed": [
        ("(uint8_t)(q[2 * j][i] | (q[2 * j + 1][i] << 4));", "(uint8_t)(q[i][2 * j] | (q[i][2 * j + 1] << 4));")],
    "R20 mean subtracted again in the dequant": [("float y = v + mean[(r % H) * d + c];",
                                                  "float y = v - mean[(r % H) * d + c];")],
    "R20 mean indexed by token instead of head": [("float y = v + mean[(r % H) * d + c];",
                                                   "float y = v + mean[(r / H % H) * d + c];")],
    "R21 2D block max over its first row only": [
        ("            for (int i = 0; i < 16; i++)\n                for (int j = 0; j < 16; j++) {",
         "            for (int i = 0; i < 1; i++)\n                for (int j = 0; j < 16; j++) {")],
}


def _run_pins(tmp_path, replacements, stop_at_first=True):
    src = open(SRC).read()
    for old, new in replacements:
        assert src.count(old) == 1, old
        src = src.replace(old, new)
    c = tmp_path / "oracle_mut.c"
    c.write_text(src)
    env = dict(os.environ, NVFP4_ORACLE_SRC=str(c), NVFP4_ORACLE_LIB=str(tmp_path / "liboracle_mut.so"))
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "not gpu", "-p", "no:cacheprovider"]
    if stop_at_first:
        cmd.append("-x")
    r = subprocess.run(cmd + PIN_FILES, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-3000:]


def test_whole_pin_suite_passes_on_an_unchanged_copy(gcc, tmp_path):
    rc, out = _run_pins(tmp_path, [], stop_at_first=False)
    assert rc == 0, out


@pytest.mark.parametrize("name", list(ORACLE_MUTATIONS))
def test_planted_mistake_in_the_oracle_fails_a_pin(gcc, tmp_path, name):
    rc, out = _run_pins(tmp_path, ORACLE_MUTATIONS[name])
    # tests ran and at least one failed (exit status 1), or a pin's input crashed the
    # modified copy (killed by a signal); not a build, collection or usage error
    assert (rc == 1 and " failed" in out) or rc < 0, f"no pin caught: {name} (exit {rc})\n{out}"


# ---------------------------------------------------------------------------
# The attention part of the oracle is Python: a mutant is the function's source
# with one mistake, compiled into the oracle module's namespace and patched in
# for the duration of the test; the attention pins are then called directly.
PY_MUTATIONS = {
    "softmax over the queries": ("attention", "p /= p.sum(axis=1, keepdims=True)",
                                 "p /= p.sum(axis=0, keepdims=True)"),
    "scores without the scale": ("attention", "s = (qf[:, h, :] @ kf[:, h, :].T) * scale",
                                 "s = (qf[:, h, :] @ kf[:, h, :].T)"),
    "keys in place of values": ("attention", "out[:, h, :] = p @ vf[:, h, :]", "out[:, h, :] = p @ kf[:, h, :]"),
    "window one chunk short": ("attention_chunks", "set(range(t - window, t))", "set(range(t - window + 1, t))"),
    "the current chunk included": ("attention_chunks", "if 0 <= c < t)", "if 0 <= c <= t)"),
    "shot sink from the first chunk": ("attention_chunks", "set(range(shot_start, shot_start + sink_shot))",
                                       "set(range(0, sink_shot))"),
}


def _py_mutant(fn_name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(oracle, fn_name)))
    assert src.count(old) == 1, old
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), f"<planted {fn_name}>", "exec"), ns)
    return ns[fn_name]


def _attention_pins():
    yield _ta.test_attention_matches_torch_sdpa_in_float64
    yield _ta.test_equal_keys_average_the_values
    yield _ta.test_a_dominant_key_selects_its_value
    for args, want in _ta._golden():
        yield lambda args=args, want=want: _ta.test_attention_chunks_hand_worked(args, want)


def _failing_attention_pins():
    failed = 0
    for pin in _attention_pins():
        try:
            pin()
        except AssertionError:
            failed += 1
    return failed


def test_attention_pins_pass_on_the_unchanged_functions():
    assert _failing_attention_pins() == 0


@pytest.mark.parametrize("name", list(PY_MUTATIONS))
def test_planted_mistake_in_the_attention_oracle_fails_a_pin(monkeypatch, name):
    fn_name, old, new = PY_MUTATIONS[name]
    monkeypatch.setattr(oracle, fn_name, _py_mutant(fn_name, old, new))
    assert _failing_attention_pins() > 0, f"no pin caught: {name}"
