"""Mutation check of the oracle's pins.

Plausible mistakes (a dropped term, a wrong sign or index, a shifted operand,
an off-by-one in a bound) are planted, one at a time, in a copy of oracle.c
built on the CPU; the pin suite in test_oracle_pins.py must fail for every
one of them.  Nothing here touches the CUDA path.
"""
import inspect
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as obuild

import test_oracle_pins as pins

# (name, text in oracle.c, replacement)
MUTANTS = [
    ("e4m3 exponent bias", "ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    ("e4m3 subnormal quantum", "v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    ("e4m3 encode ties away", "return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f + 1.0;"),
    ("bf16 truncation", "u += 0x7FFFu + lsb;", "u += 0u * lsb;"),
    ("scale tile index", "row + SMO_SCALE_OFF + 4 * (i / SMO_TILE)", "row + SMO_SCALE_OFF + 4 * (i / 256)"),
    ("scale divisor", "scale = amax / 448.0f;", "scale = amax / 480.0f;"),
    ("dequant product not rounded to bf16",
     "k[i] = smo_bf16_to_double(smo_bf16_from_float(p));", "k[i] = (double)p;"),
    ("rope offset", "smo_load_u16le(row + SMO_ROPE_OFF + 2 * i)", "smo_load_u16le(row + SMO_ROPE_OFF - 2 + 2 * i)"),
    ("softmax scale dropped", "s[j] = softmax_scale * acc;", "s[j] = acc;"),
    ("lse loses max", "sum += exp(s[j] - m);\n        l = m + log(sum);", "sum += exp(s[j] - m);\n        l = log(sum);"),
    ("combine lse loses max", "        l = m + log(sum);\n        lse[h] = l;\n        for (s = 0;",
     "        l = log(sum);\n        lse[h] = l;\n        for (s = 0;"),
    ("value columns shifted to RoPE", "oh[d] += w * K[(size_t)j * SMO_DQK + d];",
     "oh[d] += w * K[(size_t)j * SMO_DQK + d + 64];"),
    ("score over latent only", "for (d = 0; d < SMO_DQK; ++d) acc +=", "for (d = 0; d < SMO_DV; ++d) acc +="),
    ("validity bound inclusive", "valid[j] = (t >= 0 && t < seqlen) ? 1 : 0;",
     "valid[j] = (t >= 0 && t <= seqlen) ? 1 : 0;"),
    ("paged row within block", "(size_t)(phys * SMO_BLOCK + t % SMO_BLOCK)", "(size_t)(phys * SMO_BLOCK + t % 32)"),
    ("combine weights use max", "double w = exp(lse_parts[(size_t)s * h_q + h] - l);",
     "double w = exp(lse_parts[(size_t)s * h_q + h] - m);"),
    ("sched last part off by one", "int64_t last = ((int64_t)(r + 1) * n - 1) / L;",
     "int64_t last = ((int64_t)(r + 1) * n) / L;"),
    ("sched first slot offset dropped",
     "m[4] = num_splits[m[0]] + p - (int32_t)((((int64_t)m[0]) * n) / L);", "m[4] = num_splits[m[0]];"),
    ("sched tiles per part floor", "L = total > 0 ? (total + P - 1) / P : 1;\n    num_splits[0] = 0;\n    for (r = 0; r < R; ++r) {\n        int64_t first = ((int64_t)r * n) / L;",
     "L = total > 0 ? total / P + (total < P) : 1;\n    num_splits[0] = 0;\n    for (r = 0; r < R; ++r) {\n        int64_t first = ((int64_t)r * n) / L;"),
    ("causal visible length off by one", "int64_t len = causal ? (int64_t)seqlen - (s_q - 1 - t) : (int64_t)seqlen;",
     "int64_t len = causal ? (int64_t)seqlen - (s_q - t) : (int64_t)seqlen;"),
    ("bf16 row read shifted", "k[i] = smo_bf16_to_double(smo_load_u16le(row + 2 * i));",
     "k[i] = smo_bf16_to_double(smo_load_u16le(row + 2 * i + 2));"),
    ("dense bf16 row stride of the latent only", "const size_t row_bytes = kv_format ? SMO_BF16_ROW_BYTES : SMO_ROW_BYTES;",
     "const size_t row_bytes = kv_format ? 1024 : SMO_ROW_BYTES;"),
    ("dense row within block", "(size_t)(phys * SMO_BLOCK + i % SMO_BLOCK) * row_bytes",
     "(size_t)(phys * SMO_BLOCK + i % 32) * row_bytes"),
    ("varlen last part off by one", "int64_t last = ((int64_t)tile_prefix[r + 1] - 1) / L;",
     "int64_t last = ((int64_t)tile_prefix[r + 1]) / L;"),
    ("varlen first tile not relative to its request", "m[1] = (int32_t)(g0 - tile_prefix[rb]);", "m[1] = (int32_t)g0;"),
    ("varlen end request search stops early", "while (re + 1 < R && tile_prefix[re + 1] <= g1) ++re;",
     "while (re + 1 < R && tile_prefix[re + 1] < g1) ++re;"),
]


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        if name == "test_sched_meta_brute_force":
            for args in [(64, 32, 148), (7, 3, 5), (5, 7, 35), (13, 2, 3), (3, 100, 7)]:
                out.append((f"{name}{args}", lambda fn=fn, args=args: fn(*args)))
        elif name == "test_sched_meta_varlen_brute_force":
            for args in [([3, 1, 5, 2], 4), ([7, 1, 1, 1, 30, 2], 5), ([9, 9], 7), ([128] * 64, 148)]:
                out.append((f"{name}{args}", lambda fn=fn, args=args: fn(*args)))
        else:
            out.append((name, fn))
    return out


def _build_mutant(tmp, src_text):
    src = os.path.join(tmp, "oracle.c")
    lib = os.path.join(tmp, "liboracle_mutant.so")
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                    "-o", lib, src, "-lm"], check=True)
    return lib


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new):
    with open(obuild.SRC) as f:
        text = f.read()
    assert text.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        lib = _build_mutant(tmp, text.replace(old, new))
        caught = []
        with oracle.using_library(lib):
            for pin_name, fn in _pin_functions():
                try:
                    fn()
                except (AssertionError, ValueError, FloatingPointError):
                    caught.append(pin_name)
                    break
        assert caught, f"no pin fails for the planted mistake '{name}'"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
