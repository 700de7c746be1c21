"""The oracle's pins are strong enough: each plausible mistake planted in a copy of
``oracle/oracle.c`` (a dropped term, a wrong sign, index or offset, an exponent
bias off by one, the wrong rounding) makes ``tests/test_oracle.py`` fail, and
the unmodified copy makes it pass. The mutants are built with gcc into a
temporary directory and run in child processes; the oracle itself is never
touched. CPU only."""

from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# (name, text in oracle.c, planted replacement)
MUTANTS = [
    ("gqa-interleaved", "int G = Hq / Hkv, h = hq / G;", "int G = Hq / Hkv, h = hq % Hkv;"),
    ("table-index", "    int32_t blk = table[i / bs];\n    if (blk < 0 || blk >= num_blocks) return OR_ERR_BLOCK;\n    size_t row",
     "    int32_t blk = table[i % bs];\n    if (blk < 0 || blk >= num_blocks) return OR_ERR_BLOCK;\n    size_t row"),
    ("row-in-block", "size_t row = (((size_t)blk * bs + (size_t)(i % bs)) * Hkv + h) * (size_t)D;",
     "size_t row = (((size_t)blk * bs + (size_t)(i / bs)) * Hkv + h) * (size_t)D;"),
    ("scale-dropped", "s[i] = scale * dot;", "s[i] = dot;"),
    ("exp-sign", "double w = exp(s[i] - m);", "double w = exp(m - s[i]);"),
    ("not-normalised", "for (int d = 0; d < D; ++d) o[d] /= l;", "for (int d = 0; d < D; ++d) o[d] /= 1.0;"),
    ("context-short", "block_tables + (size_t)b * max_blocks, context_lens[b], Hq",
     "block_tables + (size_t)b * max_blocks, context_lens[b] - 1, Hq"),
    ("prefill-excludes-self", "pos + 1, Hq, Hkv, D, bs,", "pos, Hq, Hkv, D, bs,"),
    ("prefill-top-left", "int pos = context_lens[b] - n + (int)(t - query_start[b]);",
     "int pos = (int)(t - query_start[b]);"),
    ("merge-unweighted", "double c = exp(mj[j] - M);", "double c = 1.0;"),
    ("f16-bias", "v = ldexp((double)(f | 0x400), e - 25);", "v = ldexp((double)(f | 0x400), e - 24);"),
    ("bf16-shift", "uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    ("e4m3-bias", "v = ldexp((double)(8 + f), e - 10);", "v = ldexp((double)(8 + f), e - 11);"),
    ("e4m3-ties-away", "double v = rint(a / step) * step;", "double v = floor(a / step + 0.5) * step;"),
    ("e4m3-saturates-to-nan", "if (a >= 448.0) return sign | 0x7E;", "if (a >= 448.0) return sign | 0x7F;"),
    ("fp8-scale-multiplied", "e4m3_from_float(kx / k_scale);", "e4m3_from_float(kx * k_scale);"),
    ("scatter-row-dropped", "size_t blk = (size_t)(s / bs), off = (size_t)(s % bs);",
     "size_t blk = (size_t)(s / bs), off = 0;"),
    ("copy-v-dropped", "    memcpy((char*)vpool + d * blk, snap + (2 * (size_t)p + 1) * blk, blk);\n", ""),
    ("swap-reads-dst-index", "(const char*)src_k + s * block_bytes", "(const char*)src_k + d * block_bytes"),
    ("mixed-v-read-as-k-type", "rc = gather_head(V, vpool, vdt, vscale,", "rc = gather_head(V, vpool, kdt, vscale,"),
    ("mixed-scatter-one-scale", "float sc = which ? v_scale : k_scale;", "float sc = k_scale;"),
    ("mixed-prefill-v-unscaled", "kpool, k_dtype, k_scale, vpool, v_dtype, v_scale,\n                       block_tables",
     "kpool, k_dtype, k_scale, vpool, v_dtype, 1.0,\n                       block_tables"),
]

PLUGIN = '''
import os
import oracle

def pytest_configure(config):
    path = os.environ["ORACLE_MUTANT_LIB"]
    oracle.build = lambda force=False: path
    oracle._lib = None
'''


def _build(src_text: str, out_dir: str, name: str) -> str:
    c = os.path.join(out_dir, f"{name}.c")
    so = os.path.join(out_dir, f"lib{name}.so")
    with open(c, "w", encoding="utf-8") as f:
        f.write(src_text)
    r = subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                        "-ffp-contract=off", "-fno-fast-math", "-o", so, c, "-lm"],
                       capture_output=True, text=True)
    assert r.returncode == 0, f"{name}: {r.stderr}"
    return so


def _run_pins(so: str, plugin_dir: str) -> int:
    env = dict(os.environ, ORACLE_MUTANT_LIB=so, OMP_NUM_THREADS="2",
               PYTHONPATH=os.pathsep.join([plugin_dir, ROOT]))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "mutant_plugin",
                        "-p", "no:cacheprovider", os.path.join(ROOT, "tests", "test_oracle.py")],
                       capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
    return r.returncode


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("oracle_mutants"))
    with open(os.path.join(d, "mutant_plugin.py"), "w", encoding="utf-8") as f:
        f.write(PLUGIN)
    text = open(SRC, encoding="utf-8").read()
    libs = {"unmodified": _build(text, d, "unmodified")}
    for name, old, new in MUTANTS:
        assert text.count(old) == 1, f"{name}: the planted site must occur once"
        libs[name] = _build(text.replace(old, new), d, name.replace("-", "_"))
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        codes = dict(zip(libs, ex.map(lambda so: _run_pins(so, d), libs.values())))
    return codes


def test_unmodified_copy_passes_the_pins(outcomes):
    assert outcomes["unmodified"] == 0


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(outcomes, name):
    # pytest exit code 1: tests ran and at least one failed (not a crash or usage error)
    assert outcomes[name] == 1, f"{name}: pins exit code {outcomes[name]}"
