"""The oracle's pins catch plausible mistakes.

Each case plants one mistake (a dropped term, a wrong sign or index, a
rounding mode, a transposed operand, ...) in a temporary copy of the oracle
source, builds it, and runs the pin module against that copy in a fresh
process; the pins must fail.  An unmodified copy must pass, so a broken
harness cannot look like a success.  CPU only; the mistakes are planted in
the oracle, never in the CUDA library.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")

# name -> (text in oracle/spx_oracle.cpp, replacement)
MUTANTS = {
    # IndexPool and its bf16 store
    "pool weights reversed": (
        "acc += w[i] * bf16_to_f64(raw[(b * pool + i) * dim + d]);",
        "acc += w[pool - 1 - i] * bf16_to_f64(raw[(b * pool + i) * dim + d]);"),
    "pool token off by one": (
        "acc += w[i] * bf16_to_f64(raw[(b * pool + i) * dim + d]);",
        "acc += w[i] * bf16_to_f64(raw[(b * pool + (i + 1) % pool) * dim + d]);"),
    "bf16 truncation instead of nearest-even": (
        "double r = std::nearbyint(std::ldexp(std::fabs(v), -qe));",
        "double r = std::trunc(std::ldexp(std::fabs(v), -qe));"),
    "per-token weight of the next token": (
        "acc += wt[b * pool + i] * bf16_to_f64(raw[(b * pool + i) * dim + d]);",
        "acc += wt[b * pool + (i + 1) % pool] * bf16_to_f64(raw[(b * pool + i) * dim + d]);"),
    "per-token weights of the block's first token only": (
        "acc += wt[b * pool + i] * bf16_to_f64(raw[(b * pool + i) * dim + d]);",
        "acc += wt[b * pool] * bf16_to_f64(raw[(b * pool + i) * dim + d]);"),
    "per-token sum in fp32": (
        "      pooled[b * dim + d] = f64_to_bf16_rne(acc);\n    }\n  }\n}\n\n// Lightning",
        "      pooled[b * dim + d] = f64_to_bf16_rne(static_cast<float>(acc));\n    }\n  }\n}\n\n// Lightning"),
    # indexer score
    "score without ReLU": (
        "s += w_head[h] * (dot > 0.0 ? dot : 0.0);", "s += w_head[h] * dot;"),
    "score without head weight": (
        "s += w_head[h] * (dot > 0.0 ? dot : 0.0);", "s += (dot > 0.0 ? dot : 0.0);"),
    "score with |dot| instead of ReLU": (
        "s += w_head[h] * (dot > 0.0 ? dot : 0.0);", "s += w_head[h] * std::fabs(dot);"),
    # top-k
    "ties to the higher block": (
        "return a.second < c.second;", "return a.second > c.second;"),
    "lowest scores kept": (
        "if (a.first != c.first) return a.first > c.first;",
        "if (a.first != c.first) return a.first < c.first;"),
    "decision not on fp32 scores": (
        "for (int64_t b = 0; b < nblk; ++b) v[b] = {static_cast<float>(s[b]), b};",
        "for (int64_t b = 0; b < nblk; ++b) v[b] = {static_cast<float>(s[b] + 1e-30 * b), b};"),
    # token set and attention
    "partial tail dropped": (
        "for (int64_t t = (n_vis / pool) * pool; t < n_vis; ++t) pos_out[m++] = t;", ""),
    "softmax scale dropped": ("z[t] = sm_scale * dot;", "z[t] = dot;"),
    "lse without the max": (
        "if (lse) lse[h] = m + std::log(l);", "if (lse) lse[h] = std::log(l);"),
    "output not normalised": ("out[h * dim + d] = acc / l;", "out[h * dim + d] = acc;"),
    # INT8 cache
    "int8 ties away from zero": (
        "const double c = std::nearbyint(std::ldexp(x[i], -e));",
        "const double c = std::round(std::ldexp(x[i], -e));"),
    "int8 exponent one too high": (
        "while (e > -149 && amax <= 127.0 * std::ldexp(1.0, e - 1)) --e;",
        "while (e > -149 && amax <= 127.0 * std::ldexp(1.0, e - 1)) --e;\n    ++e;"),
    "int8 exponent one too low": (
        "while (e > -149 && amax <= 127.0 * std::ldexp(1.0, e - 1)) --e;",
        "while (e > -149 && amax <= 127.0 * std::ldexp(1.0, e - 1)) --e;\n    --e;"),
    "int8 bound 128 instead of 127": (
        "while (e > -149 && amax <= 127.0 * std::ldexp(1.0, e - 1)) --e;",
        "while (e > -149 && amax <= 128.0 * std::ldexp(1.0, e - 1)) --e;"),
    "int8 pooled sum rounded to bf16 first": (
        "      acc[d] = s;\n", "      acc[d] = bf16_to_f64(f64_to_bf16_rne(s));\n"),
    "int8 block scale dropped": ("out[b] = scale[b] * s;", "out[b] = s;"),
    "int8 head scale dropped": (
        "s += w_head[h] * qs[h] * (dot > 0.0 ? dot : 0.0);",
        "s += w_head[h] * (dot > 0.0 ? dot : 0.0);"),
    "int8 ReLU after the weight": (
        "s += w_head[h] * qs[h] * (dot > 0.0 ? dot : 0.0);",
        "s += std::max(0.0, w_head[h] * qs[h] * dot);"),
    # FP8 latent cache
    "e4m3 ties away from zero": (
        "const double r = std::ldexp(std::nearbyint(std::ldexp(std::fabs(v), -qe)), qe);",
        "const double r = std::ldexp(std::round(std::ldexp(std::fabs(v), -qe)), qe);"),
    "e4m3 one mantissa bit too many": ("int qe = E - 4;", "int qe = E - 5;"),
    "e4m3 subnormal step 2^-10": ("if (qe < -9) qe = -9;", "if (qe < -10) qe = -10;"),
    "e4m3 bound 512 instead of 448": (
        "while (e > -149 && amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;",
        "while (e > -149 && amax <= 512.0 * std::ldexp(1.0, e - 1)) --e;"),
    "e4m3 exponent one too high": (
        "while (e > -149 && amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;",
        "while (e > -149 && amax <= 448.0 * std::ldexp(1.0, e - 1)) --e;\n    ++e;"),
    "e4m3 exponent field bias 8": (
        "return sign | static_cast<uint8_t>(((E - 1 + 7) << 3) | mant);",
        "return sign | static_cast<uint8_t>(((E - 1 + 8) << 3) | mant);"),
    "int8 key operand transposed": (
        "static_cast<double>(codes[b * dim + d]);",
        "static_cast<double>(codes[d * nblk + b]);"),
}

RUNNER = """
import sys
sys.path.insert(0, {pkg_parent!r})
import oracle
assert oracle.__file__.startswith({pkg_parent!r}), oracle.__file__
try:
    oracle.build()
except Exception:
    sys.exit(3)  # a copy that does not build is a harness error, not a catch
sys.path.insert(1, {root!r})
sys.path.insert(2, {tests!r})
import pytest
sys.exit(pytest.main(["-q", "-x", "-p", "no:cacheprovider", {pins!r}]))
"""


def _run_copy(tmp_root: str, name: str, source: str) -> int:
    """Builds an oracle package with `source` under tmp_root/name and runs the
    pins against it; returns pytest's exit code."""
    parent = os.path.join(tmp_root, name.replace(" ", "_"))
    pkg = os.path.join(parent, "oracle")
    os.makedirs(pkg)
    shutil.copy(os.path.join(ORACLE_DIR, "__init__.py"), pkg)
    with open(os.path.join(pkg, "spx_oracle.cpp"), "w") as f:
        f.write(source)
    code = RUNNER.format(pkg_parent=parent, root=ROOT, tests=os.path.join(ROOT, "tests"),
                         pins=os.path.join(ROOT, "tests", "test_oracle_pins.py"))
    env = dict(os.environ, TMPDIR=parent)  # compiler temporaries stay in the scratch folder
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=600, env=env)
    return r.returncode


def test_pins_catch_planted_mistakes():
    src = open(os.path.join(ORACLE_DIR, "spx_oracle.cpp")).read()
    jobs = {"unmodified": src}
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, f"mutant {name!r} no longer matches the oracle source"
        jobs[name] = src.replace(old, new)
    # scratch inside the repository's (ignored) build folder, removed afterwards
    scratch = os.path.join(ROOT, "_build", f"oracle_mutants_{os.getpid()}")
    os.makedirs(scratch)
    try:
        workers = max(1, min(8, os.cpu_count() or 1))
        with cf.ThreadPoolExecutor(workers) as ex:
            futs = {name: ex.submit(_run_copy, scratch, name, s) for name, s in jobs.items()}
            rc = {name: f.result() for name, f in futs.items()}
    finally:
        shutil.rmtree(scratch, ignore_errors=True)
    assert rc.pop("unmodified") == 0, "the unmodified oracle copy must pass its pins"
    survived = [name for name, code in rc.items() if code != 1]
    assert not survived, f"pins did not catch: {survived}"
