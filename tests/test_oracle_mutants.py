"""The oracle's pins catch plausible mistakes (test infrastructure, CPU only).

Each mutant below is duo_oracle.c with one deliberate error of the kind a
restatement of the method could make: a band edge off by one, a dropped or
rescaled term, a wrong logarithm, a wrong head grouping, a transposed or
shifted operand, a ring read in the wrong order.  Each is compiled into a
temporary directory, and the oracle's own pin tests run against it (through
DUO_ORACLE_LIB) in a subprocess: first the fast pins (closed forms, torch
SDPA, decode against prefill rows, block decode), then, for a mutant those
pass, the brute-force attended-set simulation at the small band sizes.
Every mutant must fail at least one pin, while an unmutated copy built the
same way passes the fast pins.  Every mutant stays within its buffers: each
only filters keys, permutes indices modulo their range, or changes
arithmetic.  A mutant that no pin caught would be a gap in the pins, not in
the oracle."""
import concurrent.futures
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "duo_oracle.c")
PIN_FILES = ["tests/test_oracle_pins.py", "tests/test_oracle_decode_block.py"]
FAST = "not cache_simulation"                      # about 10 s on one core
SIMULATION = "cache_simulation and not sizes0"     # the small band sizes, L <= 321

# (what the mistake is, the text it replaces, its replacement)
MUTANTS = [
    ("streaming band one key too wide",
     "return j < p->sink || j > i - p->recent;", "return j < p->sink || j >= i - p->recent;"),
    ("sink one key too wide",
     "return j < p->sink || j > i - p->recent;", "return j <= p->sink || j > i - p->recent;"),
    ("sliding window one key too wide",
     "default: return j > i - p->window;", "default: return j >= i - p->window;"),
    ("sink logit dropped from the denominator",
     "    if (has_sink) Z += exp(sigma - m);\n", "\n"),
    ("log-sum-exp in base 2",
     "return m + log(Z);", "return m + log2(Z);"),
    ("prefill groups query heads round robin",
     "const int64_t b = r / L / Hq;\n            const int g = h / group;",
     "const int64_t b = r / L / Hq;\n            const int g = h % Hkv;"),
    ("decode groups query heads round robin",
     "const int h = (int)(r % Hq);\n            const int g = h / group;",
     "const int h = (int)(r % Hq);\n            const int g = h % Hkv;"),
    ("prefill scores not scaled",
     "s[n] = p->softmax_scale * dot_bf16(qi, kj, D);", "s[n] = dot_bf16(qi, kj, D);"),
    ("prefill sink logit scaled like a score",
     "const double sigma = has_sink ? (double)p->sink_logit[h] : 0.0;\n            lse[t] = softmax_row(n,",
     "const double sigma = has_sink ? p->softmax_scale * (double)p->sink_logit[h] : 0.0;\n"
     "            lse[t] = softmax_row(n,"),
    ("prefill values read from K",
     "vr[n] = v + ((b * L + j) * Hkv + g) * D;", "vr[n] = k + ((b * L + j) * Hkv + g) * D;"),
    ("dot product with a shifted operand",
     "acc += bf16_value(a[d]) * bf16_value(b[d]);", "acc += bf16_value(a[d]) * bf16_value(b[(d + 1) % D]);"),
    ("ring head moves backwards",
     "c->ring_head[b] = (c->ring_head[b] + 1) % R;", "c->ring_head[b] = (c->ring_head[b] + R - 1) % R;"),
    ("decode skips the oldest ring slot",
     "for (int64_t e = 0; e < cnt; ++e) {", "for (int64_t e = 1; e < cnt; ++e) {"),
    ("decode reads the ring from ring_head forward",
     "const int64_t slot = S + (((int64_t)c->ring_head[b] - cnt + e) % R + R) % R;",
     "const int64_t slot = S + (((int64_t)c->ring_head[b] + e) % R + R) % R;"),
    ("block decode keeps one cached key too old",
     "if (pos <= i - R) continue;", "if (pos < i - R) continue;"),
    ("block decode's own keys one too wide",
     "!(j < S || j > i - R)) continue;", "!(j < S || j >= i - R)) continue;"),
    ("bf16 decoded with the wrong shift",
     "uint32_t u = (uint32_t)bits << 16;", "uint32_t u = (uint32_t)bits << 15;"),
]


def _compile(text: str, out: str) -> None:
    src = out[:-3] + ".c"
    with open(src, "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", out, src, "-lm"])


def _pins(lib: str, select: str):
    env = dict(os.environ, DUO_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu", "-k", select, *PIN_FILES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:]


def _caught(lib: str):
    rc, out = _pins(lib, FAST)
    if rc == 0:
        rc, out = _pins(lib, SIMULATION)
    return rc, out


def test_every_mutant_fails_a_pin(tmp_path):
    base = open(SRC).read()
    jobs = [("unmutated", os.path.join(tmp_path, "m_ref.so"), base)]
    for idx, (what, old, new) in enumerate(MUTANTS):
        assert base.count(old) == 1, f"mutant site not unique: {what}"
        jobs.append((what, os.path.join(tmp_path, f"m{idx:02d}.so"), base.replace(old, new)))
    for _, lib, text in jobs:
        _compile(text, lib)
    workers = max(2, min(len(jobs), os.cpu_count() or 2))
    with concurrent.futures.ThreadPoolExecutor(workers) as pool:
        runs = [pool.submit(_pins, lib, FAST) if what == "unmutated" else pool.submit(_caught, lib)
                for what, lib, _ in jobs]
        results = {what: r.result() for (what, _, _), r in zip(jobs, runs)}
    rc, out = results.pop("unmutated")
    assert rc == 0, "the unmutated copy must pass its pins:\n" + out
    survivors = [what for what, (rc, out) in results.items() if rc == 0]
    assert not survivors, f"mutants no pin caught: {survivors}"
    # each mutant failed on a pin's assertion, not on a crash or a collection error
    for what, (rc, out) in results.items():
        assert rc == 1 and "failed" in out, f"{what}: pytest exited {rc}\n{out}"


# ------------------------------------------------------------ the Python parts
# (module, what the mistake is, the text it replaces, its replacement)
PY_MUTANTS = [
    ("oracle/prep.py", "rotation pairs adjacent channels",
     "a, b = y[..., : D // 2], y[..., D // 2:]", "a, b = y[..., 0::2], y[..., 1::2]"),
    ("oracle/prep.py", "rotation in the opposite direction",
     "[a * c - b * s, b * c + a * s]", "[a * c + b * s, b * c - a * s]"),
    ("oracle/prep.py", "YaRN ramp reversed",
     "base * (1.0 - ramp) + (base / factor) * ramp", "base * ramp + (base / factor) * (1.0 - ramp)"),
    ("oracle/prep.py", "YaRN lower bound rounded up",
     "lo = max(math.floor(pair_index_for_turns(beta_fast)), 0)",
     "lo = max(math.ceil(pair_index_for_turns(beta_fast)), 0)"),
    ("oracle/prep.py", "YaRN beta_fast and beta_slow swapped",
     "lo = max(math.floor(pair_index_for_turns(beta_fast)), 0)\n    hi = min(math.ceil(pair_index_for_turns(beta_slow)), d - 1)",
     "lo = max(math.floor(pair_index_for_turns(beta_slow)), 0)\n    hi = min(math.ceil(pair_index_for_turns(beta_fast)), d - 1)"),
    ("oracle/prep.py", "RMSNorm eps outside the square root",
     "np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)",
     "(np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps)"),
    ("oracle/prep.py", "attention_factor dropped",
     "b * c + a * s], axis=-1) * attention_factor", "b * c + a * s], axis=-1)"),
    ("oracle/prep.py", "bf16 rounding ties away from zero",
     "r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)",
     "r = np.ldexp(np.trunc(np.ldexp(m, 8) + np.copysign(0.5, m)), e - 8)"),
    ("oracle/prep.py", "bf16 rounding to 7 significant bits",
     "r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)", "r = np.ldexp(np.rint(np.ldexp(m, 7)), e - 7)"),
    ("oracle/__init__.py", "sigmoid of the negated gate",
     "return 1.0 / (1.0 + np.exp(-x))", "return 1.0 / (1.0 + np.exp(x))"),
    ("oracle/__init__.py", "per-head prefill gate read from the next head",
     "gv = g[b, i, h, :] if mode == GATE_PER_ELEMENT else g[b, i, h][:, None]",
     "gv = g[b, i, h, :] if mode == GATE_PER_ELEMENT else g[b, i, (h + 1) % Hq][:, None]"),
    ("oracle/__init__.py", "per-channel decode gate read from the next head",
     "gv = g[b, h, :] if mode == GATE_PER_ELEMENT else g[b, h][:, None]",
     "gv = g[b, (h + 1) % Hq, :] if mode == GATE_PER_ELEMENT else g[b, h][:, None]"),
]
PY_PINS = ["tests/test_oracle_prep.py", "tests/test_oracle_gate.py"]

# Runs the pins with one oracle module's source replaced in place: the module is
# imported, the mutated text is executed over its namespace, then pytest runs.
_BOOT = r"""
import importlib, sys
sys.path.insert(0, {root!r})
mod = importlib.import_module({module!r})
src = open(mod.__file__).read()
assert src.count({old!r}) == 1
exec(compile(src.replace({old!r}, {new!r}), mod.__file__, "exec"), mod.__dict__)
import pytest
sys.exit(pytest.main(["-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu", *{pins!r}]))
"""


def _py_pins(module_file: str, old: str, new: str):
    module = module_file[:-3].replace("/", ".").removesuffix(".__init__")
    code = _BOOT.format(root=ROOT, module=module, old=old, new=new, pins=PY_PINS)
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=600, env=dict(os.environ, OMP_NUM_THREADS="1"))
    return r.returncode, r.stdout[-2000:] + r.stderr[-1000:]


def test_every_python_mutant_fails_a_pin():
    for module_file, what, old, new in PY_MUTANTS:
        assert open(os.path.join(ROOT, module_file)).read().count(old) == 1, f"site not unique: {what}"
    jobs = [("unmutated", "oracle/prep.py", "D = 128", "D = 128")] + \
        [(what, m, old, new) for m, what, old, new in PY_MUTANTS]
    with concurrent.futures.ThreadPoolExecutor(min(len(jobs), os.cpu_count() or 2)) as pool:
        results = dict(zip([j[0] for j in jobs], pool.map(lambda j: _py_pins(*j[1:]), jobs)))
    rc, out = results.pop("unmutated")
    assert rc == 0, "the unmutated modules must pass their pins:\n" + out
    survivors = [what for what, (rc, _) in results.items() if rc == 0]
    assert not survivors, f"mutants no pin caught: {survivors}"
    for what, (rc, out) in results.items():
        assert rc == 1 and "failed" in out, f"{what}: exited {rc}\n{out}"
