"""The oracle's pins catch plausible mistakes. Each case plants one mistake in
a copy of the oracle's C source (on the CPU, in a temporary directory),
compiles it, and runs the pin tests against it: at least one pin must fail.
A control copy without a mistake must pass them all. The oracle's own source
and library are not touched."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")
PINS = [os.path.join(ROOT, "tests", "test_oracle_pins.py"),
        os.path.join(ROOT, "tests", "test_oracle_bruteforce.py"),
        os.path.join(ROOT, "tests", "test_bias_pid.py")]

# (name, text in the source, replacement, occurrences); every planted mistake
# keeps all accesses in bounds
MUTANTS = [
    ("silu_sign", "h[f] = a / (1.0 + exp(-a)) * u;", "h[f] = a / (1.0 + exp(a)) * u;", 1),
    ("ties_to_higher_id", "if (best < 0 || key > best_key) {",
     "if (best < 0 || key >= best_key) {", 1),
    ("bias_left_out_of_keys", "double key = logit[e] + (double)bias[e];",
     "double key = logit[e];", 2),
    ("w_down_transposed",
     "acc += elem(w_down, w_dtype, base + f) * h[f];",
     "acc += elem(w_down, w_dtype, (e * F + f) * d + n) * h[f];", 1),
    ("router_columns_reversed", "(double)w_r[e * d + i];", "(double)w_r[e * d + (d - 1 - i)];",
     2),
    ("identity_dropped_in_combine", "ident += gate[sl] * x[t * d + i];", "ident += 0.0;", 1),
    ("identity_dropped_in_layer", "for (int64_t i = 0; i < d; ++i) o[i] += g[j] * xt[i];",
     "(void)xt;", 1),
    ("identity_scaled_in_combine", "out[t * d + i] = s * routed + ident;",
     "out[t * d + i] = s * (routed + ident);", 1),
    ("identity_scaled_in_layer", "o[i] += g[j] * xt[i];", "o[i] += s * g[j] * xt[i];", 1),
    ("routed_part_unscaled", "o[i] += s * g[j] * y[i];", "o[i] += g[j] * y[i];", 1),
    ("gates_not_normalised", "for (int64_t j = 0; j < k; ++j) gate[j] = exp(logit[idx[j]] - m) / z;",
     "for (int64_t j = 0; j < k; ++j) gate[j] = exp(logit[idx[j]] - m);", 1),
    ("dispatch_tokens_descending",
     "for (int64_t t = 0; t < T; ++t)\n      for (int64_t j = 0; j < k; ++j)\n        if (idx[t * k + j] == e) {",
     "for (int64_t t = T - 1; t >= 0; --t)\n      for (int64_t j = 0; j < k; ++j)\n        if (idx[t * k + j] == e) {",
     1),
    ("margin_sign", "*margin = kth_key - next;", "*margin = next - kth_key;", 1),
    ("pid_integral_not_carried", "const double integral = state[0] + err;",
     "const double integral = err;", 1),
    ("pid_derivative_sign", "kd * (err - state[1]);", "kd * (state[1] - err);", 1),
    ("pid_no_clamp", "if (u > max_step) u = max_step;", "(void)max_step;", 1),
]


def _compile(text, directory, name):
    src = os.path.join(directory, name + ".c")
    lib = os.path.join(directory, name + ".so")
    with open(src, "w") as f:
        f.write(text)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                    "-fno-fast-math", "-o", lib, src, "-lm"], check=True)
    return lib


def _run_pins(lib):
    env = dict(os.environ, MOE_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           "-m", "not gpu", *PINS], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=900)


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("oracle_mutants"))
    with open(SRC) as f:
        text = f.read()
    libs = {"control": _compile(text, d, "control")}
    for name, old, new, count in MUTANTS:
        assert text.count(old) == count, (name, text.count(old))
        libs[name] = _compile(text.replace(old, new), d, name)
    with ThreadPoolExecutor(max_workers=4) as pool:
        runs = dict(zip(libs, pool.map(_run_pins, libs.values())))
    return runs


def test_control_copy_passes_every_pin(results):
    r = results["control"]
    assert r.returncode == 0, r.stdout[-3000:]


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(results, name):
    r = results[name]
    assert r.returncode == 1, f"{name}: exit {r.returncode}\n{r.stdout[-3000:]}"
    assert " failed" in r.stdout, r.stdout[-3000:]
