"""The oracle's pins catch plausible mistakes.  Each case below plants one
mistake in a copy of the oracle's C source (the copy and its build live under
oracle/_build/mutants/, ignored by git; the oracle itself is untouched), points
the oracle module at that copy in a child process, and runs the pin suite
(tests/test_oracle_pins.py) there: every planted mistake must fail at least
five pins (a planted mistake in the e4m3 or decision oracle, at least two of
their pins).  The mistakes are the ones a hand-written restatement of the
method is likely to make:

  exclusive_diagonal   a token does not see itself (own-node causality)
  missing_scale        scores without the 1/sqrt(d) factor
  decay_after_write    the gate also decays the new write beta v k^T
  erase_without_beta   the delta rule erases S k k^T without beta
  skipped_root         the root's tokens are left out of every branch's keys
  positions_no_past    isolated positions ignore the checkpointed past
  gqa_modulo           query head h reads kv head h % Hkv instead of h / G
  depth_counts_nodes   depth counts nodes instead of edges
  ctx_without_own_node context length leaves out the node's own tokens
  children_from_request_state  memoised children restart from the request's
                       state instead of their parent's end state
  resume_state_ignored a resumed request starts from zero
  gate_not_exponentiated  the decay uses 1 + g instead of exp(g)
  read_before_write    o_t reads the state before token t's update
  erase_sign           the delta rule adds S k k^T instead of erasing it

The child processes run a few at a time, one oracle thread each.
"""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "flide_oracle.c")

# one token's write and read in the GDN scan (the read must follow the write)
_STEP = ("            gdn_step(S, dk, dv, k + ((size_t)t * H + h) * dk,\n"
         "                     v + ((size_t)t * H + h) * dv,\n"
         "                     (double)g[(size_t)t * H + h],\n"
         "                     (double)beta[(size_t)t * H + h], u);\n")
_READ = "            gdn_read(S, dk, dv, q + ((size_t)t * H + h) * dk, o);\n"

MUTANTS = {
    "exclusive_diagonal": ("for (int j = node_start[n]; j <= t; ++j) {",
                           "for (int j = node_start[n]; j < t; ++j) {"),
    "missing_scale": ("s[j] = dot * scale;", "s[j] = dot;"),
    "decay_after_write": (
        "S[(size_t)i * dk + c] = alpha * (S[(size_t)i * dk + c] - w * kc) + bv * kc;",
        "S[(size_t)i * dk + c] = alpha * (S[(size_t)i * dk + c] - w * kc + bv * kc);"),
    "erase_without_beta": ("double w = beta * u[i];", "double w = u[i];"),
    "skipped_root": ("  for (int a = 0; a + 1 < cnt; ++a)\n    for (int j = 0; j < seg_len[chain[a]]; ++j) {\n"
                     "      if (m >= cap) return -1;\n      keys[m++] = node_start[chain[a]] + j;",
                     "  for (int a = 1; a + 1 < cnt; ++a)\n    for (int j = 0; j < seg_len[chain[a]]; ++j) {\n"
                     "      if (m >= cap) return -1;\n      keys[m++] = node_start[chain[a]] + j;"),
    "positions_no_past": ("int before = past_len[r];", "int before = 0;"),
    "gqa_modulo": ("int kvh = h / G;", "int kvh = h % Hkv;"),
    "depth_counts_nodes": ("depth[n] = cnt - 1;", "depth[n] = cnt;"),
    "ctx_without_own_node": ("ctx += seg_len[chain[i]];", "if (i + 1 < cnt) ctx += seg_len[chain[i]];"),
    "children_from_request_state": ("if (memoise && parent[n] >= 0) {", "if (0) {"),
    "resume_state_ignored": [("} else if (state_in_f64) {", "} else if (0) {"),
                             ("} else if (state_in) {", "} else if (0) {")],
    "gate_not_exponentiated": ("double alpha = exp(g);", "double alpha = 1.0 + g;"),
    "read_before_write": (_STEP + _READ, _READ + _STEP),
    "erase_sign": ("alpha * (S[(size_t)i * dk + c] - w * kc)", "alpha * (S[(size_t)i * dk + c] + w * kc)"),
}

MIN_FAILED = 5


def _c_job(name):
    """Child-process code that runs the pins against a copy of the C oracle
    with mistake `name` planted (the copy is written and built here)."""
    edits = MUTANTS[name] if isinstance(MUTANTS[name], list) else [MUTANTS[name]]
    src = open(SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, "the mutation site must be unique"
        src = src.replace(old, new)
    d = os.path.join(ROOT, "oracle", "_build", "mutants", name)
    os.makedirs(d, exist_ok=True)
    msrc, mso = os.path.join(d, "flide_oracle.c"), os.path.join(d, "liboracle.so")
    with open(msrc, "w") as f:
        f.write(src)
    if os.path.exists(mso):
        os.remove(mso)
    return ("import sys, oracle, pytest\n"
            f"oracle._SRC = {msrc!r}\noracle._SO = {mso!r}\n"
            "sys.exit(pytest.main(['-q', '-p', 'no:cacheprovider', 'tests/test_oracle_pins.py']))\n")


# The Python oracles (e4m3 and decision scoring): a mistake is planted by
# re-executing a mutated copy of the module's source in the module's own
# namespace in the child process (and rebinding the names the oracle package
# re-exports), so the pins see the mutated functions.
PY_MUTANTS = {
    # name: (module, pin file, old, new)
    "e4m3_bias_8": ("fp8", "test_fp8_oracle.py", "np.exp2(e - 7.0)", "np.exp2(e - 8.0)"),
    "e4m3_ties_up": ("fp8", "test_fp8_oracle.py", "m = np.rint(an * np.exp2(3.0 - e))",
                     "m = np.floor(an * np.exp2(3.0 - e) + 0.5)"),
    "e4m3_no_saturation": ("fp8", "test_fp8_oracle.py",
                           "np.where((e > 8) | ((e == 8) & (m == 15)), 0x7E, code)", "code"),
    "e4m3_attention_without_sk": ("fp8", "test_fp8_oracle.py", "c = float(scale) * sq * sk",
                                  "c = float(scale) * sq"),
    "e4m3_descale_inverted": ("fp8", "test_fp8_oracle.py", "descale = a / np.float32(E4M3_MAX)",
                              "descale = np.float32(E4M3_MAX) / a"),
    "tvd_without_half": ("decision", "test_decision_oracle.py", "0.5 * float(np.sum(",
                         "float(np.sum("),
    "path_without_ancestors": ("decision", "test_decision_oracle.py",
                               "path[n] = path[gpar[n]] + float(", "path[n] = float("),
    "logprob_without_lse": ("decision", "test_decision_oracle.py",
                            "np.asarray(targets)[rows]] - lse", "np.asarray(targets)[rows]]"),
    "softmax_over_inner_nodes": ("decision", "test_decision_oracle.py",
                                 "if gpar[n] >= 0 and not has_child[n]]", "if gpar[n] >= 0]"),
}

PY_MIN_FAILED = 2


def _py_job(name):
    mod, pins, old, new = PY_MUTANTS[name]
    path = os.path.join(ROOT, "oracle", f"{mod}.py")
    assert open(path).read().count(old) == 1, "the mutation site must be unique"
    return ("import sys, pytest, oracle\n"
            f"import oracle.{mod} as m\n"
            "orig = dict(m.__dict__)\n"
            f"src = open({path!r}).read().replace({old!r}, {new!r})\n"
            "exec(compile(src, m.__file__, 'exec'), m.__dict__)\n"
            "for k, v in list(vars(oracle).items()):  # the package re-exports some functions\n"
            "    if k in orig and orig[k] is v and m.__dict__[k] is not v:\n"
            "        setattr(oracle, k, m.__dict__[k])\n"
            f"sys.exit(pytest.main(['-q', '-p', 'no:cacheprovider', 'tests/{pins}']))\n")


def _run_all(jobs):
    """Runs the child processes a few at a time (one oracle thread each) and
    returns per job the number of failed pins and the child's output."""
    from concurrent.futures import ThreadPoolExecutor
    env = dict(os.environ, OMP_NUM_THREADS="1")

    def run(code):
        p = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                           text=True, timeout=600)
        m = re.search(r"(\d+) failed", p.stdout)
        return (int(m.group(1)) if m else 0), p.stdout[-3000:] + p.stderr[-2000:]

    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futures = {name: ex.submit(run, code) for name, code in jobs.items()}
        return {name: f.result() for name, f in futures.items()}


@pytest.fixture(scope="module")
def c_runs():
    return _run_all({name: _c_job(name) for name in MUTANTS})


@pytest.fixture(scope="module")
def py_runs():
    return _run_all({name: _py_job(name) for name in PY_MUTANTS})


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_pins(name, c_runs):
    failed, log = c_runs[name]
    assert os.path.exists(os.path.join(ROOT, "oracle", "_build", "mutants", name, "liboracle.so")), log
    print(f"{name}: {failed} pins failed")
    assert failed >= MIN_FAILED, log


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_planted_mistake_fails_python_oracle_pins(name, py_runs):
    failed, log = py_runs[name]
    print(f"{name}: {failed} pins failed")
    assert failed >= PY_MIN_FAILED, log
