"""The oracle's pins against planted mistakes (CPU).

Each mutant is a copy of oracle/moe_oracle.c with one plausible mistake - a
reversed tie rule, a dropped term, a wrong sign, index or operand, a
transposition - built into its own library and loaded in place of the
oracle by a run of tests/test_oracle_pins.py.  Every mutant must make at
least one pin fail, so none of these mistakes could sit in the oracle
unnoticed.  The unmutated copy, built the same way, must pass: the harness
itself is sound.  The mistakes are planted in copies on the CPU only; the
committed oracle is never changed."""
import atexit
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")
_OUT = []


def _out():
    """A temporary directory, outside the source tree, for the mutated copies
    and their libraries; removed when the test process exits."""
    if not _OUT:
        d = tempfile.mkdtemp(prefix="moe_oracle_mutants_")
        atexit.register(shutil.rmtree, d, True)
        _OUT.append(d)
    return _OUT[0]

# (name, exact text in the oracle, its replacement)
MUTANTS = [
    ("topk_ties_to_higher_index",
     "if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] >= l[best]) best = e;"),
    ("gate_renormalisation_inverted", "        if (norm_topk) {", "        if (!norm_topk) {"),
    ("gate_of_wrong_slot",
     "gate[t * k + j] = (float)(exp((double)l[expert_idx[t * k + j]] - m) / denom);",
     "gate[t * k + j] = (float)(exp((double)l[expert_idx[t * k]] - m) / denom);"),
    ("router_weight_transposed",
     "load_elem(W_r, dtype, (int64_t)e * d + c)", "load_elem(W_r, dtype, (int64_t)c * E + e)"),
    ("capacity_rounded_down", "return (int64_t)ceil(capacity_factor", "return (int64_t)floor(capacity_factor"),
    ("keeps_one_past_capacity", "kept[s] = rank < capacity;", "kept[s] = rank <= capacity;"),
    ("dropped_count_sign", "drop += load[e] - counts[e];", "drop += counts[e] - load[e];"),
    ("offsets_from_load_before_capacity",
     "offsets[e + 1] = offsets[e] + counts[e];", "offsets[e + 1] = offsets[e] + load[e];"),
    ("group_row_wrong_token", "if (has) { row_token[R] = (int32_t)t; ++R; }",
     "if (has) { row_token[R] = (int32_t)(T - 1 - t); ++R; }"),
    ("swiglu_operands_swapped", "v = silu(a) * b;", "v = silu(b) * a;"),
    ("gelu_without_sqrt2", "erf(z / sqrt(2.0))", "erf(z)"),
    ("bf16_truncates", "double r = rint(x * scale) / scale;", "double r = trunc(x * scale) / scale;"),
    ("down_projection_transposed",
     "acc += load_elem(W2, dtype, wrow + f) * h[f];",
     "acc += load_elem(W2, dtype, (e * F + f) * (int64_t)d + c) * h[f];"),
    ("combine_gate_of_wrong_slot",
     "acc += (double)gate[t * k + j] * load_elem(Y, dtype, (int64_t)r * d + c);",
     "acc += (double)gate[t * k] * load_elem(Y, dtype, (int64_t)r * d + c);"),
    ("precombine_first_slot_only", "for (int q = j; q < k; ++q) {", "for (int q = j; q < j + 1; ++q) {"),
    ("group_rows_counted_per_slot",
     "if (first) acc += load_elem(Y_g, dtype, (int64_t)r * d + c);",
     "acc += load_elem(Y_g, dtype, (int64_t)r * d + c);"),
    ("expert_choice_ties_to_higher_token", "return (ta > tb) - (ta < tb);", "return (ta < tb) - (ta > tb);"),
    ("logsumexp_without_max", "double lse = m + log(s);", "double lse = log(s);"),
    ("expert_choice_gate_is_log",
     "ec_gate[(int64_t)e * C + i] = (float)exp(key[(int64_t)order[i] * E + e]);",
     "ec_gate[(int64_t)e * C + i] = (float)(key[(int64_t)order[i] * E + e]);"),
    ("coselect_without_diagonal",
     "cosel[(int64_t)expert_idx[t * k + i] * E + expert_idx[t * k + j]] += 1;",
     "cosel[(int64_t)expert_idx[t * k + i] * E + expert_idx[t * k + j]] += (i != j);"),
    ("transition_transposed",
     "trans[(int64_t)idx1[t * k1 + i] * E + idx2[t * k2 + j]] += 1;",
     "trans[(int64_t)idx2[t * k2 + j] * E + idx1[t * k1 + i]] += 1;"),
    ("local_share_wrong_home", "int64_t home = t * G / T;", "int64_t home = (t * G / T + 1) % G;"),
    ("placement_seed_ties_to_higher_index",
     "if (group_of_expert[x] < 0 && (seed < 0 || mass[x] > mass[seed])) seed = x;",
     "if (group_of_expert[x] < 0 && (seed < 0 || mass[x] >= mass[seed])) seed = x;"),
    ("affinity_transposed",
     "+= trans[(int64_t)a * E + b];", "+= trans[(int64_t)b * E + a];"),
    ("home_ties_to_higher_group", "if (g == 0 || v > best_v)", "if (g == 0 || v >= best_v)"),
    ("router_logit_drops_last_term",
     "for (int c = 0; c < d; ++c) acc += load_elem(x, dtype", "for (int c = 0; c < d - 1; ++c) acc += load_elem(x, dtype"),
    ("topk_slot_order_reversed", "expert_idx[t * k + j] = best;", "expert_idx[t * k + (k - 1 - j)] = best;"),
    ("softmax_denominator_drops_last_expert",
     "for (int e = 0; e < E; ++e) denom += exp((double)l[e] - m);",
     "for (int e = 0; e < E - 1; ++e) denom += exp((double)l[e] - m);"),
    ("row_token_is_the_slot", "row_token[r] = (int32_t)(s / k);", "row_token[r] = (int32_t)(s % k);"),
    ("group_layout_ignores_capacity",
     "if (kept[s] && group_of_expert[expert_idx[s]] == g)", "if (group_of_expert[expert_idx[s]] == g)"),
    ("gelu_without_half", "return 0.5 * z * (1.0 + erf(", "return z * (1.0 + erf("),
    ("hidden_not_rounded_to_bf16", "h[f] = (dtype == ORC_BF16) ? round_to_bf16(v) : v;", "h[f] = v;"),
    ("combine_reads_row_0_for_drops",
     "int32_t r = row_map[t * k + j];\n                if (r < 0) continue;",
     "int32_t r = row_map[t * k + j];\n                if (r < 0) r = 0;"),
    ("expert_choice_combine_without_gate", "acc += (double)ec_gate[r] * load_elem", "acc += load_elem"),
    ("local_fraction_per_token", "return T > 0 ? (double)local / (double)(T * k) : 0.0;",
     "return T > 0 ? (double)local / (double)T : 0.0;"),
    ("placement_forgets_earlier_members",
     "aff[x] += cosel[(int64_t)x * E + best];", "aff[x] = cosel[(int64_t)x * E + best];"),
    ("home_from_last_expert_only",
     "for (int i = 0; i < k1; ++i) v += affinity", "for (int i = 0; i < k1; ++i) v = affinity"),
    ("bf16_subnormal_spacing_ignored", "if (ex < -125) ex = -125;", "if (ex < -125) ex = ex;"),
]


# mistakes in the oracle's Python layer (argument marshalling and the per-token layer compositions)
PY_MUTANTS = [
    ("py_norm_topk_flag_inverted", "k, int(norm_topk), idx.ctypes.data", "k, int(not norm_topk), idx.ctypes.data"),
    ("py_capacity_k_and_E_swapped", "oracle_capacity(float(capacity_factor), T, k, E)",
     "oracle_capacity(float(capacity_factor), T, E, k)"),
    ("py_layer_gate_of_slot_0", "np.float64(gate[tokens[owner[n]], slot[n]])", "np.float64(gate[tokens[owner[n]], 0])"),
    ("py_layer_shared_subtracted", "        out += ys\n", "        out -= ys\n"),
    ("py_group_layer_row_per_slot", "            if g not in seen:\n", "            if True:\n"),
    ("py_expert_choice_gates_reversed", "g = _c(ec_gate, np.float32).reshape(-1)",
     "g = _c(ec_gate, np.float32).reshape(-1)[::-1].copy()"),
    ("py_local_count_ignores_home", "        hp = home.ctypes.data\n", "        hp = None\n"),
    ("py_local_fraction_one_group_more", "goe.ctypes.data, G))", "goe.ctypes.data, G + 1))"),
    ("py_expert_choice_on_negated_logits",
     "def route_ec(logits: np.ndarray, C: int):\n    \"\"\"ExpertChoiceRouter: (ec_token [E,C], ec_gate [E,C], tok_ptr [T+1], "
     "tok_row [E*C]).\"\"\"\n    lg = _c(logits, np.float32)",
     "def route_ec(logits: np.ndarray, C: int):\n    \"\"\"ExpertChoiceRouter: (ec_token [E,C], ec_gate [E,C], tok_ptr [T+1], "
     "tok_row [E*C]).\"\"\"\n    lg = _c(-np.asarray(logits), np.float32)"),
]
PY_SRC = os.path.join(ROOT, "oracle", "oracle.py")


def _build(name, text):
    c = os.path.join(_out(), name + ".c")
    so = os.path.join(_out(), "lib" + name + ".so")
    with open(c, "w") as f:
        f.write(text)
    subprocess.run(O.CC_FLAGS + [c, "-o", so, "-lm"], check=True, capture_output=True)
    return so


def _pins(so):
    env = dict(os.environ, MOE_ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-q",
                        "-x", "-p", "no:cacheprovider", "-m", "not gpu"], capture_output=True, text=True, cwd=ROOT,
                       env=env, timeout=900)
    return r.returncode, r.stdout[-600:]


def _py_package(name, text):
    """A copy of the oracle package whose oracle.py is `text`; it builds its
    own C library next to it on first use."""
    root = os.path.join(_out(), name)
    pkg = os.path.join(root, "oracle")
    os.makedirs(pkg, exist_ok=True)
    for f in ("__init__.py", "moe_oracle.c"):
        with open(os.path.join(ROOT, "oracle", f)) as a, open(os.path.join(pkg, f), "w") as b:
            b.write(a.read())
    with open(os.path.join(pkg, "oracle.py"), "w") as b:
        b.write(text)
    return root


def _py_pins(root):
    """The pin tests with the copied package first on the import path."""
    env = dict(os.environ, PYTHONPATH=ROOT)
    env.pop("MOE_ORACLE_LIB", None)
    which = subprocess.run([sys.executable, "-c", "import oracle; print(oracle.__file__)"], capture_output=True,
                           text=True, cwd=root, env=env, timeout=300)
    assert which.stdout.strip().startswith(root), which.stdout + which.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-q",
                        "-x", "-p", "no:cacheprovider", "-m", "not gpu"], capture_output=True, text=True, cwd=root,
                       env=env, timeout=900)
    return r.returncode, r.stdout[-600:]


def test_every_planted_mistake_in_the_python_layer_fails_a_pin():
    src = open(PY_SRC).read()
    jobs = {"py_unmutated": src}
    for name, old, new in PY_MUTANTS:
        assert src.count(old) == 1, "mutation site of %s is not unique in oracle.py" % name
        jobs[name] = src.replace(old, new)
    roots = {n: _py_package(n, t) for n, t in jobs.items()}
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = dict(zip(roots, ex.map(_py_pins, roots.values())))
    rc, tail = results.pop("py_unmutated")
    assert rc == 0, "the unmutated copy fails its pins:\n" + tail
    survivors = {n: rc for n, (rc, _) in results.items() if rc != 1}
    assert not survivors, "mutants not caught by a failing pin: %s" % survivors


def test_every_planted_mistake_fails_a_pin():
    src = open(SRC).read()
    jobs = {"unmutated": src}
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, "mutation site of %s is not unique in the oracle" % name
        jobs[name] = src.replace(old, new)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        libs = dict(zip(jobs, ex.map(lambda kv: _build(*kv), jobs.items())))
        results = dict(zip(libs, ex.map(_pins, libs.values())))
    rc, tail = results.pop("unmutated")
    assert rc == 0, "the unmutated copy fails its pins:\n" + tail
    survivors = {n: (rc, tail) for n, (rc, tail) in results.items() if rc != 1}
    assert not survivors, "mutants not caught by a failing pin: %s" % {n: v[0] for n, v in survivors.items()}
