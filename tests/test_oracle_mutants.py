"""The oracle's pins catch plausible mistakes. Each case plants one mistake in a temporary copy of
``oracle/`` (never in the repository's files) and runs the pin tests against that copy. The
mutated suite must fail, and the unmutated copy must pass, so every failure comes from the mistake.

Mistakes planted: a wrong default scale, an interleaved head-to-group map, a flipped causal mask,
a window that is off by one, no maximum subtraction, no normalisation, a wrong log-sum-exp, a
dropped scale, no length slice, a merge without rescaling, a backward without the row term D, a
dK that loses its scale, an MLA value width that includes the rotary part, a page index taken
from the wrong table column, and an append one row late."""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_TESTS = ["test_oracle_pins.py", "test_oracle_window.py", "test_oracle_backward.py",
             "test_oracle_mla.py", "test_oracle_paged.py"]

# (oracle file, exact text, replacement, pin test that must fail)
MUTANTS = [
    ("attention_ref.py", "scale = 1.0 / np.sqrt(d_h)", "scale = 1.0 / d_h", "test_oracle_pins.py"),
    ("attention_ref.py", "return a // r", "return a % h_kv", "test_oracle_pins.py"),
    ("attention_ref.py", "visible = j[None, :] <= q_pos[:, None]", "visible = j[None, :] >= q_pos[:, None]",
     "test_oracle_pins.py"),
    ("attention_ref.py", "visible &= j[None, :] > q_pos[:, None] - window",
     "visible &= j[None, :] >= q_pos[:, None] - window", "test_oracle_window.py"),
    ("attention_ref.py", "m = S.max(axis=1, keepdims=True)", "m = np.zeros((S.shape[0], 1))",
     "test_oracle_pins.py"),
    ("attention_ref.py", "P = E / denom", "P = E", "test_oracle_pins.py"),
    ("attention_ref.py", "lse = m[:, 0] + np.log(denom[:, 0])", "lse = m[:, 0] + denom[:, 0]",
     "test_oracle_pins.py"),
    ("attention_ref.py", "S = (q_rows @ k.T) * scale", "S = (q_rows @ k.T)", "test_oracle_pins.py"),
    ("attention_ref.py", "k = np.asarray(k, dtype=np.float64)[:kv_len]", "k = np.asarray(k, dtype=np.float64)",
     "test_oracle_pins.py"),
    ("online_softmax.py", "u = alpha * u + w @ v", "u = u + w @ v", "test_oracle_pins.py"),
    ("online_softmax.py", "fa * np.asarray(u_a) + fb * np.asarray(u_b)", "np.asarray(u_a) + np.asarray(u_b)",
     "test_oracle_pins.py"),
    ("backward.py", "dS = P * (dP - D[:, None])", "dS = P * dP", "test_oracle_backward.py"),
    ("backward.py", "dK[b, g, :n] += scale * (dS.T @ q[b, a])", "dK[b, g, :n] += dS.T @ q[b, a]",
     "test_oracle_backward.py"),
    ("mla.py", "O[b] = (E / den) @ rows[:, :d_v]", "O[b] = (E / den) @ rows[:, -d_v:]", "test_oracle_mla.py"),
    ("paged.py", "page = int(block_table[b, t0 // page_size])", "page = int(block_table[b, t0 // page_size - 1])",
     "test_oracle_paged.py"),
    ("kv_append_ref.py", "k_cache[b, :, p:p + S_new, :] = k_new[b]", "k_cache[b, :, p + 1:p + 1 + S_new, :] = k_new[b]",
     "test_oracle_pins.py"),
]


def _copy_tree(dst):
    """The oracle, the input generators and the pin tests (with their fixtures) under ``dst``."""
    for d in ("oracle", "workloads"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(dst, d),
                        ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(dst, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for f in ["conftest.py", "_tol.py"] + PIN_TESTS:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))


def _run(dst, test):
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    env.pop("PYTHONPATH", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join("tests", test)], cwd=dst, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def pristine(tmp_path_factory):
    dst = str(tmp_path_factory.mktemp("oracle_copy"))
    _copy_tree(dst)
    return dst


def _workers():
    return max(1, min(8, (os.cpu_count() or 2) // 2))


def test_unmutated_copy_passes(pristine):
    import concurrent.futures

    tests = sorted(set(m[3] for m in MUTANTS))
    with concurrent.futures.ThreadPoolExecutor(_workers()) as ex:
        results = list(ex.map(lambda t: _run(pristine, t), tests))
    for (rc, out), test in zip(results, tests):
        assert rc == 0, f"{test} fails on the unmutated copy\n{out}"


def _caught(base, i, fname, old, new, test):
    dst = os.path.join(base, f"mutant{i}")
    os.makedirs(dst)
    _copy_tree(dst)
    path = os.path.join(dst, "oracle", fname)
    src = open(path, encoding="utf-8").read()
    if src.count(old) != 1:
        return f"mutation target not found once in {fname}: {old}"
    open(path, "w", encoding="utf-8").write(src.replace(old, new))
    rc, out = _run(dst, test)
    return None if rc != 0 else f"the pins did not catch: {fname}: {old} -> {new}\n{out}"


def test_pins_catch_every_mutant(tmp_path):
    """Each mutant runs in its own copy; the copies run side by side (separate processes)."""
    import concurrent.futures

    with concurrent.futures.ThreadPoolExecutor(_workers()) as ex:
        futs = [ex.submit(_caught, str(tmp_path), i, *m) for i, m in enumerate(MUTANTS)]
        problems = [f.result() for f in futs]
    problems = [p for p in problems if p]
    assert not problems, "\n".join(problems)
