"""The pins are sensitive: each test here plants one plausible mistake in a copy of the
oracle (on the CPU, in a temporary directory) and runs the pins that guard that part of
it, which must fail.  Every mistake changes the oracle's results."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PINS = "test_oracle_pins.py"
SHARDED = "test_oracle_sharded.py"
BACKWARD = "test_oracle_backward.py"
DOCS = "test_oracle_docs.py"

MUTATIONS = [
    # (file, original text, planted mistake, pins that must catch it)
    ("msa_oracle.py", "return p[p <= t]", "return p[p < t]", PINS),                  # causal cut
    ("msa_oracle.py", "reshape(hkv, G, d).sum(axis=1)", "reshape(G, hkv, d).sum(axis=0)",
     PINS),                                                                          # head groups
    ("msa_oracle.py", "np.lexsort((j, -scores))", "np.lexsort((j, scores))", PINS),  # rank order
    ("msa_oracle.py", "np.lexsort((j, -scores))", "np.lexsort((-j, -scores))", PINS),  # ties
    ("msa_oracle.py", "/ (hi - lo)", "/ block", PINS),                               # ragged mean
    ("msa_oracle.py", "n_take = min(topk - 1, order.shape[0])",
     "n_take = min(topk, order.shape[0])", PINS),                                    # own block
    ("msa_oracle.py", "logits = scale * (q @ k.T)", "logits = (q @ k.T)", PINS),     # scale
    ("msa_oracle.py", "m[:, 0] + np.log(den[:, 0])", "np.log(den[:, 0])", PINS),     # lse
    # the parity gate: which rows must match the oracle's selection exactly
    ("msa_oracle.py", "first_left = float(scores_past[order[n_take]])",
     "first_left = float(scores_past[order[min(n_take + 1, order.shape[0] - 1)]])",
     PINS),                                                                          # cut + 1
    ("msa_oracle.py", "last = float(scores_past[order[n_take - 1]])",
     "last = float(scores_past[order[max(n_take - 2, 0)]])", PINS),                  # cut - 1
    ("msa_oracle.py", "first_left = float(scores[order[n_take]])",
     "first_left = float(scores[order[min(n_take + 1, order.shape[0] - 1)]])",
     PINS),                                                                          # decode cut
    ("msa_oracle.py", "den = max(abs(a), abs(b))", "den = abs(a)", PINS),            # gap scale
    ("msa_oracle.py", "else (a - b) / den", "else 0.0 * (a - b) / den", PINS),       # gap = 0
    ("msa_oracle.py", 'return float("inf")', "return 0.0", PINS),                    # none left
    ("msa_sharded.py", "lo, topk + 1)", "lo, topk)", SHARDED),                       # k+1 lists
    ("msa_sharded.py", "lo = r * base + min(r, extra)", "lo = r * base", SHARDED),   # ranges
    ("msa_sharded.py", "return O, m + np.log(den)", "return O, m", SHARDED),         # lse merge
    ("msa_sharded.py", "if lo <= j < hi]", "if lo <= j <= hi]", SHARDED),            # ownership
    ("msa_backward.py", "dS = P * (dP - (g * O)", "dS = P * (dP + (g * O)", BACKWARD),
    ("msa_backward.py", "dk = scale * (dS.T @ q)", "dk = (dS.T @ q)", BACKWARD),
    ("msa_backward.py", "dv = P.T @ g", "dv = P.T @ g[::-1]", BACKWARD),
    ("msa_backward.py", "np.add.at(dK[b, :, g], p, dk)", "dK[b, p, g] = dk", BACKWARD),
    ("msa_docs.py", "pos[a:b] = np.arange(b - a)", "pos[a:b] = np.arange(a, b)", DOCS),  # no reset
    ("msa_docs.py", "theta = base ** (-2.0 * i / d)", "theta = base ** (-1.0 * i / d)", DOCS),
    ("msa_docs.py", "[a * c - b * s, b * c + a * s]", "[a * c + b * s, b * c - a * s]",
     DOCS),                                                                          # direction
    ("msa_docs.py", "a, b = x[..., :half], x[..., half:]", "a, b = x[..., 0::2], x[..., 1::2]",
     DOCS),                                                                          # pairing
    ("msa_docs.py", "res = prefill_rows(Q[None, a:b], K[None, a:b], V[None, a:b]",
     "res = prefill_rows(Q[None, a:b], K[None, 0:b - a], V[None, a:b]", DOCS),       # wrong doc
]


# the copy's conftest only puts the copy first on the path (no CUDA probing)
_CONFTEST = """import os, sys
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
"""


def _copy_and_run(tmp_path, pins, fname=None, old=None, new=None):
    for d in ("oracle", "msa_inputs"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__"))
    (tmp_path / "tests").mkdir()
    shutil.copy(os.path.join(ROOT, "tests", pins), tmp_path / "tests" / pins)
    (tmp_path / "tests" / "conftest.py").write_text(_CONFTEST)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), tmp_path / "tests" / "golden")
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    if fname is not None:
        path = tmp_path / "oracle" / fname
        src = path.read_text()
        assert old in src, f"mutation anchor missing: {old}"
        path.write_text(src.replace(old, new, 1))
    env = {k: v for k, v in os.environ.items() if k != "PYTHONPATH"}
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", f"tests/{pins}"],
                          cwd=tmp_path, env=env, capture_output=True, text=True, timeout=600)


@pytest.mark.parametrize("pins", [PINS, SHARDED, BACKWARD, DOCS])
def test_unchanged_copy_passes(tmp_path, pins):
    """Control: the copied pins pass on the unchanged oracle, so a failure below is the
    planted mistake's doing."""
    r = _copy_and_run(tmp_path, pins)
    assert r.returncode == 0, r.stdout[-1500:]


@pytest.mark.parametrize("fname,old,new,pins", MUTATIONS,
                         ids=[f"{m[0]}:{i}" for i, m in enumerate(MUTATIONS)])
def test_pins_catch_a_planted_mistake(tmp_path, fname, old, new, pins):
    r = _copy_and_run(tmp_path, pins, fname, old, new)
    assert r.returncode == 1, (r.returncode, r.stdout[-1500:])   # 1 = some test failed
