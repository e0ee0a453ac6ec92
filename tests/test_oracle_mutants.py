"""Mutation check of the oracle's pins (CPU).

Each mutant below is a plausible slip in oracle/indexcache_oracle.py (a
dropped term, a wrong sign, an off-by-one causal bound, a reversed
tie-break, a missing scale, swapped operands, a broken F/S branch).  The
mutated module is imported in a child process in place of the real one and
tests/test_oracle_pins.py is run against it: every mutant must make at least
one pin fail, and the unmutated copy must pass, so the pins are shown to
catch these mistakes rather than assumed to.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "indexcache_oracle.py")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, text in the oracle, replacement); each text must occur exactly once
MUTANTS = [
    ("indexer: ReLU dropped",
     "relu = np.maximum(dots, 0.0)", "relu = dots"),
    ("indexer: ReLU keeps the negative part",
     "relu = np.maximum(dots, 0.0)", "relu = np.minimum(dots, 0.0)"),
    ("indexer: head weights ignored",
     "out[b, r, : t + 1] = wv[b, i] @ relu", "out[b, r, : t + 1] = relu.sum(axis=0)"),
    ("indexer: a row does not see its own key",
     "dots = q[b, i] @ k[b, : t + 1].T", "dots = q[b, i] @ np.concatenate([k[b, :t], 0 * k[b, :1]]).T"),
    ("indexer: q_start ignored",
     "            t = q_start + i\n            dots", "            t = i\n            dots"),
    ("fp8: scale not applied",
     "return v * s.reshape(s.shape + (1,) * (v.ndim - s.ndim))", "return v"),
    ("fp8: subnormals decoded as normals",
     "out = np.where(e == 0, sub, nrm)", "out = nrm"),
    ("fp8: exponent bias 8",
     "np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))",
     "np.ldexp(1.0 + m / 8.0, (e - 8).astype(np.int64))"),
    ("top-k: ties to the larger position",
     "order = np.lexsort((pos, -cand))", "order = np.lexsort((-pos, -cand))"),
    ("top-k: positions in score order",
     "chosen = np.sort(pos[order[:take]])", "chosen = pos[order[:take]]"),
    ("top-k: one candidate too few",
     "take = min(k, t + 1)", "take = min(k, t)"),
    ("top-k: padded with 0",
     "out = np.full((B, n_rows, k), -1, dtype=np.int32)",
     "out = np.full((B, n_rows, k), 0, dtype=np.int32)"),
    ("attention: softmax scale missing",
     "logits = scale * (qv[b, i] @ Kv[b, J].T)", "logits = (qv[b, i] @ Kv[b, J].T)"),
    ("attention: -1 entries used as keys",
     "J = ix[b, i][ix[b, i] >= 0].astype(np.int64)", "J = ix[b, i].astype(np.int64)"),
    ("attention: keys used as values",
     "out[b, i] = p @ Vv[b, J]", "out[b, i] = p @ Kv[b, J][:, : Vv.shape[-1]]"),
    ("attention: softmax taken over heads",
     "p = e / e.sum(axis=1, keepdims=True)", "p = e / e.sum(axis=0, keepdims=True)"),
    ("dense attention: strictly causal",
     "mask = s <= t", "mask = s < t"),
    ("stack: S layers run their own indexer",
     '        if kind == "F":\n            sc = indexer_scores',
     '        if True:\n            sc = indexer_scores'),
    ("stack: S layers reuse the first F layer",
     "            idx_cache = topk_indices(sc, q_start, k, rows=rows)",
     "            idx_cache = topk_indices(sc, q_start, k, rows=rows) if idx_cache is None "
     "else idx_cache"),
    ("stack: a leading S layer is accepted",
     'if n_layers > 0 and pattern[0] != "F":', "if False:"),
]

_DRIVER = r"""
import sys
sys.path.insert(0, sys.argv[1])
sys.path.append(sys.argv[2])
import oracle
assert oracle.__file__.startswith(sys.argv[1]), oracle.__file__
import pytest
sys.exit(pytest.main([sys.argv[3], "-x", "-q", "-p", "no:cacheprovider"]))
"""


def _run_pins(workdir, source):
    pkg = os.path.join(workdir, "oracle")
    os.makedirs(pkg)
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), pkg)
    with open(os.path.join(pkg, "indexcache_oracle.py"), "w") as f:
        f.write(source)
    env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    run = subprocess.run([sys.executable, "-c", _DRIVER, workdir, ROOT, PINS], cwd=workdir,
                         capture_output=True, text=True, timeout=600, env=env)
    return run.returncode, run.stdout[-2000:]


def test_every_mutant_fails_a_pin_and_the_original_passes(tmp_path):
    original = open(SRC).read()
    jobs = [("original", original)]
    for name, old, new in MUTANTS:
        assert original.count(old) == 1, name
        jobs.append((name, original.replace(old, new)))
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        futs = {name: ex.submit(_run_pins, str(tmp_path / ("m%02d" % n)), src)
                for n, (name, src) in enumerate(jobs)}
        results = {name: f.result() for name, f in futs.items()}
    rc, out = results.pop("original")
    assert rc == 0, "unmutated oracle copy fails its pins:\n" + out
    survivors = [name for name, (rc, _) in results.items() if rc == 0]
    assert not survivors, "mutants no pin catches: %s" % survivors
    # a crash at import would also give a non-zero code: each mutant must
    # fail a test, not the collection
    crashed = [name for name, (rc, out) in results.items() if "failed" not in out]
    assert not crashed, "mutants that failed to run: %s" % crashed
