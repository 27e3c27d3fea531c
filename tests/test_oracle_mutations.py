"""Plant a mistake in a copy of the oracle (on the CPU) and check that a pin catches it.

Each case copies ``oracle/`` to a temporary directory, edits one line of the
copy, and runs the pin file that should fail against it in a subprocess.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = [
    # (file, original text, planted mistake, pin file)
    ("pctree.py", "Z = L_d[None, :] + markov", "Z = L_d[None, :] - markov",
     "test_oracle_pctree.py"),                                     # wrong sign
    ("pctree.py", "markov = E[toks] @ W", "markov = E[toks * 0] @ W",
     "test_oracle_pctree.py"),                                     # wrong parent index
    ("pctree.py", "p.s + logpi[i, v], p.path", "logpi[i, v], p.path",
     "test_oracle_pctree.py"),                                     # dropped prefix term
    ("pctree.py", "for v in order[i]]", "for v in order[i][::-1]]",
     "test_oracle_pctree.py"),                                     # top-k from the wrong end
    ("pctree.py", "key=lambda c: (-c.s, c.depth, c.path)", "key=lambda c: (c.s, c.depth, c.path)",
     "test_oracle_pctree.py"),                                     # global top-N reversed
    ("pctree.py", "score_parents(L[d - 1],", "score_parents(L[d % D],",
     "test_oracle_pctree.py"),                                     # depth off by one
    ("pctree.py", "cands.sort(key=lambda c: (-c.s, c.path))", "cands.sort(key=lambda c: (c.path,))",
     "test_oracle_pctree.py"),                                     # beam by path, not score
    ("pctree.py", "kept = sorted(_near_tie_keep(cands, beam,",
     "kept = sorted(_near_tie_keep(cands[::-1], beam,",
     "test_oracle_pctree.py"),                                     # beam keeps the worst
    ("numerics.py", "lse = m_safe + np.log(", "lse = np.log(",
     "test_oracle_numerics.py"),                                   # dropped max shift
    ("caddtree.py", "(1.0 + phi + p) / C(n + 1) <= (1.0 + phi) / C(n)",
     "(phi + p) / C(n + 1) <= (phi + 1e-300) / C(n)", "test_oracle_caddtree.py"),   # dropped 1
    ("caddtree.py", "push_child(pidx, rank + 1)", "push_child(pidx, rank + 2)",
     "test_oracle_caddtree.py"),                                   # skipped sibling
    ("caddtree.py", "return C_d + a + b * ell + c * n + e * n * n",
     "return C_d + a + b * ell + c * n + e * n", "test_oracle_caddtree.py"),   # wrong power
    ("verify.py", "tok[b, c] == am[b, u]", "tok[b, c] == am[b, c]",
     "test_oracle_verify.py"),                                     # wrong node index
    ("verify.py", "<< np.uint32(j % 32)", "<< np.uint32(j % 31)",
     "test_oracle_verify.py"),                                     # wrong bit position
    ("verify.py", "corr[b] = am[b, u]", "corr[b] = am[b, 0]",
     "test_oracle_verify.py"),                                     # correction from the root
]


def _run_mutant(tmp_path, i, fname, old, new, pin):
    base = tmp_path / f"m{i}"
    dst = base / "oracle"
    shutil.copytree(os.path.join(ROOT, "oracle"), dst,
                    ignore=shutil.ignore_patterns("__pycache__"))
    src = (dst / fname).read_text()
    assert src.count(old) == 1, f"mutation anchor not unique in {fname}: {old}"
    (dst / fname).write_text(src.replace(old, new))
    env = dict(os.environ)
    env["PYTHONPATH"] = os.pathsep.join([str(base), ROOT, env.get("PYTHONPATH", "")])
    env["PYTHONDONTWRITEBYTECODE"] = "1"
    code = ("import sys, pytest; import oracle; "
            f"assert oracle.__file__.startswith({str(base)!r}), oracle.__file__; "
            "sys.exit(pytest.main(['-x', '-q', '-p', 'no:cacheprovider', '-m', 'not gpu', "
            f"{os.path.join(ROOT, 'tests', pin)!r}]))")
    run = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True,
                         text=True, cwd=str(base), timeout=600)
    return run.returncode, run.stdout[-1500:] + run.stderr[-1500:]


def test_planted_mistakes_are_caught(tmp_path):
    workers = max(1, min(len(MUTATIONS), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futs = [ex.submit(_run_mutant, tmp_path, i, *m) for i, m in enumerate(MUTATIONS)]
        results = [f.result() for f in futs]
    for (fname, old, new, pin), (rc, out) in zip(MUTATIONS, results):
        # rc 1: tests failed; anything else (import error, usage error) is not a catch
        assert rc == 1, f"{fname}: pin {pin} did not catch '{new}' (rc={rc})\n{out}"
