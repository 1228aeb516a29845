"""The oracle pins are strong enough: each plausible mistake, planted in a temporary copy of
the oracle (CPU only), makes at least one test of tests/test_oracle_pins.py fail, while the
unmodified copy passes them all."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle")

MUTATIONS = {
    "pool mean instead of sum": (".reshape(L // stride, stride, d).sum(axis=1)",
                                 ".reshape(L // stride, stride, d).mean(axis=1)"),
    "diagonal stride dropped": ("valid = j <= i", "valid = j < i"),
    "shift ignored": ("return (h + shift) % stride", "return h % stride"),
    "GQA by modulo": ("return h // (heads_q // heads_kv)", "return h % heads_kv"),
    "no 1/m": (".sum(axis=(0, 2)) / m", ".sum(axis=(0, 2))"),
    "ties by larger J": ('order = np.argsort(-a, kind="stable")',
                         "order = np.lexsort((-np.arange(a.size), -a))"),
    "strict comparison": ("hit = np.nonzero(csum >= tau * total)[0]",
                          "hit = np.nonzero(csum > tau * total)[0]"),
    "causal mask off by one": ("allowed = keys[None, :] <= t[:, None]",
                               "allowed = keys[None, :] < t[:, None]"),
    "diagonal not kept": ("kept.add(I)                                     # diagonal always kept",
                          "pass"),
    "scale dropped": ("return scale * (qhat @ kbar[: (I + 1) * m].T)",
                      "return (qhat @ kbar[: (I + 1) * m].T)"),
    "sampled rows reversed": ("qhat = q[rows].astype(np.float64)",
                              "qhat = q[rows].astype(np.float64)[::-1]"),
    "xattn main diagonal": ("z += qs[:, t, :] @ ks[:, stride - 1 - t, :].T",
                            "z += qs[:, t, :] @ ks[:, t, :].T"),
    "xattn scale dropped": ("    return scale * z\n", "    return z\n"),
}


def _run_pins(tmp, mutation=None):
    dst = os.path.join(tmp, "oracle")
    shutil.rmtree(dst, ignore_errors=True)
    shutil.copytree(SRC, dst, ignore=shutil.ignore_patterns("__pycache__"))
    if mutation is not None:
        path = os.path.join(dst, "rr_oracle.py")
        text = open(path).read()
        assert mutation[0] in text, mutation[0]
        open(path, "w").write(text.replace(mutation[0], mutation[1]))
    env = dict(os.environ, RRA_ORACLE_OVERRIDE=tmp, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout


def test_unmodified_copy_passes(tmp_path):
    rc, out = _run_pins(str(tmp_path))
    assert rc == 0, out[-2000:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    rc, out = _run_pins(str(tmp_path), MUTATIONS[name])
    assert rc != 0, f"mistake '{name}' passed every pin:\n{out[-2000:]}"
