"""The oracle's pins must catch plausible mistakes. Each case plants one mistake in a copy
of the oracle (never in the oracle itself), runs the pin tests against that copy in a
subprocess and expects them to fail: a dropped bias, a flipped residual sign, a transposed
weight, the wrong tie rule, the wrong head slice or GQA map, a missing scale, a dropped
residual, the tanh GELU, an ignored exact tail, a block score that sums instead of averaging,
a block selection that breaks ties upwards, block means over an unclipped last block, a
quantiser that floors or uses four steps or the wrong bit order, a GELU derivative without
its x phi term, a flipped or mis-scaled gradient, a W1 gradient from the wrong rows, an
untrained b2, a fitting step that climbs.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle", "lowram_oracle.py")

MUTATIONS = {
    "residual sign": ("val[l, h] = round_storage(v[sel] - vh[sel], dtype)",
                      "val[l, h] = round_storage(vh[sel] - v[sel], dtype)"),
    "b1 dropped": ("u = kt @ np.asarray(W1, np.float64).T + np.asarray(b1, np.float64)",
                   "u = kt @ np.asarray(W1, np.float64).T"),
    "W2 layout": ("gelu(u) @ np.asarray(W2, np.float64).T",
                  "gelu(u) @ np.asarray(W2, np.float64).reshape(np.asarray(W2).shape[::-1])"),
    "b2 dropped": ("        v = v + np.asarray(b2, np.float64)", "        v = v + 0.0"),
    "ties to the higher index": ("order = np.lexsort((np.arange(T), -e))", "order = np.lexsort((-np.arange(T), -e))"),
    "head slice": ("c0 = (layer * n_kv_heads + head) * head_dim", "c0 = (head * n_kv_heads + layer) * head_dim"),
    "scale missing": ("s = (kt @ q[hq]) * scale", "s = (kt @ q[hq])"),
    "GQA map": ("hq = h * G + g", "hq = g * n_kv_heads + h"),
    "residual not added": ("v = v + r_full[S]", "v = v"),
    "tanh GELU": ("return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))",
                  "return 0.5 * x * (1.0 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))"),
    "tail ignored": ("            kt = np.concatenate([kt, np.asarray(tail_K[h], np.float64)])\n"
                     "            v = np.concatenate([v, np.asarray(tail_V[h], np.float64)])",
                     "            pass"),
    "block score sums": ("kbar = kt[j * block:min(T, (j + 1) * block)].mean(axis=0)",
                         "kbar = kt[j * block:min(T, (j + 1) * block)].sum(axis=0) / block"),
    "block ties upwards": ("order = np.lexsort((np.arange(scores.shape[1]), -scores[h]))",
                           "order = np.lexsort((-np.arange(scores.shape[1]), -scores[h]))"),
    "block means over a full block": ("out[j] = A[j * block:min(T, (j + 1) * block)].mean(axis=0)",
                                      "out[j] = A[j * block:min(T, (j + 1) * block)].sum(axis=0) / block"),
    "quantiser floors": ("codes[i] = np.clip(np.rint(t.astype(np.float32)), 0, 3).astype(np.uint8)",
                         "codes[i] = np.clip(np.floor(t.astype(np.float32)), 0, 3).astype(np.uint8)"),
    "quantiser four steps": ("st = np.float32(np.float32(h - l) / np.float32(3.0))",
                             "st = np.float32(np.float32(h - l) / np.float32(4.0))"),
    "code bit order": ("return (c4[..., 0] | (c4[..., 1] << 2) | (c4[..., 2] << 4) | (c4[..., 3] << 6)).astype(np.uint8)",
                       "return (c4[..., 3] | (c4[..., 2] << 2) | (c4[..., 1] << 4) | (c4[..., 0] << 6)).astype(np.uint8)"),
    "GELU derivative without x phi": ("    return Phi + x * phi", "    return Phi"),
    "gradient sign": ("dv = 2.0 * (vh - v) / v.size", "dv = 2.0 * (v - vh) / v.size"),
    "loss averaged over tokens only": ("dv = 2.0 * (vh - v) / v.size", "dv = 2.0 * (vh - v) / v.shape[0]"),
    "W1 gradient from the wrong side": ('out = {"W_lin": dv.T @ kt, "W1": du.T @ kt,',
                                        'out = {"W_lin": dv.T @ kt, "W1": (du.T @ kt) * 0.0 + du.T @ kt[::-1],'),
    "b2 not trained": ('        out["b2"] = dv.sum(axis=0)', '        out["b2"] = 0.0 * dv.sum(axis=0)'),
    "fit step ascends": ("            p[n] = p[n] - lr * d", "            p[n] = p[n] + lr * d"),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(ORACLE).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {name}"
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), pkg / "__init__.py")
    (pkg / "lowram_oracle.py").write_text(src.replace(old, new))
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([str(tmp_path), ROOT]))
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        "-q", "-x", "-p", "no:cacheprovider"], cwd=str(tmp_path), env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"the pins did not catch: {name}\n{r.stdout[-2000:]}"


def test_unmutated_copy_passes(tmp_path):
    """The same harness on an unchanged copy passes, so a failure above is the mutation's."""
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), pkg / "__init__.py")
    shutil.copy(ORACLE, pkg / "lowram_oracle.py")
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([str(tmp_path), ROOT]))
    where = subprocess.run([sys.executable, "-c", "import oracle.lowram_oracle as o; print(o.__file__)"],
                           cwd=str(tmp_path), env=env, capture_output=True, text=True, timeout=300)
    assert where.stdout.strip().startswith(str(tmp_path)), where.stdout  # the copy is what gets imported
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        "-q", "-p", "no:cacheprovider"], cwd=str(tmp_path), env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]
