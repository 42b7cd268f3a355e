"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle, on the CPU:
- a dropped normalisation factor;
- a transposed operand;
- a wrong tie order;
- a wrong rounding;
- a shifted bit;
- ...

It then runs the pin suite (tests/test_oracle.py) against that copy, which must fail. The real oracle
is never modified. Together these show that the pins pin the oracle to the pages and the
mathematics, not to itself.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, text in oracle/tactkv_oracle.py, replacement)
MUTATIONS = [
    ("dct: a_k = sqrt(1/L) for every k", "math.sqrt(1.0 / L), math.sqrt(2.0 / L))",
     "math.sqrt(1.0 / L), math.sqrt(1.0 / L))"),
    ("dct: half-sample shift dropped", "np.cos(np.pi * (2.0 * t + 1.0) * k / (2.0 * L))",
     "np.cos(np.pi * (2.0 * t) * k / (2.0 * L))"),
    ("dct3: H-axis matrix transposed", 'np.einsum("kh,shwc->skwc", dct_matrix(H), y)',
     'np.einsum("hk,shwc->skwc", dct_matrix(H), y)'),
    ("variance: mean removed", "return np.mean(Xf * Xf, axis=1)",
     "return np.var(Xf, axis=1)"),
    # (rounding down instead of to nearest is NOT a mistake: the +-1 greedy reaches the same top-B
    #  set from any rounding, so that change is equivalent and left out)
    ("allocation: 8-bit cap ignored by the greedy", "cand = act & (b < MAX_BITS)", "cand = act"),
    ("allocation: budget one bit short", "B = int(bits) * N\n    act", "B = int(bits) * N - 1\n    act"),
    ("allocation: greedy adds the least valuable bit", "m = key.max()",
     "m = key[np.isfinite(key)].min()"),
    ("allocation: add-ties to the highest index", "i = idx[key == m].min()                     # ties -> lowest index",
     "i = idx[key == m].max()"),
    ("quantize: ties go down", 'np.asarray(u, dtype=np.float32), side="right")',
     'np.asarray(u, dtype=np.float32), side="left")'),
    ("pack: MSB-first bit order", "out[:, q >> 3] |= (bit << (q & 7)).astype(np.uint8)",
     "out[:, q >> 3] |= (bit << (7 - (q & 7))).astype(np.uint8)"),
    ("lloyd-max: thresholds not midpoints", "return y, 0.5 * (y[1:] + y[:-1])",
     "return y, 0.45 * (y[1:] + y[:-1])"),
    ("code band: squared divisor", "return np.min(gaps / np.maximum(1.0, np.abs(thresholds_b)), axis=-1)",
     "return np.min(gaps / np.maximum(1.0, np.abs(thresholds_b)) ** 2, axis=-1)"),
    ("code band: farthest threshold", "return np.min(gaps / np.maximum(1.0, np.abs(thresholds_b)), axis=-1)",
     "return np.max(gaps / np.maximum(1.0, np.abs(thresholds_b)), axis=-1)"),
    ("rotation: Hadamard sign from the wrong bits", "return np.where(pop % 2 == 1, -1.0, 1.0)",
     "return np.where(pop % 3 == 1, -1.0, 1.0)"),
    ("rotation: decoder does not undo it", "            X = X @ rotation_matrix(n)                  # row i",
     "            X = X @ rotation_matrix(n).T                # row i"),
    ("rotation: unnormalised", "Hm = hadamard(ROTATION_GROUP) / math.sqrt(ROTATION_GROUP)",
     "Hm = hadamard(ROTATION_GROUP) / ROTATION_GROUP"),
    ("splitmix: finalizer shift", "z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m",
     "z = ((z ^ (z >> 28)) * 0x94D049BB133111EB) & m"),
    ("axis mask: H skipped when S is", "    if axes[1]:\n        y = np.einsum(\"kh,shwc->skwc\"",
     "    if axes[0]:\n        y = np.einsum(\"kh,shwc->skwc\""),
    ("uniform: nominal bits plus one", "return np.where(var > 0, int(bits), 0).astype(np.int64)",
     "return np.where(var > 0, int(bits) + 1, 0).astype(np.int64)"),
    ("head gain: heads and channels transposed",
     "hv = np.mean(X.reshape(X.shape[0], heads, head_dim) ** 2, axis=2).T",
     "hv = np.mean(X.reshape(X.shape[0], head_dim, heads) ** 2, axis=1).T"),
    ("head gain: pooled over all heads", "g = np.repeat(sig[:, i], head_dim) if flags & FLAG_HEAD_GAIN",
     "g = np.repeat(np.sqrt(np.mean(sig[:, i].astype(np.float64) ** 2)), n) if flags & FLAG_HEAD_GAIN"),
    ("head gain: decoder uses head 0's gain", "g = np.repeat(p[\"sigma\"][:, i].astype(np.float64), p[\"head_dim\"])",
     "g = np.repeat(p[\"sigma\"][0, i].astype(np.float64), p[\"heads\"] * p[\"head_dim\"])"),
    ("code band: distance to the levels", "thresholds_b = table(bits)[1]", "thresholds_b = table(bits)[0]"),
    ("code band: no relative scaling", "return np.min(gaps / np.maximum(1.0, np.abs(thresholds_b)), axis=-1)",
     "return np.min(gaps, axis=-1)"),
]


def _copy_tree(dst):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"))
    os.makedirs(os.path.join(dst, "tests"))
    for f in ("conftest.py", "test_oracle.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    shutil.copytree(os.path.join(ROOT, "dct_transform_coding_b200"), os.path.join(dst, "dct_transform_coding_b200"),
                    ignore=shutil.ignore_patterns("*.so", "_build", "csrc", "__pycache__"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), os.path.join(dst, "pytest.ini"))


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(tmp_path, name, old, new):
    _copy_tree(str(tmp_path))
    path = tmp_path / "oracle" / "tactkv_oracle.py"
    src = path.read_text()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    path.write_text(src.replace(old, new, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle.py", "-x", "-q", "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=str(tmp_path), capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin caught the planted mistake '{name}':\n{r.stdout[-2000:]}"
