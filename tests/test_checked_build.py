"""The checked build (libsta_debug.so: the same kernels with device-side
bounds and alignment checks on every index and address derived from run-time
data) runs every entry point on small ragged cases without recording a
failed check, and gives results bit-identical to the product library."""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRIPT = os.path.join(ROOT, "tests", "_checked_cases.py")


def _run(path, checked):
    env = dict(os.environ)
    env["STA_CHECKED"] = "1" if checked else "0"
    r = subprocess.run([sys.executable, SCRIPT, str(path)], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return dict(np.load(path))


@pytest.mark.gpu
def test_checked_build_records_nothing_and_matches_the_product_build(tmp_path):
    chk = _run(tmp_path / "checked.npz", True)
    prod = _run(tmp_path / "product.npz", False)
    assert int(chk.pop("debug_build")) == 1 and int(prod.pop("debug_build")) == 0
    statuses = {k: int(v) for k, v in chk.items() if k.startswith("status_")}
    assert statuses and all(v == 0 for v in statuses.values()), statuses
    assert all(int(v) == 0 for k, v in prod.items() if k.startswith("status_"))
    assert sorted(chk) == sorted(prod)
    for k in chk:
        assert chk[k].shape == prod[k].shape and np.array_equal(chk[k], prod[k], equal_nan=True), k
