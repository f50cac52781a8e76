import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def rel_err(got, ref) -> float:
    """Norm-wise relative error: max |got - ref| / max |ref| (per output tensor)."""
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    return num / den if den > 0 else num


def elem_err(got, ref):
    """Element-wise relative error against a floor of the tensor's RMS:
    max_e |got_e - ref_e| / (|ref_e| + rms(ref)).  Returns (error, worst index,
    got there, ref there)."""
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0, None, None, None
    rms = float(np.sqrt(np.mean(ref * ref)))
    den = np.abs(ref) + rms
    diff = np.abs(got - ref)
    r = np.where(den > 0, diff / np.where(den > 0, den, 1.0), diff)
    i = int(np.argmax(r))
    idx = np.unravel_index(i, ref.shape) if ref.ndim else ()
    return float(r.flat[i]), idx, float(got.flat[i]), float(ref.flat[i])


def close_errs(got, ref):
    """(norm-wise error, element-wise error) of one output tensor."""
    return rel_err(got, ref), elem_err(got, ref)[0]


def assert_close(got, ref, tol, name=""):
    """Both parity criteria at tolerance `tol`: the norm-wise
    max|got - ref| / max|ref| and the element-wise |got - ref| <= tol (|ref| +
    rms(ref)).  A failure names the worst element."""
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    ne = rel_err(got, ref)
    ee, idx, g, r = elem_err(got, ref)
    assert ne < tol and ee < tol, (
        f"{name}: norm-wise {ne:.3e}, element-wise {ee:.3e} (tol {tol:.1e}); worst element "
        f"{idx}: got {g!r}, ref {r!r}")
    return ne, ee
