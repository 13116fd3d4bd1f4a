"""The kernels decide INT2 codes by three comparisons with the exact
midpoints s/2, 3s/2, 5s/2 instead of the fp32 division of the quantiser's
definition.  This checks, in numpy fp32,
that the comparison rule gives exactly the oracle's codes, on groups built to
sit on the rounding midpoints (ties to even included) and on ordinary data.
The GPU-side counterpart runs the same groups through the kernels."""
import numpy as np

from int2_kv_cache_rotate_b200 import workloads as WL
from oracle import okv_oracle as O
from tests import gpu_helpers as H


def _rule(z, s16, m16):
    """x = fl(z - m); c = [x > s/2] + [x >= 3s/2] + [x > 5s/2] (all products exact)."""
    s = s16.astype(np.float32)[:, None]
    m = m16.astype(np.float32)[:, None]
    x = (z - m).astype(np.float32)
    f = np.float32
    c = (x > f(0.5) * s).astype(np.uint8)
    c += (x >= f(1.5) * s).astype(np.uint8)
    c += (x > f(2.5) * s).astype(np.uint8)
    return np.where(s == 0, 0, c).astype(np.uint8)


def test_threshold_rule_equals_division_at_midpoints():
    z = H.rounding_boundary_vectors(5, 1500)
    c, s16, m16 = O.quantize(z)
    s = s16.astype(np.float32)[:, None]
    x = (z - m16.astype(np.float32)[:, None]).astype(np.float32)
    q = np.divide(x, s, out=np.zeros_like(x), where=s > 0)
    assert np.isin(q, np.float32([0.5, 1.5, 2.5])).sum() > 1000  # exact ties are exercised
    assert np.array_equal(_rule(z, s16, m16), c)


def test_threshold_rule_equals_division_on_workload_data():
    z = np.concatenate([WL.sample_rotated(0, 0, 0, 0, 4096, 0, scale=sc) for sc in (1e-6, 1.0, 300.0)])
    c, s16, m16 = O.quantize(z)
    assert np.array_equal(_rule(z, s16, m16), c)
