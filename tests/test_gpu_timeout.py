"""The kernels' timeout paths, run on purpose with a test build of the
library in which every bounded wait gives up after 64 cycles
(``python -m int2_kv_cache_rotate_b200.build --short-wait``).

No wait is left unbounded and nothing faults: a wait that runs out sets
OKV_DEV_TIMEOUT in the cache's status word and the CTA winds down -- the
decode ring's warp 0 waits (with the full limit) for the bulk copies it
issued, the tcgen05 append and prefill wait for their loads and for their
last MMA commit, and TMEM is freed.  The test runs in a child process that
loads the short-wait build; it appends a prefill chunk on the tcgen05 path,
decodes through the tensor-core split-K ring and runs a prefill attention,
checks that each call raised the timeout flag, and then checks that the
CUDA context is still usable."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

CHILD = r"""
import numpy as np, torch
from int2_kv_cache_rotate_b200 import okv
from int2_kv_cache_rotate_b200 import workloads as WL
torch.cuda.set_device(0)
seed, hq, hkv, L = 61, 32, 8, 4096
r = np.random.default_rng(seed)
uk = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
uv = np.stack([WL.haar_orthogonal(r) for _ in range(hkv)]).astype(np.float32)
table, nb = WL.block_table(seed, 0, [L], extra_tokens=16)
cache = okv.Cache(hq, hkv, nb, 1, table.shape[1], uk, uv)
dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
k = dev(r.standard_normal((L, hkv, 128)).astype(np.float32)).to(torch.bfloat16)
v = dev(r.standard_normal((L, hkv, 128)).astype(np.float32)).to(torch.bfloat16)
okv.append_quantize(cache, k, v, dev(np.zeros(L, np.int32)), dev(np.arange(L, dtype=np.int32)), dev(table),
                    dev(np.array([L], np.int32)))
torch.cuda.synchronize()
s_app = cache.device_status()
cache.clear_status()
q = dev(r.standard_normal((1, hq, 128)).astype(np.float32)).to(torch.bfloat16)
out = okv.decode_attention(cache, q, dev(np.zeros(1, np.int32)), dev(table), dev(np.array([L], np.int32)))
torch.cuda.synchronize()
s_dec = cache.device_status()
cache.clear_status()
qp = dev(r.standard_normal((256, hq, 128)).astype(np.float32)).to(torch.bfloat16)
outp = okv.prefill_attention(cache, qp, 0, L, dev(table))
torch.cuda.synchronize()
s_pf = cache.device_status()
# the context survives: ordinary work still runs and returns
x = torch.arange(1 << 20, device="cuda", dtype=torch.float32)
assert float(x.sum().item()) == float((1 << 20) * ((1 << 20) - 1) // 2)
print("STATUS", s_app, s_dec, s_pf)
"""


def _short_wait_lib() -> str:
    from int2_kv_cache_rotate_b200 import build as B
    if not os.path.exists(B.SHORT_WAIT_LIB):
        B.build(out=B.SHORT_WAIT_LIB, short_wait=True)
    return B.SHORT_WAIT_LIB


def test_timeouts_wind_down_cleanly():
    lib = _short_wait_lib()
    env = dict(os.environ, OKV_LIBRARY=lib, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    res = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    line = [ln for ln in res.stdout.splitlines() if ln.startswith("STATUS")][-1]
    s_app, s_dec, s_pf = (int(x) for x in line.split()[1:])
    from int2_kv_cache_rotate_b200 import okv
    for name, s in (("append", s_app), ("decode", s_dec), ("prefill", s_pf)):
        assert s & okv.DEV_TIMEOUT, (name, s)
