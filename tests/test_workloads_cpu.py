"""The seeded synthetic inputs follow the recipe stated for them: shapes and
values of the five workloads, bf16-exact values, keys with four fixed outlier
channels (x16) per layer, queries whose covariance has the logspace(0, -3)
spectrum in a Haar basis, block tables that are permutations, and streams
that depend on every part of their seed tuple."""
import numpy as np

from int2_kv_cache_rotate_b200 import workloads as WL


def test_workload_shapes():
    w = [WL.config(i) for i in range(5)]
    assert (w[0].batch, w[0].hq, w[0].hkv, w[0].ctx) == (1, 4, 1, (2048,))
    assert (w[1].batch, w[1].hq, w[1].hkv, w[1].ctx) == (8, 32, 8, (32768,) * 8)
    assert (w[2].batch, w[2].hq, w[2].hkv, w[2].ctx, w[2].steps) == (4, 32, 8, (100000,) * 4, 64)
    assert (w[3].layers, w[3].hq, w[3].hkv, w[3].ctx) == (80, 64, 8, (131072,))
    assert w[4].batch == 64 and w[4].prefill_append == 8192
    assert all(1024 <= n <= 65536 for n in w[4].ctx)
    # log-uniform: the median sits near the geometric middle of [1K, 64K]
    assert 4000 < np.median(w[4].ctx) < 16000


def test_values_are_bf16_exact():
    for x in (WL.sample_keys(0, 0, 0, 0, 64), WL.sample_values(0, 0, 0, 0, 64),
              WL.sample_queries(0, 0, 0, 0, 64, 4)):
        bits = x.astype(np.float32).view(np.uint32)
        assert np.all(bits & 0xFFFF == 0)


def test_keys_have_four_fixed_outlier_channels():
    k = WL.sample_keys(0, 0, 0, 0, 4096).astype(np.float64)
    std = k.std(axis=0)
    out = WL.outlier_channels(0, 0, 0)
    assert len(set(out.tolist())) == 4
    assert np.all(np.abs(std[out] / 16 - 1) < 0.1)
    assert np.all(np.abs(np.delete(std, out) - 1) < 0.1)
    # the same channels for every KV head of a layer, others in another layer
    k1 = WL.sample_keys(0, 0, 0, 5, 4096).astype(np.float64)
    assert set(np.argsort(k1.std(axis=0))[-4:]) == set(out.tolist())
    assert set(WL.outlier_channels(0, 0, 1).tolist()) != set(out.tolist())


def test_query_covariance_spectrum_and_basis():
    q = WL.sample_queries(0, 0, 0, 0, 20000, 1).reshape(-1, 128).astype(np.float64)
    o = WL.query_basis(0, 0, 0, 0)
    assert np.abs(o.T @ o - np.eye(128)).max() < 1e-10
    lam = np.diag(o.T @ (q.T @ q / len(q)) @ o)
    spec = WL.query_spectrum()
    assert spec[0] == 1.0 and abs(spec[-1] - 1e-3) < 1e-15 and len(spec) == 128
    # each direction's variance within sampling error (and bf16 rounding) of the spectrum
    assert np.all(np.abs(lam / spec - 1) < 0.06 + 1e-3 / spec)


def test_block_tables_are_permutations():
    table, n = WL.block_table(3, 1, [100, 1, 0, 48], extra_tokens=16, spare_blocks=5)
    used = table[table >= 0]
    assert n == sum(WL.blocks_needed(L + 16) for L in (100, 1, 0, 48)) + 5 == 20
    assert len(np.unique(used)) == len(used) and used.max() < n
    assert [int((row >= 0).sum()) for row in table] == [8, 2, 1, 4]


def test_streams_depend_on_every_seed_part():
    base = WL.stream(1, 2, 3, 4, 5, 6).standard_normal(8)
    for args in ((0, 2, 3, 4, 5, 6), (1, 0, 3, 4, 5, 6), (1, 2, 0, 4, 5, 6), (1, 2, 3, 0, 5, 6),
                 (1, 2, 3, 4, 0, 6), (1, 2, 3, 4, 5, 0)):
        assert not np.array_equal(WL.stream(*args).standard_normal(8), base), args
    assert np.array_equal(WL.stream(1, 2, 3, 4, 5, 6).standard_normal(8), base)
