"""The seeded input drawer (paged_kv_cache_474_b200/workloads.py) follows the
named workloads' recipes: shapes, length distributions, row layouts and
windows as their titles state, blocks handed out as a permutation of the
pool, and the same tensors for the same seed.  CPU only; it holds none of the
method's arithmetic, so these are checks of the inputs both sides share."""
import numpy as np
import pytest
import torch

from paged_kv_cache_474_b200.workloads import (CONFIG_TITLES, config_lengths, config_workload,
                                               make_workload)


def test_lengths_follow_the_titles():
    s, l, w, ws = config_lengths(1)
    assert (s, l, w, ws) == ([37, 50], [1, 1], 0, None)
    s, l, w, ws = config_lengths(2)
    assert len(s) == 32 and min(s) >= 1024 and max(s) <= 8192 and l == [1] * 32
    assert w == 0 and ws is None
    s, l, w, ws = config_lengths(3)
    assert len(s) == 16 and all(2048 <= x <= 32768 for x in s[:15]) and s[15] == 300
    assert l == [1] * 12 + [2, 3, 4] + [5] and w == 4096 and ws is None
    assert config_lengths(4) == ([131072], [1], 0, None)
    s, l, w, ws = config_lengths(5)
    assert len(s) == 64 and min(s) >= 4096 and max(s) <= 65536
    assert set(l) <= {1, 2, 3, 4} and len(set(l)) == 4
    assert w == 0 and ws == [4096 if b % 2 == 0 else 0 for b in range(64)]


@pytest.mark.parametrize("cfg,hq,hkv,d,bs", [(1, 4, 2, 64, 16), (2, 32, 8, 128, 16),
                                            (3, 32, 8, 128, 16), (4, 8, 1, 128, 16),
                                            (5, 64, 8, 128, 1024)])
def test_shapes_follow_the_titles(cfg, hq, hkv, d, bs):
    # the shape table the drawer builds from (building the full pools of the
    # large workloads on the CPU would take minutes), and one small build
    from paged_kv_cache_474_b200.workloads import _SHAPES
    title = CONFIG_TITLES[cfg]
    for key, val in (("Hq", hq), ("Hkv", hkv), ("D", d), ("BS", bs)):
        assert f"{key}={val}" in title
    sh = _SHAPES[cfg]
    assert (sh["num_q_heads"], sh["num_kv_heads"], sh["head_dim"], sh["block_size"]) == \
        (hq, hkv, d, bs)
    assert f"B={len(config_lengths(cfg)[0])}" in title


def test_tiny_workload_is_built_to_its_shape():
    wl = config_workload(1)
    assert (wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size) == (4, 2, 64, 16)
    assert wl.q.shape == (2, 4, 64) and wl.q.dtype == wl.k_cache.dtype == torch.bfloat16
    assert wl.num_blocks == 3 + 4 + 1 and wl.scale == 1.0 / 8.0


def test_blocks_are_a_permutation_of_the_pool():
    wl = make_workload(seq_lens=[37, 50, 1, 160], query_lens=[1, 2, 1, 3], num_q_heads=4,
                       num_kv_heads=2, head_dim=64, block_size=16, seed=3, spare_blocks=2,
                       extra_table_cols=2)
    need = [(s + 15) // 16 for s in wl.seq_lens.tolist()]
    assert wl.num_blocks == sum(need) + 2
    used = torch.cat([wl.block_tables[b, :n] for b, n in enumerate(need)]).tolist()
    assert len(set(used)) == len(used) and all(0 <= x < wl.num_blocks for x in used)
    for b, n in enumerate(need):  # unused slots and padding columns hold 0
        assert wl.block_tables[b, n:].eq(0).all()


def test_same_seed_same_tensors_other_seed_other_tensors():
    kw = dict(seq_lens=[100, 7], query_lens=[2, 1], num_q_heads=4, num_kv_heads=2,
              head_dim=64, block_size=16)
    a, b, c = make_workload(seed=5, **kw), make_workload(seed=5, **kw), make_workload(seed=6, **kw)
    for name in ("q", "k_cache", "v_cache", "block_tables"):
        assert torch.equal(getattr(a, name), getattr(b, name))
    assert not torch.equal(a.k_cache, c.k_cache)


def test_fp8_caches_are_scaled_e4m3_codes_of_the_values():
    base = make_workload(seq_lens=[300], query_lens=[1], num_q_heads=4, num_kv_heads=2,
                         head_dim=64, block_size=16, seed=7)
    q8 = make_workload(seq_lens=[300], query_lens=[1], num_q_heads=4, num_kv_heads=2,
                       head_dim=64, block_size=16, seed=7, kv_dtype="fp8_e4m3")
    assert q8.k_cache.dtype == torch.uint8 and q8.k_scale > 0 and q8.v_scale > 0
    codes = q8.k_cache.view(torch.float8_e4m3fn).to(torch.float64) * q8.k_scale
    ref = base.k_cache.to(torch.float64)
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range
    big = ref.abs() > 2.0 ** -6 * q8.k_scale * 4
    assert torch.all((codes - ref).abs()[big] <= ref.abs()[big] * 2.0 ** -4 + 1e-12)
    assert torch.isfinite(codes).all()
    assert not np.any(np.isin(q8.k_cache.numpy(), [0x7F, 0xFF]))  # no NaN codes


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
def test_row_subset_keeps_each_rows_problem(kv_dtype):
    # Workload.subset gathers some rows into a compact pool with renumbered
    # tables (the parity tests and the bench's oracle leg use it on the large
    # workloads).  The oracle's outputs for those rows must not change at
    # all, and the gathered blocks must be exactly the ones the rows use.
    import oracle
    wl = make_workload(seq_lens=[70, 5, 33, 128, 17], query_lens=[2, 1, 0, 3, 1],
                       num_q_heads=6, num_kv_heads=2, head_dim=32, block_size=16,
                       windows=[0, 3, 9, 40, 0], seed=5, spare_blocks=3, kv_dtype=kv_dtype)
    full = oracle.decode(oracle.problem_from_workload(wl))
    L = wl.query_lens.tolist()
    qoff = np.concatenate([[0], np.cumsum(L)])
    for rows in ([3], [0, 3], [4, 1, 2], [0, 1, 2, 3, 4]):
        sub, rmap = wl.subset(rows)
        assert sorted(rmap) == sorted(set(rows)) and sub.k_scale == wl.k_scale
        nb = [(s + 15) // 16 for s in sub.seq_lens.tolist()]
        assert sub.num_blocks == sum(nb)
        for b, j in rmap.items():
            used = wl.block_tables[b, :nb[j]].long()
            assert torch.equal(sub.k_cache[sub.block_tables[j, :nb[j]].long()], wl.k_cache[used])
            assert torch.equal(sub.v_cache[sub.block_tables[j, :nb[j]].long()], wl.v_cache[used])
        got = oracle.decode(oracle.problem_from_workload(sub))
        sl = np.concatenate([[0], np.cumsum(sub.query_lens.tolist())])
        for b, j in rmap.items():
            assert np.array_equal(got[sl[j]:sl[j + 1]], full[qoff[b]:qoff[b + 1]])
