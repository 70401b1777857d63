"""Helpers shared by the GPU parity tests: host copies for the oracle,
sub-problems for sampled checks at full size, and the tolerance check.

Tolerance (reading of "max-abs 2e-2 and rel 2e-2 on every element"): each
element must satisfy |gpu - oracle| <= 2e-2 + 2e-2 * |oracle|.
"""
import numpy as np
import torch

import oracle
from paged_kv_cache_474_b200.workloads import Workload, make_workload

ATOL = 2e-2
RTOL = 2e-2


def problem(wl: Workload) -> oracle.Problem:
    """Whole workload as an oracle problem (host copies of every buffer)."""
    return oracle.problem_from_workload(wl)


def subproblem(wl: Workload, rows):
    """Oracle problem holding only the given batch rows: their q rows, the
    blocks their tables reach (gathered into a compact pool, tables
    remapped), lengths and windows.  Returns (problem, row_map) where row_map
    maps an original row to its index in the sub-problem."""
    sub, rmap = wl.subset(rows)
    return oracle.problem_from_workload(sub), rmap


def token_offsets(wl: Workload):
    L = wl.query_lens.cpu().tolist()
    return np.concatenate([[0], np.cumsum(L)]).astype(np.int64)


def assert_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU output"
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {err.size} elements out of tolerance; "
            f"worst at {i}: gpu={got[i]:.6f} oracle={ref[i]:.6f}")
    return float(err.max())


def check_full(wl: Workload, dst, what=""):
    ref = oracle.decode(problem(wl))
    return assert_close(dst.float().cpu().numpy(), ref, what)


def sample_queries(wl: Workload, n: int, seed: int = 0, rows=None):
    """n seeded (b, i, h) triples over rows with queryLen > 0 (or only `rows`)."""
    g = np.random.default_rng(seed)
    L = wl.query_lens.cpu().tolist()
    cand = [b for b in (rows if rows is not None else range(wl.batch)) if L[b] > 0]
    out = []
    for _ in range(n):
        b = int(g.choice(cand))
        out.append((b, int(g.integers(0, L[b])), int(g.integers(0, wl.num_q_heads))))
    return out


def check_sampled(wl: Workload, dst, sel, what=""):
    """Compares the outputs of the selected (b, i, h) with the oracle computed
    one by one on a sub-problem holding only the rows involved."""
    pr, rmap = subproblem(wl, [b for b, _, _ in sel])
    ref = oracle.decode_select(pr, [(rmap[b], i, h) for b, i, h in sel])
    qoff = token_offsets(wl)
    d = dst.float().cpu().numpy()
    got = np.stack([d[qoff[b] + i, h] for b, i, h in sel])
    return assert_close(got, ref, what)


def scaled_workload(cfg, seed=1, **kw):
    """The named workloads' shapes at lengths the oracle finishes in seconds,
    still spanning several stages, partitions and a ragged tail.  Extra
    keywords (kv_dtype, q_dtype) go to make_workload."""
    g = np.random.default_rng(seed)
    if cfg == 2:
        s = g.integers(100, 1500, 6).tolist()
        return make_workload(seq_lens=s, query_lens=[1] * 6, num_q_heads=32,
                             num_kv_heads=8, head_dim=128, block_size=16, seed=seed, **kw)
    if cfg == 3:
        s = g.integers(200, 2500, 7).tolist() + [300]
        return make_workload(seq_lens=s, query_lens=[1, 1, 1, 1, 2, 3, 4, 5],
                             num_q_heads=32, num_kv_heads=8, head_dim=128,
                             block_size=16, window=333, seed=seed, **kw)
    if cfg == 4:
        return make_workload(seq_lens=[9001], query_lens=[1], num_q_heads=8,
                             num_kv_heads=1, head_dim=128, block_size=16, seed=seed, **kw)
    if cfg == 5:
        s = g.integers(1100, 4200, 6).tolist()
        l = g.integers(1, 5, 6).tolist()
        return make_workload(seq_lens=s, query_lens=l, num_q_heads=64,
                             num_kv_heads=8, head_dim=128, block_size=1024,
                             windows=[700 if b % 2 == 0 else 0 for b in range(6)],
                             seed=seed, **kw)
    raise ValueError(cfg)


def host_buffer(arr, kind, offset=0):
    """A host copy of ``arr`` (a CPU tensor): pinned (read in place by the
    library's staging kernel) or pageable (copied), optionally starting
    ``offset`` bytes into a larger buffer of the same kind."""
    raw = arr.contiguous().view(torch.uint8).reshape(-1)
    buf = torch.zeros(raw.numel() + offset + 16, dtype=torch.uint8)
    if kind == "pinned":
        buf = buf.pin_memory()
    buf[offset:offset + raw.numel()] = raw
    return buf, buf.data_ptr() + offset


def poison_outside_spans(wl: Workload):
    """Writes NaN (bf16 NaN, or the e4m3 NaN code 0x7F) into every cache
    position no query token may see: before each row's earliest visible
    position, past its last token in its last block, and in every block no
    row uses; and puts out-of-pool entries (alternately too large and
    negative) in the block-table slots past each row's last block.  In
    place, on the workload's own tensors (CPU)."""
    nan = 0x7F if wl.kv_fp8 else float("nan")
    S = wl.seq_lens.tolist()
    L = wl.query_lens.tolist()
    W = wl.windows.tolist() if wl.windows is not None else [wl.window] * len(S)
    bs = wl.block_size
    for b in range(len(S)):
        nb = (S[b] + bs - 1) // bs
        first = max(0, S[b] - L[b] + 1 - W[b]) if (W[b] > 0 and L[b] > 0) else 0
        if L[b] <= 0:
            first = S[b]  # no query: nothing of the row is visible
        dead = list(range(0, first)) + list(range(S[b], nb * bs))
        if dead:
            t = torch.tensor(dead, dtype=torch.long)
            blk = wl.block_tables[b, t // bs].long()
            wl.k_cache[blk, :, t % bs] = nan
            wl.v_cache[blk, :, t % bs] = nan
        cols = wl.block_tables.shape[1]
        for j in range(nb, cols):
            wl.block_tables[b, j] = 10 ** 6 + j if j % 2 == 0 else -7 - j
    used = set(int(x) for x in wl.block_tables.flatten().tolist() if 0 <= x < wl.num_blocks)
    for blk in range(wl.num_blocks):
        if blk not in used:
            wl.k_cache[blk] = nan
            wl.v_cache[blk] = nan
