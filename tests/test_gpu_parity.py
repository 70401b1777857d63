"""GPU parity: pa_decode (through the C ABI) against the float64 oracle.

Small workloads are compared element by element; the five named workloads
at full size are compared on seeded samples the oracle computes one by one,
in the same launch configuration the bench times (host hints, workspace,
dispatcher's partitioning).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_helpers import (assert_close, check_full, check_sampled, host_buffer,
                                  problem, sample_queries, scaled_workload, token_offsets)

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_474_b200")
from paged_kv_cache_474_b200.workloads import (config_lengths, config_workload,  # noqa: E402
                                               make_workload)


@pytest.fixture(autouse=True)
def _device_status_clean(cuda_device):
    pa.pa_device_status(clear=True)
    yield
    assert pa.pa_device_status(clear=True) == 0


def dev(wl):
    return wl.to("cuda:0")


# ----------------------------------------------------------- small, full
@pytest.mark.parametrize("window", [0, 8])
@pytest.mark.parametrize("parts", [0, 1, 2, 3])
def test_tiny_workload(window, parts):
    wl = config_workload(1, window=window)
    out = pa.decode(dev(wl), force_partitions=parts)
    check_full(wl, out, f"tiny w={window} parts={parts}")


scaled = scaled_workload


VARIANTS = [pa.PA_VARIANT_AUTO, pa.PA_VARIANT_FMA, pa.PA_VARIANT_MMA]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
@pytest.mark.parametrize("parts", [0, 1, 5])
def test_scaled_named_workloads(cfg, parts, variant):
    wl = scaled(cfg)
    out = pa.decode(dev(wl), force_partitions=parts, force_variant=variant)
    check_full(wl, out, f"scaled cfg{cfg} parts={parts} variant={variant}")


def test_dispatcher_defaults_to_the_tensor_core_kernel():
    for cfg, bs in ((2, 16), (4, 16), (5, 1024)):
        _, info = pa.pa_plan(pa.params_for(dev(scaled(cfg))), bs)
        assert info.variant == pa.PA_VARIANT_MMA


@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("variant", [pa.PA_VARIANT_FMA, pa.PA_VARIANT_MMA])
@pytest.mark.parametrize("parts", [1, 2, 3, 7, 64, 200])
def test_split_k_invariance(parts, variant, head_dim):
    # 64 and 200 partitions also exercise the reduce that splits head_dim over CTAs
    wl = make_workload(seq_lens=[5000, 3333, 77], query_lens=[1, 3, 2], num_q_heads=8,
                       num_kv_heads=2, head_dim=head_dim, block_size=16, window=0, seed=7)
    d = dev(wl)
    out = pa.decode(d, force_partitions=parts, force_variant=variant)
    check_full(wl, out, f"parts={parts}")
    base = pa.decode(d, force_partitions=1, force_variant=variant).float()
    assert torch.max(torch.abs(out.float() - base)).item() < 2e-2


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("block_size", [16, 32, 64, 256, 1024])
def test_head_dims_and_block_sizes(head_dim, block_size, variant):
    wl = make_workload(seq_lens=[1, 17, 64, 65, 1500, 2049], query_lens=[1, 1, 2, 1, 4, 1],
                       num_q_heads=8, num_kv_heads=4, head_dim=head_dim,
                       block_size=block_size, window=0, seed=head_dim + block_size)
    out = pa.decode(dev(wl), force_variant=variant)
    check_full(wl, out, f"D={head_dim} BS={block_size} variant={variant}")


@pytest.mark.parametrize("variant", [pa.PA_VARIANT_FMA, pa.PA_VARIANT_MMA])
@pytest.mark.parametrize("group,qlen", [(1, 1), (2, 3), (8, 1), (8, 4), (16, 5), (64, 1)])
def test_row_tiles_and_slabs(group, qlen, variant):
    # rows per kv head from 1 to 80: padding rows, several M tiles, several slabs
    wl = make_workload(seq_lens=[700, 64, 1999], query_lens=[qlen, min(qlen, 2), qlen],
                       num_q_heads=2 * group, num_kv_heads=2, head_dim=128, block_size=16,
                       window=0, seed=group * 10 + qlen)
    out = pa.decode(dev(wl), force_variant=variant)
    check_full(wl, out, f"group={group} qlen={qlen} variant={variant}")


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("window", [1, 2, 5, 16, 100, 4096])
def test_gllm_window_batch(window, variant):
    # gllm PR #116 "Verification": a 5-token prefill chunk over a 300-token
    # context plus a decode row over 40, windows 16, 100 and 4096 (and the
    # CPU test's small windows), here with GQA.
    wl = make_workload(seq_lens=[300, 40], query_lens=[5, 1], num_q_heads=8,
                       num_kv_heads=2, head_dim=64, block_size=16, window=window,
                       seed=window)
    out = pa.decode(dev(wl), force_variant=variant)
    check_full(wl, out, f"window={window} variant={variant}")


def test_window_one_returns_own_value():
    wl = make_workload(seq_lens=[70, 3, 1000], query_lens=[3, 1, 2], num_q_heads=4,
                       num_kv_heads=2, head_dim=128, block_size=16, window=1, seed=3)
    out = pa.decode(dev(wl)).cpu()
    qoff = token_offsets(wl)
    for b, (S, L) in enumerate(zip(wl.seq_lens.tolist(), wl.query_lens.tolist())):
        for i in range(L):
            p = S - L + i
            phys = int(wl.block_tables[b, p // 16])
            for h in range(4):
                assert torch.equal(out[qoff[b] + i, h], wl.v_cache[phys, h // 2, p % 16])


def test_window_at_or_beyond_context_equals_unlimited():
    kw = dict(seq_lens=[500, 123, 2000], query_lens=[1, 2, 1], num_q_heads=8,
              num_kv_heads=1, head_dim=128, block_size=16, seed=4)
    a = pa.decode(dev(make_workload(window=0, **kw)))
    b = pa.decode(dev(make_workload(window=2000, **kw)))
    c = pa.decode(dev(make_workload(window=10 ** 6, **kw)))
    assert torch.equal(a, b) and torch.equal(a, c)


def test_rows_without_queries_and_empty_batch():
    wl = make_workload(seq_lens=[50, 900, 10, 333], query_lens=[0, 2, 0, 1], num_q_heads=4,
                       num_kv_heads=4, head_dim=64, block_size=16, seed=5)
    out = pa.decode(dev(wl))
    check_full(wl, out, "zero-length rows")
    empty = make_workload(seq_lens=[], query_lens=[], num_q_heads=4, num_kv_heads=4,
                          head_dim=64, block_size=16, seed=5)
    p = pa.params_for(empty)
    rc = pa.pa_decode(16, 16, 16, 16, 16, 16, 16, 1.0, 0, 16, p, None)
    assert rc == pa.PA_OK


@pytest.mark.parametrize("variant", [pa.PA_VARIANT_FMA, pa.PA_VARIANT_MMA])
def test_garbage_outside_spans_is_never_read(variant):
    # Slots past each row's last token, the spare block and unused table
    # entries hold NaN / out-of-range values; outputs must not see them.
    wl = make_workload(seq_lens=[37, 50, 1], query_lens=[1, 3, 1], num_q_heads=4,
                       num_kv_heads=2, head_dim=128, block_size=16, window=0, seed=9,
                       spare_blocks=2, extra_table_cols=3)
    ref = oracle.decode(problem(wl))
    for b, S in enumerate(wl.seq_lens.tolist()):
        nb = (S + 15) // 16
        last = int(wl.block_tables[b, nb - 1])
        wl.k_cache[last, :, S - (nb - 1) * 16:] = float("nan")
        wl.v_cache[last, :, S - (nb - 1) * 16:] = float("nan")
        wl.block_tables[b, nb:] = 10 ** 6
    used = set(wl.block_tables[wl.block_tables < wl.num_blocks].tolist())
    for blk in range(wl.num_blocks):
        if blk not in used:
            wl.k_cache[blk] = float("nan")
            wl.v_cache[blk] = float("nan")
    out = pa.decode(dev(wl), force_variant=variant)
    assert_close(out.float().cpu().numpy(), ref, f"garbage outside spans variant={variant}")


@pytest.mark.parametrize("variant", [pa.PA_VARIANT_FMA, pa.PA_VARIANT_MMA])
def test_windowed_garbage_before_the_window_is_never_read(variant):
    # Positions before each row's window start hold NaN: a window that starts
    # mid-block must still never let them into the output.
    wl = make_workload(seq_lens=[1000, 333, 77], query_lens=[3, 1, 2], num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=16, window=50, seed=19)
    ref = oracle.decode(problem(wl))
    for b, (S, L) in enumerate(zip(wl.seq_lens.tolist(), wl.query_lens.tolist())):
        first = max(0, S - L + 1 - 50)
        for t in range(first):
            blk = int(wl.block_tables[b, t // 16])
            wl.k_cache[blk, :, t % 16] = float("nan")
            wl.v_cache[blk, :, t % 16] = float("nan")
    out = pa.decode(dev(wl), force_variant=variant)
    assert_close(out.float().cpu().numpy(), ref, f"window garbage variant={variant}")


def test_no_hints_path_matches_hinted():
    wl = scaled(3)
    d = dev(wl)
    a = pa.decode(d, hints=True)
    b = pa.decode(d, hints=False)
    assert torch.equal(a, b)


def test_visible_ranges_match_oracle_exactly():
    cases = [config_lengths(c) for c in (1, 2, 3, 4, 5)]
    cases += [([300, 40], [5, 1], w, None) for w in (0, 1, 2, 5, 16, 100, 4096)]
    cases += [([7, 1, 9, 2500, 33] * 300, [3, 1, 0, 5, 2] * 300, 0, [2, 0, 4, 333, 1] * 300)]
    for s, l, w, ws in cases:
        S = torch.tensor(s, dtype=torch.int32, device="cuda:0")
        L = torch.tensor(l, dtype=torch.int32, device="cuda:0")
        W = None if ws is None else torch.tensor(ws, dtype=torch.int32, device="cuda:0")
        lo, hi = pa.visible_ranges(S, L, w, W)
        rlo, rhi = oracle.visible_ranges(s, l, w, ws)
        assert np.array_equal(lo.cpu().numpy(), rlo)
        assert np.array_equal(hi.cpu().numpy(), rhi)


# kinds of q / tables+lengths+windows / dst host buffers, and byte offsets of
# q, tables and dst inside their buffers (offsets that break 16-byte or 4-byte
# alignment take the narrower staging copies or the copy-back path)
HOST_CASES = {
    "pinned": (("pinned", "pinned", "pinned"), (0, 0, 0)),
    "pageable": (("pageable", "pageable", "pageable"), (0, 0, 0)),
    "mixed": (("pinned", "pageable", "pinned"), (0, 0, 0)),
    "offsets": (("pinned", "pinned", "pinned"), (2, 4, 2)),
    "offsets16": (("pinned", "pinned", "pinned"), (16, 32, 48)),
}


@pytest.mark.parametrize("case", list(HOST_CASES))
@pytest.mark.parametrize("cfg", [2, 5])
def test_host_entry_point_matches_device_path(cfg, case):
    (kq, kt, kd), (oq, ot, od) = HOST_CASES[case]
    wl = scaled(cfg)
    d = dev(wl)
    ref = pa.decode(d)
    p = pa.make_params(batch=wl.batch, num_q_heads=wl.num_q_heads,
                       num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim,
                       num_blocks=wl.num_blocks, max_blocks_per_seq=wl.max_blocks_per_seq)
    keep = []

    def host(t, kind, off=0):
        buf, ptr = host_buffer(t, kind, off)
        keep.append(buf)
        return ptr
    S = host(wl.seq_lens, kt)
    L = host(wl.query_lens, kt)
    if wl.windows is not None:
        p.windows = host(wl.windows, kt)
    n = pa.pa_host_workspace_size(p, wl.block_size, wl.window, S, L)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda:0")
    p.workspace, p.workspace_bytes = ws.data_ptr(), n
    q = host(wl.q, kq, oq)
    bt = host(wl.block_tables, kt, ot)
    out_buf, out_ptr = host_buffer(torch.full(wl.q.shape, float("nan"), dtype=torch.bfloat16),
                                    kd, od)
    for _ in range(2):   # twice: the second call overwrites the first's output in place
        rc = pa.pa_decode_host(out_ptr, q, d.k_cache.data_ptr(), d.v_cache.data_ptr(), bt, S, L,
                               wl.scale, wl.window, wl.block_size, p, pa._stream_handle())
        assert rc == pa.PA_OK, pa.pa_last_error()
        nbytes = ref.numel() * 2
        got = out_buf[od:od + nbytes].view(torch.bfloat16).reshape(ref.shape)
        assert torch.equal(got, ref.cpu())
    # bytes around dst are untouched
    assert torch.all(out_buf[:od] == 0) and torch.all(out_buf[od + nbytes:] == 0)


# ---------------------------------------------------- full size, sampled
@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_named_workload_full_size_sampled(cfg):
    wl = config_workload(cfg, device="cuda:0")
    out = pa.decode(wl)
    torch.cuda.synchronize()
    n = 48
    sel = sample_queries(wl, n, seed=cfg)
    if cfg in (3, 5):   # make sure every kind of row is sampled
        L = wl.query_lens.cpu().tolist()
        kinds = {}
        for b, l in enumerate(L):
            kinds.setdefault((l, None if wl.windows is None else int(wl.windows[b])), b)
        for b in kinds.values():
            sel += [(b, L[b] - 1, 0), (b, 0, wl.num_q_heads - 1)]
    if cfg == 5:       # keep the gathered sub-problem small: few distinct rows
        rows = sorted({b for b, _, _ in sel})[:6]
        sel = [t for t in sel if t[0] in rows]
    check_sampled(wl, out, sel, f"cfg{cfg} full size")


# ------------------------------------------------------------ error paths
def test_small_workspace_is_rejected():
    wl = dev(scaled(4))
    p = pa.params_for(wl)
    need = pa.pa_workspace_size(p, wl.block_size)
    assert need > 0
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda:0")
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    out = torch.empty_like(wl.q)
    rc = pa.pa_decode(out.data_ptr(), wl.q.data_ptr(), wl.k_cache.data_ptr(),
                      wl.v_cache.data_ptr(), wl.block_tables.data_ptr(),
                      wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(), wl.scale,
                      wl.window, wl.block_size, p, pa._stream_handle())
    assert rc == pa.PA_ERR_WORKSPACE


def _raw_decode(wl, p, out):
    return pa.pa_decode(out.data_ptr(), wl.q.data_ptr(), wl.k_cache.data_ptr(),
                        wl.v_cache.data_ptr(), wl.block_tables.data_ptr(),
                        wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(), wl.scale,
                        wl.window, wl.block_size, p, pa._stream_handle())


def test_device_detects_rows_beyond_hints_and_bad_blocks():
    wl = dev(make_workload(seq_lens=[900, 40], query_lens=[1, 1], num_q_heads=4,
                           num_kv_heads=2, head_dim=64, block_size=16, seed=2))
    # span hint smaller than the real span: the long row is skipped and flagged
    p = pa.params_for(wl)
    p.max_span_hint = 100
    ws = pa.alloc_workspace(p, 16)
    if ws is not None:
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    out = torch.zeros_like(wl.q)
    assert _raw_decode(wl, p, out) == pa.PA_OK
    assert pa.pa_device_status(clear=True) & pa.PA_DEV_HINT
    # block-table entries outside the pool (above it, or negative) are flagged,
    # not dereferenced, also in a partition's first stage, which this one-wave,
    # window-free plan issues before the lengths arrive
    for first, value in ((1, wl.num_blocks + 5), (0, -7)):
        bad = wl.block_tables.clone()
        bad[first, 0] = value
        wl2 = type(wl)(**{**wl.__dict__, "block_tables": bad})
        p = pa.params_for(wl2)
        ws = pa.alloc_workspace(p, 16)
        if ws is not None:
            p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
        assert _raw_decode(wl2, p, out) == pa.PA_OK
        assert pa.pa_device_status(clear=True) & pa.PA_DEV_BAD_BLOCK
    # a row whose queryLen exceeds its seqLen is flagged when hints skip the host check
    lens = torch.tensor([900, 2], dtype=torch.int32, device="cuda:0")
    ql = torch.tensor([1, 3], dtype=torch.int32, device="cuda:0")
    wl3 = type(wl)(**{**wl.__dict__, "query_lens": ql, "seq_lens": lens,
                      "q": torch.zeros(4, 4, 64, dtype=torch.bfloat16, device="cuda:0")})
    p = pa.params_for(wl, hints=False)
    p.max_span_hint, p.max_query_len_hint = 900, 3
    ws = pa.alloc_workspace(p, 16)
    if ws is not None:
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    out3 = torch.zeros(4, 4, 64, dtype=torch.bfloat16, device="cuda:0")
    assert _raw_decode(wl3, p, out3) == pa.PA_OK
    assert pa.pa_device_status(clear=True) & pa.PA_DEV_BAD_ROW


@pytest.mark.parametrize("seq_len", [64, 512, 4096, 16384])
def test_executorch_h100_benchmark_shape(seq_len):
    # ExecuTorch PR #18759's standalone kernel benchmark shape (B=1, H_q=16,
    # H_kv=2, D=256, one decode token), here over a paged cache
    wl = make_workload(seq_lens=[seq_len], query_lens=[1], num_q_heads=16, num_kv_heads=2,
                       head_dim=256, block_size=16, seed=seq_len)
    out = pa.decode(dev(wl))
    check_full(wl, out, f"D=256 S={seq_len}")


@pytest.mark.parametrize("block_size", [16, 1024])
@pytest.mark.parametrize("parts", [0, 3, 80])
def test_head_dim_256_mixed_rows_and_windows(block_size, parts):
    wl = make_workload(seq_lens=[3000, 77, 1500, 300], query_lens=[1, 2, 4, 5], num_q_heads=8,
                       num_kv_heads=2, head_dim=256, block_size=block_size,
                       windows=[100, 0, 700, 16], seed=block_size + parts)
    out = pa.decode(dev(wl), force_partitions=parts)
    check_full(wl, out, f"D=256 BS={block_size} parts={parts}")


def test_unreachable_blocks_match_oracle():
    cases = [config_lengths(c) for c in (1, 2, 3, 4, 5)]
    cases += [([300, 40], [5, 1], w, None) for w in (0, 1, 16, 100, 4096)]
    rng = np.random.default_rng(8)
    s = rng.integers(1, 70000, 500).tolist()
    l = [int(min(x, y)) for x, y in zip(s, rng.integers(0, 6, 500).tolist())]
    cases.append((s, l, 0, rng.choice([0, 1, 63, 64, 4096, 30000], 500).tolist()))
    for bs in (16, 64, 1024):
        for s, l, w, ws in cases:
            S = torch.tensor(s, dtype=torch.int32, device="cuda:0")
            L = torch.tensor(l, dtype=torch.int32, device="cuda:0")
            W = None if ws is None else torch.tensor(ws, dtype=torch.int32, device="cuda:0")
            got = pa.unreachable_blocks(S, L, bs, w, W).cpu().numpy()
            assert np.array_equal(got, oracle.unreachable_blocks(s, l, bs, w, ws))


# ------------------------------------------------- work-list schedule
def _wl_case(case):
    if case == "long":
        return make_workload(seq_lens=[9001], query_lens=[1], num_q_heads=8, num_kv_heads=1,
                             head_dim=128, block_size=16, seed=41)
    if case == "rows":
        return make_workload(seq_lens=[5000, 333, 77, 1], query_lens=[1, 3, 2, 1], num_q_heads=8,
                             num_kv_heads=2, head_dim=128, block_size=16, seed=42)
    if case == "windows":
        return make_workload(seq_lens=[6000, 2500, 300], query_lens=[2, 1, 5], num_q_heads=8,
                             num_kv_heads=2, head_dim=64, block_size=64, windows=[1000, 0, 16],
                             seed=43)
    if case == "slabs":
        return make_workload(seq_lens=[3000, 1200], query_lens=[5, 2], num_q_heads=32,
                             num_kv_heads=2, head_dim=128, block_size=16, seed=44)
    if case == "fp8":
        return make_workload(seq_lens=[7000, 900], query_lens=[1, 4], num_q_heads=16,
                             num_kv_heads=2, head_dim=128, block_size=1024, seed=45,
                             kv_dtype="fp8_e4m3")
    if case == "d256":
        return make_workload(seq_lens=[4000, 100], query_lens=[1, 2], num_q_heads=16,
                             num_kv_heads=2, head_dim=256, block_size=16, seed=46)
    raise ValueError(case)


@pytest.mark.parametrize("case", ["long", "rows", "windows", "slabs", "fp8", "d256"])
def test_work_list_schedule_matches_oracle(case):
    wl = _wl_case(case)
    d = dev(wl)
    _, info = pa.pa_plan(pa.params_for(d, schedule=pa.PA_SCHED_WORKLIST), wl.block_size)
    assert info.max_partitions > 1 and info.worklist
    out = pa.decode(d, schedule=pa.PA_SCHED_WORKLIST)
    check_full(wl, out, f"work list {case}")


@pytest.mark.parametrize("parts", [2, 7, 30])
def test_work_list_schedule_with_forced_partitions(parts):
    # more CTAs per unit than stages for the short rows: some claim nothing
    wl = _wl_case("rows")
    out = pa.decode(dev(wl), schedule=pa.PA_SCHED_WORKLIST, force_partitions=parts)
    check_full(wl, out, f"work list parts={parts}")


@pytest.mark.parametrize("fill", [0x00, 0xFF, "random", "reuse"])
def test_work_list_workspace_needs_no_initialisation(fill):
    # the counters are epoch-tagged: stale, garbage or reused workspaces give
    # the same result as a fresh one
    wl = _wl_case("rows")
    d = dev(wl)
    p = pa.params_for(d, schedule=pa.PA_SCHED_WORKLIST)
    ws = pa.alloc_workspace(p, wl.block_size)
    if fill == "random":
        ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device=ws.device))
    elif fill != "reuse":
        ws.fill_(fill)
    ref = oracle.decode(problem(wl))
    for _ in range(3 if fill == "reuse" else 1):
        out = pa.decode(d, workspace=ws, schedule=pa.PA_SCHED_WORKLIST)
        assert_close(out.float().cpu().numpy(), ref, f"work list workspace {fill}")


@pytest.mark.parametrize("parts", [1, 2, 3])
@pytest.mark.parametrize("head_dim,kv_dtype", [(64, "bf16"), (64, "fp8_e4m3"), (128, "bf16"),
                                               (128, "fp8_e4m3")])
def test_work_list_stage_counts_around_the_fixed_runs(head_dim, kv_dtype, parts):
    # Each CTA owns (ring depth + 2) stages outright and claims the rest from
    # the unit's counter.  Rows of parts x that many stages, give or take
    # three (ragged last stage), put the first claims and the first claim past
    # the end on either ring parity; the rings here are 3, 4 and 8 deep.
    probe = make_workload(seq_lens=[64], query_lens=[1], num_q_heads=8, num_kv_heads=2,
                          head_dim=head_dim, block_size=16, kv_dtype=kv_dtype)
    rc, info = pa.pa_plan(pa.params_for(probe, force_partitions=1,
                                        schedule=pa.PA_SCHED_WORKLIST), 16)
    assert rc == pa.PA_OK, pa.pa_last_error()
    fixed = parts * (info.stages + 2)
    S = [n * 64 - 8 for n in range(fixed - 3, fixed + 4)]
    wl = make_workload(seq_lens=S, query_lens=[1] * len(S), num_q_heads=8, num_kv_heads=2,
                       head_dim=head_dim, block_size=16, seed=78, kv_dtype=kv_dtype)
    d = dev(wl)
    _, plan = pa.pa_plan(pa.params_for(d, force_partitions=parts,
                                       schedule=pa.PA_SCHED_WORKLIST), 16)
    assert plan.worklist and plan.stages == info.stages
    out = pa.decode(d, force_partitions=parts, schedule=pa.PA_SCHED_WORKLIST)
    check_full(wl, out, f"work list D={head_dim} {kv_dtype} parts={parts}")


def test_work_list_schedule_refuses_multi_wave_grids():
    d = dev(scaled(2))
    p = pa.params_for(d, force_partitions=40, schedule=pa.PA_SCHED_WORKLIST)
    rc, _ = pa.pa_plan(p, 16)
    assert rc == pa.PA_ERR_UNSUPPORTED


def test_work_list_full_size_long_context_sampled():
    wl = config_workload(4, device="cuda:0")
    out = pa.decode(wl, schedule=pa.PA_SCHED_WORKLIST)
    torch.cuda.synchronize()
    check_sampled(wl, out, sample_queries(wl, 32, seed=77), "work list long context")


@pytest.mark.parametrize("limit", [20_000, 2_000_000])
def test_work_list_merge_wait_gives_up_and_the_next_call_is_correct(limit):
    # The work-list merge waits for its unit's arrivals on a counter other
    # CTAs bump; the wait is bounded.  The test knob raises the target by one
    # so it is never met: every merging CTA gives up after `limit` SM clocks
    # (~10 us or ~1 ms), the kernel returns, the status word says
    # PA_DEV_TIMEOUT, and no dst element is written (the single row needs
    # many partitions, so nothing takes the one-shot path).  The next normal
    # call on the same workspace, with stale counters left behind, is exact.
    wl = _wl_case("long")
    d = dev(wl)
    p = pa.params_for(d, schedule=pa.PA_SCHED_WORKLIST)
    _, info = pa.pa_plan(p, wl.block_size)
    assert info.worklist and info.max_partitions > 1
    ws = pa.alloc_workspace(p, wl.block_size)
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    p.wait_limit_cycles = limit
    p.merge_target_extra = 1
    out = torch.full(d.q.shape, float("nan"), dtype=torch.bfloat16, device="cuda:0")
    assert _raw_decode(d, p, out) == pa.PA_OK, pa.pa_last_error()
    torch.cuda.synchronize()
    assert pa.pa_device_status(clear=True) == pa.PA_DEV_TIMEOUT
    assert torch.isnan(out.float()).all()
    p.wait_limit_cycles = 0
    p.merge_target_extra = 0
    for _ in range(2):
        out = torch.full(d.q.shape, float("nan"), dtype=torch.bfloat16, device="cuda:0")
        assert _raw_decode(d, p, out) == pa.PA_OK, pa.pa_last_error()
        check_full(wl, out, "work list after a timed-out call")


def test_wait_knobs_must_not_be_negative():
    d = dev(_wl_case("long"))
    p = pa.params_for(d, schedule=pa.PA_SCHED_WORKLIST)
    p.wait_limit_cycles = -1
    assert pa.pa_plan(p, 16)[0] == pa.PA_ERR_ARG


@pytest.mark.parametrize("head_dim", [64, 128, 256])
@pytest.mark.parametrize("parts", [33, 65, 129, 300, 700, 1500])
def test_reduce_splits_over_partial_counts(head_dim, parts):
    # The reduce splits head_dim so that at most 16 warps, two partials per
    # lane, cover a row's partials: forced partition counts of one 8-row unit
    # (64-token partitions, a ragged last one) reach every split from one to
    # sixteen CTAs per row and, past 512 partials, several rounds per lane.
    S = parts * 64 - 5
    wl = make_workload(seq_lens=[S], query_lens=[1], num_q_heads=8, num_kv_heads=1,
                       head_dim=head_dim, block_size=64, seed=parts + head_dim)
    d = dev(wl)
    rc, info = pa.pa_plan(pa.params_for(d, force_partitions=parts), 64)
    # 64-token partitions: the row has `parts` of them (the plan sizes for one
    # more, the 64-token alignment of a span's start)
    assert rc == pa.PA_OK and info.partition_tokens == 64
    out = pa.decode(d, force_partitions=parts)
    check_full(wl, out, f"reduce D={head_dim} parts={parts}")
