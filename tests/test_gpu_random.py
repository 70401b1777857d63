"""GPU parity on seeded random configurations: head_dim, block size, GQA
group, batch, lengths from one token to a few thousand, query lengths 0-5,
no window / one window / per-row windows, bf16 or FP8 caches and queries,
each kernel variant that supports the draw, forced partition counts and the
no-hints path, every output element against the oracle.  The draws mix the
shapes the named workloads use with combinations none of them has.  Subsets
of the draws also run through the host entry point, on the work-list
schedule, and with every position no query may see poisoned (NaN, and
out-of-pool table slots past each row); a second, wider family of draws
takes up to 48 rows and query lengths up to 16."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_helpers import (assert_close, check_full, host_buffer, poison_outside_spans,
                                  problem)

pa = pytest.importorskip("paged_kv_cache_474_b200")
from paged_kv_cache_474_b200.workloads import make_workload  # noqa: E402

NSEEDS = 160


def draw(seed):
    """One seeded configuration: (make_workload keywords, decode keywords)."""
    g = np.random.default_rng(1000 + seed)
    D = int(g.choice([64, 128, 128, 256]))
    BS = int(g.choice([16, 16, 32, 64, 128, 256, 512, 1024]))
    hkv = int(g.choice([1, 2, 4]))
    group = int(g.choice([1, 2, 3, 4, 5, 8, 16, 32]))
    B = int(g.integers(1, 7))
    kind = g.choice(["tiny", "mid", "long", "longer"], size=B, p=[0.3, 0.35, 0.25, 0.1])
    lo_hi = {"tiny": (1, 41), "mid": (41, 601), "long": (601, 3001), "longer": (3001, 12001)}
    S = [int(g.integers(*lo_hi[k])) for k in kind]
    L = [int(min(s, g.choice([0, 1, 1, 1, 2, 3, 5]))) for s in S]
    if sum(L) == 0:
        L[0] = 1
    wmode = g.choice(["none", "one", "rows"])
    window, windows = 0, None
    if wmode == "one":
        window = int(g.choice([1, 2, 7, 64, 500, 5000]))
    elif wmode == "rows":
        windows = [int(g.choice([0, 1, 3, 16, 100, 1000])) for _ in range(B)]
    kv_fp8 = g.random() < 0.3
    q_fp8 = g.random() < 0.15
    fp8 = kv_fp8 or q_fp8
    variants = [pa.PA_VARIANT_AUTO]
    if not fp8 and D != 256:
        variants.append(pa.PA_VARIANT_FMA)
    if kv_fp8 and D == 128:
        variants.append(pa.PA_VARIANT_TC)
    variant = int(g.choice(variants))
    parts = int(g.choice([0, 0, 0, 1, 2, 3, 7]))
    hints = bool(g.random() < 0.8)
    wl_kw = dict(seq_lens=S, query_lens=L, num_q_heads=hkv * group, num_kv_heads=hkv,
                 head_dim=D, block_size=BS, window=window, windows=windows,
                 dist=str(g.choice(["normal", "uniform"])), seed=2000 + seed,
                 spare_blocks=int(g.integers(1, 4)), extra_table_cols=int(g.integers(0, 3)),
                 kv_dtype="fp8_e4m3" if kv_fp8 else "bf16",
                 q_dtype="fp8_e4m3" if q_fp8 else "bf16")
    return wl_kw, dict(force_variant=variant, force_partitions=parts, hints=hints)


def draw_wide(seed):
    """A wider seeded configuration: up to 48 rows, query lengths up to 16
    (MTP and prefill chunks), windows at and around the query length, log-
    uniform context lengths; the oracle's work is capped by shortening rows."""
    g = np.random.default_rng(5000 + seed)
    D = int(g.choice([64, 128, 256]))
    BS = int(g.choice([16, 32, 64, 128, 256, 512, 1024]))
    hkv = int(g.choice([1, 2, 8]))
    group = int(g.choice([1, 2, 4, 6, 8, 12, 16]))
    B = int(g.integers(1, 49))
    S = [int(np.exp(g.uniform(0.0, np.log(6000.0)))) + 1 for _ in range(B)]
    L = [int(min(s, 1 if g.random() < 0.5 else g.integers(0, 17))) for s in S]
    if sum(L) == 0:
        L[0] = 1
    windows = None
    if g.random() < 0.6:
        windows = [int(g.choice([0, 1, max(1, l - 1), max(1, l), l + 1, 50, 2000]))
                   for l in L]
    budget = 4e8 / (hkv * group * D)
    while sum(l * min(s, (w or s) + l) for s, l, w in
              zip(S, L, windows or [0] * B)) > budget:
        S = [max(l, s // 2) for s, l in zip(S, L)]
    kv_fp8 = g.random() < 0.3
    q_fp8 = g.random() < 0.1
    fp8 = kv_fp8 or q_fp8
    variants = [pa.PA_VARIANT_AUTO]
    if not fp8 and D != 256:
        variants.append(pa.PA_VARIANT_FMA)
    if kv_fp8 and D == 128:
        variants.append(pa.PA_VARIANT_TC)
    wl_kw = dict(seq_lens=S, query_lens=L, num_q_heads=hkv * group, num_kv_heads=hkv,
                 head_dim=D, block_size=BS, windows=windows, seed=6000 + seed,
                 kv_dtype="fp8_e4m3" if kv_fp8 else "bf16",
                 q_dtype="fp8_e4m3" if q_fp8 else "bf16")
    return wl_kw, dict(force_variant=int(g.choice(variants)),
                       force_partitions=int(g.choice([0, 0, 2, 5])),
                       hints=bool(g.random() < 0.8))


NWIDE = 64


def test_draws_cover_the_space_and_plan_on_the_host():
    # the seeds below reach every head_dim, variant, dtype mix and window
    # mode, and every draw is a valid call (the host plan accepts it)
    draws = [draw(s) for s in range(NSEEDS)]
    for w, d in draws:
        wl = make_workload(**w)
        p = pa.params_for(wl, hints=True, force_variant=d["force_variant"],
                          force_partitions=d["force_partitions"])
        rc, _ = pa.pa_plan(p, wl.block_size, num_sms=148, ctas_per_sm=2)
        assert rc == pa.PA_OK, (w, d, pa.pa_last_error())
    assert {w["head_dim"] for w, _ in draws} == {64, 128, 256}
    assert {d["force_variant"] for _, d in draws} == {pa.PA_VARIANT_AUTO, pa.PA_VARIANT_FMA,
                                                       pa.PA_VARIANT_TC}
    assert {w["kv_dtype"] for w, _ in draws} == {"bf16", "fp8_e4m3"}
    assert {w["q_dtype"] for w, _ in draws} == {"bf16", "fp8_e4m3"}
    assert any(w["windows"] is not None for w, _ in draws)
    assert any(w["window"] > 0 for w, _ in draws)
    assert any(not d["hints"] for _, d in draws)
    assert {w["block_size"] for w, _ in draws} >= {16, 1024}
    # the work-list schedule (one-wave grids only) accepts a good share of them
    ok = 0
    for w, d in draws:
        if d["force_variant"] != pa.PA_VARIANT_AUTO:
            continue
        wl = make_workload(**w)
        p = pa.params_for(wl, force_partitions=d["force_partitions"],
                          schedule=pa.PA_SCHED_WORKLIST)
        ok += pa.pa_plan(p, wl.block_size, num_sms=148, ctas_per_sm=2)[0] == pa.PA_OK
    assert ok >= 40
    wide = [draw_wide(s) for s in range(NWIDE)]
    for w, d in wide:
        wl = make_workload(**w)
        p = pa.params_for(wl, force_variant=d["force_variant"],
                          force_partitions=d["force_partitions"])
        rc, _ = pa.pa_plan(p, wl.block_size, num_sms=148, ctas_per_sm=2)
        assert rc == pa.PA_OK, (w, d, pa.pa_last_error())
    assert max(max(w["query_lens"]) for w, _ in wide) >= 12
    assert max(len(w["seq_lens"]) for w, _ in wide) >= 40
    # poisoning touches only positions no query sees: the oracle is unchanged
    for w, _ in draws[::8]:
        wl = make_workload(**w)
        ref = oracle.decode(problem(wl))
        poison_outside_spans(wl)
        assert np.array_equal(oracle.decode(problem(wl)), ref)


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(NSEEDS))
def test_random_configuration(seed, cuda_device):
    wl_kw, dec_kw = draw(seed)
    wl = make_workload(**wl_kw)
    pa.pa_device_status(clear=True)
    out = pa.decode(wl.to("cuda:0"), **dec_kw)
    assert pa.pa_device_status(clear=True) == 0
    check_full(wl, out, f"seed {seed}: {wl_kw['head_dim']=} {wl_kw['block_size']=} "
                        f"{wl_kw['seq_lens']=} {wl_kw['query_lens']=} {dec_kw}")


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(0, NSEEDS, 4))
def test_random_configuration_host_entry(seed, cuda_device):
    # pa_decode_host with q, lengths, tables, windows and dst in host memory
    # (pinned or pageable, drawn per buffer): the same bits as the device
    # entry point with the same plan, and within tolerance of the oracle
    wl_kw, dec_kw = draw(seed)
    wl = make_workload(**wl_kw)
    d = wl.to("cuda:0")
    ref = pa.decode(d, force_variant=dec_kw["force_variant"],
                    force_partitions=dec_kw["force_partitions"])
    g = np.random.default_rng(3000 + seed)
    kq, kt, kd = (str(g.choice(["pinned", "pageable"])) for _ in range(3))
    keep = []

    def host(t, kind):
        buf, ptr = host_buffer(t, kind)
        keep.append(buf)
        return ptr
    p = pa.params_for(wl, hints=False, force_variant=dec_kw["force_variant"],
                      force_partitions=dec_kw["force_partitions"])
    S = host(wl.seq_lens, kt)
    L = host(wl.query_lens, kt)
    if wl.windows is not None:
        p.windows = host(wl.windows, kt)
    n = pa.pa_host_workspace_size(p, wl.block_size, wl.window, S, L)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device="cuda:0")
    p.workspace, p.workspace_bytes = ws.data_ptr(), n
    out_buf, out_ptr = host_buffer(torch.full(wl.q.shape, float("nan"), dtype=torch.bfloat16), kd)
    pa.pa_device_status(clear=True)
    rc = pa.pa_decode_host(out_ptr, host(wl.q, kq), d.k_cache.data_ptr(), d.v_cache.data_ptr(),
                           host(wl.block_tables, kt), S, L, wl.scale, wl.window, wl.block_size,
                           p, pa._stream_handle())
    assert rc == pa.PA_OK, pa.pa_last_error()
    assert pa.pa_device_status(clear=True) == 0
    got = out_buf[:ref.numel() * 2].view(torch.bfloat16).reshape(ref.shape)
    assert torch.equal(got, ref.cpu()), f"seed {seed} ({kq}, {kt}, {kd})"
    check_full(wl, got, f"host entry seed {seed}")


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(NSEEDS))
def test_random_configuration_work_list(seed, cuda_device):
    # the work-list schedule on every draw it accepts (the default variant,
    # grids of one wave on this GPU)
    wl_kw, dec_kw = draw(seed)
    if dec_kw["force_variant"] != pa.PA_VARIANT_AUTO:
        pytest.skip("the work-list schedule runs on the default variant only")
    wl = make_workload(**wl_kw)
    d = wl.to("cuda:0")
    p = pa.params_for(d, force_partitions=dec_kw["force_partitions"],
                      schedule=pa.PA_SCHED_WORKLIST)
    rc, _ = pa.pa_plan(p, wl.block_size)
    if rc == pa.PA_ERR_UNSUPPORTED:
        pytest.skip("grid of more than one wave")
    assert rc == pa.PA_OK, pa.pa_last_error()
    pa.pa_device_status(clear=True)
    out = pa.decode(d, force_partitions=dec_kw["force_partitions"],
                    schedule=pa.PA_SCHED_WORKLIST)
    assert pa.pa_device_status(clear=True) == 0
    check_full(wl, out, f"work list seed {seed}")


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(NWIDE))
def test_wide_random_configuration(seed, cuda_device):
    wl_kw, dec_kw = draw_wide(seed)
    wl = make_workload(**wl_kw)
    pa.pa_device_status(clear=True)
    out = pa.decode(wl.to("cuda:0"), **dec_kw)
    assert pa.pa_device_status(clear=True) == 0
    check_full(wl, out, f"wide seed {seed}: {dec_kw}")


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(0, NSEEDS, 2))
def test_random_configuration_never_reads_outside_spans(seed, cuda_device):
    # every position no query may see holds NaN and every table slot past a
    # row's blocks points outside the pool: outputs match the oracle on the
    # clean inputs, and no bad block is flagged (those slots are never used)
    wl_kw, dec_kw = draw(seed)
    wl = make_workload(**wl_kw)
    ref = oracle.decode(problem(wl))
    poison_outside_spans(wl)
    pa.pa_device_status(clear=True)
    out = pa.decode(wl.to("cuda:0"), **dec_kw)
    assert pa.pa_device_status(clear=True) == 0
    assert_close(out.float().cpu().numpy(), ref, f"poisoned seed {seed}: {dec_kw}")


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(0, NSEEDS, 5))
def test_random_configuration_replays_in_a_cuda_graph(seed, cuda_device):
    # with hints set a call only enqueues kernels: captured once, replayed on
    # new queries, it gives the same bits as an eager call on those queries
    wl_kw, dec_kw = draw(seed)
    wl = make_workload(**wl_kw).to("cuda:0")
    kw = dict(force_variant=dec_kw["force_variant"], force_partitions=dec_kw["force_partitions"])
    p = pa.params_for(wl, **kw)
    ws = pa.alloc_workspace(p, wl.block_size, device="cuda:0")
    if ws is not None:
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    q = wl.q.clone()
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda:0")

    def call():
        rc = pa.pa_decode(out.data_ptr(), q.data_ptr(), wl.k_cache.data_ptr(),
                          wl.v_cache.data_ptr(), wl.block_tables.data_ptr(),
                          wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(), wl.scale,
                          wl.window, wl.block_size, p, pa._stream_handle())
        assert rc == pa.PA_OK, pa.pa_last_error()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()  # the first call on a device sets kernel attributes outside the capture
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    g = torch.Generator(device="cuda:0").manual_seed(seed)
    for k in (1, 2):
        if q.dtype == torch.uint8:  # FP8 codes: other valid codes, the heads rotated
            q.copy_(wl.q.roll(k, 1))
        else:
            q.copy_(torch.randn(q.shape, generator=g, device="cuda:0").to(torch.bfloat16))
        graph.replay()
        torch.cuda.synchronize()
        eager = pa.decode(type(wl)(**{**wl.__dict__, "q": q.clone()}), **kw)
        assert torch.equal(out, eager), f"seed {seed} replay {k}"
    assert pa.pa_device_status(clear=True) == 0
