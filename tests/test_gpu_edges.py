"""GPU parity on edge cases of the lengths: query tokens that cover the whole
context (L == S), one-token rows, windows at and around the query length,
rows without queries between rows with queries, and a large batch of short
rows (thousands of (row, kv head) units and a long query-offset scan), on
both kernel variants and with FP8 caches; and a call captured in a CUDA graph
and replayed on new queries; a decode loop whose inputs are written by the
kernel just before each call."""
import numpy as np
import pytest
import torch

from tests.parity_helpers import check_full, check_sampled, sample_queries

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_474_b200")
from paged_kv_cache_474_b200.workloads import make_workload  # noqa: E402


@pytest.fixture(autouse=True)
def _device_status_clean(cuda_device):
    pa.pa_device_status(clear=True)
    yield
    assert pa.pa_device_status(clear=True) == 0


VARIANTS = [pa.PA_VARIANT_FMA, pa.PA_VARIANT_MMA]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("window", [0, 1, 3, 5, 6])
def test_queries_cover_the_whole_context(window, variant):
    # L == S: the row is a prefill chunk from position 0; token i sees [.., i]
    wl = make_workload(seq_lens=[5, 1, 3, 70, 64], query_lens=[5, 1, 3, 5, 4],
                       num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                       window=window, seed=50 + window)
    out = pa.decode(wl.to("cuda:0"), force_variant=variant)
    check_full(wl, out, f"L==S window={window} variant={variant}")


@pytest.mark.parametrize("variant", VARIANTS)
def test_empty_rows_between_query_rows(variant):
    wl = make_workload(seq_lens=[40, 9, 700, 1, 33, 2000, 5], query_lens=[0, 3, 0, 1, 0, 2, 0],
                       num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=32,
                       windows=[7, 0, 3, 1, 0, 100, 2], seed=60)
    out = pa.decode(wl.to("cuda:0"), force_variant=variant, force_partitions=3)
    check_full(wl, out, f"empty rows variant={variant}")


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
def test_windows_at_the_query_length(kv_dtype):
    # w = L - 1, L, L + 1 for a 4-token chunk: the earliest query token's
    # range starts at, or just before, the chunk
    rows = [(200, 4, 3), (200, 4, 4), (200, 4, 5), (17, 4, 4), (4, 4, 4), (4, 4, 3)]
    wl = make_workload(seq_lens=[r[0] for r in rows], query_lens=[r[1] for r in rows],
                       num_q_heads=16, num_kv_heads=4, head_dim=128, block_size=16,
                       windows=[r[2] for r in rows], seed=61, kv_dtype=kv_dtype)
    out = pa.decode(wl.to("cuda:0"))
    check_full(wl, out, f"window around L kv={kv_dtype}")


def test_large_batch_of_short_rows():
    # 3000 rows of 1..300 tokens: 24000 units, a long offset scan per CTA
    g = np.random.default_rng(62)
    S = g.integers(1, 301, 3000).tolist()
    L = [int(min(s, x)) for s, x in zip(S, g.integers(0, 3, 3000).tolist())]
    wl = make_workload(seq_lens=S, query_lens=L, num_q_heads=8, num_kv_heads=8, head_dim=64,
                       block_size=16, windows=g.choice([0, 1, 50], 3000).tolist(), seed=62,
                       device="cuda:0")
    out = pa.decode(wl)
    torch.cuda.synchronize()
    rows = [b for b in range(3000) if L[b] > 0]
    sel = sample_queries(wl, 48, seed=62, rows=rows[-200:]) + sample_queries(wl, 16, seed=63)
    check_sampled(wl, out, sel, "3000 short rows")


def test_decode_replays_inside_a_cuda_graph():
    # With host hints set, pa_decode makes no synchronising call, so a stream
    # capture records its launches (the partition kernel and the reduce, with
    # their programmatic dependency); replays read the tensors' current values.
    import paged_kv_cache_474_b200 as pa
    from paged_kv_cache_474_b200.workloads import make_workload
    wl = make_workload(seq_lens=[3000, 700, 45], query_lens=[1, 2, 1], num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=16, seed=91, device="cuda:0")
    p = pa.params_for(wl)
    ws = pa.alloc_workspace(p, wl.block_size, device="cuda:0")
    if ws is not None:
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    out = torch.empty(wl.q.shape, dtype=torch.bfloat16, device="cuda:0")
    q = wl.q.clone()

    def call():
        rc = pa.pa_decode(out.data_ptr(), q.data_ptr(), wl.k_cache.data_ptr(),
                          wl.v_cache.data_ptr(), wl.block_tables.data_ptr(),
                          wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(), wl.scale,
                          wl.window, wl.block_size, p, pa._stream_handle())
        assert rc == pa.PA_OK, pa.pa_last_error()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()   # first call on this device sets kernel attributes outside the capture
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for seed in (1, 2, 3):
        g = torch.Generator(device="cuda:0").manual_seed(seed)
        q.copy_(torch.randn(q.shape, generator=g, device="cuda:0").to(torch.bfloat16))
        graph.replay()
        torch.cuda.synchronize()
        ref = pa.decode(type(wl)(**{**wl.__dict__, "q": q}))
        assert torch.equal(out, ref)
    assert pa.pa_device_status(clear=True) == 0


@pytest.mark.parametrize("variant", [pa.PA_VARIANT_AUTO, pa.PA_VARIANT_FMA])
@pytest.mark.parametrize("window", [0, 200])
def test_decode_loop_sees_inputs_written_just_before_each_call(variant, window):
    # A decode loop with no host synchronisation.  Steps cycle through four
    # orders, so that the kernel right before a call (the one a call may
    # overlap while it drains) writes, in turn: seq_lens (after the new K/V
    # token and q); the new K/V token (q is the previous call's dst); q; and
    # nothing of this step (no new token, q is the previous dst, the previous
    # call is the kernel before).  Each call's output is checked against the
    # oracle at that step's lengths (positions written later lie past the
    # step's context, so the final caches serve every step), and equals the
    # same call made alone after a synchronise.
    B, steps = 4, 8
    appends = [t % 4 != 3 for t in range(steps)]
    final = [900, 2500, 3100, 1700]
    wl = make_workload(seq_lens=final, query_lens=[1] * B, num_q_heads=8, num_kv_heads=2,
                       head_dim=128, block_size=16, window=window, seed=92, device="cuda:0")
    p = pa.params_for(wl, force_variant=variant)  # hints from the final lengths bound every step
    ws = pa.alloc_workspace(p, wl.block_size, device="cuda:0")
    if ws is not None:
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    g = torch.Generator(device="cuda:0").manual_seed(93)
    new_k = torch.randn((steps, B, 2, 128), generator=g, device="cuda:0").to(torch.bfloat16)
    new_v = torch.randn((steps, B, 2, 128), generator=g, device="cuda:0").to(torch.bfloat16)
    q_src = torch.randn((steps,) + tuple(wl.q.shape), generator=g,
                        device="cuda:0").to(torch.bfloat16)
    # host-side positions of each step's new token, made before the loop so
    # the loop launches only the kernels named above
    start = [s - sum(appends) for s in final]
    phys, off = [], []
    n = 0
    for t in range(steps):
        n += appends[t]
        tok = torch.tensor([s0 + n - 1 for s0 in start], dtype=torch.long)
        phys.append(wl.block_tables.cpu()[torch.arange(B), tok // 16].long().to("cuda:0"))
        off.append((tok % 16).to("cuda:0"))
    sl = torch.tensor(start, dtype=torch.int32, device="cuda:0")
    q_buf = torch.empty_like(wl.q)
    torch.cuda.synchronize()
    outs, qs, lens = [], [], []

    def call(q, out, lengths):
        rc = pa.pa_decode(out.data_ptr(), q.data_ptr(), wl.k_cache.data_ptr(),
                          wl.v_cache.data_ptr(), wl.block_tables.data_ptr(),
                          lengths.data_ptr(), wl.query_lens.data_ptr(), wl.scale,
                          wl.window, wl.block_size, p, pa._stream_handle())
        assert rc == pa.PA_OK, pa.pa_last_error()

    def append(t):
        wl.k_cache[phys[t], :, off[t], :] = new_k[t]
        wl.v_cache[phys[t], :, off[t], :] = new_v[t]

    def fresh_q(t):
        torch.add(q_src[t], 0, out=q_buf)
        return q_buf

    for t in range(steps):
        phase = t % 4
        if phase == 0:
            append(t)
            q = fresh_q(t)
            sl.add_(1)
        elif phase == 1:
            sl.add_(1)
            q = outs[-1]
            append(t)
        elif phase == 2:
            sl.add_(1)
            append(t)
            q = fresh_q(t)
        else:
            q = outs[-1]
        out = torch.empty_like(wl.q)
        call(q, out, sl)
        outs.append(out)
        qs.append(q.clone())  # stream-ordered after the call
        lens.append(sl.clone())
    torch.cuda.synchronize()
    for t in range(steps):
        wt = type(wl)(**{**wl.__dict__, "q": qs[t], "seq_lens": lens[t]})
        check_full(wt, outs[t], f"decode loop step {t} window={window} variant={variant}")
        alone = torch.empty_like(wl.q)
        call(qs[t], alone, lens[t])
        torch.cuda.synchronize()
        assert torch.equal(alone, outs[t]), f"step {t}"
    assert lens[-1].cpu().tolist() == final
    assert pa.pa_device_status(clear=True) == 0


def test_work_list_schedule_refuses_stream_capture():
    # its counters carry a per-call epoch that a graph replay would repeat
    wl = make_workload(seq_lens=[3000, 700], query_lens=[1, 1], num_q_heads=8, num_kv_heads=2,
                       head_dim=128, block_size=16, seed=94, device="cuda:0")
    p = pa.params_for(wl, schedule=pa.PA_SCHED_WORKLIST)
    ws = pa.alloc_workspace(p, wl.block_size, device="cuda:0")
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    out = torch.empty(wl.q.shape, dtype=torch.bfloat16, device="cuda:0")

    def call():
        return pa.pa_decode(out.data_ptr(), wl.q.data_ptr(), wl.k_cache.data_ptr(),
                            wl.v_cache.data_ptr(), wl.block_tables.data_ptr(),
                            wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(), wl.scale,
                            wl.window, wl.block_size, p, pa._stream_handle())
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        assert call() == pa.PA_OK, pa.pa_last_error()  # eager: fine
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out.zero_()
        rc = call()
    assert rc == pa.PA_ERR_UNSUPPORTED and "graph" in pa.pa_last_error()
    graph.replay()
    torch.cuda.synchronize()
    assert pa.pa_device_status(clear=True) == 0
