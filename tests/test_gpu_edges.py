"""GPU parity on edge cases of the lengths: query tokens that cover the whole
context (L == S), one-token rows, windows at and around the query length,
rows without queries between rows with queries, and a large batch of short
rows (thousands of (row, kv head) units and a long query-offset scan), on
both kernel variants and with FP8 caches; and a call captured in a CUDA graph
and replayed on new queries."""
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
