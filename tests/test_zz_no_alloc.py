"""pa_decode_noalloc: the decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (code under another framework's
allocator, plugins handed only their input and output buffers, hot paths that
must not allocate).  pa_decode_noalloc keeps the split-K partials in a static
array inside the library instead of a caller workspace.  These tests call it
through the C ABI and check, on two calls in a row, that its output is bit
for bit pa_decode's with a caller workspace (the same plan and kernels, only
the partials' address differs) and within the parity tolerance of the
float64 oracle; and that an oversized request is refused before any
launch.  The file sorts last so a stop-at-first-failure run has already run
every other test; it passes alone in a fresh process too.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_474_b200")
from paged_kv_cache_474_b200.workloads import make_workload  # noqa: E402

from tests.parity_helpers import check_full  # noqa: E402


def _call(fn, wl, p, out):
    return fn(out.data_ptr(), wl.q.data_ptr(), wl.k_cache.data_ptr(), wl.v_cache.data_ptr(),
              wl.block_tables.data_ptr(), wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(),
              wl.scale, wl.window, wl.block_size, p, pa._stream_handle())


@pytest.mark.parametrize("kind", ["long_single_group", "gqa_ragged_mtp", "fp8_kv"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device, kind):
    if kind == "long_single_group":
        wl = make_workload(seq_lens=[9001], query_lens=[1], num_q_heads=8, num_kv_heads=1,
                           head_dim=128, block_size=16, seed=31, device="cuda:0")
    elif kind == "fp8_kv":
        wl = make_workload(seq_lens=[6000, 300], query_lens=[1, 4], num_q_heads=16,
                           num_kv_heads=2, head_dim=128, block_size=16, seed=33,
                           device="cuda:0", kv_dtype="fp8_e4m3", q_dtype="fp8_e4m3")
    else:
        wl = make_workload(seq_lens=[3000, 777, 5120, 64], query_lens=[1, 3, 2, 1],
                           num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                           window=1500, seed=32, device="cuda:0")
    p = pa.params_for(wl)
    need = pa.pa_workspace_size(p, wl.block_size)
    assert 0 < need <= pa.PA_NOALLOC_SCRATCH_BYTES   # the split-K scratch is used
    ws = torch.empty(need, dtype=torch.uint8, device="cuda:0")
    p.workspace, p.workspace_bytes = ws.data_ptr(), need
    ref = torch.empty(wl.q.shape, dtype=torch.bfloat16, device="cuda:0")
    assert _call(pa.pa_decode, wl, p, ref) == pa.PA_OK, pa.pa_last_error()

    q = pa.params_for(wl)            # no workspace: the static array is used
    for _ in range(2):
        out = torch.full(wl.q.shape, float("nan"), dtype=torch.bfloat16, device="cuda:0")
        assert _call(pa.pa_decode_noalloc, wl, q, out) == pa.PA_OK, pa.pa_last_error()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        check_full(wl, out, f"no-alloc {kind}")
    assert pa.pa_device_status(clear=True) == 0


def test_noalloc_refuses_requests_beyond_the_static_array(cuda_device):
    wl = make_workload(seq_lens=[4096] * 8, query_lens=[4] * 8, num_q_heads=64, num_kv_heads=8,
                       head_dim=128, block_size=1024, seed=33, device="cuda:0")
    p = pa.params_for(wl, force_partitions=64)
    assert pa.pa_workspace_size(p, wl.block_size) > pa.PA_NOALLOC_SCRATCH_BYTES
    out = torch.zeros_like(wl.q)
    assert _call(pa.pa_decode_noalloc, wl, p, out) == pa.PA_ERR_WORKSPACE
    assert "needed" in pa.pa_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0      # nothing was launched
