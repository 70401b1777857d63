"""GPU parity on the five named workloads at full size, on every output element.

Each workload runs once through the C ABI in the launch configuration the
bench times (host hints, a workspace from pa_workspace_size, the
dispatcher's partitioning), and every element of dst is compared with the
float64 oracle under the parity tolerance |gpu - oracle| <= 2e-2 +
2e-2 * |oracle| (the reading of "max-abs 2e-2 and rel 2e-2 on every element";
gllm PR #116 "feat(backend): sliding-window PagedAttention", section
"Verification", compares the GPU kernel with the CPU reference on whole
outputs).  The large-block MTP workload's 9 GB pool is checked in row chunks:
each chunk's rows are gathered into a compact pool (Workload.subset) and the
oracle runs on that, which leaves each row's problem unchanged.

Each case prints the number of elements compared, the largest absolute
error and the largest relative error over elements with |oracle| > 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_helpers import ATOL, RTOL, token_offsets

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_474_b200")
from paged_kv_cache_474_b200.workloads import CONFIG_NAMES, config_workload  # noqa: E402


@pytest.fixture(autouse=True)
def _device_status_clean(cuda_device):
    pa.pa_device_status(clear=True)
    yield
    assert pa.pa_device_status(clear=True) == 0
    torch.cuda.empty_cache()


def _compare(got, ref, what):
    """Asserts the tolerance on every element; returns (n, max_abs, max_rel)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    big = np.abs(ref) > 1e-3
    max_rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {err.size} elements out of tolerance; "
                           f"max abs err {err.max():.3e}")
    return err.size, float(err.max()), max_rel


def _decode_full_size(cfg, kv_dtype):
    wl = config_workload(cfg, device="cuda:0", kv_dtype=kv_dtype)
    out = pa.decode(wl)     # host hints, workspace, dispatcher's plan: the bench's call
    torch.cuda.synchronize()
    return wl, out


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_named_workload_full_size_every_element(cfg, kv_dtype):
    wl, out = _decode_full_size(cfg, kv_dtype)
    ref = oracle.decode(oracle.problem_from_workload(wl))
    n, mabs, mrel = _compare(out.float().cpu().numpy(), ref, f"{CONFIG_NAMES[cfg]} {kv_dtype}")
    assert n == wl.num_tokens * wl.num_q_heads * wl.head_dim
    print(f"\n[full size] {CONFIG_NAMES[cfg]} {kv_dtype}: {n} elements, "
          f"max abs {mabs:.3e}, max rel {mrel:.3e}")


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8_e4m3"])
def test_large_block_mtp_full_size_every_element_in_row_chunks(kv_dtype):
    wl, out = _decode_full_size(5, kv_dtype)
    got = out.float().cpu().numpy()
    qoff = token_offsets(wl)
    n_all, mabs, mrel = 0, 0.0, 0.0
    chunk = 8
    for r0 in range(0, wl.batch, chunk):
        rows = list(range(r0, min(wl.batch, r0 + chunk)))
        sub, rmap = wl.subset(rows)
        ref = oracle.decode(oracle.problem_from_workload(sub))
        sub_off = np.concatenate([[0], np.cumsum(sub.query_lens.tolist())])
        for b in rows:
            j = rmap[b]
            n, a, r = _compare(got[qoff[b]:qoff[b + 1]], ref[sub_off[j]:sub_off[j + 1]],
                               f"mtp {kv_dtype} row {b}")
            n_all += n
            mabs, mrel = max(mabs, a), max(mrel, r)
        del sub
    assert n_all == wl.num_tokens * wl.num_q_heads * wl.head_dim
    print(f"\n[full size] mtp {kv_dtype}: {n_all} elements in {wl.batch} rows, "
          f"max abs {mabs:.3e}, max rel {mrel:.3e}")
