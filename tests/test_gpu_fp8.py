"""GPU parity of FP8 operands: pa_decode with FP8 e4m3 KV caches and/or an
FP8 query (per-tensor scales) against the float64 oracle, which decodes the
same codes from the e4m3 definition and multiplies by the same scales.

Same tolerance as the bf16 path (|gpu - oracle| <= 2e-2 + 2e-2 |oracle|):
the codes are exact inputs on both sides; only the kernel's f16 / fp32
arithmetic differs from the oracle's float64.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity_helpers import (assert_close, check_full, check_sampled, problem,
                                  sample_queries, scaled_workload, token_offsets)

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_474_b200")
from paged_kv_cache_474_b200.workloads import config_workload, make_workload  # noqa: E402

FP8 = "fp8_e4m3"
NAN_CODE = 0x7F   # e4m3 NaN (S.1111.111)


@pytest.fixture(autouse=True)
def _device_status_clean(cuda_device):
    pa.pa_device_status(clear=True)
    yield
    assert pa.pa_device_status(clear=True) == 0


def dev(wl):
    return wl.to("cuda:0")


@pytest.mark.parametrize("q_dtype", ["bf16", FP8])
@pytest.mark.parametrize("window", [0, 8])
@pytest.mark.parametrize("parts", [0, 1, 2, 3])
def test_tiny_workload_fp8_cache(window, parts, q_dtype):
    # head_dim 64: 64-byte FP8 rows, the 64-byte swizzle
    wl = config_workload(1, window=window, kv_dtype=FP8, q_dtype=q_dtype)
    out = pa.decode(dev(wl), force_partitions=parts)
    check_full(wl, out, f"tiny fp8 w={window} parts={parts} q={q_dtype}")


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
@pytest.mark.parametrize("parts", [0, 1, 5])
def test_scaled_named_workloads_fp8_cache(cfg, parts):
    wl = scaled_workload(cfg, kv_dtype=FP8)
    assert wl.k_scale != wl.v_scale
    out = pa.decode(dev(wl), force_partitions=parts)
    check_full(wl, out, f"scaled cfg{cfg} fp8 parts={parts}")


@pytest.mark.parametrize("head_dim", [64, 128, 256])
@pytest.mark.parametrize("block_size", [16, 32, 64, 256, 1024])
def test_head_dims_and_block_sizes_fp8(head_dim, block_size):
    wl = make_workload(seq_lens=[1, 17, 64, 65, 1500, 2049], query_lens=[1, 1, 2, 1, 4, 1],
                       num_q_heads=8, num_kv_heads=4, head_dim=head_dim,
                       block_size=block_size, window=0, seed=head_dim + block_size,
                       kv_dtype=FP8)
    out = pa.decode(dev(wl))
    check_full(wl, out, f"fp8 D={head_dim} BS={block_size}")


@pytest.mark.parametrize("group,qlen", [(1, 1), (2, 3), (8, 1), (8, 4), (16, 5), (64, 1)])
def test_row_tiles_and_slabs_fp8(group, qlen):
    wl = make_workload(seq_lens=[700, 64, 1999], query_lens=[qlen, min(qlen, 2), qlen],
                       num_q_heads=2 * group, num_kv_heads=2, head_dim=128, block_size=16,
                       window=0, seed=group * 10 + qlen, kv_dtype=FP8)
    out = pa.decode(dev(wl))
    check_full(wl, out, f"fp8 group={group} qlen={qlen}")


@pytest.mark.parametrize("head_dim", [64, 128, 256])
@pytest.mark.parametrize("kv_dtype", ["bf16", FP8])
def test_fp8_query(head_dim, kv_dtype):
    # FP8 query codes: converted to bf16 (bf16 caches) or f16 (FP8 caches)
    wl = make_workload(seq_lens=[300, 40, 1200], query_lens=[5, 1, 3], num_q_heads=8,
                       num_kv_heads=2, head_dim=head_dim, block_size=16,
                       windows=[16, 0, 100], seed=head_dim, kv_dtype=kv_dtype, q_dtype=FP8)
    out = pa.decode(dev(wl))
    check_full(wl, out, f"fp8 q D={head_dim} kv={kv_dtype}")


@pytest.mark.parametrize("parts", [1, 2, 7, 64, 200])
def test_split_k_invariance_fp8(parts):
    wl = make_workload(seq_lens=[5000, 3333, 77], query_lens=[1, 3, 2], num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=16, window=0, seed=7,
                       kv_dtype=FP8)
    d = dev(wl)
    out = pa.decode(d, force_partitions=parts)
    check_full(wl, out, f"fp8 parts={parts}")
    base = pa.decode(d, force_partitions=1).float()
    assert torch.max(torch.abs(out.float() - base)).item() < 2e-2


@pytest.mark.parametrize("head_dim", [64, 128])
def test_fp8_nan_codes_outside_spans_are_never_read(head_dim):
    # NaN codes past each row's last token, before each window and in blocks
    # no table reaches: the outputs must not see them.
    wl = make_workload(seq_lens=[1000, 333, 77, 50], query_lens=[3, 1, 2, 1], num_q_heads=8,
                       num_kv_heads=2, head_dim=head_dim, block_size=16,
                       windows=[50, 0, 20, 0], seed=19, spare_blocks=2, extra_table_cols=3,
                       kv_dtype=FP8)
    ref = oracle.decode(problem(wl))
    W = wl.windows.tolist()
    for b, (S, L) in enumerate(zip(wl.seq_lens.tolist(), wl.query_lens.tolist())):
        nb = (S + 15) // 16
        last = int(wl.block_tables[b, nb - 1])
        wl.k_cache[last, :, S - (nb - 1) * 16:] = NAN_CODE
        wl.v_cache[last, :, S - (nb - 1) * 16:] = NAN_CODE
        first = max(0, S - L + 1 - W[b]) if W[b] > 0 else 0
        for t in range(first):
            blk = int(wl.block_tables[b, t // 16])
            wl.k_cache[blk, :, t % 16] = NAN_CODE
            wl.v_cache[blk, :, t % 16] = NAN_CODE
        wl.block_tables[b, nb:] = 10 ** 6
    used = set(wl.block_tables[wl.block_tables < wl.num_blocks].tolist())
    for blk in range(wl.num_blocks):
        if blk not in used:
            wl.k_cache[blk] = NAN_CODE
            wl.v_cache[blk] = NAN_CODE
    out = pa.decode(dev(wl))
    assert_close(out.float().cpu().numpy(), ref, f"fp8 NaN codes outside spans D={head_dim}")


def test_fp8_window_one_returns_scaled_own_value():
    # window 1: the output is v_scale times the token's own e4m3 value
    wl = make_workload(seq_lens=[70, 3, 1000], query_lens=[3, 1, 2], num_q_heads=4,
                       num_kv_heads=2, head_dim=128, block_size=16, window=1, seed=3,
                       kv_dtype=FP8)
    out = pa.decode(dev(wl)).cpu().double()
    qoff = token_offsets(wl)
    for b, (S, L) in enumerate(zip(wl.seq_lens.tolist(), wl.query_lens.tolist())):
        for i in range(L):
            p = S - L + i
            phys = int(wl.block_tables[b, p // 16])
            for h in range(4):
                v = oracle.e4m3_decode(wl.v_cache[phys, h // 2, p % 16].numpy()) * wl.v_scale
                # left: v_scale in fp32, the fp32 product and the bf16 store
                want = torch.from_numpy(v)
                assert torch.allclose(out[qoff[b] + i, h], want, rtol=2 ** -7, atol=0)


def test_fp8_cache_with_large_bf16_queries():
    # bf16 queries meet FP8 caches as f16 operands: values far from 1 (but in
    # f16's range) must still convert exactly
    wl = make_workload(seq_lens=[900, 45], query_lens=[2, 1], num_q_heads=8, num_kv_heads=2,
                       head_dim=128, block_size=16, window=0, seed=5, kv_dtype=FP8,
                       scale=1e-3)
    wl.q = (wl.q.float() * 3000.0).to(torch.bfloat16)
    out = pa.decode(dev(wl))
    check_full(wl, out, "fp8 cache, |q| ~ 1e4")


def test_host_entry_point_fp8_query_matches_device_path():
    wl = scaled_workload(3, kv_dtype=FP8, q_dtype=FP8)
    d = dev(wl)
    ref = pa.decode(d)
    p = pa.params_for(wl, hints=False)
    S = wl.seq_lens.numpy().copy()
    L = wl.query_lens.numpy().copy()
    n = pa.pa_host_workspace_size(p, wl.block_size, wl.window, S.ctypes.data, L.ctypes.data)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda:0")
    p.workspace, p.workspace_bytes = ws.data_ptr(), n
    q_host = wl.q.contiguous().pin_memory()
    out_host = torch.empty(wl.q.shape, dtype=torch.bfloat16).pin_memory()
    bt = wl.block_tables.contiguous().numpy()
    rc = pa.pa_decode_host(out_host.data_ptr(), q_host.data_ptr(), d.k_cache.data_ptr(),
                           d.v_cache.data_ptr(), bt.ctypes.data, S.ctypes.data, L.ctypes.data,
                           wl.scale, wl.window, wl.block_size, p, pa._stream_handle())
    assert rc == pa.PA_OK, pa.pa_last_error()
    assert torch.equal(out_host, ref.cpu())


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_named_workload_full_size_sampled_fp8(cfg):
    wl = config_workload(cfg, device="cuda:0", kv_dtype=FP8)
    out = pa.decode(wl)
    torch.cuda.synchronize()
    sel = sample_queries(wl, 32, seed=100 + cfg)
    if cfg == 5:
        rows = sorted({b for b, _, _ in sel})[:6]
        sel = [t for t in sel if t[0] in rows]
    check_sampled(wl, out, sel, f"cfg{cfg} fp8 full size")


def test_missing_scale_is_rejected_before_launch():
    wl = dev(scaled_workload(2, kv_dtype=FP8))
    p = pa.params_for(wl)
    p.v_scale = 0.0
    out = torch.zeros(wl.q.shape, dtype=torch.bfloat16, device="cuda:0")
    rc = pa.pa_decode(out.data_ptr(), wl.q.data_ptr(), wl.k_cache.data_ptr(),
                      wl.v_cache.data_ptr(), wl.block_tables.data_ptr(),
                      wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(), wl.scale, wl.window,
                      wl.block_size, p, pa._stream_handle())
    assert rc == pa.PA_ERR_ARG and "v_scale" in pa.pa_last_error()
    assert not out.any()


# ------------------------------------------- tensor-memory (tcgen05) kernel
TC = pa.PA_VARIANT_TC


def _variant_of(wl, **kw):
    _, info = pa.pa_plan(pa.params_for(dev(wl), **kw), wl.block_size)
    return info.variant


@pytest.mark.parametrize("variant", [pa.PA_VARIANT_MMA, TC])
@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
@pytest.mark.parametrize("parts", [0, 1, 5])
def test_tensor_memory_kernel_on_the_named_shapes(cfg, parts, variant):
    # the forced tensor-memory kernel runs units of more than 8 rows as slabs
    wl = scaled_workload(cfg, kv_dtype=FP8, seed=3)
    assert _variant_of(wl, force_variant=variant) == variant
    out = pa.decode(dev(wl), force_partitions=parts, force_variant=variant)
    check_full(wl, out, f"cfg{cfg} parts={parts} variant={variant}")


def test_tensor_memory_kernel_runs_on_request_only():
    assert _variant_of(scaled_workload(2, kv_dtype=FP8)) == pa.PA_VARIANT_MMA
    assert _variant_of(scaled_workload(2, kv_dtype=FP8), force_variant=TC) == TC


@pytest.mark.parametrize("block_size", [16, 32, 64, 256, 1024])
@pytest.mark.parametrize("q_dtype", ["bf16", FP8])
def test_tensor_memory_kernel_block_sizes_and_queries(block_size, q_dtype):
    wl = make_workload(seq_lens=[1, 17, 64, 65, 127, 128, 129, 1500, 2049],
                       query_lens=[1, 1, 2, 1, 1, 1, 3, 4, 1], num_q_heads=8, num_kv_heads=4,
                       head_dim=128, block_size=block_size, window=0, seed=block_size,
                       kv_dtype=FP8, q_dtype=q_dtype)
    out = pa.decode(dev(wl), force_variant=TC)
    check_full(wl, out, f"tc BS={block_size} q={q_dtype}")


@pytest.mark.parametrize("group,qlen", [(1, 1), (2, 3), (4, 2), (8, 1), (8, 2), (16, 1)])
def test_tensor_memory_kernel_rows_and_slabs(group, qlen):
    wl = make_workload(seq_lens=[700, 64, 1999], query_lens=[qlen, min(qlen, 2), qlen],
                       num_q_heads=2 * group, num_kv_heads=2, head_dim=128, block_size=16,
                       windows=[100, 0, 33], seed=group * 10 + qlen, kv_dtype=FP8)
    out = pa.decode(dev(wl), force_variant=TC)
    check_full(wl, out, f"tc group={group} qlen={qlen}")


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 64, 200])
def test_tensor_memory_kernel_split_k(parts):
    wl = make_workload(seq_lens=[5000, 3333, 77], query_lens=[1, 3, 2], num_q_heads=8,
                       num_kv_heads=4, head_dim=128, block_size=16, window=0, seed=7,
                       kv_dtype=FP8)
    out = pa.decode(dev(wl), force_partitions=parts, force_variant=TC)
    check_full(wl, out, f"tc parts={parts}")


def test_tensor_memory_kernel_never_reads_outside_spans():
    wl = make_workload(seq_lens=[1000, 333, 77, 50], query_lens=[3, 1, 2, 1], num_q_heads=8,
                       num_kv_heads=4, head_dim=128, block_size=16,
                       windows=[50, 0, 20, 0], seed=19, spare_blocks=2, extra_table_cols=3,
                       kv_dtype=FP8)
    ref = oracle.decode(problem(wl))
    W = wl.windows.tolist()
    for b, (S, L) in enumerate(zip(wl.seq_lens.tolist(), wl.query_lens.tolist())):
        nb = (S + 15) // 16
        last = int(wl.block_tables[b, nb - 1])
        wl.k_cache[last, :, S - (nb - 1) * 16:] = NAN_CODE
        wl.v_cache[last, :, S - (nb - 1) * 16:] = NAN_CODE
        first = max(0, S - L + 1 - W[b]) if W[b] > 0 else 0
        for t in range(first):
            blk = int(wl.block_tables[b, t // 16])
            wl.k_cache[blk, :, t % 16] = NAN_CODE
            wl.v_cache[blk, :, t % 16] = NAN_CODE
        wl.block_tables[b, nb:] = 10 ** 6
    used = set(wl.block_tables[wl.block_tables < wl.num_blocks].tolist())
    for blk in range(wl.num_blocks):
        if blk not in used:
            wl.k_cache[blk] = NAN_CODE
            wl.v_cache[blk] = NAN_CODE
    out = pa.decode(dev(wl), force_variant=TC)
    assert_close(out.float().cpu().numpy(), ref, "tc NaN codes outside spans")


def test_tensor_memory_kernel_large_and_tiny_queries():
    # a bf16 q row is split into two e4m3 terms after a power-of-two scale:
    # rows of very different magnitudes must all come out right
    wl = make_workload(seq_lens=[900, 45, 300], query_lens=[2, 1, 1], num_q_heads=8,
                       num_kv_heads=2, head_dim=128, block_size=16, window=0, seed=5,
                       kv_dtype=FP8, scale=1e-3)
    qf = wl.q.float()
    qf[0] *= 3000.0
    qf[1] *= 1e-3
    qf[2, :4] *= 100.0
    wl.q = qf.to(torch.bfloat16)
    out = pa.decode(dev(wl), force_variant=TC)
    check_full(wl, out, "tc query magnitudes")


@pytest.mark.parametrize("cfg", [2, 4])
def test_tensor_memory_kernel_full_size_sampled(cfg):
    wl = config_workload(cfg, device="cuda:0", kv_dtype=FP8)
    assert _variant_of(wl, force_variant=TC) == TC
    out = pa.decode(wl, force_variant=TC)
    torch.cuda.synchronize()
    check_sampled(wl, out, sample_queries(wl, 32, seed=200 + cfg), f"cfg{cfg} tc full size")


@pytest.mark.parametrize("block_size", [16, 32, 64, 256, 1024])
@pytest.mark.parametrize("parts", [0, 3])
def test_fp8_one_wave_and_self_refill_rings(block_size, parts):
    # FP8 caches, units of at most 8 rows.  A one-wave grid (few units, the
    # dispatcher's own partitions) runs the six-stage ring at two CTAs per SM,
    # refilled by the copy warp; a forced partition count keeps the four-stage
    # ring, whose compute warps refill their own half stages with boxes of at
    # most 32 rows (slices of the larger blocks).
    wl = make_workload(seq_lens=[1, 63, 64, 700, 2049, 5000], query_lens=[1, 1, 1, 2, 1, 2],
                       num_q_heads=16, num_kv_heads=4, head_dim=128, block_size=block_size,
                       seed=block_size + parts, kv_dtype=FP8)
    d = dev(wl)
    rc, info = pa.pa_plan(pa.params_for(d, force_partitions=parts), block_size)
    assert rc == pa.PA_OK
    assert info.stages == (6 if parts == 0 else 4)
    out = pa.decode(d, force_partitions=parts)
    check_full(wl, out, f"fp8 ring BS={block_size} parts={parts}")


def test_fp8_self_refill_on_a_grid_of_many_units():
    # many units (several waves of CTAs): the four-stage ring with self-refill
    # chosen by the dispatcher itself, ragged rows, every element checked
    g = np.random.default_rng(21)
    S = g.integers(1, 3000, size=48).tolist()
    wl = make_workload(seq_lens=S, query_lens=[1] * 48, num_q_heads=32, num_kv_heads=8,
                       head_dim=128, block_size=16, seed=21, kv_dtype=FP8)
    d = dev(wl)
    rc, info = pa.pa_plan(pa.params_for(d), 16)
    assert rc == pa.PA_OK and info.stages == 4
    out = pa.decode(d)
    check_full(wl, out, "fp8 self-refill, many units")


@pytest.mark.parametrize("block_size", [16, 64])
def test_fp8_self_refill_never_reads_outside_spans(block_size):
    # A grid of many units takes the four-stage ring whose compute warps pick
    # and copy their own boxes.  NaN codes past each row's last token, before
    # each window and in blocks no table reaches must not reach the outputs.
    g = np.random.default_rng(23 + block_size)
    B = 48
    S = g.integers(1, 3000, size=B).tolist()
    L = g.integers(1, 3, size=B).tolist()
    W = [int(w) if g.random() < 0.6 else 0 for w in g.integers(1, 2500, size=B)]
    L = [min(l, s) for l, s in zip(L, S)]
    wl = make_workload(seq_lens=S, query_lens=L, num_q_heads=8, num_kv_heads=2, head_dim=128,
                       block_size=block_size, windows=W, seed=23 + block_size, spare_blocks=2,
                       extra_table_cols=3, kv_dtype=FP8)
    ref = oracle.decode(problem(wl))
    bs = block_size
    for b in range(B):
        nb = (S[b] + bs - 1) // bs
        last = int(wl.block_tables[b, nb - 1])
        wl.k_cache[last, :, S[b] - (nb - 1) * bs:] = NAN_CODE
        wl.v_cache[last, :, S[b] - (nb - 1) * bs:] = NAN_CODE
        first = max(0, S[b] - L[b] + 1 - W[b]) if W[b] > 0 else 0
        for t in range(first):
            blk = int(wl.block_tables[b, t // bs])
            wl.k_cache[blk, :, t % bs] = NAN_CODE
            wl.v_cache[blk, :, t % bs] = NAN_CODE
        wl.block_tables[b, nb:] = 10 ** 6
    used = set(wl.block_tables[wl.block_tables < wl.num_blocks].tolist())
    for blk in range(wl.num_blocks):
        if blk not in used:
            wl.k_cache[blk] = NAN_CODE
            wl.v_cache[blk] = NAN_CODE
    d = dev(wl)
    rc, info = pa.pa_plan(pa.params_for(d), block_size)
    assert rc == pa.PA_OK and info.stages == 4
    out = pa.decode(d)
    assert_close(out.float().cpu().numpy(), ref, f"fp8 self-refill NaN codes BS={block_size}")
