"""CPU checks of the C ABI: the library loads, exports every symbol the header
declares, validates arguments on the host, and plans partitions the way the
dispatcher promises.  No call here launches GPU work."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedattn.h")

pa = pytest.importorskip("paged_kv_cache_474_b200")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pa_decode", "pa_workspace_size", "pa_visible_ranges", "pa_last_error"):
        assert required in names


def test_every_declared_symbol_is_exported_and_bound():
    import ctypes
    lib = ctypes.CDLL(pa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in pa.SIGNATURES, name


def test_version():
    assert "sm_100a" in pa.pa_version()


def base_params(**kw):
    d = dict(batch=2, num_q_heads=4, num_kv_heads=2, head_dim=64, num_blocks=8,
             max_blocks_per_seq=4, max_span_hint=50, max_query_len_hint=1)
    d.update(kw)
    return pa.make_params(**d)


def call(p, bs=16, window=0, scale=0.125, ptrs=16):
    return pa.pa_decode(ptrs, ptrs, ptrs, ptrs, ptrs, ptrs, ptrs, scale, window, bs, p, None)


@pytest.mark.parametrize("kw,code", [
    (dict(num_q_heads=5), pa.PA_ERR_ARG),
    (dict(num_kv_heads=0), pa.PA_ERR_ARG),
    (dict(head_dim=96), pa.PA_ERR_UNSUPPORTED),
    (dict(head_dim=512), pa.PA_ERR_UNSUPPORTED),
    (dict(batch=-1), pa.PA_ERR_ARG),
    (dict(num_blocks=0), pa.PA_ERR_ARG),
    (dict(max_span_hint=-3), pa.PA_ERR_ARG),
    (dict(force_partitions=-1), pa.PA_ERR_ARG),
    (dict(force_variant=7), pa.PA_ERR_ARG),
    (dict(schedule=1), pa.PA_ERR_ARG),
    (dict(schedule=3), pa.PA_ERR_ARG),
    (dict(force_variant=4), pa.PA_ERR_ARG),
])
def test_invalid_params_are_rejected_on_the_host(kw, code):
    assert call(base_params(**kw)) == code
    assert pa.pa_last_error()


@pytest.mark.parametrize("bs", [0, 8, 48, 2048])
def test_unsupported_block_sizes(bs):
    assert call(base_params(), bs=bs) == pa.PA_ERR_UNSUPPORTED


def test_negative_window_null_and_misaligned_pointers():
    assert call(base_params(), window=-1) == pa.PA_ERR_ARG
    assert call(base_params(), ptrs=0) == pa.PA_ERR_ARG
    assert call(base_params(), ptrs=24) == pa.PA_ERR_ARG
    assert call(base_params(), scale=float("nan")) == pa.PA_ERR_ARG


def test_empty_batch_is_a_no_op():
    assert call(base_params(batch=0)) == pa.PA_OK
    assert pa.pa_last_error() == ""


def test_extents_follow_the_window_rule():
    # gllm page "Verification" batch: a 5-token chunk over 300 and a decode row over 40
    assert pa.pa_extents_host([300, 40], [5, 1], 16) == (20, 5)
    assert pa.pa_extents_host([300, 40], [5, 1], 0) == (300, 5)
    assert pa.pa_extents_host([300, 40], [5, 1], 4096) == (300, 5)
    assert pa.pa_extents_host([300, 40], [0, 1], 16) == (16, 1)
    assert pa.pa_extents_host([7, 9], [3, 1], windows=[2, 0]) == (9, 3)
    assert pa.pa_extents_host([7, 9], [3, 1], windows=[2, 5]) == (5, 3)
    with pytest.raises(pa.PagedAttnError):
        pa.pa_extents_host([3], [4], 0)


def test_extents_agree_with_oracle_ranges():
    rng = np.random.default_rng(0)
    for _ in range(50):
        B = int(rng.integers(1, 20))
        S = rng.integers(1, 5000, B)
        L = np.minimum(S, rng.integers(0, 6, B))
        W = rng.choice([0, 1, 7, 64, 4096], B)
        lo, hi = oracle.visible_ranges(S, L, windows=W)
        span, qlen = pa.pa_extents_host(S, L, windows=W)
        qoff = np.concatenate([[0], np.cumsum(L)])
        want = max([int(S[b] - lo[qoff[b]]) for b in range(B) if L[b] > 0] or [0])
        assert span == want and qlen == int(L.max())


def plan(**kw):
    bs = kw.pop("bs", 16)
    sms = kw.pop("sms", 148)
    occ = kw.pop("occ", 2)
    rc, info = pa.pa_plan(base_params(**kw), bs, sms, occ)
    assert rc == pa.PA_OK, pa.pa_last_error()
    return info


def test_plan_long_single_group_fills_one_wave():
    # B=1, H_kv=1, S=131072: partitions sized so one wave covers every SM slot
    info = plan(batch=1, num_q_heads=8, num_kv_heads=1, head_dim=128, num_blocks=8193,
                max_blocks_per_seq=8192, max_span_hint=131072)
    assert info.partition_tokens % 64 == 0
    assert info.max_partitions * info.partition_tokens >= 131072 + 63
    assert 148 * 2 * 0.9 <= info.max_partitions <= 148 * 2
    assert not info.one_shot and info.workspace_bytes > 0
    assert info.grid_x == info.max_partitions and info.grid_y == 1 and info.grid_z == 1


def test_plan_uses_the_windowed_span_not_the_context():
    wide = plan(batch=16, num_q_heads=32, num_kv_heads=8, head_dim=128, num_blocks=30000,
                max_blocks_per_seq=2048, max_span_hint=32768, max_query_len_hint=5)
    windowed = plan(batch=16, num_q_heads=32, num_kv_heads=8, head_dim=128, num_blocks=30000,
                    max_blocks_per_seq=2048, max_span_hint=4100, max_query_len_hint=5)
    assert windowed.max_partitions * windowed.partition_tokens < 8192
    assert wide.max_partitions * wide.partition_tokens >= 32768


def test_plan_one_shot_for_short_spans():
    info = plan(max_span_hint=50)
    assert info.one_shot and info.max_partitions == 1 and info.workspace_bytes == 0


def test_plan_forced_partitions_and_workspace_formula():
    info = plan(batch=3, num_q_heads=8, num_kv_heads=2, head_dim=128, num_blocks=400,
                max_blocks_per_seq=320, max_span_hint=5000, max_query_len_hint=3,
                force_partitions=7)
    assert info.partition_tokens == 768 and info.max_partitions == 7
    rows = 4 * 3
    partials = 3 * 2 * 7 * rows
    align = lambda x: (x + 255) // 256 * 256
    assert info.max_rows == rows
    assert info.workspace_bytes == align(partials * 4) + align(partials * 128 * 4)


def test_plan_row_slabs_for_many_rows():
    kw = dict(batch=4, num_q_heads=64, num_kv_heads=8, head_dim=128, num_blocks=400,
              max_blocks_per_seq=64, bs=1024, max_span_hint=65536, max_query_len_hint=4)
    mma = plan(**kw)
    assert mma.variant == pa.PA_VARIANT_MMA
    assert mma.max_rows == 32 and mma.slab_rows == 64 and mma.grid_y == 8
    fma = plan(force_variant=pa.PA_VARIANT_FMA, **kw)
    assert fma.max_rows == 32 and fma.slab_rows == 32 and fma.grid_y == 8
    kw.update(num_kv_heads=4, max_query_len_hint=5, batch=2)
    big = plan(**kw)
    assert big.max_rows == 80 and big.slab_rows == 64 and big.grid_y == 4 * 2
    big_fma = plan(force_variant=pa.PA_VARIANT_FMA, **kw)
    assert big_fma.grid_y == 4 * 3


def test_plan_variant_and_tile_width():
    # tensor-core kernel by default; one 8-row n-tile per warp up to 8 rows, two above
    sparse = plan(batch=32, num_q_heads=32, num_kv_heads=8, head_dim=128, num_blocks=20000,
                  max_blocks_per_seq=512, max_span_hint=8192)
    dense = plan(batch=1, num_q_heads=8, num_kv_heads=1, head_dim=128, num_blocks=8193,
                 max_blocks_per_seq=8192, max_span_hint=131072)
    mtp = plan(batch=2, num_q_heads=16, num_kv_heads=4, head_dim=64, num_blocks=100,
               max_blocks_per_seq=50, max_span_hint=700, max_query_len_hint=4)
    assert sparse.variant == dense.variant == mtp.variant == pa.PA_VARIANT_MMA
    assert sparse.slab_rows == dense.slab_rows == 32 and mtp.slab_rows == 64
    fma = plan(batch=32, num_q_heads=32, num_kv_heads=8, head_dim=128, num_blocks=20000,
               max_blocks_per_seq=512, max_span_hint=8192, force_variant=pa.PA_VARIANT_FMA)
    assert fma.variant == pa.PA_VARIANT_FMA and fma.slab_rows == 16
    forced = plan(batch=1, num_q_heads=8, num_kv_heads=1, head_dim=128, num_blocks=8193,
                  max_blocks_per_seq=8192, max_span_hint=131072, force_variant=pa.PA_VARIANT_FMA)
    assert forced.variant == pa.PA_VARIANT_FMA


def test_plan_rejects_tensor_maps_beyond_32bit_rows():
    rc, _ = pa.pa_plan(base_params(num_blocks=1 << 22, num_kv_heads=2, num_q_heads=16,
                                   force_variant=pa.PA_VARIANT_MMA), 1024, 148, 2)
    assert rc == pa.PA_ERR_UNSUPPORTED
    rc, info = pa.pa_plan(base_params(num_blocks=1 << 22, num_kv_heads=2, num_q_heads=16,
                                      max_query_len_hint=2), 1024, 148, 2)
    assert rc == pa.PA_OK and info.variant == pa.PA_VARIANT_FMA


def test_plan_caps_partition_at_the_table_cache():
    info = plan(batch=1, num_q_heads=1, num_kv_heads=1, head_dim=64, num_blocks=70000,
                max_blocks_per_seq=65536, max_span_hint=1 << 20, sms=1, occ=1)
    assert info.partition_tokens <= (1024 - 2) * 16


def test_plan_head_dim_256_uses_the_tensor_core_kernel():
    # the ExecuTorch page's H100 benchmark shape: B=1, H_q=16, H_kv=2, D=256
    info = plan(batch=1, num_q_heads=16, num_kv_heads=2, head_dim=256, num_blocks=1100,
                max_blocks_per_seq=1024, max_span_hint=16384, occ=1)
    assert info.variant == pa.PA_VARIANT_MMA and info.slab_rows == 32
    assert info.smem_bytes <= 227 * 1024
    rc, _ = pa.pa_plan(base_params(head_dim=256, force_variant=pa.PA_VARIANT_FMA), 16, 148, 1)
    assert rc == pa.PA_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw", [
    dict(kv_dtype=pa.PA_DTYPE_FP8_E4M3),                              # scales missing
    dict(kv_dtype=pa.PA_DTYPE_FP8_E4M3, k_scale=0.5),                 # v_scale missing
    dict(kv_dtype=pa.PA_DTYPE_FP8_E4M3, k_scale=-1.0, v_scale=1.0),
    dict(kv_dtype=pa.PA_DTYPE_FP8_E4M3, k_scale=float("nan"), v_scale=1.0),
    dict(kv_dtype=pa.PA_DTYPE_FP8_E4M3, k_scale=float("inf"), v_scale=1.0),
    dict(q_dtype=pa.PA_DTYPE_FP8_E4M3),                               # q_scale missing
    dict(q_dtype=2),
    dict(kv_dtype=-1),
])
def test_fp8_operands_need_their_scales(kw):
    # aiter PR #2914 review: FP8 tensors without their scales must be rejected
    assert call(base_params(**kw)) == pa.PA_ERR_ARG
    assert "scale" in pa.pa_last_error() or "dtype" in pa.pa_last_error()


def test_fp8_scales_of_bf16_operands_are_ignored():
    assert call(base_params(batch=0, k_scale=-5.0, q_scale=float("nan"))) == pa.PA_OK


def test_fp8_runs_on_the_tensor_core_kernel_only():
    kw = dict(kv_dtype=pa.PA_DTYPE_FP8_E4M3, k_scale=1.0, v_scale=1.0)
    assert call(base_params(force_variant=pa.PA_VARIANT_FMA, **kw)) == pa.PA_ERR_UNSUPPORTED
    kq = dict(q_dtype=pa.PA_DTYPE_FP8_E4M3, q_scale=1.0)
    assert call(base_params(force_variant=pa.PA_VARIANT_FMA, **kq)) == pa.PA_ERR_UNSUPPORTED
    rc, _ = pa.pa_plan(base_params(num_blocks=1 << 22, num_kv_heads=2, num_q_heads=16, **kw),
                       1024, 148, 2)
    assert rc == pa.PA_ERR_UNSUPPORTED


@pytest.mark.parametrize("d,stages", [(64, 8), (128, 4), (256, 3)])
def test_plan_fp8_ring(d, stages):
    info = plan(batch=8, num_q_heads=16, num_kv_heads=2, head_dim=d, num_blocks=4000,
                max_blocks_per_seq=512, max_span_hint=8192, force_variant=pa.PA_VARIANT_MMA,
                kv_dtype=pa.PA_DTYPE_FP8_E4M3, k_scale=1.0, v_scale=1.0)
    assert info.variant == pa.PA_VARIANT_MMA and info.stages == stages
    # ring = stages x (K + V) x 64 tokens x head_dim bytes
    assert info.smem_bytes >= stages * 2 * 64 * d
    assert info.smem_bytes < stages * 2 * 64 * d + 1024 + 4096


def test_plan_tensor_memory_variant_on_request():
    fp8 = dict(kv_dtype=pa.PA_DTYPE_FP8_E4M3, k_scale=1.0, v_scale=1.0)
    gqa = dict(batch=32, num_q_heads=32, num_kv_heads=8, head_dim=128, num_blocks=20000,
               max_blocks_per_seq=512, max_span_hint=8192)
    assert plan(**gqa, **fp8).variant == pa.PA_VARIANT_MMA   # not chosen by itself
    info = plan(force_variant=pa.PA_VARIANT_TC, **gqa, **fp8)
    assert info.variant == pa.PA_VARIANT_TC and info.block_threads == 320
    assert info.slab_rows == 8 and info.stages == 3
    assert info.partition_tokens % 128 == 0
    # more rows run as 8-row slabs; bf16 caches and other head dims are refused
    forced = plan(force_variant=pa.PA_VARIANT_TC, **dict(gqa, max_query_len_hint=3), **fp8)
    assert forced.variant == pa.PA_VARIANT_TC and forced.grid_y == 8 * 2
    rc, _ = pa.pa_plan(base_params(force_variant=pa.PA_VARIANT_TC, **gqa), 16, 148, 2)
    assert rc == pa.PA_ERR_UNSUPPORTED
    rc, _ = pa.pa_plan(base_params(force_variant=pa.PA_VARIANT_TC, **dict(gqa, head_dim=64),
                                   **fp8), 16, 148, 2)
    assert rc == pa.PA_ERR_UNSUPPORTED
    long_row = plan(batch=1, num_q_heads=8, num_kv_heads=1, head_dim=128, num_blocks=8193,
                    max_blocks_per_seq=8192, max_span_hint=131072,
                    force_variant=pa.PA_VARIANT_TC, **fp8)
    assert long_row.variant == pa.PA_VARIANT_TC and long_row.partition_tokens % 128 == 0


def test_plan_work_list_schedule():
    long_row = dict(batch=1, num_q_heads=8, num_kv_heads=1, head_dim=128, num_blocks=8193,
                    max_blocks_per_seq=8192, max_span_hint=131072)
    static = plan(**long_row)
    assert not static.worklist
    wl = plan(schedule=pa.PA_SCHED_WORKLIST, **long_row)
    assert wl.worklist and wl.grid_x * wl.grid_y * wl.grid_z <= 148 * 2
    align = lambda x: (x + 255) // 256 * 256
    assert wl.workspace_bytes == static.workspace_bytes + align(2 * 1 * 1 * 8)
    # more CTAs than one wave, or a variant other than MMA: refused
    many = dict(batch=32, num_q_heads=32, num_kv_heads=8, head_dim=128, num_blocks=20000,
                max_blocks_per_seq=512, max_span_hint=8192)
    rc, _ = pa.pa_plan(base_params(schedule=pa.PA_SCHED_WORKLIST, **many), 16, 148, 2)
    assert rc == pa.PA_ERR_UNSUPPORTED
    rc, _ = pa.pa_plan(base_params(schedule=pa.PA_SCHED_WORKLIST, force_variant=pa.PA_VARIANT_FMA,
                                   **long_row), 16, 148, 2)
    assert rc == pa.PA_ERR_UNSUPPORTED
    one_shot = plan(schedule=pa.PA_SCHED_WORKLIST, max_span_hint=50)
    assert one_shot.one_shot and not one_shot.worklist and one_shot.workspace_bytes == 0


def test_header_is_plain_c_and_matches_the_binding(tmp_path):
    # tests/c_abi_check.c uses the header from C11 (pedantic, warnings as
    # errors), links the library and calls its host-only entry points; its
    # results equal the same calls through the binding
    import subprocess
    libdir = os.path.dirname(pa.LIB_PATH)
    exe = tmp_path / "c_abi_check"
    subprocess.run(["gcc", "-std=c11", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe),
                    "-L", libdir, "-lpagedattn", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    # every field of both structs sits where the binding's ctypes mirror puts it
    nfield = 0
    for line in out.strip().splitlines():
        kind, rest = line.split(" ", 1)
        if kind == "offset":
            name, off = rest.split()
            struct, field = name.split(".")
            assert getattr(getattr(pa, struct), field).offset == int(off), name
            nfield += 1
        elif kind == "sizeof":
            struct, size = rest.split()
            assert ctypes.sizeof(getattr(pa, struct)) == int(size), struct
    assert nfield == len(pa.pa_params._fields_) + len(pa.pa_plan_info._fields_)
    lines = dict(line.split(" ", 1) for line in out.strip().splitlines()
                 if line.split(" ", 1)[0] not in ("offset", "sizeof"))
    S, L, W = [300, 40, 7], [5, 1, 3], [16, 100, 2]
    span, qlen = pa.pa_extents_host(S, L, windows=W)
    assert lines["extents"] == f"{span} {qlen}"
    win = np.array(W, dtype=np.int32)
    p = pa.make_params(batch=3, num_q_heads=8, num_kv_heads=2, head_dim=128, num_blocks=64,
                       max_blocks_per_seq=19, max_span_hint=span, max_query_len_hint=qlen)
    p.windows = win.ctypes.data
    rc, info = pa.pa_plan(p, 16, num_sms=148, ctas_per_sm=2)
    assert rc == pa.PA_OK
    assert lines["plan"] == " ".join(str(x) for x in (
        info.variant, info.partition_tokens, info.max_partitions, info.one_shot,
        info.max_rows, info.grid_x, info.grid_y, info.grid_z, info.workspace_bytes))
    assert lines["refused"] == f"{pa.PA_ERR_UNSUPPORTED} 1"
    assert lines["version"] == pa.pa_version()


def test_plan_invariants_on_random_params():
    # 600 seeded draws of shapes, hints, variants, partition counts and KV
    # dtypes: every plan the host accepts keeps the dispatcher's promises, and
    # the only refusals are the documented ones
    g = np.random.default_rng(5)
    align = lambda x: (x + 255) // 256 * 256
    accepted = 0
    for _ in range(600):
        D = int(g.choice([64, 128, 256]))
        BS = int(g.choice([16, 32, 64, 128, 256, 512, 1024]))
        hkv, grp = int(g.choice([1, 2, 4, 8])), int(g.choice([1, 2, 3, 4, 8, 16]))
        B, mbps, qlen = int(g.integers(1, 3000)), int(g.integers(1, 4096)), int(g.integers(1, 17))
        span = int(g.integers(1, mbps * BS + 1))
        fp8 = bool(g.random() < 0.3)
        fv, fp = int(g.choice([0, 0, 0, pa.PA_VARIANT_FMA])), int(g.choice([0, 0, 0, 2, 7, 100]))
        p = pa.make_params(batch=B, num_q_heads=hkv * grp, num_kv_heads=hkv, head_dim=D,
                           num_blocks=B * mbps + 1, max_blocks_per_seq=mbps,
                           max_span_hint=span, max_query_len_hint=qlen, force_variant=fv,
                           force_partitions=fp,
                           kv_dtype=pa.PA_DTYPE_FP8_E4M3 if fp8 else pa.PA_DTYPE_BF16,
                           k_scale=1.0 if fp8 else 0.0, v_scale=1.0 if fp8 else 0.0)
        rc, info = pa.pa_plan(p, BS, 148, 2)
        # pools past the TMA map's 32-bit rows run on the FMA kernel, which has
        # no head_dim 256 and no FP8 path
        fits = (B * mbps + 1) * hkv * BS <= 2 ** 31 - 1
        fma = fv == pa.PA_VARIANT_FMA or not fits
        if rc != pa.PA_OK:
            assert rc == pa.PA_ERR_UNSUPPORTED and fma and (D == 256 or fp8), pa.pa_last_error()
            continue
        accepted += 1
        P = info.max_partitions
        assert info.partition_tokens % 64 == 0 and 1 <= P <= 16384
        # the partitions cover the longest span plus the 64-token alignment of its start
        assert P * info.partition_tokens >= span + 63 or P == 1
        # the smem block-table slice caps a partition at its blocks plus two
        cap = max(64, (1024 - 2) * BS // 64 * 64)
        assert info.partition_tokens <= cap
        if fp:  # "~n partitions": n, or one more for the start's alignment, unless capped
            assert P <= fp + 1 or info.partition_tokens == cap
        assert info.one_shot == (P == 1)
        assert info.max_rows == grp * qlen
        nslab = -(-info.max_rows // info.slab_rows)
        assert (info.grid_x, info.grid_y, info.grid_z) == (P, hkv * nslab, B)
        assert info.block_threads == 32 * (info.consumer_warps + 1)
        assert info.smem_bytes <= 227 * 1024
        if info.one_shot:
            assert info.workspace_bytes == 0
        else:
            n = B * hkv * P * info.max_rows
            assert info.workspace_bytes == align(n * 4) + align(n * D * 4)
        assert info.variant == (pa.PA_VARIANT_FMA if fma else pa.PA_VARIANT_MMA)
    assert accepted >= 400


def test_import_fails_loudly_without_the_library(tmp_path):
    # no fallback: a copy of the package without libpagedattn.so refuses to import
    import shutil
    import subprocess
    import sys
    pkg = os.path.dirname(pa.__file__)
    dst = tmp_path / os.path.basename(pkg)
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", f"import {dst.name}"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libpagedattn.so is missing" in r.stderr
