"""Python binding of libpagedattn (paged-attention decode on one B200).

A thin ctypes layer over the C ABI in ``include/pagedattn.h``: the functions
below carry the C names and only marshal arguments; every step of the decode
runs in the library's sm_100a kernels.  There is no fallback: importing this
package fails loudly when ``libpagedattn.so`` has not been built
(``python paged_kv_cache_474_b200/_build.py`` or ``__graft_entry__.build()``).

PyTorch is used only for device memory and streams (``tensor.data_ptr()``,
``torch.cuda.current_stream()``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK = 0
PA_ERR_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_WORKSPACE = 3
PA_ERR_CUDA = 4

PA_DEV_TIMEOUT = 1
PA_DEV_BAD_ROW = 2
PA_DEV_BAD_BLOCK = 4
PA_DEV_HINT = 8

PA_VARIANT_AUTO = 0
PA_VARIANT_FMA = 1
PA_VARIANT_MMA = 2
PA_VARIANT_TC = 3

PA_DTYPE_BF16 = 0
PA_DTYPE_FP8_E4M3 = 1

PA_SCHED_STATIC = 0
PA_SCHED_WORKLIST = 2


class pa_params(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("num_blocks", ctypes.c_int),
        ("max_blocks_per_seq", ctypes.c_int),
        ("max_span_hint", ctypes.c_int),
        ("max_query_len_hint", ctypes.c_int),
        ("windows", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("force_variant", ctypes.c_int),
        ("force_partitions", ctypes.c_int),
        ("profile_events", ctypes.c_void_p),
        ("q_dtype", ctypes.c_int),
        ("kv_dtype", ctypes.c_int),
        ("q_scale", ctypes.c_float),
        ("k_scale", ctypes.c_float),
        ("v_scale", ctypes.c_float),
        ("schedule", ctypes.c_int),
        ("wait_limit_cycles", ctypes.c_longlong),
        ("merge_target_extra", ctypes.c_int),
    ]


class pa_plan_info(ctypes.Structure):
    _fields_ = [
        ("variant", ctypes.c_int),
        ("partition_tokens", ctypes.c_int),
        ("max_partitions", ctypes.c_int),
        ("one_shot", ctypes.c_int),
        ("max_rows", ctypes.c_int),
        ("slab_rows", ctypes.c_int),
        ("consumer_warps", ctypes.c_int),
        ("stages", ctypes.c_int),
        ("grid_x", ctypes.c_int),
        ("grid_y", ctypes.c_int),
        ("grid_z", ctypes.c_int),
        ("block_threads", ctypes.c_int),
        ("smem_bytes", ctypes.c_size_t),
        ("workspace_bytes", ctypes.c_size_t),
        ("num_sms", ctypes.c_int),
        ("ctas_per_sm", ctypes.c_int),
        ("worklist", ctypes.c_int),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


# Every symbol include/pagedattn.h declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_PP = ctypes.POINTER(pa_params)
SIGNATURES = {
    "pa_decode": (_I, [_P, _P, _P, _P, _P, _P, _P, _F, _I, _I, _PP, _P]),
    "pa_workspace_size": (ctypes.c_size_t, [_PP, _I]),
    "pa_plan": (_I, [_PP, _I, _I, _I, ctypes.POINTER(pa_plan_info)]),
    "pa_visible_ranges": (_I, [_P, _P, _P, _P, _I, _P, _I, _P]),
    "pa_decode_host": (_I, [_P, _P, _P, _P, _P, _P, _P, _F, _I, _I, _PP, _P]),
    "pa_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _F, _I, _I, _PP, _P]),
    "pa_host_workspace_size": (ctypes.c_size_t, [_PP, _I, _I, _P, _P]),
    "pa_unreachable_blocks": (_I, [_P, _P, _P, _I, _P, _I, _I, _P]),
    "pa_extents_host": (_I, [_P, _P, _P, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "pa_device_status": (_I, [ctypes.POINTER(ctypes.c_uint), _I, _P]),
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_version": (ctypes.c_char_p, []),
}

SIZE_ERROR = ctypes.c_size_t(-1).value


class PagedAttnError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"libpagedattn error {code}: {message}")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python paged_kv_cache_474_b200/_build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _check(rc: int) -> int:
    if rc != PA_OK:
        raise PagedAttnError(rc, pa_last_error())
    return rc


# ---------------------------------------------------------------- raw C calls
def pa_decode(dst, q, kCache, vCache, blockTables, seqLens, queryLens, scale,
              window, kvBlockSize, params, stream) -> int:
    return _lib.pa_decode(dst, q, kCache, vCache, blockTables, seqLens,
                          queryLens, float(scale), int(window), int(kvBlockSize),
                          ctypes.byref(params), stream)


def pa_decode_noalloc(dst, q, kCache, vCache, blockTables, seqLens, queryLens, scale,
                      window, kvBlockSize, params, stream) -> int:
    """pa_decode with the library's static scratch array instead of a caller
    workspace (for callers that cannot allocate device memory)."""
    return _lib.pa_decode_noalloc(dst, q, kCache, vCache, blockTables, seqLens,
                                  queryLens, float(scale), int(window), int(kvBlockSize),
                                  ctypes.byref(params), stream)


PA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def pa_workspace_size(params, kvBlockSize) -> int:
    return _lib.pa_workspace_size(ctypes.byref(params), int(kvBlockSize))


def pa_plan(params, kvBlockSize, num_sms=0, ctas_per_sm=0):
    info = pa_plan_info()
    rc = _lib.pa_plan(ctypes.byref(params), int(kvBlockSize), int(num_sms),
                      int(ctas_per_sm), ctypes.byref(info))
    return rc, info


def pa_visible_ranges(lo, hi, seqLens, queryLens, window, windows, batch, stream) -> int:
    return _lib.pa_visible_ranges(lo, hi, seqLens, queryLens, int(window), windows,
                                  int(batch), stream)


def pa_decode_host(dst_host, q_host, kCache, vCache, blockTables_host, seqLens_host,
                   queryLens_host, scale, window, kvBlockSize, params, stream) -> int:
    return _lib.pa_decode_host(dst_host, q_host, kCache, vCache, blockTables_host,
                               seqLens_host, queryLens_host, float(scale), int(window),
                               int(kvBlockSize), ctypes.byref(params), stream)


def pa_host_workspace_size(params, kvBlockSize, window, seqLens_host, queryLens_host) -> int:
    return _lib.pa_host_workspace_size(ctypes.byref(params), int(kvBlockSize), int(window),
                                       seqLens_host, queryLens_host)


def pa_device_status(clear: bool = True, stream=None) -> int:
    st = ctypes.c_uint(0)
    _check(_lib.pa_device_status(ctypes.byref(st), int(bool(clear)), stream))
    return st.value


def pa_last_error() -> str:
    return _lib.pa_last_error().decode()


def pa_version() -> str:
    return _lib.pa_version().decode()


# ------------------------------------------------------- torch conveniences
def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_params(*, batch, num_q_heads, num_kv_heads, head_dim, num_blocks,
                max_blocks_per_seq, max_span_hint=0, max_query_len_hint=0,
                windows=None, workspace=None, force_variant=PA_VARIANT_AUTO,
                force_partitions=0, q_dtype=PA_DTYPE_BF16, kv_dtype=PA_DTYPE_BF16,
                q_scale=0.0, k_scale=0.0, v_scale=0.0,
                schedule=PA_SCHED_STATIC) -> pa_params:
    p = pa_params()
    p.batch = int(batch)
    p.num_q_heads = int(num_q_heads)
    p.num_kv_heads = int(num_kv_heads)
    p.head_dim = int(head_dim)
    p.num_blocks = int(num_blocks)
    p.max_blocks_per_seq = int(max_blocks_per_seq)
    p.max_span_hint = int(max_span_hint)
    p.max_query_len_hint = int(max_query_len_hint)
    p.windows = _ptr(windows)
    if workspace is not None:
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel() * workspace.element_size()
    p.force_variant = int(force_variant)
    p.force_partitions = int(force_partitions)
    p.q_dtype = int(q_dtype)
    p.kv_dtype = int(kv_dtype)
    p.q_scale = float(q_scale)
    p.k_scale = float(k_scale)
    p.v_scale = float(v_scale)
    p.schedule = int(schedule)
    return p


def pa_extents_host(seq_lens, query_lens, window=0, windows=None):
    """(max_span, max_query_len) hints from host int sequences (the library's
    own span rule, via the C ABI)."""
    import numpy as np
    S = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    L = np.ascontiguousarray(np.asarray(query_lens, dtype=np.int32))
    W = None if windows is None else np.ascontiguousarray(np.asarray(windows, dtype=np.int32))
    span, qlen = ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.pa_extents_host(S.ctypes.data, L.ctypes.data,
                                None if W is None else W.ctypes.data, int(window),
                                int(S.shape[0]), ctypes.byref(span), ctypes.byref(qlen)))
    return span.value, qlen.value


def params_for(wl, *, workspace=None, hints=True, force_variant=PA_VARIANT_AUTO,
               force_partitions=0, schedule=PA_SCHED_STATIC) -> pa_params:
    """pa_params for a ``workloads.Workload`` (host hints from its lengths)."""
    span = qlen = 0
    if hints:
        s, l, w = wl.host_lists()
        span, qlen = pa_extents_host(s, l, windows=w)
    return make_params(batch=wl.batch, num_q_heads=wl.num_q_heads,
                       num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim,
                       num_blocks=wl.num_blocks,
                       max_blocks_per_seq=wl.max_blocks_per_seq,
                       max_span_hint=span, max_query_len_hint=qlen,
                       windows=wl.windows, workspace=workspace,
                       force_variant=force_variant,
                       force_partitions=force_partitions,
                       q_dtype=PA_DTYPE_FP8_E4M3 if wl.q_fp8 else PA_DTYPE_BF16,
                       kv_dtype=PA_DTYPE_FP8_E4M3 if wl.kv_fp8 else PA_DTYPE_BF16,
                       q_scale=wl.q_scale if wl.q_fp8 else 0.0,
                       k_scale=wl.k_scale if wl.kv_fp8 else 0.0,
                       v_scale=wl.v_scale if wl.kv_fp8 else 0.0,
                       schedule=schedule)


def alloc_workspace(params: pa_params, kv_block_size: int, device="cuda"):
    """A uint8 device tensor of pa_workspace_size() bytes (None if 0)."""
    import torch
    n = pa_workspace_size(params, kv_block_size)
    if n == SIZE_ERROR:
        raise PagedAttnError(PA_ERR_ARG, pa_last_error())
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def decode(wl, *, out=None, workspace=None, hints=True, force_variant=PA_VARIANT_AUTO,
           force_partitions=0, schedule=PA_SCHED_STATIC, stream=None):
    """Runs pa_decode on a device-resident ``Workload``; returns dst (bf16
    [sum(queryLens), H_q, D]).  Allocates the workspace when none is given."""
    import torch
    p = params_for(wl, workspace=workspace, hints=hints, force_variant=force_variant,
                   force_partitions=force_partitions, schedule=schedule)
    if workspace is None:
        # size the workspace from the real extents even when the call itself
        # runs without hints (pa_decode then reads the lengths itself)
        sizing = p if hints else params_for(wl, force_variant=force_variant,
                                            force_partitions=force_partitions,
                                            schedule=schedule)
        workspace = alloc_workspace(sizing, wl.block_size, device=wl.q.device)
        if workspace is not None:
            p.workspace = workspace.data_ptr()
            p.workspace_bytes = workspace.numel()
    if out is None:
        out = torch.empty(wl.q.shape, dtype=torch.bfloat16, device=wl.q.device)
    _check(pa_decode(out.data_ptr(), wl.q.data_ptr(), wl.k_cache.data_ptr(),
                     wl.v_cache.data_ptr(), wl.block_tables.data_ptr(),
                     wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(), wl.scale,
                     wl.window, wl.block_size, p, _stream_handle(stream)))
    return out


def pa_unreachable_blocks(count, seqLens, queryLens, window, windows, kvBlockSize, batch,
                          stream) -> int:
    return _lib.pa_unreachable_blocks(count, seqLens, queryLens, int(window), windows,
                                      int(kvBlockSize), int(batch), stream)


def unreachable_blocks(seq_lens, query_lens, kv_block_size, window=0, windows=None, stream=None):
    """int32 device tensor [batch]: leading KV blocks of each row that no query
    token can see again (pa_unreachable_blocks)."""
    import torch
    out = torch.empty(seq_lens.numel(), dtype=torch.int32, device=seq_lens.device)
    _check(pa_unreachable_blocks(out.data_ptr(), seq_lens.data_ptr(), query_lens.data_ptr(),
                                 window, _ptr(windows), kv_block_size, seq_lens.numel(),
                                 _stream_handle(stream)))
    return out


def visible_ranges(seq_lens, query_lens, window=0, windows=None, stream=None):
    """(lo, hi) int32 device tensors over every query token (pa_visible_ranges)."""
    import torch
    n = int(query_lens.sum().item())
    lo = torch.empty(max(n, 1), dtype=torch.int32, device=seq_lens.device)
    hi = torch.empty(max(n, 1), dtype=torch.int32, device=seq_lens.device)
    _check(pa_visible_ranges(lo.data_ptr(), hi.data_ptr(), seq_lens.data_ptr(),
                             query_lens.data_ptr(), window, _ptr(windows),
                             seq_lens.numel(), _stream_handle(stream)))
    return lo[:n], hi[:n]
