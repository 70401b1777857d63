"""Float64 CPU oracle for paged-attention decode (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline /
reference arm may import this package.  The product path never does: the
CUDA library fails loudly when its extension is missing instead of falling
back here.

The arithmetic lives in ``pa_oracle.c`` (plain C, float64, optional OpenMP);
this module builds it with gcc and marshals numpy arrays through ctypes.
Inputs are bf16 bit patterns (``numpy.uint16``) or FP8 e4m3 codes
(``numpy.uint8``, with per-tensor scales), exactly as the GPU sees them.

Sources: gllm PR #116 "feat(backend): sliding-window PagedAttention"
(sections "What changes" and "Verification") for the call, the window rule
and the CPU reference; ExecuTorch PR #18759 (sdpa_decode_splitk docstring and
review suggestion 5) for GQA grouping and the split-K log-sum-exp merge.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# Tests that plant a slip in a copy of the oracle point this at their build.
_LIB_OVERRIDE = os.environ.get("PA_ORACLE_LIB")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(_LIB_OVERRIDE or build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            D = ctypes.c_double
            lib.oracle_visible_range.argtypes = [I, I, I, I, P, P]
            lib.oracle_visible_range.restype = I
            lib.oracle_visible_ranges.argtypes = [P, P, P, P, P, I, I]
            lib.oracle_visible_ranges.restype = I
            lib.oracle_unreachable_blocks.argtypes = [P, P, P, P, I, I, I]
            lib.oracle_unreachable_blocks.restype = I
            lib.oracle_max_threads.argtypes = [I]
            lib.oracle_max_threads.restype = I
            common = [P, P, P, P, P, P, P, I, D, I, I, I, I, I, I, I, I, D, D, I, D]
            lib.oracle_e4m3_decode.argtypes = [P, P, I]
            lib.oracle_e4m3_decode.restype = None
            lib.oracle_pa_decode.argtypes = [P] + common + [I, I]
            lib.oracle_pa_decode.restype = I
            lib.oracle_pa_decode_select.argtypes = [P, P, I] + common + [I]
            lib.oracle_pa_decode_select.restype = I
            lib.oracle_softmax_weights.argtypes = [P, I, I, I] + common
            lib.oracle_softmax_weights.restype = I
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 inputs must be passed as numpy.uint16 bit patterns")
    return a


def _i32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


class Problem:
    """One paged-attention decode problem, as host arrays.

    q:            uint16 [sum(query_lens), H_q, D]   (bf16 bits), or uint8
                  FP8 e4m3 codes (value = e4m3 number times q_scale)
    k_cache/v_cache: uint16 [num_blocks, H_kv, block_size, D] (bf16 bits), or
                  uint8 of the same shape (FP8 e4m3 codes; the value of a code
                  is its e4m3 number times k_scale / v_scale)
    block_tables: int32 [batch, max_blocks_per_seq]
    seq_lens, query_lens: int32 [batch]
    windows:      int32 [batch] or None (then the scalar ``window`` applies)
    """

    def __init__(self, q, k_cache, v_cache, block_tables, seq_lens, query_lens,
                 scale, window=0, windows=None, k_scale=1.0, v_scale=1.0,
                 q_scale=1.0):
        q = np.ascontiguousarray(q)
        self.q_fp8 = int(q.dtype == np.uint8)
        self.q = q if self.q_fp8 else _u16(q)
        self.q_scale = float(q_scale)
        k_cache = np.ascontiguousarray(k_cache)
        v_cache = np.ascontiguousarray(v_cache)
        self.kv_fp8 = int(k_cache.dtype == np.uint8)
        if self.kv_fp8:
            if v_cache.dtype != np.uint8:
                raise TypeError("k_cache and v_cache must both be FP8 codes")
            self.k_cache, self.v_cache = k_cache, v_cache
        else:
            self.k_cache, self.v_cache = _u16(k_cache), _u16(v_cache)
        self.k_scale = float(k_scale)
        self.v_scale = float(v_scale)
        self.block_tables = _i32(block_tables)
        self.seq_lens = _i32(seq_lens)
        self.query_lens = _i32(query_lens)
        self.windows = _i32(windows)
        self.window = int(window)
        self.scale = float(scale)
        nb, hkv, bs, d = self.k_cache.shape
        self.num_blocks, self.hkv, self.bs, self.d = nb, hkv, bs, d
        self.hq = self.q.shape[1]
        self.batch = self.seq_lens.shape[0]
        self.mbps = self.block_tables.shape[1]
        if self.v_cache.shape != self.k_cache.shape:
            raise ValueError("k_cache and v_cache shapes differ")

    def _common(self):
        return [_ptr(self.q), _ptr(self.k_cache), _ptr(self.v_cache),
                _ptr(self.block_tables), _ptr(self.seq_lens),
                _ptr(self.query_lens), _ptr(self.windows), self.window,
                self.scale, self.batch, self.hq, self.hkv, self.d, self.bs,
                self.num_blocks, self.mbps, self.kv_fp8, self.k_scale, self.v_scale,
                self.q_fp8, self.q_scale]

    @property
    def num_tokens(self) -> int:
        return int(self.query_lens.sum())


def problem_from_workload(wl) -> Problem:
    """A Problem holding host copies of a workload's buffers (any object with
    the attributes of ``paged_kv_cache_474_b200.workloads.Workload``; its
    tensors may live on any device).  bf16 tensors become their uint16 bit
    patterns, FP8 code tensors stay uint8.  Marshalling only."""
    import torch

    def bits(t):
        t = t.detach().contiguous().cpu()
        if t.dtype == torch.uint8:
            return t.numpy()
        return t.view(torch.int16).numpy().view(np.uint16)

    return Problem(bits(wl.q), bits(wl.k_cache), bits(wl.v_cache),
                   wl.block_tables.cpu().numpy(), wl.seq_lens.cpu().numpy(),
                   wl.query_lens.cpu().numpy(), wl.scale, wl.window,
                   None if wl.windows is None else wl.windows.cpu().numpy(),
                   k_scale=wl.k_scale, v_scale=wl.v_scale, q_scale=wl.q_scale)


def decode(pr: Problem, parts: int = 0, nthreads: int = 0) -> np.ndarray:
    """All outputs, float64 [sum(query_lens), H_q, D].  parts=0: direct form;
    parts>0: split-K with that many partitions per row and a log-sum-exp merge."""
    lib = _load()
    out = np.zeros((pr.num_tokens, pr.hq, pr.d), dtype=np.float64)
    rc = lib.oracle_pa_decode(_ptr(out), *pr._common(), int(parts), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the problem")
    return out


def decode_select(pr: Problem, sel, nthreads: int = 0) -> np.ndarray:
    """Outputs of selected queries: sel is int [n, 3] of (b, i, h); returns
    float64 [n, D]."""
    lib = _load()
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(-1, 3))
    out = np.zeros((sel.shape[0], pr.d), dtype=np.float64)
    rc = lib.oracle_pa_decode_select(_ptr(out), _ptr(sel), sel.shape[0],
                                     *pr._common(), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the problem or the selection")
    return out


def softmax_weights(pr: Problem, b: int, i: int, h: int) -> np.ndarray:
    """Weights of query (b, i, h) over positions [0, seq_lens[b])."""
    lib = _load()
    w = np.zeros(int(pr.seq_lens[b]), dtype=np.float64)
    rc = lib.oracle_softmax_weights(_ptr(w), int(b), int(i), int(h), *pr._common())
    if rc != 0:
        raise ValueError("oracle rejected the problem or the query")
    return w


def visible_ranges(seq_lens, query_lens, window=0, windows=None):
    """(lo, hi) int32 arrays over every query token, packed in batch order."""
    lib = _load()
    seq_lens = _i32(seq_lens)
    query_lens = _i32(query_lens)
    windows = _i32(windows)
    n = int(query_lens.sum())
    lo = np.zeros(max(n, 1), dtype=np.int32)
    hi = np.zeros(max(n, 1), dtype=np.int32)
    rc = lib.oracle_visible_ranges(_ptr(lo), _ptr(hi), _ptr(seq_lens),
                                   _ptr(query_lens), _ptr(windows), int(window),
                                   int(seq_lens.shape[0]))
    if rc < 0:
        raise ValueError("oracle rejected the lengths")
    return lo[:n], hi[:n]


def max_threads(nthreads: int = 0) -> int:
    """Threads the oracle's parallel loops use (OpenMP), after setting nthreads
    when it is positive."""
    return int(_load().oracle_max_threads(int(nthreads)))


def unreachable_blocks(seq_lens, query_lens, block_size, window=0, windows=None):
    """int32 [batch]: leading blocks of each row no current or later query
    token can see."""
    lib = _load()
    seq_lens = _i32(seq_lens)
    query_lens = _i32(query_lens)
    windows = _i32(windows)
    out = np.zeros(max(int(seq_lens.shape[0]), 1), dtype=np.int32)
    rc = lib.oracle_unreachable_blocks(_ptr(out), _ptr(seq_lens), _ptr(query_lens),
                                       _ptr(windows), int(window), int(block_size),
                                       int(seq_lens.shape[0]))
    if rc != 0:
        raise ValueError("oracle rejected the lengths")
    return out[:seq_lens.shape[0]]


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of FP8 e4m3 codes (uint8), decoded by the oracle."""
    lib = _load()
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.zeros(codes.shape, dtype=np.float64)
    lib.oracle_e4m3_decode(_ptr(out), _ptr(codes), int(codes.size))
    return out
