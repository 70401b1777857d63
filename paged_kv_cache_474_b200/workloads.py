"""Seeded synthetic inputs for paged-attention decode.

This module only draws inputs: lengths, block tables and bf16 values.  It
holds none of the attention arithmetic, so the CUDA path and the float64
oracle can both take their inputs from here without sharing any of the
method.

The five named workloads follow the shapes the pages' tests and benchmarks
use (gllm PR #116 "Verification": scattered out-of-order blocks, GQA, a
5-token prefill chunk over a 300-token context; ExecuTorch PR #18759: long
single-group decode; aiter PR #2914: 1024-token KV blocks with MTP rows):

  tiny        B=2,  Hq=4,  Hkv=2, D=64,  BS=16,   S={37,50},        L=1
  gqa         B=32, Hq=32, Hkv=8, D=128, BS=16,   S~U[1024,8192],   L=1, w=0
  sliding     B=16, Hq=32, Hkv=8, D=128, BS=16,   15 rows S~U[2048,32768] + S=300,
              L = 12x1, 2, 3, 4, 5, w=4096
  long        B=1,  Hq=8,  Hkv=1, D=128, BS=16,   S=131072,         L=1, w=0
  mtp         B=64, Hq=64, Hkv=8, D=128, BS=1024, S~U[4096,65536],  L~U{1..4},
              w=4096 on even rows, 0 on odd rows

Recipe: integer draws come from a CPU ``torch.Generator`` seeded with
4740 + config number; ``U[a,b]`` is inclusive.  The KV pool holds exactly
sum(ceil(S_b/BS)) blocks plus one spare; the pool is randomly permuted and
handed out to the rows in row order; unused block-table slots hold 0.
Values are drawn as float32 (uniform(-1,1) for the tiny workload, standard
normal otherwise) on the requested device and rounded to bf16 (round to
nearest even); both sides then read the same bf16 bytes.  FP8 caches
(kv_dtype="fp8_e4m3") quantise those bf16 values per tensor: scale =
max|x| / 448, codes = round-to-nearest e4m3 of x / scale; FP8 queries
(q_dtype="fp8_e4m3") are quantised the same way.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

CONFIG_NAMES = {1: "tiny", 2: "gqa", 3: "sliding", 4: "long", 5: "mtp"}
CONFIG_TITLES = {
    1: "tiny oracle check: B=2 Hq=4 Hkv=2 D=64 BS=16 S={37,50} L=1",
    2: "GQA decode: B=32 Hq=32 Hkv=8 D=128 BS=16 S~U[1024,8192] L=1 w=0",
    3: "sliding-window mixed batch: B=16 Hq=32 Hkv=8 D=128 BS=16 S~U[2048,32768] w=4096 L=12x1,2,3,4,5(S=300)",
    4: "long-context single-KV-group decode: B=1 Hq=8 Hkv=1 D=128 BS=16 S=131072 L=1 w=0",
    5: "large-block MTP serving: B=64 Hq=64 Hkv=8 D=128 BS=1024 S~U[4096,65536] L~U{1..4} w=4096 even / 0 odd",
}


@dataclasses.dataclass
class Workload:
    """Inputs of one pa_decode call (torch tensors on one device)."""
    q: torch.Tensor              # bf16 [sum(L), Hq, D]
    k_cache: torch.Tensor        # bf16 [num_blocks, Hkv, BS, D]
    v_cache: torch.Tensor        # bf16 [num_blocks, Hkv, BS, D]
    block_tables: torch.Tensor   # int32 [B, max_blocks_per_seq]
    seq_lens: torch.Tensor       # int32 [B]
    query_lens: torch.Tensor     # int32 [B]
    windows: Optional[torch.Tensor]  # int32 [B] or None
    window: int
    scale: float
    name: str = ""
    # FP8 caches: k_cache / v_cache hold e4m3 codes (torch.uint8); a code's
    # value is its e4m3 number times k_scale / v_scale.  1.0 for bf16 caches.
    k_scale: float = 1.0
    v_scale: float = 1.0
    # FP8 queries: q holds e4m3 codes (torch.uint8) whose value is times q_scale
    q_scale: float = 1.0

    @property
    def kv_fp8(self) -> bool:
        return self.k_cache.dtype == torch.uint8

    @property
    def q_fp8(self) -> bool:
        return self.q.dtype == torch.uint8

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def num_q_heads(self) -> int:
        return int(self.q.shape[1])

    @property
    def num_kv_heads(self) -> int:
        return int(self.k_cache.shape[1])

    @property
    def head_dim(self) -> int:
        return int(self.k_cache.shape[3])

    @property
    def block_size(self) -> int:
        return int(self.k_cache.shape[2])

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def num_tokens(self) -> int:
        return int(self.q.shape[0])

    def to(self, device) -> "Workload":
        f = lambda t: None if t is None else t.to(device)
        return dataclasses.replace(
            self, q=f(self.q), k_cache=f(self.k_cache), v_cache=f(self.v_cache),
            block_tables=f(self.block_tables), seq_lens=f(self.seq_lens),
            query_lens=f(self.query_lens), windows=f(self.windows))

    def host_lists(self):
        """Lengths and windows as Python lists (host copies)."""
        s = self.seq_lens.cpu().tolist()
        l = self.query_lens.cpu().tolist()
        w = (self.windows.cpu().tolist() if self.windows is not None
             else [self.window] * len(s))
        return s, l, w

    def subset(self, rows):
        """The given batch rows as a workload of their own, on the CPU: their
        q rows, a compact pool holding only the blocks their tables reach
        (tables renumbered to match, unused slots 0), their lengths and
        windows; scales unchanged.  Data movement only.  Returns (workload,
        row_map) with row_map[original row] = its index in the subset."""
        rows = sorted(set(int(r) for r in rows))
        S, L, _ = self.host_lists()
        bs = self.block_size
        tables = self.block_tables.cpu()
        qoff = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
        phys, new_tables = [], []
        for b in rows:
            nb = (S[b] + bs - 1) // bs
            new_tables.append(list(range(len(phys), len(phys) + nb)))
            phys.extend(tables[b, :nb].tolist())
        mb = max(1, max(len(t) for t in new_tables))
        tab = torch.zeros((len(rows), mb), dtype=torch.int32)
        for j, t in enumerate(new_tables):
            tab[j, :len(t)] = torch.tensor(t, dtype=torch.int32)
        idx = torch.tensor(phys, dtype=torch.long, device=self.k_cache.device)
        sub = dataclasses.replace(
            self,
            q=torch.cat([self.q[qoff[b]:qoff[b + 1]] for b in rows]).cpu(),
            k_cache=self.k_cache.index_select(0, idx).cpu(),
            v_cache=self.v_cache.index_select(0, idx).cpu(),
            block_tables=tab,
            seq_lens=torch.tensor([S[b] for b in rows], dtype=torch.int32),
            query_lens=torch.tensor([L[b] for b in rows], dtype=torch.int32),
            windows=(None if self.windows is None
                     else self.windows.cpu()[torch.tensor(rows, dtype=torch.long)].clone()))
        return sub, {b: j for j, b in enumerate(rows)}


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a cache or q tensor's bit patterns: uint16 for bf16,
    uint8 for FP8 codes (already uint8)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.uint8:
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _values(shape, dist: str, g: torch.Generator, device):
    """float32 draws rounded to bf16.  Large tensors are drawn in chunks along
    dim 0 so the float32 staging stays under 1 GiB."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    per_row = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    step = max(1, (1 << 28) // max(per_row, 1))
    for a in range(0, shape[0], step):
        b = min(shape[0], a + step)
        sub = (b - a,) + tuple(shape[1:])
        if dist == "uniform":
            x = torch.rand(sub, generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0
        else:
            x = torch.randn(sub, generator=g, device=device, dtype=torch.float32)
        out[a:b] = x.to(torch.bfloat16)
    return out


def to_e4m3(x: torch.Tensor):
    """Per-tensor FP8 e4m3 codes of x (uint8) and their scale: the scale
    maps the largest |x| to 448, the largest finite e4m3 number; torch's
    float8_e4m3fn cast rounds to nearest."""
    amax = float(x.abs().max()) if x.numel() else 1.0
    s = (amax / 448.0) if amax > 0 else 1.0
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    per_row = int(np.prod(x.shape[1:])) if x.dim() > 1 else 1
    step = max(1, (1 << 28) // max(per_row, 1))  # float32 staging under 1 GiB
    for a in range(0, max(x.shape[0], 0), step):
        b = min(x.shape[0], a + step)
        codes[a:b] = (x[a:b].float() / s).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, s


def make_workload(*, seq_lens: Sequence[int], query_lens: Sequence[int],
                  num_q_heads: int, num_kv_heads: int, head_dim: int,
                  block_size: int, window: int = 0,
                  windows: Optional[Sequence[int]] = None,
                  scale: Optional[float] = None, dist: str = "normal",
                  seed: int = 0, device="cpu", spare_blocks: int = 1,
                  extra_table_cols: int = 0, name: str = "",
                  kv_dtype: str = "bf16", q_dtype: str = "bf16") -> Workload:
    """Build a workload with explicit lengths.  Blocks are a random permutation
    of a pool of sum(ceil(S_b/BS)) + spare_blocks blocks handed out in row
    order; unused block-table slots (and ``extra_table_cols`` padding columns)
    hold 0."""
    seq_lens = [int(s) for s in seq_lens]
    query_lens = [int(x) for x in query_lens]
    B = len(seq_lens)
    if len(query_lens) != B:
        raise ValueError("seq_lens and query_lens lengths differ")
    gi = _gen(seed, "cpu")
    nblk = [(s + block_size - 1) // block_size for s in seq_lens]
    n_used = sum(nblk)
    num_blocks = n_used + spare_blocks
    perm = torch.randperm(num_blocks, generator=gi).to(torch.int32)
    mbps = max(1, max(nblk) if nblk else 1) + extra_table_cols
    tables = torch.zeros((B, mbps), dtype=torch.int32)
    pos = 0
    for b, n in enumerate(nblk):
        tables[b, :n] = perm[pos:pos + n]
        pos += n
    gv = _gen(seed + 1, device)
    ntok = sum(query_lens)
    q = _values((max(ntok, 0), num_q_heads, head_dim), dist, gv, device)
    k = _values((num_blocks, num_kv_heads, block_size, head_dim), dist, gv, device)
    v = _values((num_blocks, num_kv_heads, block_size, head_dim), dist, gv, device)
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    win_t = None if windows is None else torch.tensor(list(windows), dtype=torch.int32)
    ks = vs = 1.0
    if kv_dtype == "fp8_e4m3":
        k, ks = to_e4m3(k)
        v, vs = to_e4m3(v)
    elif kv_dtype != "bf16":
        raise ValueError(f"unknown kv_dtype {kv_dtype}")
    qs = 1.0
    if q_dtype == "fp8_e4m3":
        q, qs = to_e4m3(q)
    elif q_dtype != "bf16":
        raise ValueError(f"unknown q_dtype {q_dtype}")
    return Workload(q=q, k_cache=k, v_cache=v, block_tables=tables.to(device),
                    seq_lens=torch.tensor(seq_lens, dtype=torch.int32).to(device),
                    query_lens=torch.tensor(query_lens, dtype=torch.int32).to(device),
                    windows=None if win_t is None else win_t.to(device),
                    window=int(window), scale=float(scale), name=name,
                    k_scale=float(ks), v_scale=float(vs), q_scale=float(qs))


def config_lengths(cfg: int):
    """(seq_lens, query_lens, window, windows) of a named workload."""
    g = _gen(4740 + cfg, "cpu")
    ri = lambda lo, hi, n: torch.randint(lo, hi + 1, (n,), generator=g).tolist()
    if cfg == 1:
        return [37, 50], [1, 1], 0, None
    if cfg == 2:
        return ri(1024, 8192, 32), [1] * 32, 0, None
    if cfg == 3:
        s = ri(2048, 32768, 15) + [300]
        l = [1] * 12 + [2, 3, 4] + [5]
        return s, l, 4096, None
    if cfg == 4:
        return [131072], [1], 0, None
    if cfg == 5:
        s = ri(4096, 65536, 64)
        l = ri(1, 4, 64)
        w = [4096 if b % 2 == 0 else 0 for b in range(64)]
        return s, l, 0, w
    raise ValueError(f"unknown workload {cfg}")


_SHAPES = {
    1: dict(num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16, dist="uniform", scale=1.0 / 8.0),
    2: dict(num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16, dist="normal"),
    3: dict(num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16, dist="normal"),
    4: dict(num_q_heads=8, num_kv_heads=1, head_dim=128, block_size=16, dist="normal"),
    5: dict(num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=1024, dist="normal"),
}


def config_workload(cfg: int, device="cpu", window: Optional[int] = None,
                    kv_dtype: str = "bf16", q_dtype: str = "bf16",
                    rows: Optional[int] = None) -> Workload:
    """One of the five named workloads.  ``window`` overrides the scalar window
    (the tiny workload is run at window 0 and window 8); kv_dtype="fp8_e4m3"
    quantises its caches to per-tensor-scaled FP8.  ``rows`` keeps only the
    first rows of the batch (their lengths and windows unchanged; the pool
    then holds only their blocks), a reduced case for profiling."""
    s, l, w, ws = config_lengths(cfg)
    if rows is not None:
        s, l = s[:rows], l[:rows]
        ws = None if ws is None else ws[:rows]
    if window is not None:
        w = int(window)
    return make_workload(seq_lens=s, query_lens=l, window=w, windows=ws,
                         seed=4740 + cfg, device=device, name=CONFIG_NAMES[cfg],
                         kv_dtype=kv_dtype, q_dtype=q_dtype, **_SHAPES[cfg])
