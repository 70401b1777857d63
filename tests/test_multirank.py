"""Multi-process checks of the N>1 path on CPU (gloo, world size 2).

Rows are independent units, so N GPUs decode disjoint rows (or, in the bench,
replicas of the workload) with no data-path exchange.  These tests run the
host logic that path relies on with two gloo ranks: each rank decodes its
own rows (with the oracle standing in for the device), the union of the ranks'
outputs equals the single-process result exactly, and the bench's
max-over-ranks timing reduction picks the slowest rank.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from paged_kv_cache_474_b200.workloads import bf16_bits, make_workload

        wl = make_workload(seq_lens=[37, 50, 300, 40, 9, 128], query_lens=[1, 2, 5, 1, 3, 1],
                           num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16,
                           window=16, seed=21)
        rows = [b for b in range(wl.batch) if b % world == rank]
        qoff = np.concatenate([[0], np.cumsum(wl.query_lens.numpy())])
        sel = [(b, i, h) for b in rows for i in range(int(wl.query_lens[b]))
               for h in range(wl.num_q_heads)]
        pr = oracle.Problem(bf16_bits(wl.q), bf16_bits(wl.k_cache), bf16_bits(wl.v_cache),
                            wl.block_tables.numpy(), wl.seq_lens.numpy(),
                            wl.query_lens.numpy(), wl.scale, wl.window)
        mine = oracle.decode_select(pr, sel, nthreads=1)
        full = np.zeros((int(qoff[-1]), wl.num_q_heads, wl.head_dim))
        for (b, i, h), v in zip(sel, mine):
            full[qoff[b] + i, h] = v
        t = torch.from_numpy(full)
        dist.all_reduce(t)          # disjoint rows: the sum is the union
        # bench-style timing: every rank reports its elapsed time, the max wins
        elapsed = torch.tensor([1.0 + rank], dtype=torch.float64)
        dist.all_reduce(elapsed, op=dist.ReduceOp.MAX)
        if rank == 0:
            np.save(os.path.join(out_dir, "sharded.npy"), t.numpy())
            np.save(os.path.join(out_dir, "single.npy"), oracle.decode(pr, nthreads=1))
            np.save(os.path.join(out_dir, "elapsed.npy"), elapsed.numpy())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_row_sharding_needs_no_exchange_and_timing_takes_the_max(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    sharded = np.load(tmp_path / "sharded.npy")
    single = np.load(tmp_path / "single.npy")
    assert np.array_equal(sharded, single)
    assert float(np.load(tmp_path / "elapsed.npy")[0]) == 2.0
