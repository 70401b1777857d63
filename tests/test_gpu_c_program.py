"""A plain C program calls pa_decode on device memory (no Python, no torch in
that process) and gets the same dst as the Python binding's call, bit for bit,
within the parity tolerance of the float64 oracle."""
import os
import subprocess

import numpy as np
import pytest
import torch

from tests.parity_helpers import check_full

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_474_b200")
from paged_kv_cache_474_b200.workloads import make_workload  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"


def _build(tmp_path):
    exe = tmp_path / "c_decode_device"
    libdir = os.path.dirname(pa.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                    os.path.join(ROOT, "tests", "c_decode_device.c"), "-o", str(exe),
                    "-L", libdir, "-lpagedattn", f"-Wl,-rpath,{libdir}",
                    "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"], check=True)
    return exe


@pytest.mark.parametrize("case", ["split", "one_shot", "windowed"])
def test_c_program_decodes_like_the_binding(cuda_device, tmp_path, case):
    if case == "split":
        wl = make_workload(seq_lens=[5000, 1200, 77], query_lens=[1, 3, 2], num_q_heads=16,
                           num_kv_heads=4, head_dim=128, block_size=16, seed=71)
    elif case == "one_shot":
        wl = make_workload(seq_lens=[40, 60], query_lens=[1, 1], num_q_heads=8,
                           num_kv_heads=2, head_dim=64, block_size=32, seed=72)
    else:
        wl = make_workload(seq_lens=[3000, 300], query_lens=[2, 5], num_q_heads=8,
                           num_kv_heads=1, head_dim=128, block_size=64, window=700, seed=73)
    exe = _build(tmp_path)
    d = tmp_path / "data"
    d.mkdir()
    span, qlen = pa.pa_extents_host(*wl.host_lists()[:2], window=wl.window)
    with open(d / "dims.txt", "w") as f:
        f.write(" ".join(str(x) for x in (
            wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
            wl.num_blocks, wl.max_blocks_per_seq, wl.window, repr(float(wl.scale)), span, qlen,
            wl.num_tokens)))
    for name, t in (("q", wl.q), ("k", wl.k_cache), ("v", wl.v_cache),
                    ("tables", wl.block_tables), ("seq_lens", wl.seq_lens),
                    ("query_lens", wl.query_lens)):
        t.contiguous().view(torch.uint8).numpy().tofile(d / f"{name}.bin")
    r = subprocess.run([str(exe), str(d)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.startswith("ok"), (r.returncode, r.stdout, r.stderr)
    got = torch.from_numpy(np.fromfile(d / "dst.bin", dtype=np.uint8)).view(torch.bfloat16)
    got = got.reshape(wl.q.shape)
    ref = pa.decode(wl.to("cuda:0")).cpu()
    assert torch.equal(got, ref)
    check_full(wl, got, f"C program {case}")
