"""Failure detection without faulting, trapping or hanging a GPU.

* GPU: a test build of the library (-DATTN_SELFTEST, a 2e6-cycle wait budget)
  runs a kernel whose bounded mbarrier wait can never complete (nothing
  arrives).  The wait must expire, set ATTN_DEV_TIMEOUT and the site id in the
  workspace status words, and the context must stay usable afterwards.
* CPU: in a 2-rank gloo job one rank dies before the collective; the other
  rank's collective must end with an error inside the process-group timeout
  instead of waiting forever.
"""

import ctypes
import datetime
import os
import socket
import subprocess
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _build_selftest_lib(tmpdir):
    from exact_io_aware_46_b200 import build as b

    so = os.path.join(tmpdir, "libattn_selftest.so")
    cmd = [b.nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           "-DATTN_SELFTEST", "-DATTN_WAIT_CYCLES=2000000LL", b.SRC, b.SRC_NOALLOC, "-o", so]
    subprocess.check_call(cmd)
    return so


def test_selftest_library_builds(tmp_path):
    so = _build_selftest_lib(str(tmp_path))
    lib = ctypes.CDLL(so)
    assert hasattr(lib, "attn_selftest_expired_wait")
    # the product library does not carry the self-test
    import exact_io_aware_46_b200 as attn

    assert not hasattr(attn.lib(), "attn_selftest_expired_wait")


@pytest.mark.gpu
def test_expired_wait_reports_timeout_and_context_survives(tmp_path):
    import torch

    import exact_io_aware_46_b200 as attn
    import synth

    so = _build_selftest_lib(str(tmp_path))
    lib = ctypes.CDLL(so)
    lib.attn_selftest_expired_wait.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.attn_selftest_expired_wait.restype = ctypes.c_int
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    t0 = time.time()
    assert lib.attn_selftest_expired_wait(ctypes.c_void_p(ws.data_ptr()), 42, stream) == 0
    torch.cuda.synchronize()
    words = ws.view(torch.int32)[:4].tolist()
    assert words[0] & attn.ATTN_DEV_TIMEOUT and words[3] == 42
    assert time.time() - t0 < 30
    # the context is still usable: an ordinary forward runs and is finite
    q = synth.to_torch_bf16(synth.normal_bf16(1, (1, 1, 64, 64))).cuda()
    O, L = attn.attn_fwd(q, q, q)
    torch.cuda.synchronize()
    assert torch.isfinite(O.float()).all() and torch.isfinite(L).all()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(0)  # this rank leaves between steps, before the collective
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, world)
        result = "completed"
    except Exception as e:  # noqa: BLE001
        result = "error:" + type(e).__name__
    with open(out, "w") as f:
        f.write(f"{result} {time.time() - t0:.1f}")


def test_dead_rank_ends_collective_with_error(tmp_path):
    import torch.multiprocessing as mp

    out = str(tmp_path / "r0")
    ctx = mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=False,
                             start_method="spawn")
    deadline = time.time() + 120
    while not ctx.join(timeout=5):
        assert time.time() < deadline, "surviving rank did not finish"
    res, secs = open(out).read().split()
    assert res.startswith("error:") and float(secs) < 60
