"""The multi-rank host path on CPU: two gloo ranks shard the sequences of a
small workload, run the VJP on their slices (the CPU oracle stands in for the
GPU kernels) and sum the codebook gradient; the result must equal the
single-process VJP of all sequences, and the step time is the maximum over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bcjr_sum_product_b200 import dist as bdist
from bcjr_sum_product_b200 import inputs as I


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import oracle
    L, k, V, T = 6, 2, 1, 0.4
    w, c, g = I.random_case(L, k, V, 7, 24, seed=123)
    a, b = bdist.shard_rows(w.shape[0], rank, world)

    def local_vjp(wl, cb, gl):
        r = oracle.vjp(wl, cb, L, k, V, T, gl, nthreads=1)
        return torch.from_numpy(r["grad_w"]), torch.from_numpy(r["grad_c"]).clone()

    gw, gc = bdist.vjp_data_parallel(local_vjp, w[a:b], c, g[a:b])
    t = bdist.max_over_ranks(float(rank + 1))
    np.save(os.path.join(out_dir, f"gw{rank}.npy"), gw.numpy())
    np.save(os.path.join(out_dir, f"gc{rank}.npy"), gc.numpy())
    np.save(os.path.join(out_dir, f"t{rank}.npy"), np.array([t, a, b]))
    dist.barrier()
    dist.destroy_process_group()


def _bench_worker(rank, world, port, out_dir, replicate):
    """bench.py's own multi-rank step (its row split and its two halves), with
    the CPU oracle as the local soft codeword and VJP."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import oracle
    inp = I.make("tiny")
    wl, T = inp.wl, inp.wl.temps[0]
    w, g, a, b = bench.local_problem(inp.w, inp.g, rank, world, replicate)
    soft_out = {}

    def soft_fn(w_, c_):
        soft_out["soft"] = oracle.soft(w_, c_, wl.L, wl.k, wl.V, T, nthreads=1)["soft"]

    def vjp_fn(w_, c_, g_):
        r = oracle.vjp(w_, c_, wl.L, wl.k, wl.V, T, g_, nthreads=1)
        return torch.from_numpy(r["grad_w"]), torch.from_numpy(r["grad_c"]).clone()

    first, second = bench.path_halves(soft_fn, vjp_fn, w, inp.c, g)
    first()
    gw, gc = second()
    np.save(os.path.join(out_dir, f"b_soft{rank}.npy"), soft_out["soft"])
    np.save(os.path.join(out_dir, f"b_gw{rank}.npy"), gw.numpy())
    np.save(os.path.join(out_dir, f"b_gc{rank}.npy"), gc.numpy())
    np.save(os.path.join(out_dir, f"b_rows{rank}.npy"), np.array([a, b]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("replicate", [False, True])
def test_bench_step_on_two_gloo_ranks(tmp_path, replicate):
    """The bench's N > 1 step on CPU: sharded, the ranks' slices tile the
    workload and the summed codebook gradient is the single-process one;
    replicated, every rank holds the whole workload and the sum is twice it."""
    import oracle
    port = _free_port()
    mp.start_processes(_bench_worker, args=(2, port, str(tmp_path), replicate), nprocs=2, join=True,
                       start_method="spawn")
    inp = I.make("tiny")
    wl, T = inp.wl, inp.wl.temps[0]
    ref_s = oracle.soft(inp.w, inp.c, wl.L, wl.k, wl.V, T, nthreads=1)["soft"]
    ref = oracle.vjp(inp.w, inp.c, wl.L, wl.k, wl.V, T, inp.g, nthreads=1)
    rows = [np.load(tmp_path / f"b_rows{r}.npy") for r in range(2)]
    if replicate:
        assert all(list(r) == [0, wl.n_seq] for r in rows)
        soft = np.load(tmp_path / "b_soft0.npy")
        gw = np.load(tmp_path / "b_gw0.npy")
        gc_expect = 2 * ref["grad_c"]
    else:
        assert rows[0][0] == 0 and rows[0][1] == rows[1][0] and rows[1][1] == wl.n_seq
        soft = np.concatenate([np.load(tmp_path / f"b_soft{r}.npy") for r in range(2)])
        gw = np.concatenate([np.load(tmp_path / f"b_gw{r}.npy") for r in range(2)])
        gc_expect = ref["grad_c"]
    np.testing.assert_allclose(soft, ref_s, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gw, ref["grad_w"], rtol=1e-12, atol=1e-12)
    for r in range(2):
        np.testing.assert_allclose(np.load(tmp_path / f"b_gc{r}.npy"), gc_expect, rtol=1e-12, atol=1e-12)


def test_shard_rows_partition():
    for n in (0, 1, 7, 16, 16384):
        for world in (1, 2, 3, 8):
            spans = [bdist.shard_rows(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_match_single_process(tmp_path):
    import oracle
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    L, k, V, T = 6, 2, 1, 0.4
    w, c, g = I.random_case(L, k, V, 7, 24, seed=123)
    ref = oracle.vjp(w, c, L, k, V, T, g, nthreads=1)
    gw = np.concatenate([np.load(tmp_path / f"gw{r}.npy") for r in range(2)])
    np.testing.assert_allclose(gw, ref["grad_w"], rtol=1e-12, atol=1e-12)
    for r in range(2):
        np.testing.assert_allclose(np.load(tmp_path / f"gc{r}.npy"), ref["grad_c"], rtol=1e-12, atol=1e-12)
        assert np.load(tmp_path / f"t{r}.npy")[0] == 2.0
