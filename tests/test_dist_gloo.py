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
