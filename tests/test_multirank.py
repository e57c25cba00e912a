"""The N > 1 host logic of bench.py on CPU with gloo (world size 2): every
rank gets its own layer (distinct seeds, same shapes), the step time is the
max over ranks, and the per-rank work needs no data exchange -- shown by each
rank quantizing a slice of its own layer with the oracle independently."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import oracle
    import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        wl = bench.rank_workload(rank)
        seeds = [m.seed for m in wl.matrices]
        shapes = [(m.out, m.inp) for m in wl.matrices]
        # a small slice of this rank's gate weight, generated and quantized locally
        W = workloads.weight(8, 512, 0.015, 0.001, 10.0, wl.matrices[0].seed)
        bits = W.view(torch.uint16).numpy()
        S, _, _ = oracle.global_scale(bits, wl.q_max)
        codes, scales, _ = oracle.sweep_quantize(bits, None, float(S), -9, 6)
        t = bench.max_over_ranks(float(rank + 1) * 0.5, ws)
        out[rank] = (seeds, shapes, t, int(scales.sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ws = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(ws, port, out), nprocs=ws, join=True, start_method="spawn")
    r0, r1 = out[0], out[1]
    assert r0[1] == r1[1]                      # same layer shapes on every rank
    assert set(r0[0]).isdisjoint(r1[0])        # but independent layers (seeds)
    assert r0[2] == r1[2] == 1.0               # step time = max over ranks
    assert r0[3] != r1[3]                      # different data, different scales


@pytest.mark.parametrize("out,n", [(28672, 8192), (100, 400), (64, 48), (64, 144), (7, 4112)])
def test_gptq_update_flops_count_every_cross_part_column_pair(out, n):
    """The GPTQ bench line's flop count: the update GEMMs make one multiply-add
    per row for every column pair i < k in different 128-column parts (pairs
    inside a part are the batch kernel's), three split products each."""
    import bench
    sizes = [min(128, n - i) for i in range(0, n, 128)]
    pairs = (n * n - sum(s * s for s in sizes)) // 2
    assert bench.gptq_update_flops(out, n) == 6.0 * out * pairs
