"""Host logic of bench.py's multi-GPU path, run as two gloo ranks on the CPU: each rank gets its
own units (weak scaling, no data-path collective), and durations reduce to the max over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from titans_long_term_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.WORKLOADS["mlp-d64-b2h4-t2k"]
        units = bench.rank_units(w, rank)
        inp = synth.make_inputs(w, units=units, T=64)
        mx = bench.max_over_ranks(10.0 + rank, torch.device("cpu"), world)
        out[rank] = (units, float(inp["k"].float().sum()), mx)
    finally:
        dist.destroy_process_group()


def test_two_ranks_disjoint_units_and_max_duration():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (u0, s0, m0), (u1, s1, m1) = out[0], out[1]
    assert set(u0).isdisjoint(u1) and len(u0) == len(u1) == 8
    assert s0 != s1  # different units draw different data
    assert m0 == m1 == 11.0


def test_single_rank_max_is_identity():
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5
