"""Data-parallel delayed scaling on two CPU ranks (gloo): the per-step amax all-reduce.

Each rank measures the amax of its shard of every tensor (what the quantize launches leave
in the rings' amax slots under fp8_set_ring_fold_mode(1)), then runs
``fold_rings_data_parallel`` -- gather, all-reduce(MAX), fold -- against a stand-in for the
library's gather and fold kernels built on the oracle's ring (test code only).  Both ranks
must end with identical rings, equal to one process folding the amax of the whole tensors.

Definitions: AstrAI compare view, astrai/extension/fp8.py (_ScaleRing: hist[idx] = amax, the
step from the window); the cross-rank maximum is the data-parallel reading of that fold.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import quantize as Q
from oracle import scaling as S

WORLD = 2
HIST = 4
STEPS = 3
RINGS = 3


class OracleRingLib:
    """Stand-in for the library's ring gather / fold kernels: oracle rings on the host."""

    @staticmethod
    def fp8_scale_ring_collect_amax(rings, amax_out, stream=None):
        for i, r in enumerate(rings):
            amax_out[i] = float(r.state[r.n + 2])

    @staticmethod
    def fp8_scale_ring_fold(rings, amax, stream=None):
        for i, r in enumerate(rings):
            r.fold(np.float32(amax[i].item()), r.scale)


def _tensor(step, ring):
    g = torch.Generator().manual_seed(1000 * step + ring)
    return (torch.randn(64, 48, generator=g) * (2.0 ** (step - ring))).numpy().astype(np.float32)


def _new_rings():
    rings = [S.Ring(HIST, "e4m3") for _ in range(RINGS)]
    for i, r in enumerate(rings):
        r.seed(_tensor(-1, i))
    return rings


def _worker(rank, port, out):
    from fp8_delayed_scaling_amax_b200 import dp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        rings = _new_rings()
        buf = torch.zeros(RINGS, dtype=torch.float32)
        for step in range(STEPS):
            for i, r in enumerate(rings):
                shard = np.array_split(_tensor(step, i), WORLD, axis=0)[rank]
                r.state[r.n + 2] = Q.amax(shard)  # what this rank's quantize leaves in the slot
            dp.fold_rings_data_parallel(rings, buf, lib=OracleRingLib)
            for r in rings:
                r.advance()
        out[rank] = np.stack([r.state.copy() for r in rings])
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_fold_the_global_amax():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    # one process over the whole tensors
    ref = _new_rings()
    for step in range(STEPS):
        for i, r in enumerate(ref):
            r.fold(Q.amax(_tensor(step, i)), r.scale)
            r.advance()
    want = np.stack([r.state for r in ref])
    for rank in range(WORLD):
        assert np.array_equal(out[rank].view(np.uint32), want.view(np.uint32)), rank
