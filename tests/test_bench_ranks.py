"""The host side of bench.py --gpus N (one process per GPU, replicas): two
gloo ranks on the CPU check that the job time is the slowest rank's on every
rank, that the throughput counts every rank's layer, and that the ranks draw
different layers (weak scaling, no data-path collective)."""

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, str(ROOT))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    import synth
    ms = bench.reduce_max_ms([5.0, 7.5][rank], world, "cpu")
    cfg = bench.rank_config(synth.get_config("toy-256"), rank)
    w = synth.make_w(cfg, cfg.sublayers[0])
    out.put((rank, ms, bench.job_throughput(cfg.weights, world, 4, ms), float(w[0, 0]), cfg.seed))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_draw_distinct_layers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, w0, s0), (r1, ms1, v1, w1, s1) = res
    assert ms0 == ms1 == 7.5                       # the slowest rank's time on both
    assert v0 == v1 == pytest.approx(65536 * 2 * 4 / 7.5e-3 / 1e6)
    assert s1 == s0 + 1 and w0 != w1                # different seeds, different layers


def test_stage_marks_attribute_each_interval_to_the_stage_it_closes():
    sys.path.insert(0, str(ROOT))
    import bench

    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    m = bench.StageMarks(stream=None)
    m.events = [("start", Ev(0.0)), ("covariance", Ev(7.0)), ("biip_sensitivity", Ev(7.5)),
                ("inverse_cholesky", Ev(10.0)), ("solver", Ev(11.25)), ("pack", Ev(11.5)),
                ("inverse_cholesky", Ev(12.0)), ("solver", Ev(12.5)), ("pack", Ev(12.75))]
    assert m.totals() == {"covariance": 7.0, "biip_sensitivity": 0.5, "inverse_cholesky": 3.0,
                          "solver": 1.75, "pack": 0.5}


def test_draw_to_device_equals_the_host_generator():
    """Ranks whose host copies would not fit draw their inputs chunk by chunk
    straight into device memory; the result is the host generator's matrix
    bit for bit (here into CPU memory with two threads, on a token count
    whose last chunk is ragged)."""
    sys.path.insert(0, str(ROOT))
    import dataclasses
    import torch
    import bench
    import synth
    cfg = dataclasses.replace(synth.get_config("toy-256"), tokens=2 * synth.CHUNK_TOKENS + 100)
    site, sub = cfg.sites[0], cfg.sublayers[0]
    X = bench.draw_to_device(lambda c: synth.x_chunk(cfg, site, c), cfg.tokens, site.width, "cpu", 2)
    G = bench.draw_to_device(lambda c: synth.g_chunk(cfg, sub, c), cfg.tokens, sub.m, "cpu", 2)
    assert torch.equal(X.view(torch.int16), torch.from_numpy(synth.make_x(cfg, site).view(np.int16)))
    assert torch.equal(G.view(torch.int16), torch.from_numpy(synth.make_g(cfg, sub).view(np.int16)))


def test_lean_inputs_only_where_the_host_copies_would_not_fit():
    """The Llama-3-70B MLP workload's inputs are 38.7 GB per rank: with their
    pinned copies one rank fits a 196 GiB host, two do not."""
    sys.path.insert(0, str(ROOT))
    import bench
    import synth
    cfg = synth.get_config("llama3-70b-mlp")
    assert bench.host_input_bytes(cfg) == 262144 * 2 * (8192 + 28672 + 28672 + 8192)
    ram = 196 * 2 ** 30
    assert not bench.needs_lean_inputs(cfg, 1, True, ram)
    assert bench.needs_lean_inputs(cfg, 2, True, ram)
    assert not bench.needs_lean_inputs(cfg, 2, False, ram)
    assert bench.needs_lean_inputs(cfg, 4, False, ram)
