"""Multi-rank host logic on CPU (gloo, world size 2): the benchmark's barrier
and max-over-ranks timing reduction.  The data path has no collective (every
rank runs its own batch), so this is the whole N > 1 protocol."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, "cpu")
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5


def test_algorithmic_work_counts():
    from synth import WORKLOADS
    w = WORKLOADS["gdn_prefill_bf16"]
    # per token-head: q,k,v bf16 (768 B) + o fp32 (512 B) + g + beta (8 B); S0 and S_T per head
    assert bench.prefill_bytes(w) == 128 * (8192 * 1288 + 2 * 128 * 128 * 4)
    assert bench.prefill_flops(w) == 128 * 8192 * (10 * 64 * 128 + 6 * 128 * 128)
    wd = WORKLOADS["decode_gdn_bf16"]
    assert bench.decode_bytes_per_step(wd) == 8192 * (2 * 65536 + 768 + 512 + 8)
