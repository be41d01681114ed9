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
    # per token-head: q,k,v bf16 (768 B) + o in the input dtype (256 B) + g + beta (8 B);
    # S0 and S_T per head -- 1.0989 GB per launch
    assert bench.prefill_bytes(w) == 128 * (8192 * 1032 + 2 * 128 * 128 * 4)
    # the fp32 o the kernel writes: 512 B per token-head
    assert bench.prefill_bytes(w, out_bytes=4) == 128 * (8192 * 1288 + 2 * 128 * 128 * 4)
    assert bench.prefill_flops(w) == 128 * 8192 * (10 * 64 * 128 + 6 * 128 * 128)
    wd = WORKLOADS["decode_gdn_bf16"]
    assert bench.decode_bytes_per_step(wd) == 8192 * (2 * 65536 + 768 + 512 + 8)


def test_roofline_fraction_uses_input_dtype_output_bytes():
    from synth import WORKLOADS
    w = WORKLOADS["gdn_prefill_bf16"]
    peaks = {"hbm_gbs": 6454.3, "bf16_tflops": 1693.9}
    rf = bench.roofline(w, 0.5, peaks, "measured")
    assert abs(rf["frac"] - 1.0989e9 / 0.5e-3 / 6454.3e9) < 1e-3
    assert rf["fp32_output"]["frac"] > rf["frac"]


def test_bench_gpus_flag_starts_that_many_ranks():
    """``bench.py --gpus 2`` run as one process starts two ranks (torchrun on
    127.0.0.1) and rank 0's line reports n_gpus = 2 (rank protocol only, gloo)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--launch-check",
                          "--steps", "4", "--warmup", "3"], capture_output=True, text=True, timeout=240, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(ln) for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["ms_per_step"] == 2.0


def test_bench_rejects_gpus_not_matching_world_size():
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="3")
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--launch-check"],
                         capture_output=True, text=True, timeout=120, env=env)
    assert out.returncode != 0
