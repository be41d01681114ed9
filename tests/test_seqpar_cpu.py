"""The exchange of the sequence-parallel prefill on CPU ranks (gloo).

Every rank holds one consecutive run of the same sequences, forms the run's
affine map with the oracle, and the package's ``gather_segment_maps`` collects
all maps in rank order.  Composing them must give each rank the oracle state at
the start of its run and every rank the oracle's final state; a mix-up of rank
order, of H and Lambda, or of the packing fails it.  (The GPU side of the same
protocol, the maps, the composition and the per-run prefill in the library's
kernels, is checked in test_gpu_segmented.py.)
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_97_b200.seqpar import gather_segment_maps


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(update, gate, BH=2, T=45, dk=8, dv=6, seed=31):
    r = np.random.default_rng(seed)
    k = r.standard_normal((BH, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = r.standard_normal((BH, T, dk))
    v = r.standard_normal((BH, T, dv))
    g = {"none": None, "scalar": r.uniform(-0.2, 0.0, (BH, T)), "channel": r.uniform(-0.2, 0.0, (BH, T, dk))}[gate]
    beta = r.uniform(0.1, 1.0, (BH, T)) if update == "delta" else None
    S0 = 0.3 * r.standard_normal((BH, dv, dk))
    return q, k, v, g, beta, S0


def _cuts(T, world):
    # uneven runs: rank r gets a different length than its neighbours
    w = np.arange(1, world + 1, dtype=np.float64)
    c = np.concatenate([[0], np.cumsum(w / w.sum() * T)]).round().astype(int)
    c[-1] = T
    return c


def _worker(rank, world, port, update, gate, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, g, beta, S0 = _inputs(update, gate)
        c = _cuts(q.shape[1], world)
        a, b = c[rank], c[rank + 1]
        sl = lambda x: None if x is None else x[:, a:b]
        H, Lam = oracle.segment_maps(update, gate, k[:, a:b], v[:, a:b], g=sl(g), beta=sl(beta))
        H_all, Lam_all = gather_segment_maps(torch.from_numpy(H), None if update == "additive" else
                                             torch.from_numpy(Lam))
        assert tuple(H_all.shape) == (world,) + H.shape
        S = S0
        starts = []
        for i in range(world):
            starts.append(S)
            L = np.eye(S0.shape[-1]) if Lam_all is None else Lam_all[i].numpy()
            S = S @ L + H_all[i].numpy()
        _, S_here = oracle.gdn_forward(update, gate, q[:, :a], k[:, :a], v[:, :a], g=None if g is None else g[:, :a],
                                       beta=None if beta is None else beta[:, :a], S0=S0) if a else (None, S0)
        _, ST = oracle.gdn_forward(update, gate, q, k, v, g=g, beta=beta, S0=S0)
        scale = np.sqrt(np.mean(ST ** 2))
        out[rank] = (float(np.max(np.abs(starts[rank] - S_here)) / scale), float(np.max(np.abs(S - ST)) / scale))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("update,gate,world", [("delta", "scalar", 2), ("delta", "channel", 3),
                                                ("additive", "none", 2), ("decay", "scalar", 3)])
def test_gathered_maps_compose_to_the_oracle(update, gate, world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, update, gate, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == list(range(world))
    for r, (e_start, e_final) in res.items():
        assert e_start < 1e-12 and e_final < 1e-12, (r, e_start, e_final)
