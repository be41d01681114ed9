"""gdn_chunk_fwd_segmented_noalloc: the segmented prefill with its scratch in
the library's fixed device array instead of a caller workspace.

CPU: the entry point is exported and rejects bad or oversized requests before
touching the device.  GPU: the same results as the workspace variant (bit for
bit: the same kernels on the same inputs), parity with the oracle, and no
device allocation during the call.
"""
import ctypes

import pytest

import gated_delta_rule_97_b200 as gdn


@pytest.fixture(scope="module")
def lib():
    gdn.build()
    return gdn.load()


def _desc(B=1, H=2, T=256, d=128):
    return gdn.make_desc(B, H, T, d, d, "delta", "scalar", gdn.BF16, gdn.F32)


def test_scratch_size_is_exported(lib):
    assert lib.gdn_noalloc_scratch_bytes() == 32 << 20


def test_rejects_before_touching_the_device(lib):
    vp = ctypes.c_void_p
    f = lib.gdn_chunk_fwd_segmented_noalloc
    args = (vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000), None, vp(0x100000), None, None)
    d = _desc()
    assert f(ctypes.byref(d), 0, *args) == -1                       # nseg < 1
    assert f(None, 2, *args) == -1                                  # no descriptor
    big = _desc(B=64, H=16, T=4096)                                 # 4096 segment-heads: 805 MB of scratch
    assert lib.gdn_segmented_workspace_bytes(ctypes.byref(big), 4) > lib.gdn_noalloc_scratch_bytes()
    assert f(ctypes.byref(big), 4, *args) == -3                     # larger than the array
    empty = _desc(B=0)
    assert f(ctypes.byref(empty), 4, *args) == 0                    # nothing to do, no device work
    # a malformed request is an argument error whatever its size, as in the
    # workspace variant: T not a multiple of nseg, too many segment-heads
    bad = _desc(B=64, H=16, T=4095)
    assert f(ctypes.byref(bad), 4, *args) == -1
    assert lib.gdn_chunk_fwd_segmented(ctypes.byref(bad), 4, *args[:-1], vp(0x7000000), 1 << 40, None) == -1
    huge = _desc(B=1 << 15, H=1 << 15, T=64)                        # 2^30 heads x 2 segments
    assert f(ctypes.byref(huge), 2, *args) == -1
    assert lib.gdn_segmented_workspace_bytes(ctypes.byref(huge), 2) == 0


@pytest.mark.gpu
def test_matches_workspace_variant_and_oracle_without_allocating():
    import torch

    import oracle
    from gpu_util import TOL, dev, np64, rel_err
    from synth import WORKLOADS, make_prefill_inputs

    assert torch.cuda.is_available()
    gdn.device_status(clear=True)
    w = WORKLOADS["gdn_prefill_bf16"].with_(B=1, H=4, T=1500, s0_std=0.05, name="noalloc")
    x = make_prefill_inputs(w)
    t = {k: (None if v is None else dev(v, torch.bfloat16 if k in ("q", "k", "v") else torch.float32))
         for k, v in x.items()}
    o1, S1 = gdn.chunk_fwd_segmented(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], update="delta",
                                     gate="scalar", nseg=5)
    o2 = torch.empty_like(o1)
    S2 = torch.empty_like(S1)
    torch.cuda.synchronize()
    gdn.chunk_fwd_segmented_noalloc(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], update="delta",
                                    gate="scalar", nseg=5, o=o2, S_T=S2)  # warm: maps the array
    o2.zero_()
    torch.cuda.synchronize()
    # torch's allocator counter, and the device's free memory (which also sees a
    # cudaMalloc / cudaMallocAsync inside the library)
    before = torch.cuda.memory_allocated()
    free_before = torch.cuda.mem_get_info()[0]
    gdn.chunk_fwd_segmented_noalloc(t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], update="delta",
                                    gate="scalar", nseg=5, o=o2, S_T=S2)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    assert torch.cuda.mem_get_info()[0] == free_before
    assert gdn.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    ro, rS = oracle.gdn_forward("delta", "scalar", x["q"], x["k"], x["v"], g=x["g"], beta=x["beta"], S0=x["S0"])
    assert rel_err(np64(o2), ro) <= TOL["bf16"] and rel_err(np64(S2), rS) <= TOL["bf16"]
