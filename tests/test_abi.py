"""C-ABI checks that need no GPU: the library loads, exports every function
declared in include/gdn.h, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

import gated_delta_rule_97_b200 as gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    gdn.build()
    return gdn.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("gdn_chunk_fwd", "gdn_decode_step", "gdn_strerror"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.lib_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (gdn_[a-z_0-9]+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_strerror_and_version(lib):
    assert gdn.version() == 7  # the chunkwise tensor-core backward joined the boundary
    for code in (0, -1, -2, -3, -4, -5, -6, 123):
        assert isinstance(gdn.strerror(code), str) and gdn.strerror(code)


def _desc(**kw):
    base = dict(B=2, H=3, T=100, dk=128, dv=128, update="delta", gate="scalar", dtype=gdn.BF16,
                out_dtype=gdn.F32)
    base.update(kw)
    return gdn.make_desc(**base)


def _call(lib, d, q=0x10000, k=0x20000, v=0x30000, g=0x40000, beta=0x50000, S0=None, o=0x9000000,
          ST=None):
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_chunk_fwd(ctypes.byref(d) if d is not None else None, vp(q), vp(k), vp(v), vp(g), vp(beta),
                             vp(S0), vp(o), vp(ST), None)


def test_rejects_bad_arguments_without_launching(lib):
    # Every call below fails validation, which happens before any CUDA call.
    assert _call(lib, None) == -1
    assert _call(lib, _desc(dk=96)) == -1
    assert _call(lib, _desc(dv=32)) == -1
    assert _call(lib, _desc(update=None) if False else gdn.Desc(2, 3, 100, 128, 128, 7, 1, 1, 0, 64, 0)) == -1
    assert _call(lib, _desc(update="additive", gate="scalar")) == -1       # additive takes no gate
    assert _call(lib, _desc(update="decay", gate="none"), g=None) == -1   # decay needs a gate
    assert _call(lib, _desc(gate="none")) == -1                           # g given but gate none
    assert _call(lib, _desc(), g=None) == -1                              # gate but no g
    assert _call(lib, _desc(), beta=None) == -1                           # delta needs beta
    assert _call(lib, _desc(), q=None) == -1
    assert _call(lib, _desc(T=-1)) == -1
    assert _call(lib, _desc(chunk=32)) == -3
    assert _call(lib, _desc(), k=0x20008) == -2                           # misaligned
    assert _call(lib, _desc(), o=0x10000 + 64) == -1                      # o overlaps q


def test_empty_batch_is_a_noop(lib):
    assert _call(lib, _desc(B=0)) == 0
    assert _call(lib, _desc(H=0), q=None, k=None, v=None, g=None, beta=None, o=None) == 0


def test_unknown_prologue_bits_are_rejected(lib):
    d = _desc(prologue=16)
    assert _call(lib, d) == -1
    d = _desc(prologue=1 | 2 | 4 | 8, B=0)
    assert _call(lib, d) == 0


def test_decode_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    d = _desc(T=17)
    assert lib.gdn_decode_step(ctypes.byref(d), vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000),
                               vp(0x100000), vp(0x6000), None) == -3   # T > GDN_DECODE_MAX_T
    d = _desc(T=-1)
    assert lib.gdn_decode_step(ctypes.byref(d), vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000),
                               vp(0x100000), vp(0x6000), None) == -1   # negative T
    d = _desc(T=0)
    assert lib.gdn_decode_step(ctypes.byref(d), vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000),
                               vp(0x100000), vp(0x6000), None) == 0    # no tokens: no-op, no launch
    d = _desc(T=1)
    assert lib.gdn_decode_step(ctypes.byref(d), vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000),
                               vp(0x100004), vp(0x6000), None) == -2   # misaligned state
    assert lib.gdn_decode_step(ctypes.byref(d), vp(0x1000), vp(0x2000), vp(0x3000), None, vp(0x5000),
                               vp(0x100000), vp(0x6000), None) == -1   # gate without g


def test_product_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    args = (vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000), None, vp(0x100000), None, None)
    lib.gdn_product_fwd.argtypes = [ctypes.c_void_p, ctypes.c_int] + [ctypes.c_void_p] * 9
    d = _desc()
    assert lib.gdn_product_fwd(ctypes.byref(d), 0, *args) == -1      # nh < 1
    assert lib.gdn_product_fwd(ctypes.byref(d), 17, *args) == -3     # nh > GDN_PRODUCT_MAX_NH
    d = _desc(update="additive", gate="none")
    assert lib.gdn_product_fwd(ctypes.byref(d), 2, *args) == -1      # only the delta rule has substeps
    d = _desc(algo="tc", dtype=gdn.F32)
    assert lib.gdn_product_fwd(ctypes.byref(d), 3, *args) == -3      # tensor-core kernel: bf16 inputs only
    d = _desc()
    d.algo = 3
    assert lib.gdn_product_fwd(ctypes.byref(d), 2, *args) == -1      # no such kernel choice
    d = _desc(B=0)
    assert lib.gdn_product_fwd(ctypes.byref(d), 2, *args) == 0       # empty batch: no-op


def test_segmented_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    lib.gdn_chunk_fwd_segmented.argtypes = [ctypes.c_void_p, ctypes.c_int] + [ctypes.c_void_p] * 9 + \
        [ctypes.c_size_t, ctypes.c_void_p]
    lib.gdn_segmented_workspace_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.gdn_segmented_workspace_bytes.restype = ctypes.c_size_t
    d = _desc(T=96)
    need = lib.gdn_segmented_workspace_bytes(ctypes.byref(d), 3)
    assert need == 2 * 3 * 3 * (2 * 128 * 128 + 128 * 128) * 4
    args = (vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000), None, vp(0x100000), None)
    assert lib.gdn_chunk_fwd_segmented(ctypes.byref(d), 0, *args, vp(0x9000000), need, None) == -1  # nseg < 1
    assert lib.gdn_chunk_fwd_segmented(ctypes.byref(d), 5, *args, vp(0x9000000), need, None) == -1  # 96 % 5
    assert lib.gdn_chunk_fwd_segmented(ctypes.byref(d), 3, *args, vp(0x9000000), need - 4, None) == -1  # small
    assert lib.gdn_chunk_fwd_segmented(ctypes.byref(d), 3, *args, None, need, None) == -1  # no workspace
    assert lib.gdn_chunk_fwd_segmented(ctypes.byref(d), 3, *args, vp(0x9000008), need, None) == -2  # misaligned


def test_segment_maps_reject_bad_arguments(lib):
    vp = ctypes.c_void_p
    lib.gdn_segment_maps.argtypes = [ctypes.c_void_p] + [ctypes.c_void_p] * 8
    d = _desc(T=96)
    ins = (vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000))
    H, L = vp(0x9000000), vp(0xA000000)
    assert lib.gdn_segment_maps(ctypes.byref(d), *ins, None, L, None) == -1           # no H
    assert lib.gdn_segment_maps(ctypes.byref(d), *ins, H, None, None) == -1           # no Lambda
    assert lib.gdn_segment_maps(ctypes.byref(d), *ins, H, vp(0xA000004), None) == -2  # misaligned
    assert lib.gdn_segment_maps(ctypes.byref(d), *ins, H, vp(0x9000010), None) == -1  # H and Lambda overlap
    assert lib.gdn_segment_maps(ctypes.byref(d), vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000),
                                vp(0x3000), L, None) == -1                             # H over v
    assert lib.gdn_segment_maps(ctypes.byref(d), None, *ins[1:], H, L, None) == -1    # q missing
    d = _desc(B=0)
    assert lib.gdn_segment_maps(ctypes.byref(d), *ins, None, None, None) == 0          # empty batch: no-op


def test_compose_segments_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    lib.gdn_compose_segments.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 6
    S0, H, L, Si, ST = vp(0x1000000), vp(0x2000000), vp(0x4000000), vp(0x6000000), vp(0x8000000)
    f = lib.gdn_compose_segments
    assert f(4, 0, 128, 128, S0, H, L, Si, ST, None) == -1        # nseg < 1
    assert f(-1, 2, 128, 128, S0, H, L, Si, ST, None) == -1       # negative count
    assert f(4, 2, 96, 128, S0, H, L, Si, ST, None) == -1         # unsupported dk
    assert f(4, 2, 128, 128, S0, None, L, Si, ST, None) == -1     # no H
    assert f(4, 2, 128, 128, S0, H, L, vp(0x6000008), ST, None) == -2  # misaligned
    assert f(4, 2, 128, 128, S0, H, L, vp(0x2000000 + 4096), ST, None) == -1  # S_in over H
    assert f(4, 2, 128, 128, S0, H, L, Si, vp(0x1000000 + 4096), None) == -1  # S_T partly over S0
    assert f(0, 2, 128, 128, S0, H, L, Si, ST, None) == 0         # no sequences: no-op


def test_host_pipeline_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    f = lib.gdn_chunk_fwd_host
    f.argtypes = [ctypes.c_void_p, ctypes.c_int] + [ctypes.c_void_p] * 9 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gdn_host_workspace_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int]
    lib.gdn_host_workspace_bytes.restype = ctypes.c_size_t
    d = _desc(T=96)
    need = lib.gdn_host_workspace_bytes(ctypes.byref(d), 4)
    # 6 heads in slices of 2: q, k, v (bf16), g, beta, S0, o (fp32), S_T per slot, each 256-aligned
    per = lambda n: (n + 255) // 256 * 256
    slot = sum(per(2 * x) for x in (96 * 128 * 2, 96 * 128 * 2, 96 * 128 * 2, 96 * 4, 96 * 4, 128 * 128 * 4,
                                    96 * 128 * 4, 128 * 128 * 4))
    assert need == 2 * slot
    args = (vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000), None, vp(0x100000), None)
    ws = vp(0x9000000)
    assert f(ctypes.byref(d), 0, *args, ws, need, None) == -1              # n_slices < 1
    assert f(ctypes.byref(d), 4, *args, ws, need - 1, None) == -1          # workspace too small
    assert f(ctypes.byref(d), 4, *args, None, need, None) == -1            # no workspace
    assert f(ctypes.byref(d), 4, *args, vp(0x9000010), need, None) == -2   # workspace not 256-aligned
    assert f(ctypes.byref(d), 4, vp(0x1000), vp(0x2000), vp(0x3000), vp(0x4000), vp(0x5000), None, vp(0x2000),
             None, ws, need, None) == -1                                   # o over an input
    d = _desc(B=0)
    assert f(ctypes.byref(d), 4, *args, None, 0, None) == 0                # empty batch: no-op


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(gdn, "_lib", None)
    monkeypatch.setattr(gdn, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        gdn.load()


def test_backward_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    f = lib.gdn_chunk_bwd
    f.argtypes = [ctypes.c_void_p] * 16 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gdn_bwd_workspace_bytes.argtypes = [ctypes.c_void_p]
    lib.gdn_bwd_workspace_bytes.restype = ctypes.c_size_t
    d = _desc(T=130)  # delta, scalar gate, B2 H3 dk=dv=128
    need = lib.gdn_bwd_workspace_bytes(ctypes.byref(d))
    assert need == 6 * 3 * 128 * 128 * 4  # six heads, three chunk-boundary states each
    ins = [vp(0x100000), vp(0x200000), vp(0x300000), vp(0x400000), vp(0x500000), None, vp(0x600000), None]
    outs = [vp(0x1000000), vp(0x1100000), vp(0x1200000), vp(0x1300000), vp(0x1400000), None]
    ws = vp(0x2000000)
    assert f(ctypes.byref(d), *ins, *outs, ws, need - 16, None) == -1          # workspace too small
    assert f(ctypes.byref(d), *ins, *outs[:4], None, None, ws, need, None) == -1  # delta without dbeta
    assert f(ctypes.byref(d), *ins, *outs[:3], None, outs[4], None, ws, need, None) == -1  # gate without dg
    bad = list(outs)
    bad[1] = vp(0x1100004)
    assert f(ctypes.byref(d), *ins, *bad, ws, need, None) == -2                # misaligned
    bad = list(outs)
    bad[2] = vp(0x100010)
    assert f(ctypes.byref(d), *ins, *bad, ws, need, None) == -1                # dv overlaps q
    assert f(ctypes.byref(d), *ins, *outs, vp(0x1100000), need, None) == -1   # workspace overlaps dk
    p = _desc(T=130)
    p.prologue = 1 | 2 | 4 | 8
    need_p = lib.gdn_bwd_workspace_bytes(ctypes.byref(p))
    ntok = 6 * 130
    extra = sum((x + 255) // 256 * 256 for x in (ntok * 128 * 4, ntok * 128 * 4, ntok * 128 * 4, ntok * 4)) + ntok * 4
    assert need_p == (need + 255) // 256 * 256 + extra  # + the mapped q, k, v, beta, g in fp32
    assert f(ctypes.byref(p), *ins, *outs, ws, need, None) == -1              # room for the mapped inputs too
    e = _desc(B=0)
    assert f(ctypes.byref(e), *ins, *outs, ws, 0, None) == 0                   # empty batch: no-op


def test_saved_state_entry_points_reject_bad_arguments(lib):
    vp = ctypes.c_void_p
    lib.gdn_chunk_fwd_states.argtypes = [ctypes.c_void_p] + [ctypes.c_void_p] * 10
    lib.gdn_chunk_bwd_states.argtypes = [ctypes.c_void_p] + [ctypes.c_void_p] * 15
    fw = lambda d, states: lib.gdn_chunk_fwd_states(ctypes.byref(d), vp(0x10000), vp(0x20000), vp(0x30000),
                                                     vp(0x40000), vp(0x50000), None, vp(0x9000000), None,
                                                     states, None)
    d = _desc()
    assert fw(d, None) == -1                                  # no states buffer
    assert fw(d, vp(0x7000008)) == -2                         # misaligned
    assert fw(d, vp(0x10000)) == -1                           # overlaps q
    assert fw(_desc(dtype=gdn.F32), vp(0x70000000)) == -3     # the tensor-core forward takes bf16 only
    d = _desc()
    d.prologue = 1
    assert fw(d, vp(0x70000000)) == -3                        # no input prologue with saved states
    bw = lambda d, states: lib.gdn_chunk_bwd_states(ctypes.byref(d), vp(0x10000), vp(0x20000), vp(0x30000),
                                                     vp(0x40000), vp(0x50000), states, None, None,
                                                     vp(0x1000000), vp(0x2000000), vp(0x3000000),
                                                     vp(0x4000000), vp(0x5000000), None, None)
    assert bw(_desc(), None) == -1                            # states required
    d = _desc()
    d.prologue = 1
    assert bw(d, vp(0x70000000)) == -3


def test_tensor_core_backward_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    lib.gdn_bwd_tc_workspace_bytes.argtypes = [ctypes.c_void_p]
    lib.gdn_bwd_tc_workspace_bytes.restype = ctypes.c_size_t
    f = lib.gdn_chunk_bwd_tc
    f.argtypes = [ctypes.c_void_p] * 16 + [ctypes.c_size_t, ctypes.c_void_p]
    d = _desc(T=130)  # delta, scalar gate, B2 H3 dk=dv=128: 18 chunk-heads
    n = 6 * 3
    cc, cd, ss = n * 64 * 64 * 4, n * 64 * 128 * 4, n * 128 * 128 * 4
    # T, A, P (.) Gamma; W, K>, Q~; the state gradients; b_C (on 256-byte boundaries)
    assert lib.gdn_bwd_tc_workspace_bytes(ctypes.byref(d)) == 3 * cc + 3 * cd + ss + 256
    a = _desc(T=130, update="additive", gate="none")
    assert lib.gdn_bwd_tc_workspace_bytes(ctypes.byref(a)) == cc + cd + ss + 256  # A, Q~ only
    need = lib.gdn_bwd_tc_workspace_bytes(ctypes.byref(d))
    ins = [vp(0x100000), vp(0x200000), vp(0x300000), vp(0x400000), vp(0x500000), vp(0x600000), None, None]
    outs = [vp(0x1000000), vp(0x1100000), vp(0x1200000), vp(0x1300000), vp(0x1400000), None]
    ws = vp(0x20000000)
    assert f(ctypes.byref(d), *ins, *outs, ws, need - 16, None) == -1          # workspace too small
    assert f(ctypes.byref(d), *ins, *outs, None, need, None) == -1             # no workspace
    no_states = list(ins)
    no_states[5] = None
    assert f(ctypes.byref(d), *no_states, *outs, ws, need, None) == -1         # states required
    bad = list(outs)
    bad[0] = vp(0x1000008)
    assert f(ctypes.byref(d), *ins, *bad, ws, need, None) == -2                # misaligned
    assert f(ctypes.byref(d), *ins, *outs, vp(0x1100000), need, None) == -1   # workspace overlaps dk
    for unsupported in (_desc(T=130, gate="channel"), _desc(T=130, dk=64, dv=64), _desc(B=65536, H=1, T=130)):
        assert lib.gdn_bwd_tc_workspace_bytes(ctypes.byref(unsupported)) == 0
        assert f(ctypes.byref(unsupported), *ins, *outs, ws, need, None) == -3
    p = _desc(T=130)
    p.prologue = 1
    assert f(ctypes.byref(p), *ins, *outs, ws, need, None) == -3              # no input prologue
    e = _desc(B=0)
    assert f(ctypes.byref(e), *ins, *outs, ws, 0, None) == 0                   # empty batch: no-op
    # gdn_chunk_bwd with GDN_ALGO_TC: the forward's states, then the same workspace
    lib.gdn_bwd_workspace_bytes.argtypes = [ctypes.c_void_p]
    lib.gdn_bwd_workspace_bytes.restype = ctypes.c_size_t
    b = lib.gdn_chunk_bwd
    b.argtypes = [ctypes.c_void_p] * 16 + [ctypes.c_size_t, ctypes.c_void_p]
    t = _desc(T=130, algo="tc")
    need_t = lib.gdn_bwd_workspace_bytes(ctypes.byref(t))
    assert need_t == ss + need  # 18 chunk states of 64 KB (256-byte multiple), then the tensor-core workspace
    bins = [vp(0x100000), vp(0x200000), vp(0x300000), vp(0x400000), vp(0x500000), None, None, None]
    assert b(ctypes.byref(t), *bins, *outs, ws, need_t - 16, None) == -1       # workspace too small
    for unsupported in (_desc(T=130, gate="channel", algo="tc"), _desc(T=130, dtype=gdn.F32, algo="tc")):
        assert lib.gdn_bwd_workspace_bytes(ctypes.byref(unsupported)) == 0
        assert b(ctypes.byref(unsupported), *bins, *outs, ws, need_t, None) == -3


def test_checked_prefill_rejects_bad_arguments(lib):
    f = lib.gdn_chunk_fwd_checked
    f.argtypes = [ctypes.c_void_p] * 10
    vp = ctypes.c_void_p
    d = _desc()
    args = [vp(0x10000), vp(0x20000), vp(0x30000), vp(0x40000), vp(0x50000)]
    assert f(ctypes.byref(d), *args, vp(0x7000000), vp(0x9000000), vp(0x7000000), None) == -1  # S_T is S0
    assert f(None, *args, None, vp(0x9000000), None, None) == -1                               # no desc
    bad = _desc()
    bad.update = 7
    assert f(ctypes.byref(bad), *args, None, vp(0x9000000), None, None) == -1


def test_wait_limit_hook(lib):
    lib.gdn_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    assert lib.gdn_set_wait_limit_ns(5) == 0
    assert lib.gdn_set_wait_limit_ns(0) == 0  # back to the default bound
